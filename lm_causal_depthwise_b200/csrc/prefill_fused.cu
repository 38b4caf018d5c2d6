// prefill_fused.cu -- fused sm_100a prefill of the RG-LRU block core (bf16 I/O, fp32 state).
//
// One persistent kernel, launched as clusters of two CTAs per head: CTA rank r
// owns channels [128 r, 128 r + 128) of the head (one TMEM lane per channel).
// Both CTAs of a cluster walk the same sequence of tiles (32 tokens of one
// sequence, claimed in order from the head's ticket counter by rank 0, which
// writes each tile descriptor into both CTAs).  Per tile:
//   conv warps   thread = channel: causal depthwise conv (k=4, document mask)
//                of its channel over the tile in fp32; xc / 2 goes to TMEM (fp32)
//                for the scan, its bf16 copy into the MMA B tile of BOTH
//                CTAs (the two halves of the head's 256 input channels meet in
//                each CTA's shared memory through the cluster).
//   MMA thread   both block-diagonal gate projections on the tensor cores:
//                D[128 out x 32 tok] = W[128 x 256] * xc^T with A (this half's
//                rows of W_a or W_x) resident in TMEM, written once by the scan
//                warps, and B in shared memory; fp32 accumulators in TMEM.
//   scan warps   thread = channel, two groups taking alternate tiles.  Pass 1:
//                sigmoid gates, a = sigmoid(Lambda)^(8 r), sqrt(1-a^2)
//                normaliser, resets, GELU_tanh(g) (the g tile arrives by one
//                tensor load); the local scan from h = 0 gives the tile
//                aggregate (prod a, h_end) and, per token, the output without
//                the carried-in state, y_loc = G h_loc, and its coefficient
//                q = G prod a, stashed in shared memory as f16 pairs (the
//                accumulators and xc are free again at once).
//   look-back    publish each tile aggregate as soon as pass 1 ends, walk back
//   warps        over predecessor tiles of the sequence to the nearest anchor
//                (a published inclusive prefix, or a tile holding a reset: A =
//                0), fold h <- A h + H forward from it in sequence order
//                (decoupled look-back with a fixed combination order, so
//                results are bit-reproducible), publish the inclusive prefix,
//                then pass 2 of the tile: y = y_loc + q h_in from the stash,
//                4 channels per lane, stored straight to global memory.
//   scheduler    rank 0 claims tiles and fills both CTAs' descriptor rings;
//                each CTA TMA-loads its own channels of x (tile + 3 halo rows).
// Every wait is bounded: a wait that runs out records RGLRU_ERR_TIMEOUT in the
// workspace header and the CTA unwinds (waiting, bounded, for its own copies
// and MMAs in flight), meets its peer at the final cluster barrier and frees
// its TMEM.
//
// Block structure: "Gemma explained: RecurrentGemma architecture",
// RecurrentGemmaRecurrentBlock printout (Conv1d k=4, padding=3, groups=D; GELU
// tanh) and section "Residual block with recurrent block"; RG-LRU equations of
// Griffin / RecurrentGemma (arXiv 2404.07839).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <mutex>
#include <type_traits>

#include "internal.h"
#include "sm100.cuh"

namespace rglru {
namespace {

using namespace sm100;

constexpr int NT = 32;          // tokens per tile (MMA N)
constexpr int kHalf = 128;      // channels per CTA (MMA M, TMEM lanes)
constexpr int NX = 4;           // xc/2 slots in TMEM (conv -> pass 1), fp32
constexpr int NA = 2;           // accumulator slots in TMEM (MMA -> pass 1), one per scan group
constexpr int NS = 6;           // stash slots in shared memory (pass 1 -> look-back and pass 2)
constexpr int NB = 2;           // B tiles in shared memory (conv -> MMA, both CTAs)
constexpr int XRING = 2;        // x tiles in shared memory (TMA -> conv)
constexpr int INFO_RING = 16;   // tile descriptors in flight
constexpr int kClaimBatch = 4;  // consecutive tickets claimed by one atomic
constexpr int kScanGroups = 2;  // scan warp groups, alternate tiles
constexpr int kScanWarps = 4 * kScanGroups, kConvWarps = 4;
constexpr int kConvWarp0 = kScanWarps;
constexpr int kMmaWarp = kConvWarp0 + kConvWarps, kSchedWarp = kMmaWarp + 1;
constexpr int kLbWarp0 = kMmaWarp + 2, kLbWarps = 6;
constexpr int kThreads = 32 * (kLbWarp0 + kLbWarps);
constexpr int kGroupThreads = 128;  // threads of one scan group or of the conv warps (one per channel)
constexpr int kEndMarkers = kLbWarps > kScanGroups ? kLbWarps : kScanGroups;
// every barrier array is visited one phase at a time by each waiter: a scan
// group's tiles use only its own accumulator and stash slots, a look-back
// warp's tiles revisit a stash slot every lcm(kLbWarps, NS) = NS tiles
static_assert(NA % kScanGroups == 0 && NS % kScanGroups == 0 && NS % kLbWarps == 0, "slot residues");
static_assert(kEndMarkers <= INFO_RING, "end markers fit the ring");

// TMEM columns (512): this half's rows of W_a then W_x (the MMA's A operand,
// bf16 pairs: K-step kk of a gate at column 8 kk), accumulators
// [pre_r | pre_i], xc/2 in fp32 (one column per token)
constexpr uint32_t kColW = 0, kColsWGate = 128;
constexpr uint32_t kColAcc = kColW + 2 * kColsWGate, kColsAcc = 2 * NT;
constexpr uint32_t kColXh = kColAcc + NA * kColsAcc, kColsXh = NT;
static_assert(kColXh + NX * kColsXh <= 512, "TMEM budget");

// Shared memory map (offsets from a 1024-byte aligned base)
// B tile (bf16 xc/2 of all 256 channels of the head), N-major: 8 channels x
// NT tokens per group of core matrices
constexpr int kBGroup = 8 * NT * 2;             // 512 bytes
constexpr int kBTile = 32 * kBGroup;            // 16 KB
constexpr int kBHalf = 16 * kBGroup;            // one CTA's 128 channels: 8 KB, contiguous
constexpr int kXRows = NT + 3;
constexpr int kXTile = kXRows * kHalf * 2;      // bf16 x of this half, 3 halo rows first
constexpr int OFF_B = 0;
constexpr int OFF_X = OFF_B + NB * kBTile;
constexpr int kGTile = NT * kHalf * 2;          // bf16 GELU branch of this half: [token][channel]
constexpr int OFF_G = OFF_X + XRING * kXTile;   // one per scan group
// stash slots: per token t and channel c, (y_loc, q) as an f16 pair at
// (t * 128 + c) * 4 (a look-back lane reads its 4 channels of a token at once)
constexpr int kStash = NT * kHalf * 4;
constexpr int OFF_ST = OFF_G + kScanGroups * kGTile;
// per stash slot: (prod a, h_end) per channel from pass 1
constexpr int OFF_AGG = OFF_ST + NS * kStash;
constexpr int OFF_INFO = OFF_AGG + NS * kHalf * 8;
constexpr int OFF_BAR = OFF_INFO + INFO_RING * 32;
// barrier arrays: [first index, count]
enum {
    B_INFO_FULL = 0,
    B_INFO_EMPTY = B_INFO_FULL + INFO_RING,
    B_X_FULL = B_INFO_EMPTY + INFO_RING,
    B_X_EMPTY = B_X_FULL + XRING,
    B_XH_FREE = B_X_EMPTY + XRING,
    B_BCONV = B_XH_FREE + NX,
    B_BFREE = B_BCONV + NB,
    B_MMA = B_BFREE + NB,
    B_ACC_FREE = B_MMA + NA,
    B_PASS1 = B_ACC_FREE + NA,
    B_STASH_FREE = B_PASS1 + NS,   // the look-back warp is done with the stash slot (and its aggregate)
    B_BHALF = B_STASH_FREE + NS,   // this CTA's half of a B tile written (before the copy to the peer)
    B_W_FULL = B_BHALF + NB,
    B_GFULL = B_W_FULL + 1,           // per scan group: the GELU-branch tile of its next tile has landed
    B_GFREE = B_GFULL + kScanGroups,  // per scan group: pass 1 has read the GELU-branch tile
    B_COUNT = B_GFREE + kScanGroups
};
constexpr int OFF_MISC = OFF_BAR + B_COUNT * 8;
constexpr int kSmemUsed = OFF_MISC + 16;
constexpr int kSmemBytes = kSmemUsed + 1024;    // slack for the 1024-byte alignment
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(OFF_B % 1024 == 0 && kBTile % 1024 == 0 && kXTile % 128 == 0, "alignment");

constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s per wait

struct TileInfo {
    int u;        // tile index inside the head's sequence of tiles, -1 = no more work
    int b, t0, valid;
    uint32_t reset_mask;  // bit t: segment_pos == 0 at token t0 + t (conv tap of lag 1 dropped, h reset)
    uint32_t m2, m3;      // bit t: segment_pos < 2 (< 3): conv tap of lag 2 (3) dropped
    int first_last;       // bit 0: first tile of the sequence, bit 1: last tile
};
static_assert(sizeof(TileInfo) == 32, "TileInfo size");

struct FusedParams {
    int B, T, D, C, tiles_per_head;
    const __nv_bfloat16 *x, *g;
    const float *conv_w, *conv_b;
    const float *b_a, *b_x, *lambda;
    const __nv_bfloat16 *w_a, *w_x;  // [D rows][256] (row = output channel)
    const int32_t *segpos;
    __nv_bfloat16 *conv_state;
    float *h_state;
    __nv_bfloat16 *y;
    WsHeader *hdr;
    uint32_t *flags;   // [2 H][tiles_per_head]: one scan chain per (head, half)
    float2 *agg;       // [2 H][tiles_per_head][128]  (prod a, h_end) from h = 0
    float *prefix;     // [2 H][tiles_per_head][128]  h after the tile
    unsigned long long *trace;  // RGLRU_TRACE builds only: per-role timestamps
};

// Tracing (compiled in with -DRGLRU_TRACE only): CTAs below kTraceCtas record
// %globaltimer at each role's milestones for their first kTraceTiles tiles,
// into trace[(cta * kTraceTiles + tile) * kTraceEvents + event].
enum TraceEvent {
    TR_SCHED_INFO, TR_CONV_START, TR_CONV_DONE, TR_MMA_ISSUED, TR_P1_START, TR_P1_END, TR_LB_START,
    TR_LB_HIN, TR_LB_DONE, TR_P2_START, TR_P2_END, TR_TILE_U, TR_MMA_TFREE, TR_MMA_TMA, TR_MMA_CONV,
    TR_CONV_GO, TR_CONV_LOOP, TR_P1_G, TR_P1_LD, TR_LB_ANC, TR_LB_K, kTraceEvents
};
#ifdef RGLRU_TRACE
constexpr int kTraceCtas = 4, kTraceTiles = 192;
#define RGLRU_TR(ev, j, val)                                                                                   \
    do {                                                                                                      \
        if (p.trace != nullptr && blockIdx.x < kTraceCtas && (j) < kTraceTiles)                               \
            p.trace[((size_t)blockIdx.x * kTraceTiles + (j)) * kTraceEvents + (ev)] = (val);                  \
    } while (0)
#else
#define RGLRU_TR(ev, j, val) \
    do {                     \
    } while (0)
#endif

constexpr uint32_t F_AGG = 1u, F_PREFIX = 2u, F_RESET = 4u;

__device__ __forceinline__ void raise_timeout(volatile int *abort_flag, WsHeader *hdr, int where)
{
    atomicCAS(&hdr->status, 0, (int)RGLRU_ERR_TIMEOUT);
    atomicCAS(&hdr->detail, 0, (int)(blockIdx.x << 8) | (where + 1));
    *abort_flag = 1;
}

// Bounded wait on an mbarrier phase; false on timeout or when the CTA is aborting.
__device__ __noinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag, WsHeader *hdr,
                                      int where)
{
    if (mbar_try_wait_cl(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        // suspended in hardware until the phase completes (or a time limit
        // passes); the abort and timeout checks run every 16th round
        if (mbar_try_wait_sleep_cl(bar, parity, 20000u)) return true;
        if ((it & 15u) == 0) {
            if (*abort_flag) return false;
            if (*(volatile int *)&hdr->status != 0) {
                *abort_flag = 1;
                return false;
            }
            if (globaltimer() - t0 > kTimeoutNs) {
                raise_timeout(abort_flag, hdr, where);
                return false;
            }
        }
    }
}

// Bounded spin on a global flag by one thread; 0 on timeout/abort.
__device__ __noinline__ uint32_t wait_flag(const uint32_t *f, uint32_t need, volatile int *abort_flag,
                                           WsHeader *hdr, int where)
{
    uint32_t v = ld_acquire_u32(f);
    if (v & need) return v;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        __nanosleep(64);
        v = ld_acquire_u32(f);
        if (v & need) return v;
        if ((it & 31u) == 0) {
            if (*abort_flag) return 0;
            if (*(volatile int *)&hdr->status != 0) {
                *abort_flag = 1;
                return 0;
            }
            if (globaltimer() - t0 > kTimeoutNs) {
                raise_timeout(abort_flag, hdr, where);
                return 0;
            }
        }
    }
}

// Warp-collective forms: lane 0 waits, the result is broadcast, then every lane
// performs its own (already satisfied) acquire so that the warp stays converged
// for the .sync.aligned tcgen05 instructions that follow.
__device__ __noinline__ bool warp_wait_bar_slow(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                                WsHeader *hdr, int where)
{
    uint32_t ok = 1;
    if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, abort_flag, hdr, where) ? 1u : 0u;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) {
        // the phase is complete, so each lane's own test passes at once unless
        // the barrier had already moved on a further phase (a logic error,
        // reported rather than waited on)
        bool seen = false;
        for (uint32_t it = 0; it < (1u << 20) && !(seen = mbar_try_wait_cl(bar, parity)); ++it) {
        }
        if (!__all_sync(0xffffffffu, seen)) {
            if ((threadIdx.x & 31) == 0) raise_timeout(abort_flag, hdr, where + 32);
            ok = 0;
        }
    }
    return ok != 0;
}

// Fast path: a phase that is already complete costs one test per lane and a vote.
__device__ __forceinline__ bool warp_wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                              WsHeader *hdr, int where)
{
    if (__all_sync(0xffffffffu, mbar_try_wait_cl(bar, parity))) return true;
    return warp_wait_bar_slow(bar, parity, abort_flag, hdr, where);
}

// Flags only gain bits during a launch; the value lane 0 saw drives every lane's
// control flow, each lane's own acquire load orders its later data loads.
__device__ __forceinline__ uint32_t warp_wait_flag(const uint32_t *f, uint32_t need, volatile int *abort_flag,
                                                   WsHeader *hdr, int where)
{
    uint32_t v = 0;
    if ((threadIdx.x & 31) == 0) v = wait_flag(f, need, abort_flag, hdr, where);
    v = __shfl_sync(0xffffffffu, v, 0);
    if (v) (void)ld_acquire_u32(f);
    return v;
}

// Decoupled look-back, first half: walking back from tile `hi` (>= seq_first),
// find the nearest anchor -- a tile whose inclusive prefix is published, or a
// tile holding a reset (A = 0: its prefix is its own H) -- such that every tile
// between the anchor and `hi` has published its aggregate.  Lane l examines
// tile hi - l, so 32 flags cost one round trip.  The first tile of the
// sequence is an anchor only once its prefix (or its reset) is out.
// Warp-collective; false on timeout or abort.
__device__ __noinline__ bool find_anchor(const uint32_t *flags, int hi, int seq_first, int &anchor,
                                         uint32_t &anchor_flag, volatile int *abort_flag, WsHeader *hdr)
{
    const int lane = threadIdx.x & 31;
    uint64_t t0 = 0;
    for (uint32_t spins = 0;;) {
        const int pu = hi - lane;
        const bool in = pu >= seq_first;
        const uint32_t f = in ? ld_acquire_u32(flags + pu) : 0u;
        const uint32_t anchors = __ballot_sync(0xffffffffu, in && (f & (F_PREFIX | F_RESET)));
        const uint32_t ready = __ballot_sync(0xffffffffu, in && (f & F_AGG));
        if (anchors) {
            const int la = __ffs(anchors) - 1;
            const uint32_t span = la ? ((1u << la) - 1u) : 0u;
            if ((ready & span) == span) {
                anchor = hi - la;
                anchor_flag = __shfl_sync(0xffffffffu, f, la);
                return true;
            }
        } else if (ready == 0xffffffffu && hi - 31 > seq_first) {
            hi -= 32;  // 32 aggregates, no anchor yet, the sequence start not reached: look further back
            continue;
        }
        if (t0 == 0) t0 = globaltimer();
        __nanosleep(64);
        if ((++spins & 31u) == 0) {
            uint32_t stop = 0;
            if (lane == 0) {
                if (*abort_flag) {
                    stop = 1;
                } else if (*(volatile int *)&hdr->status != 0) {
                    *abort_flag = 1;
                    stop = 1;
                } else if (globaltimer() - t0 > kTimeoutNs) {
                    raise_timeout(abort_flag, hdr, 12);
                    stop = 1;
                }
            }
            if (__shfl_sync(0xffffffffu, stop, 0)) return false;
        }
    }
}

// 1 - exp(2l) = -(exp(2l) - 1) for -1/8 < l <= 0 by its Taylor series
// -2l (1 + l + 2/3 l^2 + 1/3 l^3 + ...), cut after l^3: the first term left
// out is 2/15 l^4, under 3.3e-5 relative for |l| < 1/8.
__device__ __forceinline__ float one_minus_exp2l_small(float l)
{
    float s = fmaf(l, 1.f / 3.f, 2.f / 3.f);
    s = fmaf(l, s, 1.f);
    s = fmaf(l, s, 1.f);
    return (-2.f * l) * s;
}

// GELU_tanh of two values: the polynomial argument in fp32 pairs, the tanh on
// the f16x2 unit (its error, under 2^-10 relative, is well below the bf16
// rounding of the product the result feeds)
__device__ __forceinline__ f2_t gelu2(f2_t g)
{
    const f2_t k0 = f2_splat(0.7978845608028654f), k1 = f2_splat(0.7978845608028654f * 0.044715f);
    const f2_t u = f2_mul(g, f2_fma(f2_mul(k1, g), g, k0));
    float t0, t1;
    tanh2_f16(f2_lo(u), f2_hi(u), t0, t1);
    const f2_t hg = f2_mul(f2_splat(0.5f), g);
    return f2_fma(hg, f2_make(t0, t1), hg);
}

// two fp32 rounded to nearest-even as a bf16 pair / an f16 pair (element 0 low)
__device__ __forceinline__ uint32_t pack_bf16_pair(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float gelu_tanh_fast(float g)
{
    const float k0 = 0.7978845608028654f, k1 = 0.7978845608028654f * 0.044715f;
    const float u = g * fmaf(k1 * g, g, k0);
    const float hg = 0.5f * g;
    return fmaf(hg, tanh_approx(u), hg);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
rglru_prefill_fused_kernel(const FusedParams p, const __grid_constant__ CUtensorMap tmap_x,
                           const __grid_constant__ CUtensorMap tmap_g)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t half = cluster_ctarank(), peer = half ^ 1u;
    const int nheads = p.D / 256;
    const int head = (int)(blockIdx.x >> 1) % nheads;
    const int group = 2 * head + (int)half;  // scan chain of this CTA: (head, half)
    const int ch0 = head * 256 + (int)half * kHalf;  // first channel of this CTA
    TileInfo *info = reinterpret_cast<TileInfo *>(smem + OFF_INFO);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    auto bar = [&](int kind, int i) { return bars + kind + i; };
    // the peer CTA's barrier at the same offset, for remote arrivals
    auto peer_bar = [&](int kind, int i) { return mapa_shared(smem_u32(bars + kind + i), peer); };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
    WsHeader *hdr = p.hdr;

    // ------------------------------------------------------------------ setup
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_holder, 512);
        if (lane == 0) {
            for (int i = 0; i < INFO_RING; ++i) {
                mbar_init(bar(B_INFO_FULL, i), 1);
                mbar_init(bar(B_INFO_EMPTY, i), 2);  // the tile's look-back warps of both CTAs (rank 0's ring only)
            }
            for (int i = 0; i < XRING; ++i) {
                mbar_init(bar(B_X_FULL, i), 1);
                mbar_init(bar(B_X_EMPTY, i), kGroupThreads);
            }
            for (int i = 0; i < NX; ++i) mbar_init(bar(B_XH_FREE, i), kGroupThreads);
            for (int i = 0; i < NB; ++i) {
                // this CTA's conv threads (one of them also expects the peer's half
                // of the tile: a bulk copy that completes the transaction count)
                mbar_init(bar(B_BCONV, i), kGroupThreads);
                mbar_init(bar(B_BFREE, i), 2);                  // MMA commits of both CTAs
                mbar_init(bar(B_BHALF, i), kGroupThreads);
            }
            for (int i = 0; i < NA; ++i) {
                mbar_init(bar(B_MMA, i), 1);
                mbar_init(bar(B_ACC_FREE, i), kGroupThreads);
            }
            for (int i = 0; i < NS; ++i) {
                mbar_init(bar(B_PASS1, i), kGroupThreads);
                mbar_init(bar(B_STASH_FREE, i), 32);
            }
            for (int i = 0; i < kScanGroups; ++i) {
                mbar_init(bar(B_GFULL, i), 1);
                mbar_init(bar(B_GFREE, i), kGroupThreads);
            }
            mbar_init(bar(B_W_FULL, 0), 2 * kGroupThreads);  // both scan groups' weight rows in TMEM
            *abort_flag = 0;
            mbar_fence_init();
        }
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers initialised before any remote arrival
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
#ifdef RGLRU_TRACE
    if (threadIdx.x == 0) {
        uint32_t smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        RGLRU_TR(0, kTraceTiles - 1, (unsigned long long)smid);
    }
#endif
    const int debug_unit = *(volatile int *)&hdr->debug_unit_plus1 - 1;

    if (warp == kSchedWarp) {
        // ------------------------------------------------------------ scheduler
        // Rank 0 claims the head's tiles, one ahead of the ring, and writes
        // each descriptor into both CTAs; each CTA then loads its own
        // channels of x: rows t0 - 3 .. t0 + 31 (rows before t = 0 arrive
        // zero-filled; the conv reads conv_state there).  Ticket k is tile
        // k / B of sequence k % B: consecutive tickets go to different
        // sequences, so a tile's predecessor in its sequence was claimed B
        // tickets earlier and has usually published its aggregate (and its
        // prefix) by the time the tile's own look-back starts.  The look-back
        // indexes tiles by u = b C + c, their order inside the sequence.
        // Claims come in batches of kClaimBatch consecutive tickets: one
        // atomicAdd per batch, issued a batch ahead, and the batch's
        // segment_pos loads issued together, so the round trips overlap the
        // x loads instead of pacing them.
        int k_pending = -1;  // lane 0: ticket of the next batch (atomic in flight)
        const int nbatch = min(kClaimBatch, p.B);
        auto fetch = [&]() {
            if (lane == 0 && !*abort_flag) k_pending = (int)atomicAdd(&hdr->ticket[head], (unsigned)nbatch);
            else if (lane == 0) k_pending = 0x3fffffff;  // past every ticket: no more tiles
        };
        TileInfo batch[kClaimBatch];
        int batch_i = kClaimBatch;
        auto claim_batch = [&]() {
            const int k0 = __shfl_sync(0xffffffffu, k_pending, 0);
            fetch();
            int sp[kClaimBatch];
#pragma unroll
            for (int q = 0; q < kClaimBatch; ++q) {
                const int k = k0 + q;
                TileInfo ti{};
                ti.u = -1;
                sp[q] = 3;
                if (q < nbatch && k >= 0 && k < p.tiles_per_head) {
                    ti.b = k % p.B;
                    const int c = k / p.B;
                    ti.u = ti.b * p.C + c;
                    ti.t0 = c * NT;
                    ti.valid = min(NT, p.T - ti.t0);
                    ti.first_last = (c == 0 ? 1 : 0) | (c == p.C - 1 ? 2 : 0);
                    if (lane < ti.valid) sp[q] = p.segpos[(size_t)ti.b * p.T + ti.t0 + lane];
                }
                batch[q] = ti;
            }
#pragma unroll
            for (int q = 0; q < kClaimBatch; ++q) {
                batch[q].reset_mask = __ballot_sync(0xffffffffu, sp[q] < 1);
                batch[q].m2 = __ballot_sync(0xffffffffu, sp[q] < 2);
                batch[q].m3 = __ballot_sync(0xffffffffu, sp[q] < 3);
            }
            batch_i = 0;
        };
        auto claim = [&]() -> TileInfo {
            if (batch_i >= nbatch) claim_batch();
            TileInfo ti{};
#pragma unroll
            for (int q = 0; q < kClaimBatch; ++q)
                if (q == batch_i) ti = batch[q];
            ++batch_i;
            return ti;
        };
        if (half == 0) fetch();
        TileInfo next{};
        if (half == 0) next = claim();
        int ends = 0, x_issued = 0;
#pragma unroll 1
        for (int j = 0;; ++j) {
            const int ir = j % INFO_RING;
            bool ok = true;
            TileInfo ti;
            if (half == 0) {
                if (j >= INFO_RING)
                    ok = warp_wait_bar(bar(B_INFO_EMPTY, ir), (uint32_t)((j / INFO_RING) - 1) & 1u, abort_flag, hdr, 1);
                if (!ok) next.u = -1;
                ti = next;
                if (lane == 0) {
                    const uint4 *w = reinterpret_cast<const uint4 *>(&ti);
                    reinterpret_cast<uint4 *>(info + ir)[0] = w[0];
                    reinterpret_cast<uint4 *>(info + ir)[1] = w[1];
                    const uint32_t remote = mapa_shared(smem_u32(info + ir), peer);
                    st_cluster_v4(remote, w[0]);
                    st_cluster_v4(remote + 16, w[1]);
                    mbar_arrive(bar(B_INFO_FULL, ir));
                    mbar_arrive_cluster(peer_bar(B_INFO_FULL, ir));
                    RGLRU_TR(TR_SCHED_INFO, j, globaltimer());
                    RGLRU_TR(TR_TILE_U, j, (unsigned long long)(unsigned)ti.u);
                }
                if (ti.u < 0) {
                    if (++ends == kEndMarkers || !ok) break;
                    continue;
                }
            } else {
                if (!warp_wait_bar(bar(B_INFO_FULL, ir), (uint32_t)(j / INFO_RING) & 1u, abort_flag, hdr, 2)) break;
                ti = info[ir];
                if (ti.u < 0) break;
            }
            const int xr = j % XRING;
            if (j >= XRING && !warp_wait_bar(bar(B_X_EMPTY, xr), (uint32_t)((j / XRING) - 1) & 1u, abort_flag, hdr, 3)) {
                if (half == 0) {
                    next.u = -1;
                    continue;  // still write the end markers
                }
                break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(B_X_FULL, xr), kXTile);
                tma_load_3d(smem + OFF_X + xr * kXTile, &tmap_x, bar(B_X_FULL, xr), ch0, ti.t0 - 3, ti.b);
                // the GELU branch of this tile, read by pass 1 some microseconds later
                tma_prefetch_l2_3d(&tmap_g, ch0, ti.t0, ti.b);
            }
            ++x_issued;
            if (half == 0) next = claim();
        }
        // on abort, wait (bounded) for the x loads still in flight
        if (lane == 0 && *abort_flag) {
            for (int k = max(0, x_issued - XRING); k < x_issued; ++k) {
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(bar(B_X_FULL, k % XRING), (uint32_t)(k / XRING) & 1u) &&
                       globaltimer() - t0 < kTimeoutNs) {
                }
            }
        }
    } else if (warp >= kConvWarp0 && warp < kConvWarp0 + kConvWarps) {
        // ------------------------------------------------------------ conv warps
        // thread = channel c of this half (its TMEM lane); 32 tokens in order.
        // The conv produces xh = xc / 2 (halving is exact): the MMA then yields
        // half pre-activations, which is what sigmoid(z) = (1 + tanh(z/2)) / 2
        // needs, and the scan's i*xc becomes one FMA on xh.
        const int c = (warp - kConvWarp0) * 32 + lane;
        const int d = ch0 + c;
        const float w0 = 0.5f * p.conv_w[d], w1 = 0.5f * p.conv_w[(size_t)p.D + d];
        const float w2 = 0.5f * p.conv_w[2 * (size_t)p.D + d], w3 = 0.5f * p.conv_w[3 * (size_t)p.D + d];
        const float cb = 0.5f * p.conv_b[d];
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        // B tile, N-major without swizzle: the thread's channel k of the head
        // holds 8 tokens per 16-byte row of a core matrix at
        // (k / 8) * kBGroup + (k % 8) * 16 + (t / 8) * 128
        const int kidx = (int)half * kHalf + c;
        const uint32_t b_local = smem_u32(smem + OFF_B) + (uint32_t)(kidx >> 3) * kBGroup + (uint32_t)(kidx & 7) * 16;
        // this half's 128 channels of a B tile: 8 KB, contiguous, sent to the peer in one copy
        const int half_off = (int)half * kBHalf;
        const bool sender = warp == kConvWarp0 && lane == 0;
#pragma unroll 1
        for (int j = 0;; ++j) {
            const int ir = j % INFO_RING, xr = j % XRING, sx = j % NX, sb = j % NB;
            if (!warp_wait_bar(bar(B_INFO_FULL, ir), (uint32_t)(j / INFO_RING) & 1u, abort_flag, hdr, 4)) break;
            const TileInfo ti = info[ir];
            if (ti.u < 0) break;
            if (lane == 0 && warp == kConvWarp0) RGLRU_TR(TR_CONV_START, j, globaltimer());
            if (!warp_wait_bar(bar(B_X_FULL, xr), (uint32_t)(j / XRING) & 1u, abort_flag, hdr, 5)) break;
            if (j >= NX && !warp_wait_bar(bar(B_XH_FREE, sx), (uint32_t)((j / NX) - 1) & 1u, abort_flag, hdr, 6)) break;
            if (j >= NB && !warp_wait_bar(bar(B_BFREE, sb), (uint32_t)((j / NB) - 1) & 1u, abort_flag, hdr, 7)) break;
            if (lane == 0 && warp == kConvWarp0) RGLRU_TR(TR_CONV_GO, j, globaltimer());
            const __nv_bfloat16 *xs = reinterpret_cast<const __nv_bfloat16 *>(smem + OFF_X + xr * kXTile) + c;
            float xm3, xm2, xm1;  // tokens t - 3, t - 2, t - 1
            if (ti.t0 == 0) {     // sequence start: the carried conv state
                const __nv_bfloat16 *cs = p.conv_state + (size_t)ti.b * 3 * p.D + d;
                xm3 = __bfloat162float(cs[0]);
                xm2 = __bfloat162float(cs[p.D]);
                xm1 = __bfloat162float(cs[2 * (size_t)p.D]);
            } else {
                xm3 = __bfloat162float(xs[0]);
                xm2 = __bfloat162float(xs[kHalf]);
                xm1 = __bfloat162float(xs[2 * kHalf]);
            }
            const uint32_t bl = b_local + sb * kBTile;
            const uint32_t xh_col = tmem + lane_off + kColXh + sx * kColsXh;
            // a tile with no document start and all 32 tokens valid needs no masks
            const bool clean = (ti.reset_mask | ti.m2 | ti.m3) == 0u && ti.valid == NT;
            auto run = [&](auto clean_tag) {
                constexpr bool kClean = decltype(clean_tag)::value;
                // one token: the four taps (lag k dropped when segment_pos < k)
                auto conv1 = [&](int t, float m3, float m2, float m1, float x0) -> float {
                    if constexpr (kClean) {
                        return fmaf(w3, x0, fmaf(w2, m1, fmaf(w1, m2, fmaf(w0, m3, cb))));
                    } else {
                        float v = cb;
                        if (!((ti.m3 >> t) & 1u)) v = fmaf(w0, m3, v);
                        if (!((ti.m2 >> t) & 1u)) v = fmaf(w1, m2, v);
                        if (!((ti.reset_mask >> t) & 1u)) v = fmaf(w2, m1, v);
                        v = fmaf(w3, x0, v);
                        return t < ti.valid ? v : 0.f;
                    }
                };
#pragma unroll 1
                for (int t8 = 0; t8 < NT; t8 += 8) {
                    uint32_t xq[8], bq[4];
#pragma unroll
                    for (int k = 0; k < 8; k += 2) {
                        const int t = t8 + k;
                        const float x0 = __bfloat162float(xs[(t + 3) * kHalf]);
                        const float x1 = __bfloat162float(xs[(t + 4) * kHalf]);
                        const float v0 = conv1(t, xm3, xm2, xm1, x0);
                        const float v1 = conv1(t + 1, xm2, xm1, x0, x1);
                        bq[k >> 1] = pack_bf16_pair(v0, v1);
                        xq[k] = __float_as_uint(v0);
                        xq[k + 1] = __float_as_uint(v1);
                        xm3 = xm1;
                        xm2 = x0;
                        xm1 = x1;
                    }
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(bl + (uint32_t)(t8 >> 3) * 128), "r"(bq[0]),
                                 "r"(bq[1]), "r"(bq[2]), "r"(bq[3])
                                 : "memory");
                    tmem_st8(xh_col + (uint32_t)t8, xq);
                }
            };
            if (clean)
                run(std::true_type{});
            else
                run(std::false_type{});
            if (lane == 0 && warp == kConvWarp0) RGLRU_TR(TR_CONV_LOOP, j, globaltimer());
            tmem_wait_st();
            tc_fence_before();
            // this half of the B tile before the async proxy's reads (the MMA,
            // the copy to the peer)
            fence_proxy_async_smem();
            mbar_arrive(bar(B_X_EMPTY, xr));
            if (sender)
                mbar_arrive_expect_tx(bar(B_BCONV, sb), kBHalf);  // the peer's half, arriving by copy
            else
                mbar_arrive(bar(B_BCONV, sb));
            mbar_arrive(bar(B_BHALF, sb));
            if (warp == kConvWarp0) {
                // all of this half written: one bulk copy into the peer's tile
                if (!warp_wait_bar(bar(B_BHALF, sb), (uint32_t)(j / NB) & 1u, abort_flag, hdr, 20)) break;
                if (sender) {
                    uint8_t *src = smem + OFF_B + sb * kBTile + half_off;
                    bulk_copy_to_cluster(mapa_shared(smem_u32(src), peer), src, kBHalf, peer_bar(B_BCONV, sb));
                }
            }
            if (lane == 0 && warp == kConvWarp0) RGLRU_TR(TR_CONV_DONE, j, globaltimer());
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t idesc = umma_idesc_bf16_bn(kHalf, NT);
        bool w_ready = false;
        int issued = 0;
#pragma unroll 1
        for (int j = 0;; ++j) {
            const int ir = j % INFO_RING, sb = j % NB, sa = j % NA;
            if (!warp_wait_bar(bar(B_INFO_FULL, ir), (uint32_t)(j / INFO_RING) & 1u, abort_flag, hdr, 8)) break;
            if (info[ir].u < 0) break;
            if (j >= NA && !warp_wait_bar(bar(B_ACC_FREE, sa), (uint32_t)((j / NA) - 1) & 1u, abort_flag, hdr, 9)) break;
            if (lane == 0) RGLRU_TR(TR_MMA_TFREE, j, globaltimer());
            if (!warp_wait_bar(bar(B_BCONV, sb), (uint32_t)(j / NB) & 1u, abort_flag, hdr, 10)) break;
            if (lane == 0) RGLRU_TR(TR_MMA_CONV, j, globaltimer());
            if (!w_ready) {
                if (!warp_wait_bar(bar(B_W_FULL, 0), 0u, abort_flag, hdr, 11)) break;
                w_ready = true;
            }
            // the whole (converged) warp runs the issue loop; elect.sync picks
            // the lane that issues each MMA and commit
            tc_fence_after();
            {
                const uint32_t bt = smem_u32(smem + OFF_B + sb * kBTile);
                const uint32_t d_r = tmem + kColAcc + sa * kColsAcc, d_i = d_r + NT;
                const uint64_t bd0 = umma_desc_mn_noswizzle(bt, kBGroup, 128);
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) {
                    // A (16 input channels of this half's weight rows) from TMEM;
                    // 16 input channels = two 8-channel groups of the N-major B
                    // tile (the descriptor's start address counts 16-byte units)
                    const uint64_t bd = bd0 + (uint64_t)((kk * 2 * kBGroup) >> 4);
                    umma_ts_warp(d_r, tmem + kColW + kk * 8, bd, idesc, kk > 0);
                    umma_ts_warp(d_i, tmem + kColW + kColsWGate + kk * 8, bd, idesc, kk > 0);
                }
                umma_commit_warp(bar(B_MMA, sa));
                umma_commit_cluster_warp(bar(B_BFREE, sb), 0x3);  // this B slot is free in both CTAs' view
            }
            if (lane == 0) RGLRU_TR(TR_MMA_ISSUED, j, globaltimer());
            __syncwarp();
            ++issued;
        }
        // Before the final cluster barrier: the commits of both CTAs for the
        // last tiles have landed on this CTA's B-slot barriers (so no arrival
        // reaches a CTA that has exited).
        if (lane == 0) {
            for (int k = max(0, issued - NB); k < issued; ++k) {
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait_cl(bar(B_BFREE, k % NB), (uint32_t)(k / NB) & 1u) && globaltimer() - t0 < kTimeoutNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp < kScanWarps) {
        // ------------------------------------------------------------ scan warps
        const int sg = warp / 4;  // scan group: tiles j with j % kScanGroups == sg
        const int c = threadIdx.x % kGroupThreads;
        const int d = ch0 + c;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        {
            // this channel's row of W_a (group 0) or W_x (group 1) into its TMEM
            // lane: 256 bf16 = 128 columns, read once from global memory
            const uint4 *src = reinterpret_cast<const uint4 *>((sg == 0 ? p.w_a : p.w_x) + (size_t)d * 256);
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                uint32_t r[32];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint4 v = __ldg(src + q * 8 + k);
                    r[4 * k] = v.x;
                    r[4 * k + 1] = v.y;
                    r[4 * k + 2] = v.z;
                    r[4 * k + 3] = v.w;
                }
                tmem_st32(tmem + lane_off + kColW + sg * kColsWGate + q * 32, r);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(B_W_FULL, 0));
        }
        const float hba = 0.5f * p.b_a[d], hbx = 0.5f * p.b_x[d];
        const float lam = p.lambda[d];
        const float ls = lam >= 0.f ? -log1pf(expf(-lam)) : lam - log1pf(expf(lam));  // log sigmoid(Lambda)
        const float kl = kC * ls;                       // log a per unit r (<= 0)
        // r = (1 + tr) / 2 with tr = tanh(half pre-activation): log a = tr * hkl + hkl
        const float hkl = 0.5f * kl;
        const float hkl2 = hkl * 1.4426950408889634f;  // same in log2
        const f2_t hba2 = f2_splat(hba), hbx2 = f2_splat(hbx), hkl_2 = f2_splat(hkl), hkl2_2 = f2_splat(hkl2);
        const f2_t one_2 = f2_splat(1.f);
        // GELU branch of the group's next tile into its shared-memory buffer
        // [token][channel] by one tensor load (the tile was prefetched into L2
        // with its x; rows past the sequence end arrive zero-filled), issued
        // once pass 1 of the group's previous tile has read the buffer.
        __nv_bfloat16 *gbuf = reinterpret_cast<__nv_bfloat16 *>(smem + OFF_G + sg * kGTile);
        int g_loads = 0;  // tensor loads issued into gbuf (the k-th completes phase k of B_GFULL)
        auto load_g = [&](const TileInfo &ti) {
            if (c == 0) {
                if (g_loads == 0 || wait_bar(bar(B_GFREE, sg), (uint32_t)(g_loads - 1) & 1u, abort_flag, hdr, 24)) {
                    mbar_arrive_expect_tx(bar(B_GFULL, sg), kGTile);
                    tma_load_3d(gbuf, &tmap_g, bar(B_GFULL, sg), ch0, ti.t0, ti.b);
                    ++g_loads;
                }
            }
            __syncwarp();
        };
        auto pack_h2 = [](float lo, float hi) -> uint32_t {
            __half2 v = __floats2half2_rn(lo, hi);
            return *reinterpret_cast<uint32_t *>(&v);
        };

        auto pass1 = [&](int j, const TileInfo &ti) -> bool {
            const int sa = j % NA, ss = j % NS, sx = j % NX;
            if (!warp_wait_bar(bar(B_MMA, sa), (uint32_t)(j / NA) & 1u, abort_flag, hdr, 12)) return false;
            // the look-back warp of the slot's previous tile is done with it
            if (j >= NS && !warp_wait_bar(bar(B_STASH_FREE, ss), (uint32_t)((j / NS) - 1) & 1u, abort_flag, hdr, 14))
                return false;
            if (c == 0) RGLRU_TR(TR_P1_START, j, globaltimer());
            tc_fence_after();
            const uint32_t acc = tmem + lane_off + kColAcc + sa * kColsAcc;
            const uint32_t xhc = tmem + lane_off + kColXh + sx * kColsXh;
            const uint32_t stc = smem_u32(smem + OFF_ST + ss * kStash) + (uint32_t)c * 4;
            float hl = 0.f, P = 1.f;  // local scan state from h = 0, running prod a
            // this tile's GELU branch (the group's (j / kScanGroups)-th load)
            if (!warp_wait_bar(bar(B_GFULL, sg), (uint32_t)(j / kScanGroups) & 1u, abort_flag, hdr, 23)) return false;
            if (c == 0) RGLRU_TR(TR_P1_G, j, globaltimer());
            const uint16_t *gs = reinterpret_cast<const uint16_t *>(gbuf) + c;
#pragma unroll 1
            for (int t8 = 0; t8 < NT; t8 += 8) {
                uint32_t ar[8], ai[8], xq[8];
                tmem_ld8(acc + t8, ar);
                tmem_ld8(acc + NT + t8, ai);
                tmem_ld8(xhc + t8, xq);
                tmem_wait_ld();
                if (c == 0 && t8 == 0) RGLRU_TR(TR_P1_LD, j, globaltimer());
                uint16_t gcur[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) gcur[k] = gs[(t8 + k) * kHalf];
                uint32_t st[8];
                const bool clean = ((ti.reset_mask >> t8) & 0xffu) == 0u && t8 + 8 <= ti.valid;
                if (clean) {
#pragma unroll
                    for (int k = 0; k < 8; k += 2) {
                        const f2_t zr = f2_add(f2_make(__uint_as_float(ar[k]), __uint_as_float(ar[k + 1])), hba2);
                        const f2_t zi = f2_add(f2_make(__uint_as_float(ai[k]), __uint_as_float(ai[k + 1])), hbx2);
                        const f2_t tr = f2_make(tanh_approx(f2_lo(zr)), tanh_approx(f2_hi(zr)));
                        const f2_t tg = f2_make(tanh_approx(f2_lo(zi)), tanh_approx(f2_hi(zi)));
                        const f2_t la = f2_fma(tr, hkl2_2, hkl2_2);  // log2 a
                        const float a0 = ex2_approx(f2_lo(la)), a1 = ex2_approx(f2_hi(la));
                        // 1 - a^2 directly: with a good to ~2^-22 relative, its
                        // absolute error is under 5e-7, so sqrt(1 - a^2) errs by at
                        // most ~6e-5 absolute even as a -> 1 (small r), where the
                        // term it scales is itself that small
                        const f2_t a2 = f2_make(a0, a1);
                        const f2_t om = f2_fma(f2_mul(a2, f2_splat(-1.f)), a2, one_2);
                        const f2_t nrm = f2_make(sqrt_approx(f2_lo(om)), sqrt_approx(f2_hi(om)));
                        const f2_t xh2 = f2_make(__uint_as_float(xq[k]), __uint_as_float(xq[k + 1]));
                        const f2_t v = f2_mul(nrm, f2_fma(tg, xh2, xh2));  // sqrt(1-a^2) * i * xc
                        const float h0 = fmaf(a0, hl, f2_lo(v));
                        const float P0 = P * a0;
                        hl = fmaf(a1, h0, f2_hi(v));
                        P = P0 * a1;
                        const f2_t G = gelu2(f2_make(__uint_as_float((uint32_t)gcur[k] << 16),
                                                     __uint_as_float((uint32_t)gcur[k + 1] << 16)));
                        const f2_t yl = f2_mul(G, f2_make(h0, hl));
                        const f2_t qq = f2_mul(G, f2_make(P0, P));
                        st[k] = pack_h2(f2_lo(yl), f2_lo(qq));
                        st[k + 1] = pack_h2(f2_hi(yl), f2_hi(qq));
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int t = t8 + k;
                        const float xh = __uint_as_float(xq[k]);
                        const float tr = tanh_approx(__uint_as_float(ar[k]) + hba);
                        const float tg = tanh_approx(__uint_as_float(ai[k]) + hbx);
                        const float ell = fmaf(tr, hkl, hkl);
                        float a = ex2_approx(fmaf(tr, hkl2, hkl2));
                        const float om = ell > -0.125f ? one_minus_exp2l_small(ell) : fmaf(-a, a, 1.f);
                        const float uu = fmaf(tg, xh, xh);  // i * xc
                        float v = sqrt_approx(om) * uu;
                        if ((ti.reset_mask >> t) & 1u) {
                            a = 0.f;
                            v = uu;
                        }
                        if (t >= ti.valid) {
                            a = 1.f;
                            v = 0.f;
                        }
                        hl = fmaf(a, hl, v);
                        P *= a;
                        const float G = gelu_tanh_fast(__uint_as_float((uint32_t)gcur[k] << 16));
                        st[k] = pack_h2(G * hl, G * P);
                    }
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) st_shared_u32(stc + (uint32_t)(t8 + k) * (kHalf * 4), st[k]);
            }
            tc_fence_before();  // the accumulator and xc loads above, before the slots are handed back
            mbar_arrive(bar(B_GFREE, sg));
            mbar_arrive(bar(B_ACC_FREE, sa));
            mbar_arrive(bar(B_XH_FREE, sx));
            reinterpret_cast<float2 *>(smem + OFF_AGG + ss * kHalf * 8)[c] = make_float2(P, hl);
            mbar_arrive(bar(B_PASS1, ss));
            if (c == 0) RGLRU_TR(TR_P1_END, j, globaltimer());
            return true;
        };

        // this group's tiles: j = sg, sg + kScanGroups, ...
        int j = sg;
        bool ok = warp_wait_bar(bar(B_INFO_FULL, j % INFO_RING), (uint32_t)(j / INFO_RING) & 1u, abort_flag, hdr, 17);
        TileInfo cur{};
        if (ok) {
            cur = info[j % INFO_RING];
            if (cur.u >= 0) load_g(cur);
        }
#pragma unroll 1
        for (; ok && cur.u >= 0; j += kScanGroups) {
            ok = pass1(j, cur);
            if (!ok) break;
            const int jn = j + kScanGroups;
            ok = warp_wait_bar(bar(B_INFO_FULL, jn % INFO_RING), (uint32_t)(jn / INFO_RING) & 1u, abort_flag, hdr, 17);
            if (!ok) break;
            cur = info[jn % INFO_RING];
            if (cur.u >= 0) load_g(cur);  // lands while the group waits for the tile's MMA
        }
        if (c == 0 && g_loads > 0) {
            // a GELU-branch load still in flight (after an abort) lands before the CTA exits
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(bar(B_GFULL, sg), (uint32_t)(g_loads - 1) & 1u) && globaltimer() - t0 < kTimeoutNs) {
            }
        }
    } else if (warp >= kLbWarp0) {
        // ------------------------------------------------------------ look-back warps
        // Warp w serves the tiles j = w, w + kLbWarps, ...; their stash slots
        // recur every NS tiles, so each barrier is waited on one phase at a
        // time.  Per tile: publish the aggregate (later tiles of the sequence
        // may combine it before this tile's own look-back has finished), find
        // the anchor, fold, publish the inclusive prefix, then pass 2 of the
        // tile: y = y_loc + q h_in from the stash, 4 channels per lane, and at
        // a sequence end the new states.  These warps are the only ones that
        // fence for the aggregates and prefixes.
        const int ch = lane * 4;  // 4 channels per lane
        const size_t dch = (size_t)ch0 + ch;
        const size_t gbase = (size_t)group * p.tiles_per_head;
        constexpr int kFoldBatch = 4;  // aggregates loaded per round trip
#pragma unroll 1
        for (int j = warp - kLbWarp0;; j += kLbWarps) {
            const int ss = j % NS, ir = j % INFO_RING;
            if (!warp_wait_bar(bar(B_INFO_FULL, ir), (uint32_t)(j / INFO_RING) & 1u, abort_flag, hdr, 18)) break;
            const TileInfo ti = info[ir];
            if (ti.u < 0) break;
            if (!warp_wait_bar(bar(B_PASS1, ss), (uint32_t)(j / NS) & 1u, abort_flag, hdr, 19)) break;
            if (lane == 0) RGLRU_TR(TR_LB_START, j, globaltimer());
            const float4 *sagg = reinterpret_cast<const float4 *>(smem + OFF_AGG + ss * kHalf * 8);
            const float4 g01 = sagg[lane * 2], g23 = sagg[lane * 2 + 1];  // (A,H) of 4 channels
            const float A[4] = {g01.x, g01.z, g23.x, g23.z};
            const float Hh[4] = {g01.y, g01.w, g23.y, g23.w};
            const size_t gu = gbase + ti.u;
            const uint32_t rbit = ti.reset_mask ? F_RESET : 0u;
            const bool suppress = (int)gu == debug_unit;
            if (!suppress) {
                float4 *dst = reinterpret_cast<float4 *>(p.agg + gu * kHalf + ch);
                dst[0] = g01;
                dst[1] = g23;
                __threadfence();
                __syncwarp();
                if (lane == 0) atom_or_release_u32(p.flags + gu, F_AGG | rbit);
            }
            float hin[4];
            bool ok = true;
            if (ti.first_last & 1) {
                const float4 hs = *reinterpret_cast<const float4 *>(p.h_state + (size_t)ti.b * p.D + dch);
                hin[0] = hs.x; hin[1] = hs.y; hin[2] = hs.z; hin[3] = hs.w;
            } else {
                int anchor = -1;
                uint32_t aflag = 0;
                ok = find_anchor(p.flags + gbase, ti.u - 1, ti.b * p.C, anchor, aflag, abort_flag, hdr);
                if (lane == 0) {
                    RGLRU_TR(TR_LB_ANC, j, globaltimer());
                    RGLRU_TR(TR_LB_K, j, (unsigned long long)(ti.u - anchor) | ((unsigned long long)aflag << 32));
                }
                if (ok) {
                    // carried-in state = the chain h <- A h + H folded forward in
                    // sequence order from the anchor, the same order whichever
                    // prefixes happened to be published (bit-reproducible)
                    if (aflag & F_PREFIX) {
                        const float4 pr = ld_relaxed_f4(reinterpret_cast<const float4 *>(p.prefix + (gbase + anchor) * kHalf + ch));
                        hin[0] = pr.x; hin[1] = pr.y; hin[2] = pr.z; hin[3] = pr.w;
                    } else {  // a tile holding a reset: A = 0, its prefix is its H
                        const float4 *src = reinterpret_cast<const float4 *>(p.agg + (gbase + anchor) * kHalf + ch);
                        const float4 a01 = ld_relaxed_f4(src), a23 = ld_relaxed_f4(src + 1);
                        hin[0] = a01.y; hin[1] = a01.w; hin[2] = a23.y; hin[3] = a23.w;
                    }
#pragma unroll 1
                    for (int p0 = anchor + 1; p0 < ti.u; p0 += kFoldBatch) {
                        float4 dd[kFoldBatch][2];
#pragma unroll
                        for (int k = 0; k < kFoldBatch; ++k) {
                            if (p0 + k < ti.u) {
                                const float4 *src = reinterpret_cast<const float4 *>(p.agg + (gbase + p0 + k) * kHalf + ch);
                                dd[k][0] = ld_relaxed_f4(src);
                                dd[k][1] = ld_relaxed_f4(src + 1);
                            }
                        }
#pragma unroll
                        for (int k = 0; k < kFoldBatch; ++k) {
                            if (p0 + k < ti.u) {
                                hin[0] = fmaf(dd[k][0].x, hin[0], dd[k][0].y);
                                hin[1] = fmaf(dd[k][0].z, hin[1], dd[k][0].w);
                                hin[2] = fmaf(dd[k][1].x, hin[2], dd[k][1].y);
                                hin[3] = fmaf(dd[k][1].z, hin[3], dd[k][1].w);
                            }
                        }
                    }
                }
            }
            if (!ok) break;
            if (lane == 0) RGLRU_TR(TR_LB_HIN, j, globaltimer());
            float pre[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) pre[e] = fmaf(A[e], hin[e], Hh[e]);
            if (!suppress) {
                *reinterpret_cast<float4 *>(p.prefix + gu * kHalf + ch) = make_float4(pre[0], pre[1], pre[2], pre[3]);
                __threadfence();
                __syncwarp();
                if (lane == 0) atom_or_release_u32(p.flags + gu, F_AGG | F_PREFIX | rbit);
            }
            if (lane == 0) RGLRU_TR(TR_P2_START, j, globaltimer());
            // pass 2: token t of this lane's 4 channels is one 16-byte stash word;
            // y goes out as 8 bytes per lane (256 contiguous bytes per warp)
            {
                const uint32_t stw = smem_u32(smem + OFF_ST + ss * kStash) + (uint32_t)ch * 4;
                __nv_bfloat16 *yrow = p.y + ((size_t)ti.b * p.T + ti.t0) * p.D + dch;
#pragma unroll 4
                for (int t = 0; t < ti.valid; ++t) {
                    uint32_t w0, w1, w2, w3;
                    ld_shared_v4(stw + (uint32_t)t * (kHalf * 4), w0, w1, w2, w3);
                    const float2 q0 = __half22float2(*reinterpret_cast<const __half2 *>(&w0));
                    const float2 q1 = __half22float2(*reinterpret_cast<const __half2 *>(&w1));
                    const float2 q2 = __half22float2(*reinterpret_cast<const __half2 *>(&w2));
                    const float2 q3 = __half22float2(*reinterpret_cast<const __half2 *>(&w3));
                    uint2 yv;
                    yv.x = pack_bf16_pair(fmaf(q0.y, hin[0], q0.x), fmaf(q1.y, hin[1], q1.x));
                    yv.y = pack_bf16_pair(fmaf(q2.y, hin[2], q2.x), fmaf(q3.y, hin[3], q3.x));
                    *reinterpret_cast<uint2 *>(yrow + (size_t)t * p.D) = yv;
                }
            }
            if (ti.first_last & 2) {
                // The old states are read by the first tile of this sequence (its
                // conv and its look-back, in this CTA's half of the channels):
                // wait until that tile's prefix is published before overwriting.
                const uint32_t *f_first = p.flags + gbase + (size_t)ti.b * p.C;
                if (warp_wait_flag(f_first, F_PREFIX, abort_flag, hdr, 16) == 0) break;
                *reinterpret_cast<float4 *>(p.h_state + (size_t)ti.b * p.D + dch) = make_float4(pre[0], pre[1], pre[2], pre[3]);
                uint2 ncs[3];
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    const int ts = p.T - 3 + k;
                    ncs[k] = ts >= 0 ? *reinterpret_cast<const uint2 *>(p.x + ((size_t)ti.b * p.T + ts) * p.D + dch)
                                     : *reinterpret_cast<const uint2 *>(p.conv_state + ((size_t)ti.b * 3 + 3 + ts) * p.D + dch);
                }
#pragma unroll
                for (int k = 0; k < 3; ++k) *reinterpret_cast<uint2 *>(p.conv_state + ((size_t)ti.b * 3 + k) * p.D + dch) = ncs[k];
            }
            // the stash slot (and its aggregate) may be reused, and the descriptor
            // once both CTAs' look-back warps are done with it
            mbar_arrive(bar(B_STASH_FREE, ss));
            __syncwarp();
            if (lane == 0) {
                // relaxed: the reuse needs no ordering of this warp's y stores
                if (half == 0)
                    mbar_arrive(bar(B_INFO_EMPTY, ir));
                else
                    mbar_arrive_cluster_relaxed(peer_bar(B_INFO_EMPTY, ir));
                RGLRU_TR(TR_P2_END, j, globaltimer());
            }
            if (lane == 0) RGLRU_TR(TR_LB_DONE, j, globaltimer());
        }
    }

    // ------------------------------------------------------------------ teardown
    // No thread of either CTA writes into or arrives on the other after this.
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- host side

struct Layout {
    int C, G, tpg;
    size_t flags_off, flags_bytes, agg_off, prefix_off, trace_off, total;
};

Layout layout_of(int B, int T, int D)
{
    Layout L;
    L.C = (T + NT - 1) / NT;
    L.G = 2 * (D / kHead);
    L.tpg = B * L.C;
    const size_t tiles = (size_t)L.G * L.tpg;
    L.flags_off = kWsHeaderBytes;
    L.flags_bytes = align_up(tiles * 4, 256);
    L.agg_off = L.flags_off + L.flags_bytes;
    L.prefix_off = L.agg_off + align_up(tiles * kHalf * 8, 256);
    L.total = L.prefix_off + align_up(tiles * kHalf * 4, 256);
#ifdef RGLRU_TRACE
    L.trace_off = L.total;
    L.total += align_up((size_t)kTraceCtas * kTraceTiles * kTraceEvents * 8, 256);
#else
    L.trace_off = 0;
#endif
    return L;
}

}  // namespace

size_t fused_workspace_bytes(int B, int T, int D) { return layout_of(B, T, D).total; }

rglru_status fused_prefill(const PrefillArgs &a)
{
    const Layout L = layout_of(a.B, a.T, a.D);
    const int H = a.D / kHead;
    if ((size_t)L.tpg > 0x7fffffffu / 2 || H > (int)(sizeof(WsHeader::ticket) / sizeof(unsigned int)))
        return RGLRU_ERR_UNSUPPORTED;
    auto encode = encode_fn();
    if (!encode) return RGLRU_ERR_CUDA;

    const cuuint32_t estride[3] = {1, 1, 1};
    // x [B, T, D]: this half's 128 channels x (32 + 3) tokens of one sequence
    CUtensorMap tmap_x;
    const cuuint64_t xdim[3] = {(cuuint64_t)a.D, (cuuint64_t)a.T, (cuuint64_t)a.B};
    const cuuint64_t xstride[2] = {(cuuint64_t)a.D * 2, (cuuint64_t)a.T * a.D * 2};
    const cuuint32_t xbox[3] = {(cuuint32_t)kHalf, (cuuint32_t)kXRows, 1};
    if (encode(&tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(a.x), xdim, xstride, xbox, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return RGLRU_ERR_CUDA;
    // GELU branch [B, T, D]: this half's 128 channels x 32 tokens (L2 prefetch boxes)
    CUtensorMap tmap_g;
    const cuuint32_t gbox[3] = {(cuuint32_t)kHalf, (cuuint32_t)NT, 1};
    if (encode(&tmap_g, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(a.g), xdim, xstride, gbox, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return RGLRU_ERR_CUDA;

    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RGLRU_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return RGLRU_ERR_CUDA;
    static PerDeviceFlag smem_set;
    const rglru_status st = set_smem_limit_once((const void *)rglru_prefill_fused_kernel, kSmemBytes, smem_set);
    if (st != RGLRU_OK) return st;

    char *ws = static_cast<char *>(a.ws);
    // tickets and flags start at zero; the status word and the test hook are kept
    if (cudaMemsetAsync(ws + offsetof(WsHeader, ticket), 0,
                        L.flags_off - offsetof(WsHeader, ticket) + L.flags_bytes, a.stream) != cudaSuccess)
        return RGLRU_ERR_CUDA;

    FusedParams p;
    p.B = a.B; p.T = a.T; p.D = a.D; p.C = L.C; p.tiles_per_head = L.tpg;
    p.x = static_cast<const __nv_bfloat16 *>(a.x);
    p.g = static_cast<const __nv_bfloat16 *>(a.g);
    p.conv_w = a.conv_w; p.conv_b = a.conv_b;
    p.b_a = a.b_a; p.b_x = a.b_x;
    p.lambda = a.lambda; p.segpos = a.segpos;
    p.w_a = static_cast<const __nv_bfloat16 *>(a.W_a);
    p.w_x = static_cast<const __nv_bfloat16 *>(a.W_x);
    p.conv_state = static_cast<__nv_bfloat16 *>(a.conv_state);
    p.h_state = a.h_state;
    p.y = static_cast<__nv_bfloat16 *>(a.y);
    p.hdr = reinterpret_cast<WsHeader *>(ws);
    p.flags = reinterpret_cast<uint32_t *>(ws + L.flags_off);
    p.agg = reinterpret_cast<float2 *>(ws + L.agg_off);
    p.prefix = reinterpret_cast<float *>(ws + L.prefix_off);
    p.trace = L.trace_off ? reinterpret_cast<unsigned long long *>(ws + L.trace_off) : nullptr;

    // one cluster of two CTAs (the two halves of a head) per SM pair; the same
    // number of clusters per head, which claim that head's tiles in order
    const int per_head = max(1, (sms / 2) / H);
    const long long grid = 2LL * per_head * H;
    if (grid > 0x7fffffffLL) return RGLRU_ERR_UNSUPPORTED;
    rglru_prefill_fused_kernel<<<(unsigned)grid, kThreads, kSmemBytes, a.stream>>>(p, tmap_x, tmap_g);
    return cuda_status(cudaGetLastError());
}

}  // namespace rglru
