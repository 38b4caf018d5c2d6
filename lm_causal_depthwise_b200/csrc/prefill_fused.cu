// prefill_fused.cu -- fused sm_100a prefill of the RG-LRU block core (bf16 I/O, fp32 state).
//
// One persistent kernel does, per tile of 32 tokens of one (sequence, head, half
// of the head's 256 channels):
//   conv warps   causal depthwise conv (k=4, document mask) of all 256 input
//                channels of the head, in fp32; bf16 copy into the MMA B tile
//                (128-byte swizzled, K-major), fp32 copy of this half's channels
//                for the scan.
//   MMA thread   both block-diagonal gate projections on the tensor cores:
//                D[128 out x 32 tok] = W[128 x 256] (A, resident in TMEM) * xc^T
//                (B, shared memory), fp32 accumulators in TMEM.
//   scan warps   one thread per output channel (= TMEM lane).  Pass 1: sigmoid
//                gates, a = sigmoid(Lambda)^(8 r), sqrt(1-a^2) normaliser,
//                resets; local scan from h = 0 gives the tile aggregate
//                (prod a, h_end), published at once; (a, v) are written back
//                over the accumulators.  Pass 2 (two tiles later): re-run the
//                scan from the carried-in state, multiply by GELU_tanh(g),
//                store y.
//   look-back    one warp per slot, so that the look-backs of consecutive
//   warps        tiles overlap.  Publishes the tile aggregate as soon as pass 1
//                ends, walks back over predecessor tiles of the same sequence
//                to the nearest anchor (a published inclusive prefix, or a tile
//                that holds a reset: A = 0), folds h <- A h + H forward from it
//                in sequence order (decoupled look-back with a fixed
//                combination order, so results are bit-reproducible), hands
//                the carried-in state to pass 2, then publishes the tile's
//                inclusive prefix.
//   producer     claims tiles in order from a per-(head, half) ticket counter,
//                TMA-loads the GELU-branch tile, issues the MMAs.
// Every wait is bounded: a wait that runs out records RGLRU_ERR_TIMEOUT in the
// workspace header and the CTA unwinds (waiting, bounded, for its own copies
// and MMAs in flight) and frees its TMEM.
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

constexpr int NT = 32;       // tokens per tile (MMA N)
constexpr int SLOTS = 4;     // tiles in flight per CTA
constexpr int kHalf = 128;   // output channels per CTA (MMA M, TMEM lanes)
constexpr int INFO_RING = 8; // tile descriptors in flight (claimed ahead)
constexpr int kScanGroups = 2;  // scan warp groups, alternate tiles
constexpr int kScanWarps = 4 * kScanGroups, kConvWarps = 4;
constexpr int kConvWarp0 = kScanWarps;
constexpr int kMmaWarp = kConvWarp0 + kConvWarps, kSchedWarp = kMmaWarp + 1;
constexpr int kLbWarp0 = kMmaWarp + 2, kLbWarps = SLOTS;  // look-back warp s serves slot s
constexpr int kThreads = 32 * (kLbWarp0 + kLbWarps);
constexpr int kGroupThreads = 128;  // threads of one scan group (one per channel)

// TMEM columns (512 allocated): W_a half-head rows, W_x rows, then per slot
// [pre_r | pre_i] accumulators that pass 1 overwrites with [a | v].
constexpr uint32_t kColWa = 0, kColWx = 128, kColSlot0 = 256, kColPerSlot = 2 * NT;

// Shared memory map (offsets from a 1024-byte aligned base)
constexpr int kBTile = NT * 256 * 2;            // bf16 xc, 4 K-blocks of 64 channels
constexpr int kBBlock = NT * 128;               // one K-block: NT rows x 128 B
constexpr int kXcsTile = NT * kHalf * 4;        // fp32 xc / 2 of this half
constexpr int kGTile = NT * kHalf * 2;          // bf16 gate-branch tile (TMA box)
constexpr int XRING = 3;                         // x tiles (32 rows + 3 halo rows) in flight
constexpr int kXRows = NT + 3;
constexpr int kXTile = kXRows * 256 * 2;         // bf16, all 256 channels of the head
constexpr int OFF_B = 0;
constexpr int OFF_XCS = OFF_B + SLOTS * kBTile;
constexpr int OFF_G = OFF_XCS + SLOTS * kXcsTile;
constexpr int OFF_X = OFF_G + SLOTS * kGTile;
constexpr int OFF_AGG = OFF_X + XRING * kXTile;
constexpr int OFF_HIN = OFF_AGG + SLOTS * kHalf * 8;
constexpr int OFF_INFO = OFF_HIN + SLOTS * kHalf * 4;
constexpr int OFF_BAR = OFF_INFO + INFO_RING * 32;
// per-slot barriers (slot = tile % SLOTS)
enum { BAR_CONV, BAR_SMEM_FREE, BAR_MMA, BAR_TMEM_FREE, BAR_PASS1, BAR_LB, BAR_G, BAR_PUB, BAR_KINDS };
constexpr int OFF_RING_BAR = OFF_BAR + BAR_KINDS * SLOTS * 8;  // INFO_FULL[8], INFO_EMPTY[8]
constexpr int OFF_XBAR = OFF_RING_BAR + 2 * INFO_RING * 8;         // X_FULL[3], X_EMPTY[3]
constexpr int OFF_MISC = OFF_XBAR + 2 * XRING * 8;
constexpr int kSmemUsed = OFF_MISC + 16 + SLOTS * 4;
constexpr int kSmemBytes = kSmemUsed + 1024;    // slack for the 1024-byte alignment
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s per wait

struct TileInfo {
    int u;        // tile index inside the (head, half) group, -1 = no more work
    int b, t0, valid;
    uint32_t reset_mask;  // bit t: segment_pos == 0 at token t0 + t (conv tap of lag 1 dropped, h reset)
    uint32_t m2, m3;      // bit t: segment_pos < 2 (< 3): conv tap of lag 2 (3) dropped
    int first_last;       // bit 0: first tile of the sequence, bit 1: last tile
};
static_assert(sizeof(TileInfo) == 32, "TileInfo size");
static_assert(SLOTS * 2 == INFO_RING, "ring sizes");

struct FusedParams {
    int B, T, D, C, G, tiles_per_group;
    const __nv_bfloat16 *x;
    const float *conv_w, *conv_b;
    const __nv_bfloat16 *W_a;
    const float *b_a;
    const __nv_bfloat16 *W_x;
    const float *b_x, *lambda;
    const int32_t *segpos;
    __nv_bfloat16 *conv_state;
    float *h_state;
    __nv_bfloat16 *y;
    WsHeader *hdr;
    uint32_t *flags;   // [G][tiles_per_group]
    float2 *agg;       // [G][tiles_per_group][128]  (prod a, h_end) from h = 0
    float *prefix;     // [G][tiles_per_group][128]  h after the tile
    unsigned long long *trace;  // RGLRU_TRACE builds only: per-role timestamps
};

// Tracing (compiled in with -DRGLRU_TRACE only): CTAs below kTraceCtas record
// %globaltimer at each role's milestones for their first kTraceTiles tiles,
// into trace[(cta * kTraceTiles + tile) * kTraceEvents + event].
enum TraceEvent {
    TR_SCHED_INFO, TR_CONV_START, TR_CONV_DONE, TR_MMA_ISSUED, TR_P1_START, TR_P1_END, TR_LB_START,
    TR_LB_HIN, TR_LB_DONE, TR_P2_START, TR_P2_END, TR_TILE_U, TR_MMA_TFREE, TR_MMA_TMA, TR_MMA_CONV,
    TR_CONV_GO, kTraceEvents
};
#ifdef RGLRU_TRACE
constexpr int kTraceCtas = 4, kTraceTiles = 128;
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
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        // suspended in hardware until the phase completes (or 20 us pass)
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        {
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
        for (uint32_t it = 0; it < (1u << 20) && !(seen = mbar_try_wait(bar, parity)); ++it) {
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
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
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

__device__ __forceinline__ float gelu_tanh_fast(float g)
{
    const float k0 = 0.7978845608028654f, k1 = 0.7978845608028654f * 0.044715f;
    const float u = g * fmaf(k1 * g, g, k0);
    const float hg = 0.5f * g;
    return fmaf(hg, tanh_approx(u), hg);
}

__global__ void __launch_bounds__(kThreads, 1)
rglru_prefill_fused_kernel(const FusedParams p, const __grid_constant__ CUtensorMap tmap_g,
                           const __grid_constant__ CUtensorMap tmap_x)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int group = blockIdx.x % p.G;
    const int head = group >> 1, half = group & 1;
    TileInfo *info = reinterpret_cast<TileInfo *>(smem + OFF_INFO);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *ring_bars = reinterpret_cast<uint64_t *>(smem + OFF_RING_BAR);
    auto bar = [&](int kind, int s) { return bars + kind * SLOTS + s; };
    auto info_full = [&](int i) { return ring_bars + i; };
    auto info_empty = [&](int i) { return ring_bars + INFO_RING + i; };
    uint64_t *xbars = reinterpret_cast<uint64_t *>(smem + OFF_XBAR);
    auto x_full = [&](int i) { return xbars + i; };
    auto x_empty = [&](int i) { return xbars + XRING + i; };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
    WsHeader *hdr = p.hdr;

    // ------------------------------------------------------------------ setup
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_holder, 512);
        if (lane == 0) {
            for (int s = 0; s < SLOTS; ++s) {
                mbar_init(bar(BAR_CONV, s), kConvWarps * 32);
                mbar_init(bar(BAR_SMEM_FREE, s), kGroupThreads);
                mbar_init(bar(BAR_MMA, s), 1);
                mbar_init(bar(BAR_TMEM_FREE, s), kGroupThreads);
                mbar_init(bar(BAR_PASS1, s), kGroupThreads);
                mbar_init(bar(BAR_LB, s), 32);
                mbar_init(bar(BAR_G, s), 1);
                mbar_init(bar(BAR_PUB, s), 32);
            }
            for (int i = 0; i < INFO_RING; ++i) {
                mbar_init(info_full(i), 1);
                mbar_init(info_empty(i), kGroupThreads);
            }
            for (int i = 0; i < XRING; ++i) {
                mbar_init(x_full(i), 1);
                mbar_init(x_empty(i), kConvWarps * 32);
            }
            *abort_flag = 0;
            mbar_fence_init();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp < kScanWarps) {
        // TMEM lane = output channel c of the half; scan group g loads the rows
        // of gate g (W_a, W_x) for its channel
        const int c = threadIdx.x % kGroupThreads;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const size_t row = (size_t)head * 256 + half * kHalf + c;
#pragma unroll 1
        for (int gate = warp / 4; gate < 2; gate += kScanGroups) {
            const uint4 *src = reinterpret_cast<const uint4 *>((gate == 0 ? p.W_a : p.W_x) + row * 256);
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                uint32_t r[32];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint4 v = src[q * 8 + k];
                    r[4 * k] = v.x;
                    r[4 * k + 1] = v.y;
                    r[4 * k + 2] = v.z;
                    r[4 * k + 3] = v.w;
                }
                tmem_st32(tmem + lane_off + (gate == 0 ? kColWa : kColWx) + q * 32, r);
            }
        }
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const int debug_unit = *(volatile int *)&hdr->debug_unit_plus1 - 1;

    if (warp == kSchedWarp) {
        // ------------------------------------------------------------ scheduler
        // Claims tiles in order from this group's ticket counter, one tile ahead
        // of the ring, so that the atomic and the segment_pos read overlap the
        // wait for a free ring entry.
        auto claim = [&]() -> TileInfo {
            int u = -1;
            if (lane == 0 && !*abort_flag) {
                u = (int)atomicAdd(&hdr->ticket[group], 1u);
                if (u >= p.tiles_per_group) u = -1;
            }
            u = __shfl_sync(0xffffffffu, u, 0);
            TileInfo ti{};
            ti.u = u;
            if (u >= 0) {
                ti.b = u / p.C;
                const int c = u % p.C;
                ti.t0 = c * NT;
                ti.valid = min(NT, p.T - ti.t0);
                ti.first_last = (c == 0 ? 1 : 0) | (c == p.C - 1 ? 2 : 0);
                const int sp = lane < ti.valid ? p.segpos[(size_t)ti.b * p.T + ti.t0 + lane] : 3;
                ti.reset_mask = __ballot_sync(0xffffffffu, sp < 1);
                ti.m2 = __ballot_sync(0xffffffffu, sp < 2);
                ti.m3 = __ballot_sync(0xffffffffu, sp < 3);
            }
            return ti;
        };
        TileInfo next = claim();
        // end markers: one per scan group and one per look-back warp (each of
        // those reads only its own residue class of tiles)
        constexpr int kEndMarkers = kScanGroups > kLbWarps ? kScanGroups : kLbWarps;
        static_assert(kEndMarkers <= INFO_RING, "end markers fit the ring");
        int ends = 0;
        int x_issued = 0;  // x-tile TMA loads issued
#pragma unroll 1
        for (int j = 0;; ++j) {
            const int ir = j % INFO_RING;
            bool ok = true;
            if (j >= INFO_RING)
                ok = warp_wait_bar(info_empty(ir), (uint32_t)((j / INFO_RING) - 1) & 1u, abort_flag, hdr, 1);
            if (!ok) next.u = -1;
            if (lane == 0) {
                info[ir] = next;
                mbar_arrive(info_full(ir));
                RGLRU_TR(TR_SCHED_INFO, j, globaltimer());
                RGLRU_TR(TR_TILE_U, j, (unsigned long long)(unsigned)next.u);
            }
            if (next.u < 0) {
                if (++ends == kEndMarkers || !ok) break;
                continue;
            }
            // x rows t0-3 .. t0+31 of all 256 channels of the head into the x ring
            // (rows before t = 0 arrive zero-filled; the conv reads conv_state there)
            const int xr = j % XRING;
            if (j >= XRING && !warp_wait_bar(x_empty(xr), (uint32_t)((j / XRING) - 1) & 1u, abort_flag, hdr, 15)) {
                next.u = -1;
                continue;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(x_full(xr), kXTile);
                tma_load_3d(smem + OFF_X + xr * kXTile, &tmap_x, x_full(xr), head * 256, next.t0 - 3, next.b);
            }
            ++x_issued;
            next = claim();
        }
        // on abort, wait (bounded) for the x loads still in flight
        if (lane == 0 && *abort_flag) {
            for (int k = max(0, x_issued - XRING); k < x_issued; ++k) {
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(x_full(k % XRING), (uint32_t)(k / XRING) & 1u) && globaltimer() - t0 < kTimeoutNs) {
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer (+ GELU-branch TMA)
        const uint32_t idesc = umma_idesc_bf16(kHalf, NT);
        int issued = 0;
#pragma unroll 1
        for (int j = 0;; ++j) {
            const int s = j % SLOTS, ir = j % INFO_RING;
            const uint32_t ph = (uint32_t)(j / SLOTS) & 1u;
            if (!warp_wait_bar(info_full(ir), (uint32_t)(j / INFO_RING) & 1u, abort_flag, hdr, 2)) break;
            const TileInfo ti = info[ir];
            if (ti.u < 0) break;
            if (j >= SLOTS && !warp_wait_bar(bar(BAR_TMEM_FREE, s), ph ^ 1u, abort_flag, hdr, 3)) break;
            if (lane == 0) RGLRU_TR(TR_MMA_TFREE, j, globaltimer());
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(BAR_G, s), kGTile);
                tma_load_3d(smem + OFF_G + s * kGTile, &tmap_g, bar(BAR_G, s), head * 256 + half * kHalf, ti.t0,
                            ti.b);
            }
            if (lane == 0) RGLRU_TR(TR_MMA_TMA, j, globaltimer());
            ++issued;
            if (!warp_wait_bar(bar(BAR_CONV, s), ph, abort_flag, hdr, 4)) break;
            if (lane == 0) RGLRU_TR(TR_MMA_CONV, j, globaltimer());
            if (lane == 0) {
                tc_fence_after();
                const uint32_t b_base = smem_u32(smem + OFF_B + s * kBTile);
                const uint32_t d_r = tmem + kColSlot0 + s * kColPerSlot;
                const uint32_t d_i = d_r + NT;
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) {
                    const uint64_t bd = umma_desc_sw128(b_base + (kk >> 2) * kBBlock + (kk & 3) * 32);
                    umma_ts(d_r, tmem + kColWa + kk * 8, bd, idesc, kk > 0);
                    umma_ts(d_i, tmem + kColWx + kk * 8, bd, idesc, kk > 0);
                }
                umma_commit(bar(BAR_MMA, s));
                RGLRU_TR(TR_MMA_ISSUED, j, globaltimer());
            }
            __syncwarp();
        }
        // on abort, wait (bounded) for this CTA's copies and MMAs in flight
        if (lane == 0 && *abort_flag) {
            for (int k = max(0, issued - SLOTS); k < issued; ++k) {
                const int s = k % SLOTS;
                const uint32_t ph = (uint32_t)(k / SLOTS) & 1u;
                uint64_t t0 = globaltimer();
                while (!mbar_try_wait(bar(BAR_G, s), ph) && globaltimer() - t0 < kTimeoutNs) {
                }
                t0 = globaltimer();
                while (!mbar_try_wait(bar(BAR_MMA, s), ph) && globaltimer() - t0 < kTimeoutNs / 4) {
                }
            }
        }
    } else if (warp >= kConvWarp0 && warp < kConvWarp0 + kConvWarps) {
        // ------------------------------------------------------------ conv warps
        // Warp kb covers the head's channels [64 kb, 64 kb + 64) (one K-block of
        // the B tile); lane = (token half q, group of 4 channels cg), so each
        // lane runs 16 consecutive tokens of 4 channels, in fp32 pairs.
        const int kb = warp - kConvWarp0;
        const int cg = lane & 15;
        const int q = lane >> 4;
        const int dl = kb * 64 + cg * 4;  // channel within the head
        const size_t d0 = (size_t)head * 256 + dl;
        // The conv produces xh = xc / 2 (halving is exact): the MMA then yields
        // half pre-activations, which is what sigmoid(z) = (1 + tanh(z/2)) / 2
        // needs, and the scan's i*xc becomes one FMA on xh.
        f2_t w2[4][2], cb2[2];
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int e = 0; e < 2; ++e)
                w2[k][e] = f2_make(0.5f * p.conv_w[(size_t)k * p.D + d0 + 2 * e],
                                   0.5f * p.conv_w[(size_t)k * p.D + d0 + 2 * e + 1]);
#pragma unroll
        for (int e = 0; e < 2; ++e) cb2[e] = f2_make(0.5f * p.conv_b[d0 + 2 * e], 0.5f * p.conv_b[d0 + 2 * e + 1]);
        const bool own = (kb >> 1) == half;
        const int xcs_c = (kb & 1) * 64 + cg * 4;  // channel within this half
#pragma unroll 1
        for (int j = 0;; ++j) {
            const int s = j % SLOTS, ir = j % INFO_RING;
            const uint32_t ph = (uint32_t)(j / SLOTS) & 1u;
            if (!warp_wait_bar(info_full(ir), (uint32_t)(j / INFO_RING) & 1u, abort_flag, hdr, 5)) break;
            const TileInfo ti = info[ir];
            if (ti.u < 0) break;
            if (lane == 0 && kb == 0) RGLRU_TR(TR_CONV_START, j, globaltimer());
            const int xr = j % XRING;
            if (!warp_wait_bar(x_full(xr), (uint32_t)(j / XRING) & 1u, abort_flag, hdr, 16)) break;
            if (j >= SLOTS && !warp_wait_bar(bar(BAR_SMEM_FREE, s), ph ^ 1u, abort_flag, hdr, 6)) break;
            if (lane == 0 && kb == 0) RGLRU_TR(TR_CONV_GO, j, globaltimer());
            const int n0 = q * 16;
            uint8_t *xt = smem + OFF_X + xr * kXTile + dl * 2;  // row r = token t0 - 3 + r
            if (ti.t0 == 0 && q == 0) {
                // sequence start: rows 0..2 (tokens -3..-1, zero-filled by the
                // load) are the carried conv state; each lane patches the 4
                // channels it reads itself
#pragma unroll
                for (int r = 0; r < 3; ++r)
                    *reinterpret_cast<uint2 *>(xt + r * 512) =
                        *reinterpret_cast<const uint2 *>(p.conv_state + ((size_t)ti.b * 3 + r) * p.D + d0);
            }
            auto xrow = [&](int r, f2_t (&f)[2]) {
                const uint2 v = *reinterpret_cast<const uint2 *>(xt + r * 512);
                f[0] = f2_from_bf16x2(v.x);
                f[1] = f2_from_bf16x2(v.y);
            };
            uint8_t *btile = smem + OFF_B + s * kBTile + kb * kBBlock;
            // fp32 xh of this half, token pairs interleaved: [t / 2][channel][t % 2]
            float *xcs = reinterpret_cast<float *>(smem + OFF_XCS + s * kXcsTile);
            // a tile with no document start and all 32 tokens valid needs no masks
            const bool clean = (ti.reset_mask | ti.m2 | ti.m3) == 0u && ti.valid == NT;
            auto run = [&](auto clean_tag) {
                constexpr bool kClean = decltype(clean_tag)::value;
                f2_t xm3[2], xm2[2], xm1[2], prev[2];
                xrow(n0, xm3);
                xrow(n0 + 1, xm2);
                xrow(n0 + 2, xm1);
#pragma unroll 4
                for (int i = 0; i < 16; ++i) {
                    f2_t x0[2];
                    xrow(n0 + i + 3, x0);
                    const int n = n0 + i;
                    f2_t acc[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        if constexpr (kClean) {
                            acc[e] = f2_fma(w2[3][e], x0[e],
                                            f2_fma(w2[2][e], xm1[e], f2_fma(w2[1][e], xm2[e], f2_fma(w2[0][e], xm3[e], cb2[e]))));
                        } else {
                            // tap of lag k dropped when segment_pos < k (document start)
                            f2_t v = cb2[e];
                            if (!((ti.m3 >> n) & 1u)) v = f2_fma(w2[0][e], xm3[e], v);
                            if (!((ti.m2 >> n) & 1u)) v = f2_fma(w2[1][e], xm2[e], v);
                            if (!((ti.reset_mask >> n) & 1u)) v = f2_fma(w2[2][e], xm1[e], v);
                            v = f2_fma(w2[3][e], x0[e], v);
                            acc[e] = n < ti.valid ? v : 0ull;
                        }
                    }
                    // B tile row n: 4 channels = the (cg & 1) half of 16-byte chunk cg >> 1
                    *reinterpret_cast<uint2 *>(btile + n * 128 + (((cg >> 1) ^ (n & 7)) << 4) + (cg & 1) * 8) =
                        make_uint2(f2_to_bf16x2(acc[0]), f2_to_bf16x2(acc[1]));
                    if ((i & 1) && own) {
                        float4 *dst = reinterpret_cast<float4 *>(xcs + ((n >> 1) * kHalf + xcs_c) * 2);
                        dst[0] = make_float4(f2_lo(prev[0]), f2_lo(acc[0]), f2_hi(prev[0]), f2_hi(acc[0]));
                        dst[1] = make_float4(f2_lo(prev[1]), f2_lo(acc[1]), f2_hi(prev[1]), f2_hi(acc[1]));
                    }
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        prev[e] = acc[e];
                        xm3[e] = xm2[e];
                        xm2[e] = xm1[e];
                        xm1[e] = x0[e];
                    }
                }
            };
            if (clean)
                run(std::true_type{});
            else
                run(std::false_type{});
            // generic writes (B tile, patched x rows) before the async proxy's
            // next accesses (the MMA, the next load into this x slot)
            fence_proxy_async_smem();
            mbar_arrive(x_empty(xr));
            mbar_arrive(bar(BAR_CONV, s));
            if (lane == 0 && kb == 0) RGLRU_TR(TR_CONV_DONE, j, globaltimer());
        }
    } else if (warp < kScanWarps) {
        // ------------------------------------------------------------ scan warps
        const int sg = warp / 4;                 // scan group: tiles j with j % kScanGroups == sg
        const int c = threadIdx.x % kGroupThreads;
        const int d = head * 256 + half * kHalf + c;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const float hba = 0.5f * p.b_a[d], hbx = 0.5f * p.b_x[d];
        const float lam = p.lambda[d];
        const float ls = lam >= 0.f ? -log1pf(expf(-lam)) : lam - log1pf(expf(lam));  // log sigmoid(Lambda)
        const float kl = kC * ls;                       // log a per unit r (<= 0)
        // r = (1 + tr) / 2 with tr = tanh(half pre-activation): log a = tr * hkl + hkl
        const float hkl = 0.5f * kl;
        const float hkl2 = hkl * 1.4426950408889634f;  // same in log2
        // every log a of this channel lies in [kl, 0]: the short series for
        // 1 - a^2 applies to all of them when kl > -1/8
        const bool series_ok = kl > -0.125f;
        const f2_t hba2 = f2_splat(hba), hbx2 = f2_splat(hbx), hkl_2 = f2_splat(hkl), hkl2_2 = f2_splat(hkl2);
        const f2_t c13_2 = f2_splat(1.f / 3.f), c23_2 = f2_splat(2.f / 3.f), one_2 = f2_splat(1.f),
                   mtwo_2 = f2_splat(-2.f);

        auto pass1 = [&](int j) -> bool {
            const int s = j % SLOTS;
            const uint32_t ph = (uint32_t)(j / SLOTS) & 1u;
            const TileInfo ti = info[j % INFO_RING];
            if (!warp_wait_bar(bar(BAR_MMA, s), ph, abort_flag, hdr, 7)) return false;
            if (c == 0) RGLRU_TR(TR_P1_START, j, globaltimer());
            tc_fence_after();
            const uint32_t col = tmem + lane_off + kColSlot0 + s * kColPerSlot;
            // xh of tokens (2m, 2m + 1) of this channel: one 8-byte load
            const float2 *xcs2 = reinterpret_cast<const float2 *>(smem + OFF_XCS + s * kXcsTile) + c;
            float hl = 0.f, P = 1.f;
            f2_t lsum = 0ull;  // clean chunks: sum of log2 a (P = 2^sum at the end)
#pragma unroll 1
            for (int t8 = 0; t8 < NT; t8 += 8) {
                uint32_t ar[8], ai[8];
                tmem_ld8(col + t8, ar);
                tmem_ld8(col + NT + t8, ai);
                tmem_wait_ld();
                const bool clean = ((ti.reset_mask >> t8) & 0xffu) == 0u && t8 + 8 <= ti.valid && series_ok;
                if (clean) {
#pragma unroll
                    for (int k = 0; k < 8; k += 2) {
                        const float2 xh = xcs2[((t8 + k) >> 1) * kHalf];
                        const f2_t zr = f2_add(f2_make(__uint_as_float(ar[k]), __uint_as_float(ar[k + 1])), hba2);
                        const f2_t zi = f2_add(f2_make(__uint_as_float(ai[k]), __uint_as_float(ai[k + 1])), hbx2);
                        const f2_t tr = f2_make(tanh_approx(f2_lo(zr)), tanh_approx(f2_hi(zr)));
                        const f2_t tg = f2_make(tanh_approx(f2_lo(zi)), tanh_approx(f2_hi(zi)));
                        const f2_t ell = f2_fma(tr, hkl_2, hkl_2);    // log a
                        const f2_t la = f2_fma(tr, hkl2_2, hkl2_2);  // log2 a
                        lsum = f2_add(lsum, la);
                        const float a0 = ex2_approx(f2_lo(la)), a1 = ex2_approx(f2_hi(la));
                        // 1 - exp(2 ell) by its series (see one_minus_exp2l_small)
                        f2_t sr = f2_fma(ell, c13_2, c23_2);
                        sr = f2_fma(ell, sr, one_2);
                        sr = f2_fma(ell, sr, one_2);
                        const f2_t om = f2_mul(f2_mul(ell, mtwo_2), sr);
                        const f2_t nrm = f2_make(sqrt_approx(f2_lo(om)), sqrt_approx(f2_hi(om)));
                        const f2_t xh2 = f2_make(xh.x, xh.y);
                        const f2_t v = f2_mul(nrm, f2_fma(tg, xh2, xh2));  // sqrt(1-a^2) * i * xc
                        hl = fmaf(a0, hl, f2_lo(v));
                        hl = fmaf(a1, hl, f2_hi(v));
                        ar[k] = __float_as_uint(a0);
                        ar[k + 1] = __float_as_uint(a1);
                        ai[k] = __float_as_uint(f2_lo(v));
                        ai[k + 1] = __float_as_uint(f2_hi(v));
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int t = t8 + k;
                        const float xh = reinterpret_cast<const float *>(xcs2 + (t >> 1) * kHalf)[t & 1];
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
                        ar[k] = __float_as_uint(a);
                        ai[k] = __float_as_uint(v);
                    }
                }
                tmem_st8(col + t8, ar);
                tmem_st8(col + NT + t8, ai);
            }
            P *= ex2_approx(f2_lo(lsum) + f2_hi(lsum));
            mbar_arrive(bar(BAR_SMEM_FREE, s));  // xcs (and, via the MMA wait, the B tile) consumed
            tmem_wait_st();
            // the look-back warp must have copied out this slot's previous aggregate
            if (j >= SLOTS && !warp_wait_bar(bar(BAR_PUB, s), ph ^ 1u, abort_flag, hdr, 17)) return false;
            reinterpret_cast<float2 *>(smem + OFF_AGG + s * kHalf * 8)[c] = make_float2(P, hl);
            mbar_arrive(bar(BAR_PASS1, s));
            if (c == 0) RGLRU_TR(TR_P1_END, j, globaltimer());
            return true;
        };

        auto pass2 = [&](int j) -> bool {
            const int s = j % SLOTS, ir = j % INFO_RING;
            const uint32_t ph = (uint32_t)(j / SLOTS) & 1u;
            const TileInfo ti = info[ir];
            if (!warp_wait_bar(bar(BAR_LB, s), ph, abort_flag, hdr, 8)) return false;
            float h = reinterpret_cast<const float *>(smem + OFF_HIN + s * kHalf * 4)[c];
            if (!warp_wait_bar(bar(BAR_G, s), ph, abort_flag, hdr, 9)) return false;
            if (c == 0) RGLRU_TR(TR_P2_START, j, globaltimer());
            tc_fence_after();
            const uint32_t col = tmem + lane_off + kColSlot0 + s * kColPerSlot;
            const __nv_bfloat16 *gs = reinterpret_cast<const __nv_bfloat16 *>(smem + OFF_G + s * kGTile) + c;
            __nv_bfloat16 *yp = p.y + ((size_t)ti.b * p.T + ti.t0) * p.D + d;
            const size_t ystep = p.D;
#pragma unroll 1
            for (int t8 = 0; t8 < NT; t8 += 8) {
                uint32_t aa[8], vv[8];
                tmem_ld8(col + t8, aa);
                tmem_ld8(col + NT + t8, vv);
                tmem_wait_ld();
                if (t8 + 8 <= ti.valid) {
#pragma unroll
                    for (int k = 0; k < 8; k += 2) {
                        h = fmaf(__uint_as_float(aa[k]), h, __uint_as_float(vv[k]));
                        const float h0 = h;
                        h = fmaf(__uint_as_float(aa[k + 1]), h, __uint_as_float(vv[k + 1]));
                        const f2_t gv = f2_make(__bfloat162float(gs[(t8 + k) * kHalf]), __bfloat162float(gs[(t8 + k + 1) * kHalf]));
                        const uint32_t yy = f2_to_bf16x2(f2_mul(gelu2(gv), f2_make(h0, h)));
                        const __nv_bfloat162 y2 = *reinterpret_cast<const __nv_bfloat162 *>(&yy);
                        yp[(size_t)(t8 + k) * ystep] = y2.x;
                        yp[(size_t)(t8 + k + 1) * ystep] = y2.y;
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int t = t8 + k;
                        h = fmaf(__uint_as_float(aa[k]), h, __uint_as_float(vv[k]));
                        if (t < ti.valid) {
                            const float gv = __bfloat162float(gs[t * kHalf]);
                            yp[(size_t)t * ystep] = __float2bfloat16_rn(gelu_tanh_fast(gv) * h);
                        }
                    }
                }
            }
            if (ti.first_last & 2) {
                // The old states are read by the first tile of this sequence (its
                // conv in both halves of the head, its look-back for h): wait until
                // those reads are published before overwriting the states.
                const size_t u0 = (size_t)ti.b * p.C;
                const uint32_t *f_own = p.flags + (size_t)group * p.tiles_per_group + u0;
                const uint32_t *f_oth = p.flags + (size_t)(group ^ 1) * p.tiles_per_group + u0;
                if (warp_wait_flag(f_own, F_PREFIX, abort_flag, hdr, 10) == 0) return false;
                if (warp_wait_flag(f_oth, F_AGG, abort_flag, hdr, 11) == 0) return false;
                p.h_state[(size_t)ti.b * p.D + d] = h;
                __nv_bfloat16 ncs[3];
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    const int ts = p.T - 3 + k;
                    ncs[k] = ts >= 0 ? p.x[((size_t)ti.b * p.T + ts) * p.D + d]
                                     : p.conv_state[((size_t)ti.b * 3 + 3 + ts) * p.D + d];
                }
#pragma unroll
                for (int k = 0; k < 3; ++k) p.conv_state[((size_t)ti.b * 3 + k) * p.D + d] = ncs[k];
            }
            tc_fence_before();
            mbar_arrive(bar(BAR_TMEM_FREE, s));
            mbar_arrive(info_empty(ir));
            if (c == 0) RGLRU_TR(TR_P2_END, j, globaltimer());
            return true;
        };

        // this group's tiles: j = sg, sg + kScanGroups, ...; pass 2 of a tile runs
        // after pass 1 of the group's next tile (the look-back has that long)
#pragma unroll 1
        for (int j = sg;; j += kScanGroups) {
            const int ir = j % INFO_RING;
            bool end = !warp_wait_bar(info_full(ir), (uint32_t)(j / INFO_RING) & 1u, abort_flag, hdr, 12);
            if (!end) end = info[ir].u < 0;
            bool ok = true;
            if (!end) ok = pass1(j);
            if (ok && j >= kScanGroups) ok = pass2(j - kScanGroups);
            if (!ok || end) break;
        }
    } else if (warp >= kLbWarp0) {
        // ------------------------------------------------------------ look-back warps
        // Warp s serves the tiles of slot s (j = s, s + SLOTS, ...), so it waits on
        // its slot's barriers one phase at a time.  Per tile: publish the
        // aggregate (later tiles of the sequence may combine it before this
        // tile's own look-back has finished), find the anchor, fold, hand the
        // carried-in state to pass 2, publish the inclusive prefix.  These warps
        // are the only ones that fence for the aggregates and prefixes.
        const int s = warp - kLbWarp0;
        const int ch = lane * 4;  // 4 channels per lane
        const size_t dch = (size_t)head * 256 + half * kHalf + ch;
        const size_t gbase = (size_t)group * p.tiles_per_group;
        constexpr int kFoldBatch = 4;  // aggregates loaded per round trip
#pragma unroll 1
        for (int j = s;; j += SLOTS) {
            const int ir = j % INFO_RING;
            const uint32_t ph = (uint32_t)(j / SLOTS) & 1u;
            if (!warp_wait_bar(info_full(ir), (uint32_t)(j / INFO_RING) & 1u, abort_flag, hdr, 13)) break;
            const TileInfo ti = info[ir];
            if (ti.u < 0) break;
            if (!warp_wait_bar(bar(BAR_PASS1, s), ph, abort_flag, hdr, 14)) break;
            if (lane == 0) RGLRU_TR(TR_LB_START, j, globaltimer());
            const float4 *sagg = reinterpret_cast<const float4 *>(smem + OFF_AGG + s * kHalf * 8);
            const float4 g01 = sagg[lane * 2], g23 = sagg[lane * 2 + 1];  // (A,H) of 4 channels
            mbar_arrive(bar(BAR_PUB, s));  // the slot's aggregate buffer is free again
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
            // pass 2 needs only the carried-in state: hand it over before publishing
            *reinterpret_cast<float4 *>(smem + OFF_HIN + s * kHalf * 4 + ch * 4) =
                make_float4(hin[0], hin[1], hin[2], hin[3]);
            mbar_arrive(bar(BAR_LB, s));
            if (!suppress) {
                float pre[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) pre[e] = fmaf(A[e], hin[e], Hh[e]);
                *reinterpret_cast<float4 *>(p.prefix + gu * kHalf + ch) = make_float4(pre[0], pre[1], pre[2], pre[3]);
                __threadfence();
                __syncwarp();
                if (lane == 0) atom_or_release_u32(p.flags + gu, F_AGG | F_PREFIX | rbit);
            }
            if (lane == 0) RGLRU_TR(TR_LB_DONE, j, globaltimer());
        }
    }

    // ------------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

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
    if ((size_t)L.tpg > 0x7fffffffu / 2 || L.G > (int)(sizeof(WsHeader::ticket) / sizeof(unsigned int)))
        return RGLRU_ERR_UNSUPPORTED;
    auto encode = encode_fn();
    if (!encode) return RGLRU_ERR_CUDA;

    CUtensorMap tmap;
    const cuuint64_t gdim[3] = {(cuuint64_t)a.D, (cuuint64_t)a.T, (cuuint64_t)a.B};
    const cuuint64_t gstride[2] = {(cuuint64_t)a.D * 2, (cuuint64_t)a.T * a.D * 2};
    const cuuint32_t box[3] = {kHalf, NT, 1};
    const cuuint32_t estride[3] = {1, 1, 1};
    if (encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(a.g), gdim, gstride, box, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return RGLRU_ERR_CUDA;
    CUtensorMap tmap_x;
    const cuuint32_t xbox[3] = {256, kXRows, 1};
    if (encode(&tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(a.x), gdim, gstride, xbox, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return RGLRU_ERR_CUDA;

    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RGLRU_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return RGLRU_ERR_CUDA;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(rglru_prefill_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kSmemBytes);
    });
    if (attr_err != cudaSuccess) return RGLRU_ERR_CUDA;

    char *ws = static_cast<char *>(a.ws);
    // tickets and flags start at zero; the status word and the test hook are kept
    if (cudaMemsetAsync(ws + offsetof(WsHeader, ticket), 0,
                        L.flags_off - offsetof(WsHeader, ticket) + L.flags_bytes, a.stream) != cudaSuccess)
        return RGLRU_ERR_CUDA;

    FusedParams p;
    p.B = a.B; p.T = a.T; p.D = a.D; p.C = L.C; p.G = L.G; p.tiles_per_group = L.tpg;
    p.x = static_cast<const __nv_bfloat16 *>(a.x);
    p.conv_w = a.conv_w; p.conv_b = a.conv_b;
    p.W_a = static_cast<const __nv_bfloat16 *>(a.W_a); p.b_a = a.b_a;
    p.W_x = static_cast<const __nv_bfloat16 *>(a.W_x); p.b_x = a.b_x;
    p.lambda = a.lambda; p.segpos = a.segpos;
    p.conv_state = static_cast<__nv_bfloat16 *>(a.conv_state);
    p.h_state = a.h_state;
    p.y = static_cast<__nv_bfloat16 *>(a.y);
    p.hdr = reinterpret_cast<WsHeader *>(ws);
    p.flags = reinterpret_cast<uint32_t *>(ws + L.flags_off);
    p.agg = reinterpret_cast<float2 *>(ws + L.agg_off);
    p.prefix = reinterpret_cast<float *>(ws + L.prefix_off);
    p.trace = L.trace_off ? reinterpret_cast<unsigned long long *>(ws + L.trace_off) : nullptr;

    const int per_group = max(1, sms / L.G);
    const int grid = per_group * L.G;
    rglru_prefill_fused_kernel<<<grid, kThreads, kSmemBytes, a.stream>>>(p, tmap, tmap_x);
    return cuda_status(cudaGetLastError());
}

}  // namespace rglru
