// decode.cu -- batched single-token step of the RG-LRU block core (bf16 I/O,
// fp32 state) on sm_100a.
//
// One step for B sequences.  Per sequence b and channel d the conv window is
// conv_state[b, 0..2, d] followed by x[b, d]; the gates are the block-diagonal
// projections of the conv output; h_state[b, d] advances one step and
// y[b, d] = GELU_tanh(g[b, d]) * h.  With one token per sequence the B rows of
// a head are the token dimension of its gate GEMM.
//
// Grid: one cluster of two CTAs per (head, block of kTok = 48 batch rows); CTA
// rank r owns channels [128 r, 128 r + 128) of the head.  Thread = one channel
// (its TMEM lane) and 16 rows, for the conv and the epilogue alike:
//   1. one thread TMA-loads this half's x and conv_state tiles and its 128 rows
//      of W_a and W_x (128-byte swizzled, K-major: the tensor core's A
//      operands); every thread prefetches the h_state and GELU-branch values
//      of its rows into registers;
//   2. the conv of the thread's channel keeps xc / 2 in registers, writes its
//      bf16 copy into this CTA's half of the B tile, and shifts the conv_state
//      tile in shared memory (rows 1, 2, x become rows 0, 1, 2), which a TMA
//      store writes back; one bulk copy sends the half to the peer CTA, whose
//      mbarrier counts its bytes;
//   3. one thread issues the 2 x 16 MMAs D[128 out x kTok rows] = W * xc^T;
//   4. the epilogue applies the gates, a = sigmoid(Lambda)^(8 r), the
//      normalised one-step update (a reset when segment_pos == 0) and the GELU
//      product; y goes out through shared memory and a TMA store, h directly.
// The launch allows programmatic dependent launch: barrier and TMEM set-up,
// and the loads of the parameters (gate weights and conv taps, which no
// kernel of this library writes), may overlap the previous kernel's tail;
// every other global access follows griddepcontrol.wait.
// Each CTA reads and writes only its own channels of the states, so the two
// CTAs never race.  Waits on mbarriers are bounded (RGLRU_ERR_TIMEOUT in the
// workspace header); the cluster barrier at set-up and the split one at the
// end (arrive once the peer's copy has landed, wait before exiting) are reached
// exactly once by every thread of both CTAs.
//
// Block structure: "Gemma explained: RecurrentGemma architecture",
// RecurrentGemmaRecurrentBlock printout (Conv1d k=4, groups=D; GELU tanh) and
// section "Residual block with recurrent block"; RG-LRU equations of Griffin /
// RecurrentGemma (arXiv 2404.07839).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace rglru {
namespace {

using namespace sm100;

constexpr int kTok = 48;        // batch rows per cluster: the MMA N (B = 256: 6 blocks, 120 CTAs)
constexpr int kHalfCh = 128;    // channels per CTA: the MMA M and TMEM lanes
constexpr int kRows = 16;                  // rows per thread
constexpr int kRowGroups = kTok / kRows;   // 3
constexpr int kThreads = 128 * kRowGroups;  // 12 warps: lane quarter (warp & 3), row group (warp >> 2)
static_assert(kTok % kRows == 0 && kTok % 16 == 0, "row blocks");

constexpr int kWBlock = kHalfCh * 128;          // 128 weight rows x 64 channels (bf16): 16 KB
constexpr int kWGate = 4 * kWBlock;             // one gate, K = 256: 64 KB
constexpr int kBBlock = kTok * 128;             // kTok rows x 64 channels (bf16): 6 KB
static_assert(kBBlock % 1024 == 0, "B blocks are whole 128-byte swizzle atoms");
constexpr int kXTile = kTok * kHalfCh * 2;      // [kTok][128] bf16: 12 KB
constexpr int kCsTile = 3 * kXTile;             // [kTok][3][128] bf16: 36 KB
constexpr int OFF_W = 0;                        // W_a rows, then W_x rows
constexpr int OFF_B = OFF_W + 2 * kWGate;       // B tile: 4 K-blocks (all 256 channels of the head)
constexpr int OFF_X = OFF_B + 4 * kBBlock;      // x tile, later the y tile
constexpr int OFF_CS = OFF_X + kXTile;          // conv_state tile
constexpr int OFF_SP = OFF_CS + kCsTile;        // segment_pos of the block's rows
constexpr int OFF_BAR = OFF_SP + kTok * 4;      // x and conv_state loaded, W loaded, MMA done, peer's B half in
constexpr int OFF_MISC = OFF_BAR + 4 * 8;       // TMEM base address
constexpr int kSmemUsed = OFF_MISC + 16;
constexpr int kSmemBytes = kSmemUsed + 1024;    // slack for the 1024-byte alignment
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
constexpr uint32_t kTmemCols = 128;             // D_r at column 0, D_i at column kTok (2 kTok <= 128)
static_assert(2 * kTok <= (int)kTmemCols, "TMEM columns");
constexpr uint64_t kTimeoutNs = 2000000000ull;

// Tracing (compiled in with -DRGLRU_TRACE only): CTAs below kTraceCtas record
// %globaltimer at each phase into trace[cta * kTraceEvents + event].
enum DecTraceEvent {
    DT_START, DT_WAITED, DT_INPUTS, DT_CONV, DT_CLUSTER, DT_WEIGHTS, DT_MMA, DT_EPI0, DT_EPI1, DT_END, kTraceEvents
};
#ifdef RGLRU_TRACE
constexpr int kTraceCtas = 8;
#define DEC_TR(ev)                                                                                     \
    do {                                                                                              \
        if (blockIdx.x < kTraceCtas)                                                                  \
            reinterpret_cast<unsigned long long *>(reinterpret_cast<char *>(p.hdr) + kWsHeaderBytes)  \
                [blockIdx.x * kTraceEvents + (ev)] = globaltimer();                                   \
    } while (0)
#else
#define DEC_TR(ev) \
    do {           \
    } while (0)
#endif

struct DecodeParams {
    int B, D, nblk;
    const __nv_bfloat16 *g;
    const float *conv_w, *conv_b, *b_a, *b_x, *lambda;
    const int32_t *segpos;
    float *h_state;
    WsHeader *hdr;
};

struct DecodeMaps {
    CUtensorMap wa, wx;  // [D rows, 256] bf16, 64 x 128 boxes, 128-byte swizzle
    CUtensorMap x, y;    // [B, D] bf16, 128 x kTok boxes
    CUtensorMap cs;      // conv_state [B, 3, D] bf16, 128 x 3 x kTok boxes
};

// Bounded wait on an mbarrier phase by every lane of a warp; false (and the
// status recorded) if it does not complete within kTimeoutNs.
__device__ __noinline__ bool dec_wait_slow(uint64_t *bar, uint32_t parity, WsHeader *hdr, int where)
{
    bool seen = mbar_try_wait(bar, parity);
    if (!seen) {
        const uint64_t t0 = globaltimer();
        while (!(seen = mbar_try_wait_sleep(bar, parity, 20000u)) && globaltimer() - t0 < kTimeoutNs) {
        }
    }
    if (!__all_sync(0xffffffffu, seen)) {
        if ((threadIdx.x & 31) == 0) {
            atomicCAS(&hdr->status, 0, (int)RGLRU_ERR_TIMEOUT);
            atomicCAS(&hdr->detail, 0, (int)(blockIdx.x << 8) | (where + 1));
        }
        return false;
    }
    return true;
}

// A phase that is already complete costs one inline test per lane and a vote.
__device__ __forceinline__ bool dec_wait(uint64_t *bar, uint32_t parity, WsHeader *hdr, int where)
{
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    return dec_wait_slow(bar, parity, hdr, where);
}

// 1 - exp(2l) for -1/8 < l <= 0 by its Taylor series -2l (1 + l + 2/3 l^2 + 1/3 l^3),
// cut after l^3 (the first term left out, 2/15 l^4, is under 3.3e-5 relative).
__device__ __forceinline__ float one_minus_exp2l(float l)
{
    float s = fmaf(l, 1.f / 3.f, 2.f / 3.f);
    s = fmaf(l, s, 1.f);
    s = fmaf(l, s, 1.f);
    return (-2.f * l) * s;
}

__device__ __forceinline__ float gelu_tanh(float g)
{
    const float k0 = 0.7978845608028654f, k1 = 0.7978845608028654f * 0.044715f;
    const float u = g * fmaf(k1 * g, g, k0);
    const float hg = 0.5f * g;
    return fmaf(hg, tanh_approx(u), hg);
}


__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
rglru_decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tm_wa,
                    const __grid_constant__ CUtensorMap tm_wx, const __grid_constant__ CUtensorMap tm_x,
                    const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_cs)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t half = cluster_ctarank();
    const int cluster = blockIdx.x >> 1;
    const int head = cluster / p.nblk, blk = cluster % p.nblk;
    const int b0 = blk * kTok;
    const int nb = min(kTok, p.B - b0);                // valid rows of this block
    const int ch0 = head * 256 + (int)half * kHalfCh;  // first channel of this CTA
    uint64_t *bar_in = reinterpret_cast<uint64_t *>(smem + OFF_BAR), *bar_w = bar_in + 1, *bar_mma = bar_in + 2;
    uint64_t *bar_bx = bar_in + 3;  // the peer's half of the B tile has landed (bulk copy)
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    int32_t *sp_s = reinterpret_cast<int32_t *>(smem + OFF_SP);
    const __nv_bfloat16 *x_s = reinterpret_cast<const __nv_bfloat16 *>(smem + OFF_X);  // [kTok][128]
    __nv_bfloat16 *cs_s = reinterpret_cast<__nv_bfloat16 *>(smem + OFF_CS);            // [kTok][3][128]

    // thread = channel c of this half (TMEM lane c) and rows [n0, n0 + kRows)
    const int c = (warp & 3) * 32 + lane;
    const int d = ch0 + c;
    const int n0 = (warp >> 2) * kRows;

    if (tid == 0) DEC_TR(DT_START);
    // ---- 0. set-up that touches no global memory, which may overlap the tail
    // of the previous kernel on the stream (programmatic dependent launch)
    if (tid == 32) {
        mbar_init(bar_in, 1);
        mbar_init(bar_w, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_bx, 1);
        mbar_fence_init();
        // the peer's 128 channels of the B tile arrive as one bulk copy
        mbar_arrive_expect_tx(bar_bx, 2 * kBBlock);
        // this half's rows of W_a and W_x (parameters: read before the wait)
        mbar_arrive_expect_tx(bar_w, 2 * kWGate);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
            tma_load_2d(smem + OFF_W + kb * kWBlock, &tm_wa, bar_w, kb * 64, ch0);
            tma_load_2d(smem + OFF_W + kWGate + kb * kWBlock, &tm_wx, bar_w, kb * 64, ch0);
        }
    }
    if (warp == 0) tmem_alloc(tmem_holder, kTmemCols);
    const float w0 = 0.5f * p.conv_w[d], w1 = 0.5f * p.conv_w[(size_t)p.D + d],
                w2 = 0.5f * p.conv_w[2 * (size_t)p.D + d], w3 = 0.5f * p.conv_w[3 * (size_t)p.D + d];
    const float cb = 0.5f * p.conv_b[d];
    griddep_launch_dependents();
    griddep_wait();  // every global read below sees the previous kernel's writes
    if (tid == 0) DEC_TR(DT_WAITED);

    // ---- 1. loads
    if (tid == 32) {
        mbar_arrive_expect_tx(bar_in, kXTile + kCsTile);  // whole boxes: rows past B arrive zero-filled
        tma_load_2d(smem + OFF_X, &tm_x, bar_in, ch0, b0);
        tma_load_3d(smem + OFF_CS, &tm_cs, bar_in, ch0, 0, b0);
    }
    if (tid < kTok) sp_s[tid] = tid < nb ? p.segpos[b0 + tid] : 3;
    // (kept as loaded, one register each, so that nothing waits for them
    // before the epilogue uses them)
    float hprev[kRows];
    uint16_t graw[kRows];
#pragma unroll
    for (int k = 0; k < kRows; ++k) {
        const int n = n0 + k;
        const size_t e = (size_t)(b0 + n) * p.D + d;
        graw[k] = n < nb ? __bfloat16_as_ushort(p.g[e]) : (uint16_t)0;
        hprev[k] = n < nb ? p.h_state[e] : 0.f;
    }
    // the peer CTA must be running before its shared memory is written
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    // ---- 2. conv: xh = xc / 2 (halving is exact: the MMA then gives half
    // pre-activations for sigmoid(z) = (1 + tanh(z / 2)) / 2)
    bool ok = dec_wait(bar_in, 0, p.hdr, 0);
    if (tid == 0) DEC_TR(DT_INPUTS);
    float xh[kRows];
    {
        const int k = (int)half * kHalfCh + c;  // channel within the head = K index of the B tile
        const uint32_t b_local = smem_u32(smem + OFF_B + (k >> 6) * kBBlock);
        const int j = k & 63;
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
            const int n = n0 + i;
            const int sp = sp_s[n];
            __nv_bfloat16 *cr = cs_s + n * 3 * kHalfCh + c;
            const __nv_bfloat16 xr = x_s[n * kHalfCh + c], c1 = cr[kHalfCh], c2 = cr[2 * kHalfCh];
            // tap of lag k dropped when segment_pos < k (document start)
            float v = cb;
            if (sp >= 3) v = fmaf(w0, __bfloat162float(cr[0]), v);
            if (sp >= 2) v = fmaf(w1, __bfloat162float(c1), v);
            if (sp >= 1) v = fmaf(w2, __bfloat162float(c2), v);
            v = fmaf(w3, __bfloat162float(xr), v);
            xh[i] = v;
            // the window moves one step: rows (1, 2, x) become rows (0, 1, 2)
            cr[0] = c1;
            cr[kHalfCh] = c2;
            cr[2 * kHalfCh] = xr;
            const uint32_t off = n * 128 + (((j >> 3) ^ (n & 7)) << 4) + (j & 7) * 2;
            const uint16_t bv = __bfloat16_as_ushort(__float2bfloat16_rn(v));
            asm volatile("st.shared.b16 [%0], %1;" ::"r"(b_local + off), "h"(bv) : "memory");
        }
    }
    if (tid == 0) DEC_TR(DT_CONV);
    fence_proxy_async_smem();  // this half of the B tile and the conv_state tile, for the async proxy
    tc_fence_before();
    __syncthreads();           // this CTA's half of the B tile written
    tc_fence_after();
    // test hook (rglru_debug_suppress_publish): the CTA it names keeps its half,
    // so that its peer's bounded wait for it runs out
    const bool suppress = *(volatile int *)&p.hdr->debug_unit_plus1 == (int)blockIdx.x + 1;
    if (tid == 32 && !suppress) {
        // this half (K blocks 2 half, 2 half + 1: contiguous) into the peer's B tile
        uint8_t *src = smem + OFF_B + (int)half * 2 * kBBlock;
        bulk_copy_to_cluster(mapa_shared(smem_u32(src), half ^ 1u), src, 2 * kBBlock,
                             mapa_shared(smem_u32(bar_bx), half ^ 1u));
    }
    if (tid == 0) DEC_TR(DT_CLUSTER);

    // ---- 3. conv_state write-back and the gate projections
    if (warp == 1) {
        if (lane == 0) {
            tma_store_3d(&tm_cs, smem + OFF_CS, ch0, 0, b0);  // rows past B are clipped
            bulk_commit();
        }
        ok = dec_wait(bar_w, 0, p.hdr, 1) && ok;
        ok = dec_wait(bar_bx, 0, p.hdr, 3) && ok;  // the peer's half of the B tile
        if (lane == 0) DEC_TR(DT_WEIGHTS);
        if (ok && lane == 0) {
            tc_fence_after();
            const uint32_t idesc = umma_idesc_bf16(kHalfCh, kTok);
            const uint32_t wa = smem_u32(smem + OFF_W), wx = wa + kWGate, bt = smem_u32(smem + OFF_B);
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) {
                const uint32_t ko = (kk >> 2) * kWBlock + (kk & 3) * 32;
                const uint64_t bd = umma_desc_sw128(bt + (kk >> 2) * kBBlock + (kk & 3) * 32);
                umma_ss(tmem, umma_desc_sw128(wa + ko), bd, idesc, kk > 0);
                umma_ss(tmem + kTok, umma_desc_sw128(wx + ko), bd, idesc, kk > 0);
            }
            umma_commit(bar_mma);
            DEC_TR(DT_MMA);
        }
        __syncwarp();
    }

    // ---- 4. epilogue
    ok = dec_wait(bar_mma, 0, p.hdr, 2) && ok;
    {
        // the peer's copy into this CTA has landed (the MMA waited for it;
        // bounded here for the timeout path): tell the peer, whose exit waits
        // for it, and wait for the same news before this CTA exits
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(bar_bx, 0) && globaltimer() - t0 < kTimeoutNs) {
        }
        cluster_arrive();
    }
    if (tid == 0) DEC_TR(DT_EPI0);
    tc_fence_after();
    __nv_bfloat16 *y_s = reinterpret_cast<__nv_bfloat16 *>(smem + OFF_X);  // the x tile is dead
    if (ok) {
        const float hba = 0.5f * p.b_a[d], hbx = 0.5f * p.b_x[d];
        const float lam = p.lambda[d];
        const float ls = lam >= 0.f ? -log1pf(expf(-lam)) : lam - log1pf(expf(lam));  // log sigmoid(Lambda)
        const float hkl = 0.5f * kC * ls;               // log a = (1 + tr) * hkl, tr = tanh(half pre-activation)
        const float hkl2 = hkl * 1.4426950408889634f;  // the same in log2
        const uint32_t lane_col = tmem + ((uint32_t)((warp & 3) * 32) << 16) + n0;
#pragma unroll
        for (int k8 = 0; k8 < kRows; k8 += 8) {
            uint32_t ar[8], ai[8];
            tmem_ld8(lane_col + k8, ar);
            tmem_ld8(lane_col + kTok + k8, ai);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int i = k8 + k, n = n0 + i;
                const float tr = tanh_approx(__uint_as_float(ar[k]) + hba);
                const float tg = tanh_approx(__uint_as_float(ai[k]) + hbx);
                const float ell = fmaf(tr, hkl, hkl);
                const float a = ex2_approx(fmaf(tr, hkl2, hkl2));
                const float om = ell > -0.125f ? one_minus_exp2l(ell) : fmaf(-a, a, 1.f);
                const float uu = fmaf(tg, xh[i], xh[i]);  // i * xc
                const float h = sp_s[n] == 0 ? uu : fmaf(a, hprev[i], sqrt_approx(om) * uu);
                const float gv = __uint_as_float((uint32_t)graw[i] << 16);
                y_s[n * kHalfCh + c] = __float2bfloat16_rn(gelu_tanh(gv) * h);
                if (n < nb) p.h_state[(size_t)(b0 + n) * p.D + d] = h;
            }
        }
    }
    if (tid == 0) DEC_TR(DT_EPI1);
    fence_proxy_async_smem();  // y tile, for the async proxy
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 32) {
        if (ok) {
            tma_store_2d(&tm_y, smem + OFF_X, ch0, b0);  // rows past B are clipped
            bulk_commit();
        }
        bulk_wait_read_all();  // shared memory stays valid until the stores have read it
        DEC_TR(DT_END);
    }
    if (warp == 0) {
        if (!ok) {
            // a timed-out wait: give the MMAs in flight a bounded time to finish first
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(bar_mma, 0) && globaltimer() - t0 < kTimeoutNs) {
            }
        }
        tmem_dealloc(tmem, kTmemCols);
    }
    cluster_wait();  // this CTA's copy into the peer has landed before it exits
}

}  // namespace

#ifdef RGLRU_TRACE
size_t decode_workspace_bytes(int, int) { return kWsHeaderBytes + kTraceCtas * kTraceEvents * 8; }
#else
size_t decode_workspace_bytes(int, int) { return kWsHeaderBytes; }
#endif

rglru_status decode_step(const PrefillArgs &a)
{
    auto encode = encode_fn();
    if (!encode) return RGLRU_ERR_CUDA;
    CUtensorMap tm_wa, tm_wx, tm_x, tm_y, tm_cs;
    // gate matrices [D rows, 256]: 128-row x 64-channel boxes in the 128-byte
    // swizzle of the tensor core's K-major operand
    const cuuint64_t wdim[2] = {256, (cuuint64_t)a.D}, wstride[1] = {256 * 2};
    const cuuint32_t wbox[2] = {64, (cuuint32_t)kHalfCh};
    // [B, D] rows: 128 channels x kTok rows
    const cuuint64_t rdim[2] = {(cuuint64_t)a.D, (cuuint64_t)a.B}, rstride[1] = {(cuuint64_t)a.D * 2};
    const cuuint32_t rbox[2] = {(cuuint32_t)kHalfCh, (cuuint32_t)kTok};
    // conv_state [B, 3, D]: 128 channels x 3 rows x kTok sequences
    const cuuint64_t cdim[3] = {(cuuint64_t)a.D, 3, (cuuint64_t)a.B};
    const cuuint64_t cstride[2] = {(cuuint64_t)a.D * 2, (cuuint64_t)a.D * 6};
    const cuuint32_t cbox[3] = {(cuuint32_t)kHalfCh, 3, (cuuint32_t)kTok};
    if (!encode_bf16(encode, &tm_wa, a.W_a, 2, wdim, wstride, wbox, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_bf16(encode, &tm_wx, a.W_x, 2, wdim, wstride, wbox, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_bf16(encode, &tm_x, a.x, 2, rdim, rstride, rbox, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_bf16(encode, &tm_y, a.y, 2, rdim, rstride, rbox, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_bf16(encode, &tm_cs, a.conv_state, 3, cdim, cstride, cbox, CU_TENSOR_MAP_SWIZZLE_NONE))
        return RGLRU_ERR_CUDA;
    static PerDeviceFlag smem_set;
    const rglru_status st = set_smem_limit_once((const void *)rglru_decode_kernel, kSmemBytes, smem_set);
    if (st != RGLRU_OK) return st;

    DecodeParams p;
    p.B = a.B;
    p.D = a.D;
    p.nblk = (a.B + kTok - 1) / kTok;
    p.g = static_cast<const __nv_bfloat16 *>(a.g);
    p.conv_w = a.conv_w;
    p.conv_b = a.conv_b;
    p.b_a = a.b_a;
    p.b_x = a.b_x;
    p.lambda = a.lambda;
    p.segpos = a.segpos;
    p.h_state = a.h_state;
    p.hdr = reinterpret_cast<WsHeader *>(a.ws);
    const long long clusters = (long long)(a.D / kHead) * p.nblk;
    if (clusters * 2 > 0x7fffffffLL) return RGLRU_ERR_UNSUPPORTED;
    // programmatic stream serialization: the kernel may be scheduled while the
    // previous one on the stream finishes; it reads only the parameters (gate
    // weights, conv taps) before griddepcontrol.wait
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(clusters * 2));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, rglru_decode_kernel, p, tm_wa, tm_wx, tm_x, tm_y, tm_cs));
}

}  // namespace rglru
