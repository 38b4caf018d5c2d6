// decode.cu -- batched single-token step of the RG-LRU block core (bf16 I/O,
// fp32 state) on sm_100a.
//
// One step for B sequences.  Per sequence b and channel d the conv window is
// conv_state[b, 0..2, d] followed by x[b, d]; the gates are the block-diagonal
// projections of the conv output; h_state[b, d] advances one step and
// y[b, d] = GELU_tanh(g[b, d]) * h.  With one token per sequence the B rows of
// a head are the token dimension of its gate GEMM.
//
// Grid: one cluster of two CTAs per (head, block of kTok batch rows); CTA rank r
// owns channels [128 r, 128 r + 128) of the head:
//   1. every thread prefetches the h_state and GELU-branch values its epilogue
//      needs (independent of everything else, so their latency overlaps the rest);
//   2. one thread TMA-loads this half's 128 rows of W_a and W_x (128-byte
//      swizzled, K-major: the tensor core's A operands);
//   3. all threads run the conv of this half's channels for the block's rows,
//      keep xc / 2 in fp32 for the epilogue, write its bf16 copy into the B
//      tile of both CTAs of the cluster (this half's two K-blocks), and shift
//      this half's conv_state rows; a cluster barrier completes both B tiles;
//   4. one thread issues the 2 x 16 MMAs D[128 out x kTok rows] = W * xc^T;
//   5. every warp reads its TMEM lane quarter for half of the rows and applies
//      the gates, a = sigmoid(Lambda)^(8 r), the normalised one-step update (a
//      reset when segment_pos == 0) and the GELU product.
// Each CTA reads and writes only its own channels of the states, so the two
// CTAs never race.  Waits on mbarriers are bounded (RGLRU_ERR_TIMEOUT in the
// workspace header); the cluster barrier is reached exactly once by every
// thread of both CTAs.
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

constexpr int kTok = 64;        // batch rows per cluster: the MMA N
constexpr int kHalfCh = 128;    // channels per CTA: the MMA M and TMEM lanes
constexpr int kThreads = 256;   // 8 warps
constexpr int kRowsPerWarp = kTok / 2;  // epilogue: warps w and w + 4 share a lane quarter

constexpr int kWBlock = kHalfCh * 128;          // 128 weight rows x 64 channels (bf16): 16 KB
constexpr int kWGate = 4 * kWBlock;             // one gate, K = 256: 64 KB
constexpr int kBBlock = kTok * 128;             // kTok rows x 64 channels (bf16): 8 KB
constexpr int OFF_W = 0;                        // W_a rows, then W_x rows
constexpr int OFF_B = OFF_W + 2 * kWGate;       // B tile: 4 K-blocks (all 256 channels of the head)
constexpr int OFF_XC = OFF_B + 4 * kBBlock;     // fp32 xc / 2 of this half: [kTok][128]
constexpr int OFF_SP = OFF_XC + kTok * kHalfCh * 4;  // segment_pos of the block's rows
constexpr int OFF_BAR = OFF_SP + kTok * 4;      // W loaded, MMA done
constexpr int OFF_MISC = OFF_BAR + 2 * 8;       // TMEM base address
constexpr int kSmemUsed = OFF_MISC + 16;
constexpr int kSmemBytes = kSmemUsed + 1024;    // slack for the 1024-byte alignment
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
constexpr uint32_t kTmemCols = 2 * kTok;        // D_r then D_i
constexpr uint64_t kTimeoutNs = 2000000000ull;

struct DecodeParams {
    int B, D, nblk;
    const __nv_bfloat16 *x, *g;
    const float *conv_w, *conv_b, *b_a, *b_x, *lambda;
    const int32_t *segpos;
    __nv_bfloat16 *conv_state;
    float *h_state;
    __nv_bfloat16 *y;
    WsHeader *hdr;
};

// Bounded wait on an mbarrier phase by every lane of a warp; false (and the
// status recorded) if it does not complete within kTimeoutNs.
__device__ __noinline__ bool dec_wait(uint64_t *bar, uint32_t parity, WsHeader *hdr, int where)
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
rglru_decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_wa,
                    const __grid_constant__ CUtensorMap tmap_wx)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t half = cluster_ctarank();
    const int cluster = blockIdx.x >> 1;
    const int head = cluster / p.nblk, blk = cluster % p.nblk;
    const int b0 = blk * kTok;
    const int nb = min(kTok, p.B - b0);  // valid rows of this block
    const int ch0 = head * 256 + (int)half * kHalfCh;  // first channel of this CTA
    uint64_t *bar_w = reinterpret_cast<uint64_t *>(smem + OFF_BAR), *bar_mma = bar_w + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    int32_t *sp_s = reinterpret_cast<int32_t *>(smem + OFF_SP);
    float *xcs = reinterpret_cast<float *>(smem + OFF_XC);

    // ---- 1. epilogue operands: lane quarter (warp & 3) = channels, rows [32 (warp >> 2), +32)
    const int c = (warp & 3) * 32 + lane;
    const int d = ch0 + c;
    const int n_base = (warp >> 2) * kRowsPerWarp;
    float hprev[kRowsPerWarp];
    uint32_t graw[kRowsPerWarp / 2];  // bf16 pairs of consecutive rows
#pragma unroll
    for (int k = 0; k < kRowsPerWarp; k += 2) {
        const int n = n_base + k;
        const size_t e0 = (size_t)(b0 + n) * p.D + d, e1 = e0 + p.D;
        const uint32_t g0 = n < nb ? (uint32_t)__bfloat16_as_ushort(p.g[e0]) : 0u;
        const uint32_t g1 = n + 1 < nb ? (uint32_t)__bfloat16_as_ushort(p.g[e1]) : 0u;
        graw[k / 2] = g0 | (g1 << 16);
        hprev[k] = n < nb ? p.h_state[e0] : 0.f;
        hprev[k + 1] = n + 1 < nb ? p.h_state[e1] : 0.f;
    }

    // ---- 2. TMEM, barriers, weights
    if (warp == 0) tmem_alloc(tmem_holder, kTmemCols);
    if (tid == 32) {
        mbar_init(bar_w, 1);
        mbar_init(bar_mma, 1);
        mbar_fence_init();
        mbar_arrive_expect_tx(bar_w, 2 * kWGate);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
            tma_load_2d(smem + OFF_W + kb * kWBlock, &tmap_wa, bar_w, kb * 64, ch0);
            tma_load_2d(smem + OFF_W + kWGate + kb * kWBlock, &tmap_wx, bar_w, kb * 64, ch0);
        }
    }

    // the peer CTA must be running before its shared memory is written
    tc_fence_before();
    cluster_sync();

    // ---- 3. conv of this half: lane = 4 channels, warp = 8 rows
    {
        const int cg = lane;                 // channels ch0 + 4 cg .. + 3
        const size_t dc = (size_t)ch0 + cg * 4;
        f2_t w2[4][2], cb2[2];
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int e = 0; e < 2; ++e)
                w2[k][e] = f2_make(0.5f * p.conv_w[(size_t)k * p.D + dc + 2 * e],
                                   0.5f * p.conv_w[(size_t)k * p.D + dc + 2 * e + 1]);
#pragma unroll
        for (int e = 0; e < 2; ++e) cb2[e] = f2_make(0.5f * p.conv_b[dc + 2 * e], 0.5f * p.conv_b[dc + 2 * e + 1]);
        // this half's channels are K-blocks 2 half + (cg >> 4) of the B tile
        const int kb = 2 * (int)half + (cg >> 4);
        const uint32_t b_local = smem_u32(smem + OFF_B + kb * kBBlock);
        const uint32_t b_peer = mapa_shared(b_local, half ^ 1u);
        const int chunk = (cg & 15) >> 1;
#pragma unroll 2
        for (int i = 0; i < kTok / 8; ++i) {
            const int n = warp * (kTok / 8) + i;
            const int b = b0 + n;
            f2_t acc[2] = {0ull, 0ull};
            if (n < nb) {
                const int sp = p.segpos[b];
                const uint2 xv = *reinterpret_cast<const uint2 *>(p.x + (size_t)b * p.D + dc);
                __nv_bfloat16 *cs = p.conv_state + (size_t)b * 3 * p.D + dc;
                const uint2 s0 = *reinterpret_cast<const uint2 *>(cs);
                const uint2 s1 = *reinterpret_cast<const uint2 *>(cs + p.D);
                const uint2 s2 = *reinterpret_cast<const uint2 *>(cs + 2 * (size_t)p.D);
                const uint32_t xw[2] = {xv.x, xv.y}, w0[2] = {s0.x, s0.y}, w1[2] = {s1.x, s1.y},
                               w2r[2] = {s2.x, s2.y};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    // tap of lag k dropped when segment_pos < k (document start)
                    f2_t v = cb2[e];
                    if (sp >= 3) v = f2_fma(w2[0][e], f2_from_bf16x2(w0[e]), v);
                    if (sp >= 2) v = f2_fma(w2[1][e], f2_from_bf16x2(w1[e]), v);
                    if (sp >= 1) v = f2_fma(w2[2][e], f2_from_bf16x2(w2r[e]), v);
                    acc[e] = f2_fma(w2[3][e], f2_from_bf16x2(xw[e]), v);
                }
                // the window moves one step: rows (1, 2, x) become rows (0, 1, 2)
                *reinterpret_cast<uint2 *>(cs) = s1;
                *reinterpret_cast<uint2 *>(cs + p.D) = s2;
                *reinterpret_cast<uint2 *>(cs + 2 * (size_t)p.D) = xv;
                if (cg == 0) sp_s[n] = sp;
            }
            *reinterpret_cast<float4 *>(xcs + n * kHalfCh + cg * 4) =
                make_float4(f2_lo(acc[0]), f2_hi(acc[0]), f2_lo(acc[1]), f2_hi(acc[1]));
            const uint32_t off = n * 128 + ((chunk ^ (n & 7)) << 4) + (cg & 1) * 8;
            const uint32_t lo = f2_to_bf16x2(acc[0]), hi = f2_to_bf16x2(acc[1]);
            asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(b_local + off), "r"(lo), "r"(hi) : "memory");
            st_cluster_v2(b_peer + off, lo, hi);
        }
    }
    fence_proxy_async_cluster();
    cluster_sync();  // both halves of both B tiles written
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    // ---- 4. gate projections
    bool ok = true;
    if (warp == 1) {
        ok = dec_wait(bar_w, 0, p.hdr, 0);
        if (ok && lane == 0) {
            fence_proxy_async_smem();
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
        }
        __syncwarp();
    }

    // ---- 5. epilogue: thread = channel d (its TMEM lane), rows n_base .. n_base + 31
    ok = dec_wait(bar_mma, 0, p.hdr, 1) && ok;
    tc_fence_after();
    if (ok) {
        const float hba = 0.5f * p.b_a[d], hbx = 0.5f * p.b_x[d];
        const float lam = p.lambda[d];
        const float ls = lam >= 0.f ? -log1pf(expf(-lam)) : lam - log1pf(expf(lam));  // log sigmoid(Lambda)
        const float hkl = 0.5f * kC * ls;               // log a = (1 + tr) * hkl, tr = tanh(half pre-activation)
        const float hkl2 = hkl * 1.4426950408889634f;  // the same in log2
        const uint32_t lane_col = tmem + ((uint32_t)((warp & 3) * 32) << 16) + n_base;
#pragma unroll
        for (int k8 = 0; k8 < kRowsPerWarp; k8 += 8) {
            uint32_t ar[8], ai[8];
            tmem_ld8(lane_col + k8, ar);
            tmem_ld8(lane_col + kTok + k8, ai);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int n = n_base + k8 + k;
                if (n < nb) {
                    const float xh = xcs[n * kHalfCh + c];
                    const float tr = tanh_approx(__uint_as_float(ar[k]) + hba);
                    const float tg = tanh_approx(__uint_as_float(ai[k]) + hbx);
                    const float ell = fmaf(tr, hkl, hkl);
                    const float a = ex2_approx(fmaf(tr, hkl2, hkl2));
                    const float om = ell > -0.125f ? one_minus_exp2l(ell) : fmaf(-a, a, 1.f);
                    const float uu = fmaf(tg, xh, xh);  // i * xc
                    const float h = sp_s[n] == 0 ? uu : fmaf(a, hprev[k8 + k], sqrt_approx(om) * uu);
                    const uint32_t gw = graw[(k8 + k) / 2];
                    const float gv = __uint_as_float(((k8 + k) & 1) ? (gw & 0xffff0000u) : (gw << 16));
                    const size_t e = (size_t)(b0 + n) * p.D + d;
                    p.y[e] = __float2bfloat16_rn(gelu_tanh(gv) * h);
                    p.h_state[e] = h;
                }
            }
        }
    }

    // ---- teardown: TMEM reads done (or abandoned after a timeout) before the free
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
        if (!ok) {
            // a timed-out wait: give the MMAs in flight a bounded time to finish first
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(bar_mma, 0) && globaltimer() - t0 < kTimeoutNs) {
            }
        }
        tmem_dealloc(tmem, kTmemCols);
    }
}

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

// [H * 256 rows, 256 channels] bf16 gate matrix, loaded as 128-row x 64-channel
// boxes in the 128-byte swizzle the tensor core's K-major operand expects
bool encode_weights(CUtensorMap *m, const void *W, int D)
{
    auto encode = encode_fn();
    if (!encode) return false;
    const cuuint64_t gdim[2] = {256, (cuuint64_t)D};
    const cuuint64_t gstride[1] = {256 * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kHalfCh};
    const cuuint32_t estride[2] = {1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(W), gdim, gstride, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t decode_workspace_bytes(int, int) { return kWsHeaderBytes; }

rglru_status decode_step(const PrefillArgs &a)
{
    CUtensorMap tmap_wa, tmap_wx;
    if (!encode_weights(&tmap_wa, a.W_a, a.D) || !encode_weights(&tmap_wx, a.W_x, a.D)) return RGLRU_ERR_CUDA;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(rglru_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    });
    if (attr_err != cudaSuccess) return RGLRU_ERR_CUDA;

    DecodeParams p;
    p.B = a.B;
    p.D = a.D;
    p.nblk = (a.B + kTok - 1) / kTok;
    p.x = static_cast<const __nv_bfloat16 *>(a.x);
    p.g = static_cast<const __nv_bfloat16 *>(a.g);
    p.conv_w = a.conv_w;
    p.conv_b = a.conv_b;
    p.b_a = a.b_a;
    p.b_x = a.b_x;
    p.lambda = a.lambda;
    p.segpos = a.segpos;
    p.conv_state = static_cast<__nv_bfloat16 *>(a.conv_state);
    p.h_state = a.h_state;
    p.y = static_cast<__nv_bfloat16 *>(a.y);
    p.hdr = reinterpret_cast<WsHeader *>(a.ws);
    const long long clusters = (long long)(a.D / kHead) * p.nblk;
    if (clusters * 2 > 0x7fffffffLL) return RGLRU_ERR_UNSUPPORTED;
    rglru_decode_kernel<<<(unsigned)(clusters * 2), kThreads, kSmemBytes, a.stream>>>(p, tmap_wa, tmap_wx);
    return cuda_status(cudaGetLastError());
}

}  // namespace rglru
