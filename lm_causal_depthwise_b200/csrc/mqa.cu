// mqa.cu -- the local sliding-window MQA temporal block on sm_100a: RoPE, the
// attention itself on the tensor cores, and the block (projections around it).
//
// What it computes: "Gemma explained: RecurrentGemma architecture", the
// RecurrentGemmaSdpaAttention printout (q_proj Linear(2560, 2560, bias=False),
// k_proj and v_proj Linear(2560, 256, bias=False), o_proj Linear(2560, 2560,
// bias=True), rotary_emb) and sections "Residual block with local MQA" (10
// query heads of 256 share one key/value head; each position attends only a
// fixed number of past tokens) and "Local attention window size" (2k tokens).
// The readings where the pages are silent: rotate-half RoPE over the full head
// (pairs i and i + 128, frequency 10000^(-2i/256), position = segment_pos),
// scores scaled by 1/16 = 1/sqrt(256), query t attends keys s with
// t - window < s <= t inside its document and inside the call.
//
// Layouts (bf16, row-major):
//   qkv  [B, T, (H + 2) * 256]: q heads 0..H-1, then k, then v (one projection
//        launch of the concatenated weights writes it);
//   v_t  [B, 256, Tp], Tp = T rounded up to 8: v transposed, token fastest,
//        so that it is a K-major operand of the second GEMM;
//   out  [B, T, H * 256].
//
// rglru_mqa_rope_kernel (memory bound): RoPE on q and k in place and v_t.
// Angles are pos * 10000^(-i/128) reduced modulo 2 pi in fp64 (exact to far
// beyond any position), then sine and cosine in fp32.
//
// rglru_mqa_attention_kernel: one CTA per (head, 128-query tile, sequence),
// 192 threads:
//   warp 4     TMA producer: lane 0 the K tiles (4 boxes [64 keys x 64
//              channels], 128-byte swizzle), lane 1 the V^T tiles ([256 x 64
//              keys]), each into a 3-deep ring;
//   warp 5     MMA issuer (the converged warp, one lane elected per MMA):
//              S = Q K^T (M=128, N=64, 16 K-steps) with Q read from TMEM,
//              then O += P V (M=128, N=256, 4 K-steps) with P read from TMEM;
//              S of tile j + 1 is issued as soon as the softmax has read S of
//              tile j, so it runs under the softmax of tile j;
//   warps 0-3  softmax: thread = query row = TMEM lane.  Each first writes its
//              row of the Q tile into TMEM (the A operand of S).  Scores in
//              log2 units, the window / document / causal limits applied only
//              on tiles that cross them; the running max used for the
//              exponentials is raised only when a row's max grows by more
//              than 8 (a factor 256), and only then is O (in TMEM) rescaled,
//              after the MMAs that wrote it have completed.  P goes to TMEM as
//              bf16 pairs; at the end O / l is written as bf16.
// TMEM: O 256 columns, Q 128, S 64, P 2 x 32 (all 512, one CTA per SM).
// Every mbarrier wait is bounded (2 s): one that runs out records
// RGLRU_ERR_TIMEOUT in the workspace header and the CTA unwinds.  A wait whose
// phase is already complete costs one inline test.
#include <climits>
#include <cmath>

#include "internal.h"
#include "sm100.cuh"

namespace rglru {
namespace {

using namespace sm100;

constexpr int kHd = 256;             // head dimension
constexpr int kQT = 128;             // query rows per CTA
constexpr int kKT = 64;              // keys per tile
constexpr int kThreads = 192;
constexpr int kKBox = kKT * 64 * 2;  // 8 KB: [64 keys x 64 channels]
constexpr int kKBytes = 4 * kKBox;   // 32 KB
constexpr int kVBytes = kHd * kKT * 2;  // 32 KB: [256 channels x 64 keys]
constexpr int kStages = 3;
constexpr int OFF_K = 0, OFF_V = OFF_K + kStages * kKBytes;
constexpr int OFF_BAR = OFF_V + kStages * kVBytes;
enum {
    B_QFULL = 0,                  // the Q tile is in TMEM (128 arrivals)
    B_KFULL = 1,
    B_KFREE = B_KFULL + kStages,
    B_VFULL = B_KFREE + kStages,
    B_VFREE = B_VFULL + kStages,
    B_SFULL = B_VFREE + kStages,  // scores of tile j complete
    B_SFREE = B_SFULL + 1,        // ... read by the softmax warps (128 arrivals)
    B_PFULL = B_SFREE + 1,        // P of tile j in buffer j % 2 (128 arrivals)
    B_PVDONE = B_PFULL + 2,       // O += P V of tile j complete (P buffer free, O settled)
    B_DRAIN = B_PVDONE + 2,
    B_N = B_DRAIN + 1
};
constexpr int OFF_MISC = OFF_BAR + B_N * 8;
constexpr int kSmemBytes = OFF_MISC + 16 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
// TMEM columns: O (fp32) 256, the Q tile (bf16 pairs, the A operand of S) 128,
// S (fp32) 64, P (bf16 pairs, the A operand of O) 2 x 32
constexpr uint32_t kColO = 0, kColQ = 256, kColS = 384, kColP = 448;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kRescaleLog2 = 8.f;  // raise the reference max when the row max exceeds it by 2^8

struct AttnParams {
    int B, T, H, window, ntiles;
    const __nv_bfloat16 *qkv;
    const int32_t *segpos;
    __nv_bfloat16 *out;
    WsHeader *hdr;
};

__device__ __noinline__ bool attn_wait_slow(uint64_t *bar, uint32_t parity, WsHeader *hdr, int where)
{
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if ((it & 15u) == 0) {
            if (*(volatile int *)&hdr->status != 0) return false;
            if (globaltimer() - t0 > kTimeoutNs) {
                atomicCAS(&hdr->status, 0, (int)RGLRU_ERR_TIMEOUT);
                atomicCAS(&hdr->detail, 0, (int)(blockIdx.x << 8) | (where + 1));
                return false;
            }
        }
    }
}

// a phase that is already complete costs one inline test; only a wait that
// has to poll calls out
__device__ __forceinline__ bool attn_wait(uint64_t *bar, uint32_t parity, WsHeader *hdr, int where)
{
    if (mbar_try_wait(bar, parity)) return true;
    return attn_wait_slow(bar, parity, hdr, where);
}

// every lane of the warp waits; the warp's verdict is unanimous
__device__ __forceinline__ bool attn_warp_wait(uint64_t *bar, uint32_t parity, WsHeader *hdr, int where)
{
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = attn_wait(bar, parity, hdr, where);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (ok) {
        while (!mbar_try_wait(bar, parity)) {
        }
    }
    return ok;
}

// bounded wait used only while unwinding (no status is recorded)
__device__ void drain_wait(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity) && globaltimer() - t0 < kTimeoutNs) {
    }
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// first key query t may attend: its document start, the window, the call's first token
__device__ __forceinline__ int row_lo(const AttnParams &p, int b, int t)
{
    const int lo = max(max(t - p.segpos[(size_t)b * p.T + t], t - p.window + 1), 0);
    return min(lo, t);
}

__global__ void __launch_bounds__(kThreads, 1)
rglru_mqa_attention_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_MISC);

    // CTA -> (head, query tile, sequence): the heads of one tile run side by
    // side (they read the same K and V), the tiles with the most keys first
    const int h = blockIdx.x % p.H;
    const int y = blockIdx.x / p.H;
    const int b = y % p.B;
    const int t0 = (p.ntiles - 1 - y / p.B) * kQT;
    const int t_last = min(t0 + kQT, p.T) - 1;
    // key tiles j0 .. j0 + n - 1 cover every key of every row of the tile
    int lo_min = INT_MAX;
    for (int r = lane; r < kQT; r += 32)
        if (t0 + r < p.T) lo_min = min(lo_min, row_lo(p, b, t0 + r));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lo_min = min(lo_min, __shfl_xor_sync(0xffffffffu, lo_min, o));
    const int j0 = lo_min / kKT;
    const int n = t_last / kKT - j0 + 1;

    if (warp == 5) {
        tmem_alloc(tmem_holder, 512);
        if (lane == 0) {
            mbar_init(bars + B_QFULL, 4 * 32);
            for (int s = 0; s < kStages; ++s) {
                mbar_init(bars + B_KFULL + s, 1);
                mbar_init(bars + B_KFREE + s, 1);
                mbar_init(bars + B_VFULL + s, 1);
                mbar_init(bars + B_VFREE + s, 1);
            }
            mbar_init(bars + B_SFULL, 1);
            mbar_init(bars + B_SFREE, 4 * 32);
            for (int s = 0; s < 2; ++s) {
                mbar_init(bars + B_PFULL + s, 4 * 32);
                mbar_init(bars + B_PVDONE + s, 1);
            }
            mbar_init(bars + B_DRAIN, 1);
            mbar_fence_init();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        // lane 0 loads the K tiles, lane 1 the V tiles: a wait for a V slot
        // never holds back the next K load
        if (lane < 2) {
            const bool is_k = lane == 0;
            const int full = is_k ? B_KFULL : B_VFULL, freeb = is_k ? B_KFREE : B_VFREE;
            bool ok = true;
            int issued = 0;
            for (int j = 0; j < n && ok; ++j) {
                const int s = j % kStages, s0 = (j0 + j) * kKT;
                if (j >= kStages &&
                    !(ok = attn_wait(bars + freeb + s, (uint32_t)((j / kStages) - 1) & 1u, p.hdr, is_k ? 0 : 1)))
                    break;
                if (is_k) {
                    mbar_arrive_expect_tx(bars + full + s, kKBytes);
                    for (int kb = 0; kb < 4; ++kb)
                        tma_load_3d(smem + OFF_K + s * kKBytes + kb * kKBox, &tm_k, bars + full + s,
                                    p.H * kHd + kb * 64, s0, b);
                } else {
                    mbar_arrive_expect_tx(bars + full + s, kVBytes);
                    tma_load_3d(smem + OFF_V + s * kVBytes, &tm_v, bars + full + s, s0, 0, b);
                }
                ++issued;
            }
            if (!ok) {
                // the loads already issued land before the CTA exits
                for (int k = max(0, issued - kStages); k < issued; ++k)
                    drain_wait(bars + full + k % kStages, (uint32_t)(k / kStages) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        // the whole (converged) warp runs the loop, so descriptors and TMEM
        // addresses stay warp-uniform; elect.sync picks the lane that issues
        const uint32_t idesc_s = umma_idesc_bf16(kQT, kKT), idesc_o = umma_idesc_bf16(kQT, kHd);
        bool ok = attn_warp_wait(bars + B_QFULL, 0, p.hdr, 2);
        for (int j = 0; ok && j <= n; ++j) {
            if (j < n) {
                const int s = j % kStages;
                if (!(ok = attn_warp_wait(bars + B_KFULL + s, (uint32_t)(j / kStages) & 1u, p.hdr, 3))) break;
                // the single score buffer: tile j - 1 has been read
                if (j >= 1 && !(ok = attn_warp_wait(bars + B_SFREE, (uint32_t)(j - 1) & 1u, p.hdr, 4))) break;
                tc_fence_after();
                const uint64_t kd0 = umma_desc_sw128(smem_u32(smem + OFF_K + s * kKBytes));
#pragma unroll
                for (int kk = 0; kk < kHd / 16; ++kk) {
                    // A: 16 channels of Q from TMEM (8 columns); B: 64-channel box kk / 4,
                    // 16-channel step kk % 4 (32 bytes into each swizzled row; the
                    // descriptor's start field counts 16-byte units)
                    const uint32_t off = (uint32_t)(kk >> 2) * kKBox + (uint32_t)(kk & 3) * 32;
                    umma_ts_warp(tmem + kColS, tmem + kColQ + (uint32_t)kk * 8, kd0 + (off >> 4), idesc_s, kk > 0);
                }
                umma_commit_warp(bars + B_SFULL);
                umma_commit_warp(bars + B_KFREE + s);
            }
            if (j >= 1) {
                const int i = j - 1, pb = i % 2, s = i % kStages;
                if (!(ok = attn_warp_wait(bars + B_PFULL + pb, (uint32_t)(i / 2) & 1u, p.hdr, 5))) break;
                if (!(ok = attn_warp_wait(bars + B_VFULL + s, (uint32_t)(i / kStages) & 1u, p.hdr, 6))) break;
                tc_fence_after();
                const uint64_t vd0 = umma_desc_sw128(smem_u32(smem + OFF_V + s * kVBytes));
#pragma unroll
                for (int kk = 0; kk < kKT / 16; ++kk)
                    umma_ts_warp(tmem + kColO, tmem + kColP + (uint32_t)(pb * 32 + kk * 8), vd0 + (uint64_t)(kk * 2),
                                 idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
                umma_commit_warp(bars + B_PVDONE + pb);
                umma_commit_warp(bars + B_VFREE + s);
            }
            __syncwarp();
        }
        if (!ok) {
            // the MMAs in flight finish before TMEM is freed
            umma_commit_warp(bars + B_DRAIN);
            if (lane == 0) drain_wait(bars + B_DRAIN, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax warps
        const int row = warp * 32 + lane;
        const int t = t0 + row;
        const bool live = t < p.T;
        const int lo = live ? row_lo(p, b, t) : INT_MAX;
        const int hi = live ? t : -1;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        {
            // this row of the Q tile into its TMEM lane: 256 bf16 = 128 columns
            const uint4 *src = reinterpret_cast<const uint4 *>(
                p.qkv + ((size_t)b * p.T + (live ? t : 0)) * (size_t)((p.H + 2) * kHd) + (size_t)h * kHd);
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                uint32_t r[32];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint4 v = live ? __ldg(src + q * 8 + k) : make_uint4(0, 0, 0, 0);
                    r[4 * k] = v.x;
                    r[4 * k + 1] = v.y;
                    r[4 * k + 2] = v.z;
                    r[4 * k + 3] = v.w;
                }
                tmem_st32(tmem + lane_off + kColQ + (uint32_t)(q * 32), r);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bars + B_QFULL);
        }
        const float kScale = 1.4426950408889634f / 16.f;  // log2(e) / sqrt(256)
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
#pragma unroll 1
        for (int j = 0; j < n; ++j) {
            const int pb = j % 2, s0 = (j0 + j) * kKT;
            if (!(ok = attn_warp_wait(bars + B_SFULL, (uint32_t)j & 1u, p.hdr, 7))) break;
            tc_fence_after();
            uint32_t ra[32], rb[32];
            tmem_ld32(tmem + lane_off + kColS, ra);
            tmem_ld32(tmem + lane_off + kColS + 32, rb);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(bars + B_SFREE);
            float v[64];  // raw scores; the scale is folded into the exponent below
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                v[e] = __uint_as_float(ra[e]);
                v[e + 32] = __uint_as_float(rb[e]);
            }
            const bool inside = s0 >= lo && s0 + kKT - 1 <= hi;
            if (!__all_sync(0xffffffffu, inside)) {
#pragma unroll
                for (int e = 0; e < 64; ++e)
                    if (s0 + e < lo || s0 + e > hi) v[e] = -INFINITY;
            }
            float m8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) m8[e] = v[e];
#pragma unroll
            for (int e = 8; e < 64; ++e) m8[e & 7] = fmaxf(m8[e & 7], v[e]);
            const float mt = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * kScale;
            const float m_new = fmaxf(m_ref, mt);
            const bool grow = m_new > m_ref + kRescaleLog2;  // false while the row has no key yet
            const bool rescale = grow && m_ref != -INFINITY;
            float f = 1.f;
            if (rescale) {
                f = ex2_approx(m_ref - m_new);
                l *= f;
            }
            if (grow) m_ref = m_new;
            if (__any_sync(0xffffffffu, rescale)) {
                // O holds tiles 0 .. j-1: wait for the last of them, then scale in place
                if (!(ok = attn_warp_wait(bars + B_PVDONE + (j - 1) % 2, (uint32_t)((j - 1) / 2) & 1u, p.hdr, 8)))
                    break;
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < kHd; c += 32) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_off + kColO + (uint32_t)c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
                    tmem_st32(tmem + lane_off + kColO + (uint32_t)c, o);
                }
                tmem_wait_st();
            }
            const float mu = m_ref == -INFINITY ? 0.f : m_ref;
            uint32_t pk[32];
            float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float p0 = ex2_approx(fmaf(v[2 * e], kScale, -mu));
                const float p1 = ex2_approx(fmaf(v[2 * e + 1], kScale, -mu));
                l4[e & 3] += p0 + p1;
                pk[e] = pack_bf16(p0, p1);
            }
            l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
            // P buffer pb was last read by the MMAs of tile j - 2
            if (j >= 2 && !(ok = attn_warp_wait(bars + B_PVDONE + pb, (uint32_t)((j / 2) - 1) & 1u, p.hdr, 9)))
                break;
            tc_fence_after();
            tmem_st32(tmem + lane_off + kColP + (uint32_t)(pb * 32), pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bars + B_PFULL + pb);
        }
        if (ok && n > 0 && attn_warp_wait(bars + B_PVDONE + (n - 1) % 2, (uint32_t)((n - 1) / 2) & 1u, p.hdr, 10)) {
            tc_fence_after();
            const float inv = live ? 1.f / l : 0.f;
            __nv_bfloat16 *orow = p.out + ((size_t)b * p.T + (live ? t : 0)) * (size_t)(p.H * kHd) + (size_t)h * kHd;
#pragma unroll 1
            for (int c = 0; c < kHd; c += 32) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_off + kColO + (uint32_t)c, o);
                tmem_wait_ld();
                if (live) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_uint4(pack_bf16(__uint_as_float(o[8 * q]) * inv, __uint_as_float(o[8 * q + 1]) * inv),
                                            pack_bf16(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv),
                                            pack_bf16(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv),
                                            pack_bf16(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- RoPE and v_t
constexpr int kRopeTok = 32;  // tokens per CTA
constexpr int kRopeThreads = 256;

__global__ void __launch_bounds__(kRopeThreads)
rglru_mqa_rope_kernel(int T, int H, int Tp, __nv_bfloat16 *__restrict__ qkv, const int32_t *__restrict__ segpos,
                      __nv_bfloat16 *__restrict__ vt)
{
    __shared__ double inv_freq[kHd / 2];
    __shared__ float2 cs[kRopeTok][kHd / 2];  // (cos, sin) per token and pair
    const int b = blockIdx.y, tb = blockIdx.x * kRopeTok;
    const size_t W = (size_t)(H + 2) * kHd;
    if (threadIdx.x < kHd / 2) inv_freq[threadIdx.x] = exp2(-(double)threadIdx.x * (13.287712379549449 / 128.0));
    __syncthreads();
    for (int e = threadIdx.x; e < kRopeTok * (kHd / 2); e += kRopeThreads) {
        const int tt = e / (kHd / 2), i = e % (kHd / 2), t = tb + tt;
        float c = 1.f, s = 0.f;
        if (t < T) {
            // turns of the angle, reduced to [0, 1) in fp64
            double turns = (double)segpos[(size_t)b * T + t] * inv_freq[i] * 0.15915494309189535;
            turns -= floor(turns);
            sincospif((float)(2.0 * turns), &s, &c);
        }
        cs[tt][i] = make_float2(c, s);
    }
    __syncthreads();
    // q heads and k: thread = (token, pair), pairs (x[i], x[i + 128]) of every head
    for (int e = threadIdx.x; e < kRopeTok * (kHd / 2); e += kRopeThreads) {
        const int tt = e / (kHd / 2), i = e % (kHd / 2), t = tb + tt;
        if (t >= T) continue;
        const float2 r = cs[tt][i];
        __nv_bfloat16 *row = qkv + ((size_t)b * T + t) * W + i;
#pragma unroll 1
        for (int hh = 0; hh <= H; ++hh) {
            const float x1 = __bfloat162float(row[hh * kHd]), x2 = __bfloat162float(row[hh * kHd + kHd / 2]);
            row[hh * kHd] = __float2bfloat16_rn(x1 * r.x - x2 * r.y);
            row[hh * kHd + kHd / 2] = __float2bfloat16_rn(x2 * r.x + x1 * r.y);
        }
    }
    // v transposed: thread = channel, 8 tokens per 16-byte store
    const int d = threadIdx.x;
    const __nv_bfloat16 *vcol = qkv + (size_t)(H + 1) * kHd + d;
#pragma unroll 1
    for (int g = 0; g < kRopeTok; g += 8) {
        const int tg = tb + g;
        if (tg >= T) break;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int ta = tg + 2 * q, tb2 = ta + 1;
            const uint32_t lo = ta < T ? __bfloat16_as_ushort(vcol[((size_t)b * T + ta) * W]) : 0u;
            const uint32_t hi = tb2 < T ? __bfloat16_as_ushort(vcol[((size_t)b * T + tb2) * W]) : 0u;
            w[q] = lo | (hi << 16);
        }
        *reinterpret_cast<uint4 *>(vt + ((size_t)b * kHd + d) * Tp + tg) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}
static_assert(kRopeThreads == kHd, "one thread per v channel");

// ---------------------------------------------------------------- decode step
// One token per sequence at document position pos attends the cached keys of
// positions max(0, pos - window + 1) .. pos; the cache keeps position q at
// slot q % window.  HBM bound (1 KB of K and V per key and sequence), so it
// runs on the CUDA cores: a split over 256-key chunks, one CTA per (chunk,
// sequence), then a combine kernel.  Every CTA of a sequence rotates q and k
// itself; the CTA whose chunk holds pos first writes this token's rotated k
// and its v into the cache slot, and only it reads that slot.
constexpr int kDecKeys = 256;   // keys per CTA
constexpr int kDecThreads = 256;
constexpr int kDecMaxH = 16;

struct DecParams {
    int B, H, window, nch;
    const __nv_bfloat16 *qkv;   // [B, (H + 2) * 256]
    const int32_t *segpos;      // [B]
    __nv_bfloat16 *kc, *vc;     // [B, window, 256]
    float *part_o;              // [B, nch, H, 256]
    float *part_ml;             // [B, nch, H, 2]: chunk max (log2 units) and sum
    __nv_bfloat16 *out;         // [B, H * 256]
};

__device__ __forceinline__ f2_t bf16x2_to_f2(uint32_t w)
{
    return f2_make(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__global__ void __launch_bounds__(kDecThreads)
rglru_mqa_decode_kernel(const DecParams p)
{
    __shared__ __align__(16) float qs[kDecMaxH][kHd];       // rotated q (bf16 values) in fp32
    __shared__ __align__(16) float ps[kDecMaxH][kDecKeys];  // probabilities; later the second half's O
    __shared__ float red[kDecThreads / 32][kDecMaxH];
    __shared__ float mch[kDecMaxH], lch[kDecMaxH];
    __shared__ float2 cs[kHd / 2];
    const int b = blockIdx.y, c = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = p.H, W = p.window;
    const int pos = max(p.segpos[b], 0);
    const int n = min(pos + 1, W);
    const int i0 = c * kDecKeys;
    if (i0 >= n) return;  // the whole CTA
    const int lo = pos - n + 1;
    const size_t C = (size_t)(H + 2) * kHd;
    const __nv_bfloat16 *row = p.qkv + (size_t)b * C;
    if (tid < kHd / 2) {
        const double inv = exp2(-(double)tid * (13.287712379549449 / 128.0));
        double turns = (double)pos * inv * 0.15915494309189535;
        turns -= floor(turns);
        float sn, co;
        sincospif((float)(2.0 * turns), &sn, &co);
        cs[tid] = make_float2(co, sn);
    }
    __syncthreads();
    const bool owner = c == (n - 1) / kDecKeys;  // this CTA's chunk holds position pos
    __nv_bfloat16 *kslot = p.kc + ((size_t)b * W + pos % W) * kHd;
    for (int e = tid; e < (H + 1) * (kHd / 2); e += kDecThreads) {
        const int hh = e / (kHd / 2), i = e % (kHd / 2);
        const float x1 = __bfloat162float(row[hh * kHd + i]), x2 = __bfloat162float(row[hh * kHd + i + kHd / 2]);
        const float2 r = cs[i];
        const __nv_bfloat16 y1 = __float2bfloat16_rn(x1 * r.x - x2 * r.y);
        const __nv_bfloat16 y2 = __float2bfloat16_rn(x2 * r.x + x1 * r.y);
        if (hh < H) {
            qs[hh][i] = __bfloat162float(y1);
            qs[hh][i + kHd / 2] = __bfloat162float(y2);
        } else if (owner) {
            kslot[i] = y1;
            kslot[i + kHd / 2] = y2;
        }
    }
    if (owner) p.vc[((size_t)b * W + pos % W) * kHd + tid] = row[(H + 1) * kHd + tid];
    __syncthreads();  // the slot's k and v (global) and q (shared) are visible to the CTA

    // scores: thread = key
    const float kScale = 1.4426950408889634f / 16.f;
    const int key = i0 + tid;
    const bool have = key < n;
    float sc[kDecMaxH];
    {
        f2_t acc[kDecMaxH];
#pragma unroll
        for (int h = 0; h < kDecMaxH; ++h) acc[h] = 0ull;
        if (have) {
            const uint4 *kr = reinterpret_cast<const uint4 *>(p.kc + ((size_t)b * W + (lo + key) % W) * kHd);
#pragma unroll 2
            for (int c8 = 0; c8 < kHd / 8; ++c8) {
                const uint4 kv = kr[c8];
                const f2_t k01 = bf16x2_to_f2(kv.x), k23 = bf16x2_to_f2(kv.y);
                const f2_t k45 = bf16x2_to_f2(kv.z), k67 = bf16x2_to_f2(kv.w);
#pragma unroll
                for (int h = 0; h < kDecMaxH; ++h) {
                    if (h < H) {
                        const float4 qa = *reinterpret_cast<const float4 *>(&qs[h][c8 * 8]);
                        const float4 qb = *reinterpret_cast<const float4 *>(&qs[h][c8 * 8 + 4]);
                        acc[h] = f2_fma(k01, f2_make(qa.x, qa.y), acc[h]);
                        acc[h] = f2_fma(k23, f2_make(qa.z, qa.w), acc[h]);
                        acc[h] = f2_fma(k45, f2_make(qb.x, qb.y), acc[h]);
                        acc[h] = f2_fma(k67, f2_make(qb.z, qb.w), acc[h]);
                    }
                }
            }
        }
#pragma unroll
        for (int h = 0; h < kDecMaxH; ++h) sc[h] = have ? (f2_lo(acc[h]) + f2_hi(acc[h])) * kScale : -INFINITY;
    }
    // chunk max and sum per head
#pragma unroll
    for (int h = 0; h < kDecMaxH; ++h) {
        if (h < H) {
            float m = sc[h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) red[warp][h] = m;
        }
    }
    __syncthreads();
    if (tid < H) {
        float m = red[0][tid];
        for (int w = 1; w < kDecThreads / 32; ++w) m = fmaxf(m, red[w][tid]);
        mch[tid] = m;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < kDecMaxH; ++h) {
        if (h < H) {
            const float pr = have ? ex2_approx(sc[h] - mch[h]) : 0.f;
            ps[h][tid] = pr;
            float l = pr;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
            if (lane == 0) red[warp][h] = l;
        }
    }
    __syncthreads();
    if (tid < H) {
        float l = 0.f;
        for (int w = 0; w < kDecThreads / 32; ++w) l += red[w][tid];
        lch[tid] = l;
    }

    // O partial: thread = (channel pair dp, half of the chunk's keys)
    const int dp = tid % (kHd / 2), half = tid / (kHd / 2);
    const int kb = half * (kDecKeys / 2), ke = min(kb + kDecKeys / 2, n - i0);
    f2_t o[kDecMaxH];
#pragma unroll
    for (int h = 0; h < kDecMaxH; ++h) o[h] = 0ull;
    if (kb < ke) {
        int slot = (lo + i0 + kb) % W;
#pragma unroll 2
        for (int kk = kb; kk < ke; ++kk) {
            const uint32_t vv = *reinterpret_cast<const uint32_t *>(p.vc + ((size_t)b * W + slot) * kHd + 2 * dp);
            const f2_t v2 = bf16x2_to_f2(vv);
#pragma unroll
            for (int h = 0; h < kDecMaxH; ++h)
                if (h < H) o[h] = f2_fma(f2_splat(ps[h][kk]), v2, o[h]);
            slot = slot + 1 == W ? 0 : slot + 1;
        }
    }
    __syncthreads();  // every thread is done with ps: the second half's O goes there
    float2 *oh = reinterpret_cast<float2 *>(&ps[0][0]);  // [kDecMaxH][128] float2
    if (half == 1) {
#pragma unroll
        for (int h = 0; h < kDecMaxH; ++h)
            if (h < H) oh[h * (kHd / 2) + dp] = make_float2(f2_lo(o[h]), f2_hi(o[h]));
    }
    __syncthreads();
    if (half == 0) {
        const size_t base = ((size_t)b * p.nch + c) * H;
#pragma unroll
        for (int h = 0; h < kDecMaxH; ++h) {
            if (h < H) {
                const float2 q2 = oh[h * (kHd / 2) + dp];
                reinterpret_cast<float2 *>(p.part_o + (base + h) * kHd)[dp] =
                    make_float2(f2_lo(o[h]) + q2.x, f2_hi(o[h]) + q2.y);
            }
        }
    }
    if (tid < H) {
        const size_t base = ((size_t)b * p.nch + c) * H + tid;
        p.part_ml[2 * base] = mch[tid];
        p.part_ml[2 * base + 1] = lch[tid];
    }
}

// out[b, h] = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c over the chunks of sequence b
__global__ void __launch_bounds__(kHd)
rglru_mqa_decode_combine_kernel(const DecParams p)
{
    const int b = blockIdx.x, d = threadIdx.x, H = p.H;
    const int pos = max(p.segpos[b], 0);
    const int n = min(pos + 1, p.window);
    const int nc = (n + kDecKeys - 1) / kDecKeys;
    for (int h = 0; h < H; ++h) {
        float M = -INFINITY;
        for (int c = 0; c < nc; ++c) M = fmaxf(M, p.part_ml[2 * (((size_t)b * p.nch + c) * H + h)]);
        float num = 0.f, den = 0.f;
        for (int c = 0; c < nc; ++c) {
            const size_t base = ((size_t)b * p.nch + c) * H + h;
            const float f = ex2_approx(p.part_ml[2 * base] - M);
            num = fmaf(f, p.part_o[base * kHd + d], num);
            den = fmaf(f, p.part_ml[2 * base + 1], den);
        }
        p.out[(size_t)b * H * kHd + (size_t)h * kHd + d] = __float2bfloat16_rn(num / den);
    }
}

size_t dec_part_bytes(int B, int H, int window)
{
    const size_t nch = (size_t)((window + kDecKeys - 1) / kDecKeys);
    return align_up((size_t)B * nch * H * kHd * 4, 256) + align_up((size_t)B * nch * H * 2 * 4, 256);
}

bool al16(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
constexpr int64_t kMaxRows = int64_t(1) << 30;

bool mqa_sizes_ok(int B, int T, int H)
{
    return B >= 1 && T >= 1 && H >= 1 && H <= 64 && (int64_t)B * T <= kMaxRows &&
           (int64_t)B * ((T + kQT - 1) / kQT) * H <= 0x7fffffffLL && B <= 65535;
}

size_t vt_elems(int B, int T) { return (size_t)B * kHd * (size_t)((T + 7) / 8 * 8); }

}  // namespace

rglru_status mqa_rope_launch(int B, int T, int H, void *qkv, const int32_t *segpos, void *vt, cudaStream_t stream)
{
    const dim3 grid((unsigned)((T + kRopeTok - 1) / kRopeTok), (unsigned)B);
    rglru_mqa_rope_kernel<<<grid, kRopeThreads, 0, stream>>>(T, H, (T + 7) / 8 * 8, static_cast<__nv_bfloat16 *>(qkv),
                                                             segpos, static_cast<__nv_bfloat16 *>(vt));
    return cuda_status(cudaGetLastError());
}

rglru_status mqa_attention_launch(int B, int T, int H, int window, const void *qkv, const void *vt,
                                  const int32_t *segpos, void *out, void *ws, cudaStream_t stream)
{
    auto encode = encode_fn();
    if (!encode) return RGLRU_ERR_CUDA;
    const int Tp = (T + 7) / 8 * 8;
    const cuuint64_t cols = (cuuint64_t)(H + 2) * kHd;
    CUtensorMap tm_k, tm_v;
    const cuuint64_t kdim[3] = {cols, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t kstride[2] = {cols * 2, cols * 2 * (cuuint64_t)T};
    const cuuint32_t kbox[3] = {64, kKT, 1};
    if (!encode_bf16(encode, &tm_k, qkv, 3, kdim, kstride, kbox, CU_TENSOR_MAP_SWIZZLE_128B)) return RGLRU_ERR_CUDA;
    const cuuint64_t vdim[3] = {(cuuint64_t)Tp, (cuuint64_t)kHd, (cuuint64_t)B};
    const cuuint64_t vstride[2] = {(cuuint64_t)Tp * 2, (cuuint64_t)Tp * 2 * kHd};
    const cuuint32_t vbox[3] = {kKT, kHd, 1};
    if (!encode_bf16(encode, &tm_v, vt, 3, vdim, vstride, vbox, CU_TENSOR_MAP_SWIZZLE_128B)) return RGLRU_ERR_CUDA;

    AttnParams p;
    p.B = B;
    p.T = T;
    p.H = H;
    p.window = window;
    p.ntiles = (T + kQT - 1) / kQT;
    p.qkv = static_cast<const __nv_bfloat16 *>(qkv);
    p.segpos = segpos;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.hdr = static_cast<WsHeader *>(ws);
    static PerDeviceFlag smem_set;
    const rglru_status st = set_smem_limit_once((const void *)rglru_mqa_attention_kernel, kSmemBytes, smem_set);
    if (st != RGLRU_OK) return st;
    const unsigned grid = (unsigned)((int64_t)B * p.ntiles * H);
    rglru_mqa_attention_kernel<<<grid, kThreads, kSmemBytes, stream>>>(p, tm_k, tm_v);
    return cuda_status(cudaGetLastError());
}

}  // namespace rglru

using namespace rglru;

extern "C" {

RGLRU_API size_t rglru_mqa_vt_size(int B, int T)
{
    if (B < 1 || T < 1) return 0;
    return vt_elems(B, T) * 2;
}

RGLRU_API rglru_status rglru_mqa_rope(int B, int T, int H, void *qkv, const int32_t *segment_pos, void *v_t,
                                      cudaStream_t stream)
{
    if (!mqa_sizes_ok(B, T, H)) return RGLRU_ERR_UNSUPPORTED;
    if (!al16(qkv) || !al16(v_t) || segment_pos == nullptr) return RGLRU_ERR_INVALID_ARG;
    const uintptr_t q0 = reinterpret_cast<uintptr_t>(qkv), q1 = q0 + (size_t)B * T * (H + 2) * kHd * 2;
    const uintptr_t v0 = reinterpret_cast<uintptr_t>(v_t), v1 = v0 + vt_elems(B, T) * 2;
    if (q0 < v1 && v0 < q1) return RGLRU_ERR_INVALID_ARG;
    return mqa_rope_launch(B, T, H, qkv, segment_pos, v_t, stream);
}

RGLRU_API rglru_status rglru_mqa_attention(int B, int T, int H, int window, const void *qkv, const void *v_t,
                                           const int32_t *segment_pos, void *out, void *workspace,
                                           size_t workspace_bytes, cudaStream_t stream)
{
    if (!mqa_sizes_ok(B, T, H)) return RGLRU_ERR_UNSUPPORTED;
    if (window < 1) return RGLRU_ERR_INVALID_ARG;
    if (!al16(qkv) || !al16(v_t) || !al16(out) || segment_pos == nullptr) return RGLRU_ERR_INVALID_ARG;
    if (workspace == nullptr || !al16(workspace) || workspace_bytes < kWsHeaderBytes) return RGLRU_ERR_WORKSPACE;
    const uintptr_t o0 = reinterpret_cast<uintptr_t>(out), o1 = o0 + (size_t)B * T * H * kHd * 2;
    const struct {
        const void *p;
        size_t n;
    } ins[] = {{qkv, (size_t)B * T * (H + 2) * kHd * 2}, {v_t, vt_elems(B, T) * 2},
               {segment_pos, (size_t)B * T * 4}, {workspace, workspace_bytes}};
    for (const auto &s : ins) {
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(s.p), a1 = a0 + s.n;
        if (a0 < o1 && o0 < a1) return RGLRU_ERR_INVALID_ARG;
    }
    return mqa_attention_launch(B, T, H, window, qkv, v_t, segment_pos, out, workspace, stream);
}

RGLRU_API size_t rglru_mqa_block_workspace_size(int B, int T, int D)
{
    if (B < 1 || T < 1 || D < kHd || D % kHd != 0) return 0;
    const size_t M = (size_t)B * T;
    return kWsHeaderBytes + align_up(M * (D + 2 * kHd) * 2, 256) + align_up(vt_elems(B, T) * 2, 256) +
           align_up(M * D * 2, 256);
}

RGLRU_API rglru_status rglru_mqa_block_prefill(int B, int T, int D, int window, const void *u, const void *W_qkv,
                                               const void *W_o, const float *b_o, const int32_t *segment_pos,
                                               void *out, void *workspace, size_t workspace_bytes,
                                               cudaStream_t stream)
{
    const size_t need = rglru_mqa_block_workspace_size(B, T, D);
    if (need == 0) return RGLRU_ERR_INVALID_ARG;
    const int H = D / kHd;
    if (!mqa_sizes_ok(B, T, H)) return RGLRU_ERR_UNSUPPORTED;
    if (window < 1) return RGLRU_ERR_INVALID_ARG;
    if (workspace == nullptr || !al16(workspace) || workspace_bytes < need) return RGLRU_ERR_WORKSPACE;
    if (!al16(u) || !al16(W_qkv) || !al16(W_o) || !al16(out) || segment_pos == nullptr) return RGLRU_ERR_INVALID_ARG;
    const size_t M = (size_t)B * T, act = M * D * 2;
    const uintptr_t o0 = reinterpret_cast<uintptr_t>(out), o1 = o0 + act;
    const struct {
        const void *p;
        size_t n;
    } ins[] = {{u, act}, {W_qkv, (size_t)(D + 2 * kHd) * D * 2}, {W_o, (size_t)D * D * 2},
               {b_o, b_o ? (size_t)D * 4 : 0}, {segment_pos, M * 4}, {workspace, workspace_bytes}};
    for (const auto &s : ins) {
        if (s.p == nullptr) continue;
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(s.p), a1 = a0 + s.n;
        if (a0 < o1 && o0 < a1) return RGLRU_ERR_INVALID_ARG;
    }
    {
        const uintptr_t u0 = reinterpret_cast<uintptr_t>(u), w0 = reinterpret_cast<uintptr_t>(workspace);
        if (u0 < w0 + workspace_bytes && w0 < u0 + act) return RGLRU_ERR_INVALID_ARG;
    }
    char *ws = static_cast<char *>(workspace);
    void *qkv = ws + kWsHeaderBytes;
    void *vt = static_cast<char *>(qkv) + align_up(M * (D + 2 * kHd) * 2, 256);
    void *att = static_cast<char *>(vt) + align_up(vt_elems(B, T) * 2, 256);
    rglru_status st = rglru_linear((int)M, D + 2 * kHd, D, u, W_qkv, nullptr, qkv, ws, kWsHeaderBytes, stream);
    if (st != RGLRU_OK) return st;
    st = mqa_rope_launch(B, T, H, qkv, segment_pos, vt, stream);
    if (st != RGLRU_OK) return st;
    st = mqa_attention_launch(B, T, H, window, qkv, vt, segment_pos, att, ws, stream);
    if (st != RGLRU_OK) return st;
    return rglru_linear((int)M, D, D, att, W_o, b_o, out, ws, kWsHeaderBytes, stream);
}

RGLRU_API size_t rglru_mqa_decode_workspace_size(int B, int H, int window)
{
    if (B < 1 || B > 65535 || H < 1 || H > kDecMaxH || window < 1 || window > (1 << 20)) return 0;
    return kWsHeaderBytes + dec_part_bytes(B, H, window);
}

RGLRU_API rglru_status rglru_mqa_decode_step(int B, int H, int window, const void *qkv, const int32_t *segment_pos,
                                             void *k_cache, void *v_cache, void *out, void *workspace,
                                             size_t workspace_bytes, cudaStream_t stream)
{
    const size_t need = rglru_mqa_decode_workspace_size(B, H, window);
    if (need == 0) return RGLRU_ERR_UNSUPPORTED;
    if (!al16(qkv) || !al16(k_cache) || !al16(v_cache) || !al16(out) || segment_pos == nullptr)
        return RGLRU_ERR_INVALID_ARG;
    if (workspace == nullptr || !al16(workspace) || workspace_bytes < need) return RGLRU_ERR_WORKSPACE;
    const size_t cache = (size_t)B * window * kHd * 2;
    const struct {
        const void *p;
        size_t n;
    } bufs[] = {{qkv, (size_t)B * (H + 2) * kHd * 2}, {segment_pos, (size_t)B * 4}, {k_cache, cache},
                {v_cache, cache}, {out, (size_t)B * H * kHd * 2}, {workspace, workspace_bytes}};
    // the caches, out and the workspace are written: none may overlap another buffer
    for (int i = 0; i < 6; ++i)
        for (int j = i + 1; j < 6; ++j) {
            const bool written = i >= 2 || j >= 2;
            const uintptr_t a0 = reinterpret_cast<uintptr_t>(bufs[i].p), a1 = a0 + bufs[i].n;
            const uintptr_t b0 = reinterpret_cast<uintptr_t>(bufs[j].p), b1 = b0 + bufs[j].n;
            if (written && a0 < b1 && b0 < a1) return RGLRU_ERR_INVALID_ARG;
        }
    DecParams p;
    p.B = B;
    p.H = H;
    p.window = window;
    p.nch = (window + kDecKeys - 1) / kDecKeys;
    p.qkv = static_cast<const __nv_bfloat16 *>(qkv);
    p.segpos = segment_pos;
    p.kc = static_cast<__nv_bfloat16 *>(k_cache);
    p.vc = static_cast<__nv_bfloat16 *>(v_cache);
    char *ws = static_cast<char *>(workspace) + kWsHeaderBytes;
    p.part_o = reinterpret_cast<float *>(ws);
    p.part_ml = reinterpret_cast<float *>(ws + align_up((size_t)B * p.nch * H * kHd * 4, 256));
    p.out = static_cast<__nv_bfloat16 *>(out);
    rglru_mqa_decode_kernel<<<dim3((unsigned)p.nch, (unsigned)B), kDecThreads, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return RGLRU_ERR_CUDA;
    rglru_mqa_decode_combine_kernel<<<(unsigned)B, kHd, 0, stream>>>(p);
    return cuda_status(cudaGetLastError());
}

}  // extern "C"
