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
//   warp 4     TMA producer: the Q tile once (4 boxes [128 x 64], 128-byte
//              swizzle), then per 64-key tile the K tile (4 boxes [64 x 64])
//              and the V^T tile ([256 x 64]) into 2-deep rings;
//   warp 5     MMA issuer (one thread): S = Q K^T (M=128, N=64, 16 K-steps)
//              into one of two TMEM score buffers, then O += P V (M=128,
//              N=256, 4 K-steps) with P read from TMEM (bf16 pairs); S of
//              tile j + 1 is issued before O of tile j, so the softmax of tile
//              j overlaps the tensor cores;
//   warps 0-3  softmax: thread = query row = TMEM lane.  Scores in log2
//              units, the window / document / causal limits applied only on
//              tiles that cross them; the running max used for the
//              exponentials is raised only when a row's max grows by more
//              than 8 (a factor 256), and only then is O (in TMEM) rescaled,
//              after the MMAs that wrote it have completed.  P goes to TMEM as
//              bf16 pairs; at the end O / l is written as bf16.
// TMEM: O 256 columns, S 2 x 64, P 2 x 32 (512 allocated, one CTA per SM).
// Every mbarrier wait is bounded (2 s): one that runs out records
// RGLRU_ERR_TIMEOUT in the workspace header and the CTA unwinds.
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
constexpr int kQBox = kQT * 64 * 2;  // 16 KB: [128 rows x 64 channels]
constexpr int kQBytes = 4 * kQBox;   // 64 KB
constexpr int kKBox = kKT * 64 * 2;  // 8 KB: [64 keys x 64 channels]
constexpr int kKBytes = 4 * kKBox;   // 32 KB
constexpr int kVBytes = kHd * kKT * 2;  // 32 KB: [256 channels x 64 keys]
constexpr int kStages = 2;
constexpr int OFF_Q = 0, OFF_K = OFF_Q + kQBytes, OFF_V = OFF_K + kStages * kKBytes;
constexpr int OFF_BAR = OFF_V + kStages * kVBytes;
enum {
    B_Q = 0,
    B_KFULL = 1,
    B_KFREE = B_KFULL + kStages,
    B_VFULL = B_KFREE + kStages,
    B_VFREE = B_VFULL + kStages,
    B_SFULL = B_VFREE + kStages,  // scores of tile j in buffer j % 2
    B_SFREE = B_SFULL + 2,        // ... read by the softmax warps
    B_PFULL = B_SFREE + 2,        // P of tile j in buffer j % 2
    B_PVDONE = B_PFULL + 2,       // O += P V of tile j complete (P buffer free, O settled)
    B_DRAIN = B_PVDONE + 2,
    B_N = B_DRAIN + 1
};
constexpr int OFF_MISC = OFF_BAR + B_N * 8;
constexpr int kSmemBytes = OFF_MISC + 16 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
constexpr uint32_t kColO = 0, kColS = 256, kColP = 384;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kRescaleLog2 = 8.f;  // raise the reference max when the row max exceeds it by 2^8

struct AttnParams {
    int B, T, H, window, ntiles;
    const int32_t *segpos;
    __nv_bfloat16 *out;
    WsHeader *hdr;
};

__device__ __noinline__ bool attn_wait(uint64_t *bar, uint32_t parity, WsHeader *hdr, int where)
{
    if (mbar_try_wait(bar, parity)) return true;
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

// every lane of the warp waits; the warp's verdict is unanimous
__device__ __forceinline__ bool attn_warp_wait(uint64_t *bar, uint32_t parity, WsHeader *hdr, int where)
{
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
rglru_mqa_attention_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v)
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
            mbar_init(bars + B_Q, 1);
            for (int s = 0; s < kStages; ++s) {
                mbar_init(bars + B_KFULL + s, 1);
                mbar_init(bars + B_KFREE + s, 1);
                mbar_init(bars + B_VFULL + s, 1);
                mbar_init(bars + B_VFREE + s, 1);
            }
            for (int s = 0; s < 2; ++s) {
                mbar_init(bars + B_SFULL + s, 1);
                mbar_init(bars + B_SFREE + s, 4 * 32);
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
        if (lane == 0) {
            mbar_arrive_expect_tx(bars + B_Q, kQBytes);
            for (int kb = 0; kb < 4; ++kb)
                tma_load_3d(smem + OFF_Q + kb * kQBox, &tm_q, bars + B_Q, h * kHd + kb * 64, t0, b);
            bool ok = true;
            int jk = 0, jv = 0;  // K and V tiles issued
            for (int j = 0; j < n && ok; ++j) {
                const int s = j % kStages, s0 = (j0 + j) * kKT;
                const uint32_t ph = (uint32_t)((j / kStages) - 1) & 1u;
                if (j >= kStages && !(ok = attn_wait(bars + B_KFREE + s, ph, p.hdr, 0))) break;
                mbar_arrive_expect_tx(bars + B_KFULL + s, kKBytes);
                for (int kb = 0; kb < 4; ++kb)
                    tma_load_3d(smem + OFF_K + s * kKBytes + kb * kKBox, &tm_k, bars + B_KFULL + s,
                                p.H * kHd + kb * 64, s0, b);
                ++jk;
                if (j >= kStages && !(ok = attn_wait(bars + B_VFREE + s, ph, p.hdr, 1))) break;
                mbar_arrive_expect_tx(bars + B_VFULL + s, kVBytes);
                tma_load_3d(smem + OFF_V + s * kVBytes, &tm_v, bars + B_VFULL + s, s0, 0, b);
                ++jv;
            }
            if (!ok) {
                // the loads already issued land before the CTA exits
                drain_wait(bars + B_Q, 0);
                for (int k = max(0, jk - kStages); k < jk; ++k)
                    drain_wait(bars + B_KFULL + k % kStages, (uint32_t)(k / kStages) & 1u);
                for (int k = max(0, jv - kStages); k < jv; ++k)
                    drain_wait(bars + B_VFULL + k % kStages, (uint32_t)(k / kStages) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = umma_idesc_bf16(kQT, kKT), idesc_o = umma_idesc_bf16(kQT, kHd);
            const uint32_t q_base = smem_u32(smem + OFF_Q);
            bool ok = attn_wait(bars + B_Q, 0, p.hdr, 2);
            for (int j = 0; ok && j <= n; ++j) {
                if (j < n) {
                    const int s = j % 2;
                    if (!(ok = attn_wait(bars + B_KFULL + s, (uint32_t)(j / 2) & 1u, p.hdr, 3))) break;
                    if (j >= 2 && !(ok = attn_wait(bars + B_SFREE + s, (uint32_t)((j / 2) - 1) & 1u, p.hdr, 4)))
                        break;
                    tc_fence_after();
                    const uint32_t k_base = smem_u32(smem + OFF_K + s * kKBytes);
#pragma unroll
                    for (int kk = 0; kk < kHd / 16; ++kk) {
                        // 64-channel box kk / 4, 16-channel step kk % 4 (32 bytes into each swizzled row)
                        const uint32_t off = (uint32_t)(kk >> 2), in = (uint32_t)(kk & 3) * 32;
                        umma_ss(tmem + kColS + (uint32_t)(s * kKT), umma_desc_sw128(q_base + off * kQBox + in),
                                umma_desc_sw128(k_base + off * kKBox + in), idesc_s, kk > 0);
                    }
                    umma_commit(bars + B_SFULL + s);
                    umma_commit(bars + B_KFREE + s);
                }
                if (j >= 1) {
                    const int i = j - 1, s = i % 2;
                    if (!(ok = attn_wait(bars + B_PFULL + s, (uint32_t)(i / 2) & 1u, p.hdr, 5))) break;
                    if (!(ok = attn_wait(bars + B_VFULL + s, (uint32_t)(i / 2) & 1u, p.hdr, 6))) break;
                    tc_fence_after();
                    const uint32_t v_base = smem_u32(smem + OFF_V + s * kVBytes);
#pragma unroll
                    for (int kk = 0; kk < kKT / 16; ++kk)
                        umma_ts(tmem + kColO, tmem + kColP + (uint32_t)(s * 32 + kk * 8),
                                umma_desc_sw128(v_base + (uint32_t)kk * 32), idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(bars + B_PVDONE + s);
                    umma_commit(bars + B_VFREE + s);
                }
            }
            if (!ok) {
                // the MMAs in flight finish before TMEM is freed
                umma_commit(bars + B_DRAIN);
                drain_wait(bars + B_DRAIN, 0);
            }
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
        const float kScale = 1.4426950408889634f / 16.f;  // log2(e) / sqrt(256)
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
#pragma unroll 1
        for (int j = 0; j < n; ++j) {
            const int s = j % 2, s0 = (j0 + j) * kKT;
            if (!(ok = attn_warp_wait(bars + B_SFULL + s, (uint32_t)(j / 2) & 1u, p.hdr, 7))) break;
            tc_fence_after();
            uint32_t ra[32], rb[32];
            tmem_ld32(tmem + lane_off + kColS + (uint32_t)(s * kKT), ra);
            tmem_ld32(tmem + lane_off + kColS + (uint32_t)(s * kKT + 32), rb);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(bars + B_SFREE + s);
            float v[64];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                v[e] = __uint_as_float(ra[e]) * kScale;
                v[e + 32] = __uint_as_float(rb[e]) * kScale;
            }
            const bool inside = s0 >= lo && s0 + kKT - 1 <= hi;
            if (!__all_sync(0xffffffffu, inside)) {
#pragma unroll
                for (int e = 0; e < 64; ++e)
                    if (s0 + e < lo || s0 + e > hi) v[e] = -INFINITY;
            }
            float mt = v[0];
#pragma unroll
            for (int e = 1; e < 64; ++e) mt = fmaxf(mt, v[e]);
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
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float p0 = ex2_approx(v[2 * e] - mu), p1 = ex2_approx(v[2 * e + 1] - mu);
                l += p0 + p1;
                pk[e] = pack_bf16(p0, p1);
            }
            // P buffer s was last read by the MMAs of tile j - 2
            if (j >= 2 && !(ok = attn_warp_wait(bars + B_PVDONE + s, (uint32_t)((j / 2) - 1) & 1u, p.hdr, 9))) break;
            tc_fence_after();
            tmem_st32(tmem + lane_off + kColP + (uint32_t)(s * 32), pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bars + B_PFULL + s);
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
    CUtensorMap tm_q, tm_k, tm_v;
    const cuuint64_t qdim[3] = {cols, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t qstride[2] = {cols * 2, cols * 2 * (cuuint64_t)T};
    const cuuint32_t qbox[3] = {64, kQT, 1}, kbox[3] = {64, kKT, 1};
    if (!encode_bf16(encode, &tm_q, qkv, 3, qdim, qstride, qbox, CU_TENSOR_MAP_SWIZZLE_128B)) return RGLRU_ERR_CUDA;
    if (!encode_bf16(encode, &tm_k, qkv, 3, qdim, qstride, kbox, CU_TENSOR_MAP_SWIZZLE_128B)) return RGLRU_ERR_CUDA;
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
    p.segpos = segpos;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.hdr = static_cast<WsHeader *>(ws);
    static PerDeviceFlag smem_set;
    const rglru_status st = set_smem_limit_once((const void *)rglru_mqa_attention_kernel, kSmemBytes, smem_set);
    if (st != RGLRU_OK) return st;
    const unsigned grid = (unsigned)((int64_t)B * p.ntiles * H);
    rglru_mqa_attention_kernel<<<grid, kThreads, kSmemBytes, stream>>>(p, tm_q, tm_k, tm_v);
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

}  // extern "C"
