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
// 224 threads:
//   warp 4     TMA producer: lane 0 the K tiles (4 boxes [64 keys x 64
//              channels], 128-byte swizzle), lane 1 the V^T tiles ([256 x 64
//              keys]), each into a 3-deep ring;
//   warp 5     S issuer (the converged warp, one lane elected per MMA):
//              S = Q K^T (M=128, N=64, 16 K-steps) with Q read from TMEM; S of
//              tile j + 1 goes out as soon as the softmax has read S of tile j,
//              so it runs under the softmax of tile j;
//   warp 6     P V issuer: O += P V (M=128, N=256, 4 K-steps) with P read from
//              TMEM, as soon as P of the tile is written (two issuing warps, so
//              neither kind of MMA waits behind the other's barriers);
//   warps 0-3  softmax: thread = query row = TMEM lane.  Each loads its row of
//              the Q tile at kernel start (all 32 loads in flight under the
//              setup) and writes it into TMEM (the A operand of S).  Scores in
//              log2 units, the window / document / causal limits applied only
//              on tiles that cross them; the running max used for the
//              exponentials is raised only when a row's max grows by more
//              than 8 (a factor 256), and only then is O (in TMEM) rescaled,
//              after the MMAs that wrote it have completed.  P goes to TMEM as
//              bf16 pairs; at the end O / l is written as bf16.
// TMEM: O 256 columns, Q 128, S 64, P 2 x 32 (all 512, one CTA per SM).
// The decode step (rglru_mqa_decode_kernel, further down) has its own notes.
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
constexpr int kThreads = 224;
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
    B_DRAIN = B_PVDONE + 2,       // per issuing warp: its MMAs have finished (error path)
    B_N = B_DRAIN + 2
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
    // the softmax warps' rows of the Q tile: every 16-byte load in flight now,
    // under the key-range scan, the barrier setup and the TMEM allocation
    uint4 qv[32];
    if (warp < 4) {
        const int tq = t0 + warp * 32 + lane;
        const uint4 *src = reinterpret_cast<const uint4 *>(
            p.qkv + ((size_t)b * p.T + (tq < p.T ? tq : 0)) * (size_t)((p.H + 2) * kHd) + (size_t)h * kHd);
#pragma unroll
        for (int k = 0; k < 32; ++k) qv[k] = tq < p.T ? __ldg(src + k) : make_uint4(0, 0, 0, 0);
    }
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
            mbar_init(bars + B_DRAIN + 1, 1);
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
        // ------------------------------------------------------------ S issuer
        // S of tile j as soon as K_j has landed and the score buffer is free
        // (the converged warp runs the loop; elect.sync picks the issuing lane)
        const uint32_t idesc_s = umma_idesc_bf16(kQT, kKT);
        bool ok = attn_warp_wait(bars + B_QFULL, 0, p.hdr, 2);
        for (int j = 0; ok && j < n; ++j) {
            const int s = j % kStages;
            if (!(ok = attn_warp_wait(bars + B_KFULL + s, (uint32_t)(j / kStages) & 1u, p.hdr, 3))) break;
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
            __syncwarp();
        }
        if (!ok) {
            // this warp's MMAs finish before TMEM is freed
            umma_commit_warp(bars + B_DRAIN);
            if (lane == 0) drain_wait(bars + B_DRAIN, 0);
        }
        __syncwarp();
    } else if (warp == 6) {
        // ------------------------------------------------------------ P V issuer
        // O += P_i V_i as soon as P_i is in TMEM and V_i has landed
        const uint32_t idesc_o = umma_idesc_bf16(kQT, kHd);
        bool ok = true;
        for (int i = 0; ok && i < n; ++i) {
            const int pb = i % 2, s = i % kStages;
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
            __syncwarp();
        }
        if (!ok) {
            umma_commit_warp(bars + B_DRAIN + 1);
            if (lane == 0) drain_wait(bars + B_DRAIN + 1, 0);
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
            // this row of the Q tile (loaded at the start) into its TMEM lane: 128 columns
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t r[32];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    r[4 * k] = qv[q * 8 + k].x;
                    r[4 * k + 1] = qv[q * 8 + k].y;
                    r[4 * k + 2] = qv[q * 8 + k].z;
                    r[4 * k + 3] = qv[q * 8 + k].w;
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
constexpr int kRopeTok = 16;  // tokens per CTA
constexpr int kRopeThreads = 256;

__device__ __forceinline__ uint32_t rot_pair(uint32_t a, uint32_t c, float2 r0, float2 r1, bool second)
{
    // elements 2e, 2e+1 of the first half (a) or of the second half (c)
    const float a0 = __uint_as_float(a << 16), a1 = __uint_as_float(a & 0xffff0000u);
    const float c0 = __uint_as_float(c << 16), c1 = __uint_as_float(c & 0xffff0000u);
    float y0, y1;
    if (!second) {
        y0 = a0 * r0.x - c0 * r0.y;
        y1 = a1 * r1.x - c1 * r1.y;
    } else {
        y0 = c0 * r0.x + a0 * r0.y;
        y1 = c1 * r1.x + a1 * r1.y;
    }
    uint32_t o;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o) : "f"(y1), "f"(y0));
    return o;
}

__global__ void __launch_bounds__(kRopeThreads)
rglru_mqa_rope_kernel(int T, int H, int Tp, __nv_bfloat16 *__restrict__ qkv, const int32_t *__restrict__ segpos,
                      __nv_bfloat16 *__restrict__ vt)
{
    __shared__ double inv_freq[kHd / 2];
    __shared__ __align__(16) float2 cs[kRopeTok][kHd / 2];            // (cos, sin) per token and pair
    __shared__ __align__(16) __nv_bfloat16 vs[kRopeTok][kHd + 8];     // the v rows, padded
    const int b = blockIdx.y, tb = blockIdx.x * kRopeTok, tid = threadIdx.x;
    const size_t W = (size_t)(H + 2) * kHd;
    if (tid < kHd / 2) inv_freq[tid] = exp2(-(double)tid * (13.287712379549449 / 128.0));
    // the v rows of the CTA's tokens into shared memory (16-byte loads, all in flight)
    for (int e = tid; e < kRopeTok * (kHd / 8); e += kRopeThreads) {
        const int tt = e / (kHd / 8), c = e % (kHd / 8), t = tb + tt;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (t < T) v = *reinterpret_cast<const uint4 *>(qkv + ((size_t)b * T + t) * W + (size_t)(H + 1) * kHd + c * 8);
        *reinterpret_cast<uint4 *>(&vs[tt][c * 8]) = v;
    }
    __syncthreads();
    for (int e = tid; e < kRopeTok * (kHd / 2); e += kRopeThreads) {
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
    // q heads and k: unit = (token, head, 8 pairs): 16-byte loads of x[i..i+8] and
    // x[i+128..i+136], rotated, 16-byte stores back
    const int units = kRopeTok * (H + 1) * 16;
    for (int u = tid; u < units; u += kRopeThreads) {
        const int c8 = u % 16, rest = u / 16, hh = rest % (H + 1), tt = rest / (H + 1), t = tb + tt;
        if (t >= T) continue;
        __nv_bfloat16 *rowp = qkv + ((size_t)b * T + t) * W + (size_t)hh * kHd + c8 * 8;
        const uint4 a = *reinterpret_cast<const uint4 *>(rowp);
        const uint4 c = *reinterpret_cast<const uint4 *>(rowp + kHd / 2);
        const float4 *cp = reinterpret_cast<const float4 *>(&cs[tt][c8 * 8]);
        const float4 r01 = cp[0], r23 = cp[1], r45 = cp[2], r67 = cp[3];
        const float2 r[8] = {make_float2(r01.x, r01.y), make_float2(r01.z, r01.w), make_float2(r23.x, r23.y),
                             make_float2(r23.z, r23.w), make_float2(r45.x, r45.y), make_float2(r45.z, r45.w),
                             make_float2(r67.x, r67.y), make_float2(r67.z, r67.w)};
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, cw[4] = {c.x, c.y, c.z, c.w};
        uint32_t o1[4], o2[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            o1[q] = rot_pair(aw[q], cw[q], r[2 * q], r[2 * q + 1], false);
            o2[q] = rot_pair(aw[q], cw[q], r[2 * q], r[2 * q + 1], true);
        }
        *reinterpret_cast<uint4 *>(rowp) = make_uint4(o1[0], o1[1], o1[2], o1[3]);
        *reinterpret_cast<uint4 *>(rowp + kHd / 2) = make_uint4(o2[0], o2[1], o2[2], o2[3]);
    }
    // v transposed: thread = channel, 8 tokens per 16-byte store
    const int d = tid;
#pragma unroll 1
    for (int g = 0; g < kRopeTok; g += 8) {
        const int tg = tb + g;
        if (tg >= T) break;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            w[q] = (uint32_t)__bfloat16_as_ushort(vs[g + 2 * q][d]) |
                   ((uint32_t)__bfloat16_as_ushort(vs[g + 2 * q + 1][d]) << 16);
        *reinterpret_cast<uint4 *>(vt + ((size_t)b * kHd + d) * Tp + tg) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}
static_assert(kRopeThreads == kHd, "one thread per v channel");

// ---------------------------------------------------------------- decode step
// One token per sequence at document position pos attends the cached keys of
// positions lo = max(0, pos - window + 1) .. pos.  The rings keep position q
// at slot q % window: k_cache [B, window, 256] (rotated keys) and v_cache
// transposed, [B, 256, window], so that both tiles below are K-major operands.
// One CTA per (sequence, block of 128 positions aligned to 128), 128 threads:
//   TMA loads the block's K tile (4 boxes [128 keys x 64 channels], 128-byte
//   swizzle) while the threads rotate q and write it (heads padded to 16,
//   bf16) into a swizzled tile;
//   S^T = K Q^T        M = 128 keys, N = 16 heads, K = 256   (tcgen05, TMEM);
//   once S is done the same 64 KB buffer receives the V^T tile (4 boxes
//   [128 channels x 64 keys]) while the softmax runs over the block's keys
//   per head (thread = key, keys outside [lo, pos] masked; P^T written bf16
//   into a swizzled tile);
//   O^T = V^T P^T      M = 128 channels (two halves), N = 16, K = 128 keys;
// one 64 KB tile buffer per CTA lets two CTAs share an SM, so one CTA's loads
// run under the other's arithmetic;
// then the block's (max, sum, O) per head go to the workspace and a combine
// kernel merges the blocks.  The CTA whose block holds pos writes this token's
// rotated k and its v into its tiles (after the loads land) and into the rings.
// The rings must hold finite values in every slot (zero-filled at first use):
// masked keys enter the products with probability 0.
constexpr int kDecKeys = 128;                    // keys per CTA (TMEM lanes)
constexpr int kDecThreads = 128;
constexpr int kDecMaxH = 16;                     // heads padded to the MMA's N
constexpr int kDecKBox = kDecKeys * 64 * 2;      // 16 KB: [128 keys x 64 channels]
constexpr int kDecVBox = 128 * 64 * 2;           // 16 KB: [128 channels x 64 keys]
constexpr int kDecQBox = kDecMaxH * 128;         // 2 KB:  [16 heads x 64 channels]
constexpr int kDecPBox = kDecMaxH * 128;         // 2 KB:  [16 heads x 64 keys]
static_assert(kDecKBox == kDecVBox, "K and V^T tiles share one buffer");
constexpr int DOFF_K = 0, DOFF_V = 0, DOFF_Q = DOFF_K + 4 * kDecKBox;
constexpr int DOFF_P = DOFF_Q + 4 * kDecQBox, DOFF_BAR = DOFF_P + 2 * kDecPBox, DOFF_MISC = DOFF_BAR + 4 * 8;
constexpr int kDecSmem = DOFF_MISC + 16 + 1024;
static_assert(kDecSmem <= 227 * 1024, "shared memory budget");
constexpr uint32_t kDecCols = 64;                // TMEM: S^T 16 columns, O^T 2 x 16
constexpr uint64_t kDecTimeoutNs = 2000000000ull;

struct DecParams {
    int B, H, window, nch;
    const __nv_bfloat16 *qkv;   // [B, (H + 2) * 256]
    const int32_t *segpos;      // [B]
    __nv_bfloat16 *kc;          // [B, window, 256]
    __nv_bfloat16 *vtc;         // [B, 256, window]
    float *part_o;              // [B, nch, H, 256]
    float *part_ml;             // [B, nch, H, 2]: block max (log2 units) and sum
    __nv_bfloat16 *out;         // [B, H * 256]
    WsHeader *hdr;
};

// Byte offset of element (row, k) of a K-major tile of 64-element (128-byte)
// rows in the 128-byte swizzled layout a TMA load writes: the 16-byte chunk
// index is XORed with the row's index within its 8-row atom.
__device__ __forceinline__ uint32_t sw128(int row, int k)
{
    return (uint32_t)row * 128u + ((uint32_t)(((k >> 3) ^ row) & 7) << 4) + (uint32_t)(k & 7) * 2u;
}

// bounded wait by every thread of the CTA; false (status recorded) on timeout
__device__ bool mqd_wait(uint64_t *bar, uint32_t parity, WsHeader *hdr, int where)
{
    bool done = mbar_try_wait(bar, parity);
    if (!done) {
        const uint64_t t0 = globaltimer();
        while (!(done = mbar_try_wait_sleep(bar, parity, 20000u)) && globaltimer() - t0 < kDecTimeoutNs) {
        }
    }
    if (!__syncthreads_and(done ? 1 : 0)) {
        if (threadIdx.x == 0) {
            atomicCAS(&hdr->status, 0, (int)RGLRU_ERR_TIMEOUT);
            atomicCAS(&hdr->detail, 0, (int)((blockIdx.y * gridDim.x + blockIdx.x) << 8) | (where + 1));
        }
        return false;
    }
    return true;
}

__global__ void __launch_bounds__(kDecThreads, 2)
rglru_mqa_decode_kernel(const DecParams p, const __grid_constant__ CUtensorMap tm_kc,
                        const __grid_constant__ CUtensorMap tm_vt)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + DOFF_BAR);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + DOFF_MISC);
    __shared__ float2 cs[kHd / 2];
    __shared__ double inv_freq[kHd / 2];
    __shared__ __align__(16) __nv_bfloat16 rowbuf[(kDecMaxH + 2) * kHd];  // the token's q, k, v
    __shared__ __align__(16) __nv_bfloat16 kv_tok[2][kHd];  // this token's rotated k and its v
    __shared__ float red[kDecThreads / 32][kDecMaxH];
    __shared__ float mh[kDecMaxH], lh[kDecMaxH];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = p.H, W = p.window;
    inv_freq[tid] = exp2(-(double)tid * (13.287712379549449 / 128.0));  // 10000^(-2i/256)

    if (warp == 0) {
        tmem_alloc(tmem_holder, kDecCols);
        if (lane == 0) {
            for (int i = 0; i < 4; ++i) mbar_init(bars + i, 1);
            mbar_fence_init();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    uint8_t *Kt = smem + DOFF_K, *Vt = smem + DOFF_V, *Qt = smem + DOFF_Q, *Pt = smem + DOFF_P;
    const uint32_t idesc = umma_idesc_bf16(kDecKeys, kDecMaxH);
    const float kScale = 1.4426950408889634f / 16.f;

    // items (block c, sequence b), block-major; the CTA's k-th processed item
    // uses phase k & 1 of each of its four barriers
    bool ok = true;
    uint32_t ph = 0;
    for (int w = blockIdx.x; ok && w < p.B * p.nch; w += gridDim.x) {
        const int b = w % p.B, c = w / p.B;
        const int pos = max(p.segpos[b], 0);
        const int n = min(pos + 1, W);
        const int lo = pos - n + 1;
        const int mblk = (lo >> 7) + c;  // this item's block of 128 positions
        if (mblk > (pos >> 7)) continue;  // (uniform in the CTA)
        const int p0 = mblk << 7;
        const int slot0 = p0 % W;  // window is a multiple of 128: the block's slots are contiguous
        const bool owner = mblk == (pos >> 7);

        if (tid == 0) {
            mbar_arrive_expect_tx(bars + 0, 4 * kDecKBox);
            for (int kb = 0; kb < 4; ++kb) tma_load_2d(Kt + kb * kDecKBox, &tm_kc, bars + 0, kb * 64, b * W + slot0);
        }
        // the token's qkv row into shared memory: all 16-byte loads issued at once
        {
            const uint4 *src = reinterpret_cast<const uint4 *>(p.qkv + (size_t)b * (H + 2) * kHd);
            uint4 *dst = reinterpret_cast<uint4 *>(rowbuf);
            const int nv = (H + 2) * kHd / 8;
            uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0, v2 = v0, v3 = v0, v4 = v0;
            if (tid < nv) v0 = __ldg(src + tid);
            if (tid + 128 < nv) v1 = __ldg(src + tid + 128);
            if (tid + 256 < nv) v2 = __ldg(src + tid + 256);
            if (tid + 384 < nv) v3 = __ldg(src + tid + 384);
            if (tid + 512 < nv) v4 = __ldg(src + tid + 512);
            if (tid < nv) dst[tid] = v0;
            if (tid + 128 < nv) dst[tid + 128] = v1;
            if (tid + 256 < nv) dst[tid + 256] = v2;
            if (tid + 384 < nv) dst[tid + 384] = v3;
            if (tid + 512 < nv) dst[tid + 512] = v4;
        }
        // RoPE angles of this position (reduced modulo 2 pi in fp64), one pair per thread
        {
            double turns = (double)pos * inv_freq[tid] * 0.15915494309189535;
            turns -= floor(turns);
            float sn, co;
            sincospif((float)(2.0 * turns), &sn, &co);
            cs[tid] = make_float2(co, sn);
        }
        __syncthreads();
        const __nv_bfloat16 *row = rowbuf;
        // Q^T tile: rows = heads (16, zero past H), K = channels, 4 boxes of 64
        // channels; row H of the token is its key (into kv_tok; with 16 heads that
        // row lies past the tile)
        for (int e = tid; e < (kDecMaxH + 1) * (kHd / 2); e += kDecThreads) {
            const int hh = e / (kHd / 2), i = e % (kHd / 2);
            __nv_bfloat16 y1 = __float2bfloat16_rn(0.f), y2 = y1;
            if (hh <= H) {
                const float x1 = __bfloat162float(row[hh * kHd + i]), x2 = __bfloat162float(row[hh * kHd + i + kHd / 2]);
                const float2 r = cs[i];
                y1 = __float2bfloat16_rn(x1 * r.x - x2 * r.y);
                y2 = __float2bfloat16_rn(x2 * r.x + x1 * r.y);
            }
            if (hh == H) {  // the key
                kv_tok[0][i] = y1;
                kv_tok[0][i + kHd / 2] = y2;
                y1 = y2 = __float2bfloat16_rn(0.f);
            }
            if (hh < kDecMaxH) {
                const int d1 = i, d2 = i + kHd / 2;
                *reinterpret_cast<__nv_bfloat16 *>(Qt + (d1 >> 6) * kDecQBox + sw128(hh, d1 & 63)) = y1;
                *reinterpret_cast<__nv_bfloat16 *>(Qt + (d2 >> 6) * kDecQBox + sw128(hh, d2 & 63)) = y2;
            }
        }
        kv_tok[1][tid] = row[(H + 1) * kHd + tid];
        kv_tok[1][tid + 128] = row[(H + 1) * kHd + tid + 128];
        // the K tile has landed (a timeout ends the loop; TMEM is freed below)
        if (!(ok = mqd_wait(bars + 0, ph, p.hdr, 0))) break;
        if (owner) {
            // this token's key into the tile (over the ring's stale slot) and both into the rings
            const int r = pos - p0, sl = pos % W;
            for (int d = tid; d < kHd; d += kDecThreads) {
                const __nv_bfloat16 kk = kv_tok[0][d];
                *reinterpret_cast<__nv_bfloat16 *>(Kt + (d >> 6) * kDecKBox + sw128(r, d & 63)) = kk;
                p.kc[((size_t)b * W + sl) * kHd + d] = kk;
                p.vtc[((size_t)b * kHd + d) * W + sl] = kv_tok[1][d];
            }
        }
        fence_proxy_async_smem();  // the generic writes of the tiles, before the tensor cores read them
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint64_t kd = umma_desc_sw128(smem_u32(Kt)), qd = umma_desc_sw128(smem_u32(Qt));
#pragma unroll
            for (int kk = 0; kk < kHd / 16; ++kk) {
                const uint32_t off_k = (uint32_t)(kk >> 2) * kDecKBox + (uint32_t)(kk & 3) * 32;
                const uint32_t off_q = (uint32_t)(kk >> 2) * kDecQBox + (uint32_t)(kk & 3) * 32;
                umma_ss(tmem, kd + (off_k >> 4), qd + (off_q >> 4), idesc, kk > 0);
            }
            umma_commit(bars + 1);
        }
        if (!(ok = mqd_wait(bars + 1, ph, p.hdr, 1))) break;
        tc_fence_after();
        // S is complete, so the K tile has been read: the V^T tile goes into the same buffer
        if (tid == 0) {
            mbar_arrive_expect_tx(bars + 3, 4 * kDecVBox);
            for (int dh = 0; dh < 2; ++dh)
                for (int kh = 0; kh < 2; ++kh)
                    tma_load_3d(Vt + (dh * 2 + kh) * kDecVBox, &tm_vt, bars + 3, slot0 + 64 * kh, 128 * dh, b);
        }
        uint32_t sr[16];
        tmem_ld16(lane_base, sr);
        tmem_wait_ld();
        const int kp = p0 + tid;  // this thread's key position
        const bool valid = kp >= lo && kp <= pos;
        float sc[kDecMaxH];
#pragma unroll
        for (int h = 0; h < kDecMaxH; ++h) sc[h] = (valid && h < H) ? __uint_as_float(sr[h]) * kScale : -INFINITY;
#pragma unroll
        for (int h = 0; h < kDecMaxH; ++h) {
            float m = sc[h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) red[warp][h] = m;
        }
        __syncthreads();
        if (tid < kDecMaxH) mh[tid] = fmaxf(fmaxf(red[0][tid], red[1][tid]), fmaxf(red[2][tid], red[3][tid]));
        __syncthreads();
        float pr[kDecMaxH];
#pragma unroll
        for (int h = 0; h < kDecMaxH; ++h) {
            pr[h] = (valid && h < H) ? ex2_approx(sc[h] - mh[h]) : 0.f;
            float l = pr[h];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
            if (lane == 0) red[warp][h] = l;
        }
        // P^T tile: rows = heads, K = this block's keys (2 boxes of 64)
#pragma unroll
        for (int h = 0; h < kDecMaxH; ++h)
            *reinterpret_cast<__nv_bfloat16 *>(Pt + (tid >> 6) * kDecPBox + sw128(h, tid & 63)) =
                __float2bfloat16_rn(pr[h]);
        __syncthreads();
        if (tid < kDecMaxH) lh[tid] = (red[0][tid] + red[1][tid]) + (red[2][tid] + red[3][tid]);
        if (!(ok = mqd_wait(bars + 3, ph, p.hdr, 3))) break;  // the V^T tile has landed
        if (owner) {
            const int r = pos - p0;
            for (int d = tid; d < kHd; d += kDecThreads)
                *reinterpret_cast<__nv_bfloat16 *>(Vt + ((d >> 7) * 2 + (r >> 6)) * kDecVBox + sw128(d & 127, r & 63)) =
                    kv_tok[1][d];
        }
        fence_proxy_async_smem();  // P^T and the token's value, before the tensor cores read them
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint64_t pd = umma_desc_sw128(smem_u32(Pt));
#pragma unroll
            for (int dh = 0; dh < 2; ++dh) {
                const uint64_t vd = umma_desc_sw128(smem_u32(Vt + dh * 2 * kDecVBox));
#pragma unroll
                for (int kk = 0; kk < kDecKeys / 16; ++kk) {
                    const uint32_t off_v = (uint32_t)(kk >> 2) * kDecVBox + (uint32_t)(kk & 3) * 32;
                    const uint32_t off_p = (uint32_t)(kk >> 2) * kDecPBox + (uint32_t)(kk & 3) * 32;
                    umma_ss(tmem + 16 + 16 * dh, vd + (off_v >> 4), pd + (off_p >> 4), idesc, kk > 0);
                }
            }
            umma_commit(bars + 2);
        }
        if (!(ok = mqd_wait(bars + 2, ph, p.hdr, 2))) break;
        tc_fence_after();
        uint32_t o0[16], o1[16];
        tmem_ld16(lane_base + 16, o0);
        tmem_ld16(lane_base + 32, o1);
        tmem_wait_ld();
        const size_t base = ((size_t)b * p.nch + c) * H;
#pragma unroll
        for (int h = 0; h < kDecMaxH; ++h) {
            if (h < H) {
                p.part_o[(base + h) * kHd + tid] = __uint_as_float(o0[h]);
                p.part_o[(base + h) * kHd + 128 + tid] = __uint_as_float(o1[h]);
            }
        }
        if (tid < H) {
            p.part_ml[2 * (base + tid)] = mh[tid];
            p.part_ml[2 * (base + tid) + 1] = lh[tid];
        }
        // the next item rewrites the tiles, cs, kv_tok and TMEM only after every
        // thread has finished with this one
        tc_fence_before();
        __syncthreads();
        ph ^= 1u;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kDecCols);
}

// out[b, h] = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c over the blocks of
// sequence b (at most 17: window <= 2048).  One CTA per (sequence, head):
// every warp finds the weights (lane c holds block c's max and sum), then each
// thread (= channel) sums its channel over the blocks.
__global__ void __launch_bounds__(kHd)
rglru_mqa_decode_combine_kernel(const DecParams p)
{
    const int b = blockIdx.x, h = blockIdx.y, d = threadIdx.x, H = p.H, lane = d & 31;
    const int pos = max(p.segpos[b], 0);
    const int lo = pos - min(pos + 1, p.window) + 1;
    const int nc = (pos >> 7) - (lo >> 7) + 1;
    const bool in = lane < nc;
    const size_t base = ((size_t)b * p.nch + lane) * H + h;
    const float m = in ? p.part_ml[2 * base] : -INFINITY, l = in ? p.part_ml[2 * base + 1] : 0.f;
    float M = m;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float f = in ? ex2_approx(m - M) : 0.f;
    float den = f * l;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float *po = p.part_o + ((size_t)b * p.nch * H + h) * kHd + d;
    const size_t cstride = (size_t)H * kHd;
    float num = 0.f;
#pragma unroll 4
    for (int c = 0; c < nc; ++c) num = fmaf(__shfl_sync(0xffffffffu, f, c), po[c * cstride], num);
    p.out[(size_t)b * H * kHd + (size_t)h * kHd + d] = __float2bfloat16_rn(num / den);
}

size_t dec_part_bytes(int B, int H, int window)
{
    const size_t nch = (size_t)(window / kDecKeys + 1);
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
    if (B < 1 || B > 65535 || H < 1 || H > kDecMaxH || window < kDecKeys || window % kDecKeys != 0 ||
        window > 16 * kDecKeys)
        return 0;
    return kWsHeaderBytes + dec_part_bytes(B, H, window);
}

RGLRU_API rglru_status rglru_mqa_decode_step(int B, int H, int window, const void *qkv, const int32_t *segment_pos,
                                             void *k_cache, void *v_cache_t, void *out, void *workspace,
                                             size_t workspace_bytes, cudaStream_t stream)
{
    const size_t need = rglru_mqa_decode_workspace_size(B, H, window);
    if (need == 0) return RGLRU_ERR_UNSUPPORTED;
    if (!al16(qkv) || !al16(k_cache) || !al16(v_cache_t) || !al16(out) || segment_pos == nullptr)
        return RGLRU_ERR_INVALID_ARG;
    if (workspace == nullptr || !al16(workspace) || workspace_bytes < need) return RGLRU_ERR_WORKSPACE;
    const size_t cache = (size_t)B * window * kHd * 2;
    const struct {
        const void *p;
        size_t n;
    } bufs[] = {{qkv, (size_t)B * (H + 2) * kHd * 2}, {segment_pos, (size_t)B * 4}, {k_cache, cache},
                {v_cache_t, cache}, {out, (size_t)B * H * kHd * 2}, {workspace, workspace_bytes}};
    // the rings, out and the workspace are written: none may overlap another buffer
    for (int i = 0; i < 6; ++i)
        for (int j = i + 1; j < 6; ++j) {
            const bool written = i >= 2 || j >= 2;
            const uintptr_t a0 = reinterpret_cast<uintptr_t>(bufs[i].p), a1 = a0 + bufs[i].n;
            const uintptr_t b0 = reinterpret_cast<uintptr_t>(bufs[j].p), b1 = b0 + bufs[j].n;
            if (written && a0 < b1 && b0 < a1) return RGLRU_ERR_INVALID_ARG;
        }
    auto encode = encode_fn();
    if (!encode) return RGLRU_ERR_CUDA;
    CUtensorMap tm_kc, tm_vt;
    const cuuint64_t kdim[2] = {(cuuint64_t)kHd, (cuuint64_t)B * window}, kstride[1] = {(cuuint64_t)kHd * 2};
    const cuuint32_t kbox[2] = {64, kDecKeys};
    if (!encode_bf16(encode, &tm_kc, k_cache, 2, kdim, kstride, kbox, CU_TENSOR_MAP_SWIZZLE_128B)) return RGLRU_ERR_CUDA;
    const cuuint64_t vdim[3] = {(cuuint64_t)window, (cuuint64_t)kHd, (cuuint64_t)B};
    const cuuint64_t vstride[2] = {(cuuint64_t)window * 2, (cuuint64_t)window * 2 * kHd};
    const cuuint32_t vbox[3] = {64, 128, 1};
    if (!encode_bf16(encode, &tm_vt, v_cache_t, 3, vdim, vstride, vbox, CU_TENSOR_MAP_SWIZZLE_128B))
        return RGLRU_ERR_CUDA;
    DecParams p;
    p.B = B;
    p.H = H;
    p.window = window;
    p.nch = window / kDecKeys + 1;
    p.qkv = static_cast<const __nv_bfloat16 *>(qkv);
    p.segpos = segment_pos;
    p.kc = static_cast<__nv_bfloat16 *>(k_cache);
    p.vtc = static_cast<__nv_bfloat16 *>(v_cache_t);
    char *ws = static_cast<char *>(workspace) + kWsHeaderBytes;
    p.part_o = reinterpret_cast<float *>(ws);
    p.part_ml = reinterpret_cast<float *>(ws + align_up((size_t)B * p.nch * H * kHd * 4, 256));
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.hdr = static_cast<WsHeader *>(workspace);
    static PerDeviceFlag smem_set;
    const rglru_status st = set_smem_limit_once((const void *)rglru_mqa_decode_kernel, kDecSmem, smem_set);
    if (st != RGLRU_OK) return st;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return RGLRU_ERR_CUDA;
    const long long items = (long long)B * p.nch;
    const unsigned grid = (unsigned)(items < 2LL * sms ? items : 2LL * sms);  // two per SM, persistent
    rglru_mqa_decode_kernel<<<grid, kDecThreads, kDecSmem, stream>>>(p, tm_kc, tm_vt);
    if (cudaGetLastError() != cudaSuccess) return RGLRU_ERR_CUDA;
    rglru_mqa_decode_combine_kernel<<<dim3((unsigned)B, (unsigned)H), kHd, 0, stream>>>(p);
    return cuda_status(cudaGetLastError());
}

RGLRU_API size_t rglru_mqa_residual_block_workspace_size(int B, int T, int D, int F)
{
    if (B < 1 || T < 1 || D < kHd || D % kHd != 0 || F < 128 || F % 128 != 0 || F > (1 << 20)) return 0;
    const size_t M = (size_t)B * T, act = align_up(M * D * 2, 256);
    return kWsHeaderBytes + 3 * act + align_up(M * (D + 2 * kHd) * 2, 256) + align_up(vt_elems(B, T) * 2, 256) +
           align_up(M * F * 2, 256);
}

RGLRU_API rglru_status rglru_mqa_residual_block_prefill(
    int B, int T, int D, int F, int window, const void *u, const float *w_temporal_norm, const void *W_qkv,
    const void *W_o, const float *b_o, const int32_t *segment_pos, const float *w_channel_norm, const void *W_gate,
    const float *b_gate, const void *W_up, const float *b_up, const void *W_down, const float *b_down, float eps,
    void *out, void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    const size_t need = rglru_mqa_residual_block_workspace_size(B, T, D, F);
    if (need == 0) return RGLRU_ERR_INVALID_ARG;
    const int H = D / kHd;
    if (!mqa_sizes_ok(B, T, H) || !(eps > 0.f)) return RGLRU_ERR_UNSUPPORTED;
    if (window < 1) return RGLRU_ERR_INVALID_ARG;
    if (workspace == nullptr || !al16(workspace) || workspace_bytes < need) return RGLRU_ERR_WORKSPACE;
    // every operand checked before the first launch, so that a bad argument leaves out untouched
    if (!al16(u) || !al16(out) || !al16(W_qkv) || !al16(W_o) || !al16(w_temporal_norm) || !al16(w_channel_norm) ||
        !al16(W_gate) || !al16(b_gate) || !al16(W_up) || !al16(b_up) || !al16(W_down) || segment_pos == nullptr)
        return RGLRU_ERR_INVALID_ARG;
    for (const float *bias : {b_o, b_down})
        if (bias != nullptr && !al16(bias)) return RGLRU_ERR_INVALID_ARG;
    const size_t M = (size_t)B * T, act = M * D * 2;
    const struct {
        const void *p;
        size_t n;
    } ins[] = {{u, act}, {workspace, workspace_bytes}, {W_qkv, (size_t)(D + 2 * kHd) * D * 2},
               {W_o, (size_t)D * D * 2}, {W_gate, (size_t)F * D * 2}, {W_up, (size_t)F * D * 2},
               {W_down, (size_t)D * F * 2}, {segment_pos, M * 4}};
    const uintptr_t o0 = reinterpret_cast<uintptr_t>(out), o1 = o0 + act;
    for (const auto &b : ins) {
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(b.p), a1 = a0 + b.n;
        if (a0 < o1 && o0 < a1) return RGLRU_ERR_INVALID_ARG;
    }
    {
        const uintptr_t u0 = reinterpret_cast<uintptr_t>(u), w0 = reinterpret_cast<uintptr_t>(workspace);
        if (u0 < w0 + workspace_bytes && w0 < u0 + act) return RGLRU_ERR_INVALID_ARG;
    }
    char *ws = static_cast<char *>(workspace);
    const size_t a = align_up(act, 256);
    char *n = ws + kWsHeaderBytes, *h = n + a, *att = h + a;
    char *qkv = att + a;
    char *vt = qkv + align_up(M * (D + 2 * kHd) * 2, 256);
    char *m = vt + align_up(vt_elems(B, T) * 2, 256);
    // temporal_pre_norm -> q/k/v projections -> RoPE -> local MQA -> o_proj + residual
    rglru_status st = rglru_rmsnorm((int)M, D, u, w_temporal_norm, eps, n, stream);
    if (st == RGLRU_OK) st = rglru_linear((int)M, D + 2 * kHd, D, n, W_qkv, nullptr, qkv, ws, kWsHeaderBytes, stream);
    if (st == RGLRU_OK) st = mqa_rope_launch(B, T, H, qkv, segment_pos, vt, stream);
    if (st == RGLRU_OK) st = mqa_attention_launch(B, T, H, window, qkv, vt, segment_pos, att, ws, stream);
    if (st == RGLRU_OK) st = rglru_linear_residual((int)M, D, D, att, W_o, b_o, u, h, ws, kWsHeaderBytes, stream);
    // channel_pre_norm -> GELU-gated up projection -> down projection + residual
    if (st == RGLRU_OK) st = rglru_rmsnorm((int)M, D, h, w_channel_norm, eps, n, stream);
    if (st == RGLRU_OK)
        st = rglru_linear_geglu((int)M, F, D, n, W_gate, b_gate, W_up, b_up, m, ws, kWsHeaderBytes, stream);
    if (st == RGLRU_OK) st = rglru_linear_residual((int)M, D, F, m, W_down, b_down, h, out, ws, kWsHeaderBytes, stream);
    return st;
}

}  // extern "C"
