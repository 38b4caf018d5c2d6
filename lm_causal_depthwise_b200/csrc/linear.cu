// linear.cu -- dense projections of the recurrent block on sm_100a tensor cores:
// out[M, N] = A[M, K] W[N, K]^T + bias (torch Linear layout, bf16 operands,
// fp32 accumulation, bf16 out), with the epilogues the block needs.
//
// Where they sit: "Gemma explained: RecurrentGemma architecture", the
// RecurrentGemmaRecurrentBlock printout (linear_y, linear_x, linear_out:
// Linear(2560, 2560, bias=True)) and section "Residual block with recurrent
// block": the block input feeds linear_x (then the conv and the RG-LRU) and
// linear_y (the GELU branch); the product of the branches feeds linear_out.
// The same page's RecurrentGemmaMlp printout (gate_proj, up_proj 2560 -> 7680,
// down_proj 7680 -> 2560, GELU tanh) gives the MLP that follows each
// temporal block.
//
// One persistent kernel, one CTA per SM, 192 threads:
//   warp 0      TMA producer: per K-block of 64, the A tile [128 x 64] and the
//               W tile [256 x 64] (128-byte swizzle, K-major) into a 4-deep
//               shared-memory ring;
//   warp 1      MMA issuer (one thread): 4 x tcgen05.mma (M=128, N=256, K=16)
//               per K-block into one of two TMEM accumulators (256 columns
//               each), committing the ring slot back to the producer and the
//               finished accumulator to the epilogue;
//   warps 2..5  epilogue: thread = output row (TMEM lane), 32 columns per
//               tcgen05.ld; bias (and the residual or the GELU gate) in fp32,
//               bf16 stores straight from registers.  The accumulator is free
//               for the tile after next as soon as it has been read, so the
//               epilogue of tile i overlaps the MMAs of tile i + 1.
// Tiles are taken in order t = blockIdx.x + i * gridDim.x with the N block
// fastest, so the CTAs running at once share A tiles (and all of W) in L2.
// Every mbarrier wait is bounded (2 s): one that runs out records
// RGLRU_ERR_TIMEOUT in the workspace header and the CTA unwinds; all threads
// meet at the final CTA barrier before TMEM is freed.
#include "internal.h"
#include "sm100.cuh"

namespace rglru {
namespace {

using namespace sm100;

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int kThreads = 192;
constexpr int kATile = BM * BK * 2;     // 16 KB
constexpr int kBTile = BN * BK * 2;     // 32 KB
constexpr int kStage = kATile + kBTile;
constexpr int OFF_BAR = STAGES * kStage;
enum { BAR_FULL = 0, BAR_EMPTY = BAR_FULL + STAGES, BAR_ACC_FULL = BAR_EMPTY + STAGES, BAR_ACC_EMPTY = BAR_ACC_FULL + 2,
       BAR_DRAIN = BAR_ACC_EMPTY + 2, BAR_N = BAR_DRAIN + 1 };
constexpr int OFF_MISC = OFF_BAR + BAR_N * 8;
constexpr int kSmemBytes = OFF_MISC + 16 + 1024;  // + slack for the 1024-byte alignment
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
constexpr uint64_t kTimeoutNs = 2000000000ull;

// Epilogue kinds.
enum Epilogue : int {
    EPI_BIAS = 0,           // out = acc + bias
    EPI_BIAS_RESIDUAL = 1,  // out = acc + bias + residual            (residual [M, N] bf16)
    EPI_GEGLU = 2,          // out[:, j] = GELU_tanh(acc_g + b_g) * (acc_u + b_u): the W tile is
                            // 128 rows of W_gate then 128 rows of W_up, out has N / 2 columns
};

struct LinearParams {
    int M, N, K;             // N: columns of the accumulator (W rows used per launch)
    int n_split;             // N blocks below n_split use set 0, the rest set 1 (columns restart at 0)
    int epi;
    const float *bias0, *bias1;
    const __nv_bfloat16 *res0;
    __nv_bfloat16 *out0, *out1;
    int ld_out;              // columns of each output matrix
    WsHeader *hdr;
};

__device__ __noinline__ bool lin_wait_slow(uint64_t *bar, uint32_t parity, WsHeader *hdr, int where)
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
__device__ __forceinline__ bool lin_wait(uint64_t *bar, uint32_t parity, WsHeader *hdr, int where)
{
    if (mbar_try_wait(bar, parity)) return true;
    return lin_wait_slow(bar, parity, hdr, where);
}

// every lane of the warp waits; the warp's verdict is unanimous
__device__ __forceinline__ bool lin_warp_wait(uint64_t *bar, uint32_t parity, WsHeader *hdr, int where)
{
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = lin_wait(bar, parity, hdr, where);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (ok) {
        // complete already: each lane's own test passes, giving it the acquire
        while (!mbar_try_wait(bar, parity)) {
        }
    }
    return ok;
}

__device__ __forceinline__ float gelu_tanh_f(float g)
{
    const float k0 = 0.7978845608028654f, k1 = 0.7978845608028654f * 0.044715f;
    const float u = g * fmaf(k1 * g, g, k0);
    const float hg = 0.5f * g;
    return fmaf(hg, tanh_approx(u), hg);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__global__ void __launch_bounds__(kThreads, 1)
rglru_linear_kernel(const LinearParams p, const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_b0, const __grid_constant__ CUtensorMap tm_b1)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    const int num_m = (p.M + BM - 1) / BM, num_n = p.N / BN, num_k = p.K / BK;
    const int tiles = num_m * num_n;

    if (warp == 1) {
        tmem_alloc(tmem_holder, 512);
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(bars + BAR_FULL + s, 1);
                mbar_init(bars + BAR_EMPTY + s, 1);
            }
            for (int a = 0; a < 2; ++a) {
                mbar_init(bars + BAR_ACC_FULL + a, 1);
                mbar_init(bars + BAR_ACC_EMPTY + a, 4 * 32);
            }
            mbar_init(bars + BAR_DRAIN, 1);
            mbar_fence_init();
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const int nb = t % num_n, mb = t / num_n;
                const bool set1 = nb >= p.n_split;
                const int ncol = (set1 ? nb - p.n_split : nb) * BN;
                const CUtensorMap *tb = set1 ? &tm_b1 : &tm_b0;
                for (int kb = 0; kb < num_k; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (it >= STAGES && !(ok = lin_wait(bars + BAR_EMPTY + s, (uint32_t)((it / STAGES) - 1) & 1u, p.hdr, 0)))
                        break;
                    uint8_t *st = smem + s * kStage;
                    mbar_arrive_expect_tx(bars + BAR_FULL + s, kStage);
                    tma_load_2d(st, &tm_a, bars + BAR_FULL + s, kb * BK, mb * BM);
                    if (p.epi == EPI_GEGLU) {
                        // 128 rows of W_gate, then the same 128 rows of W_up
                        tma_load_2d(st + kATile, &tm_b0, bars + BAR_FULL + s, kb * BK, nb * (BN / 2));
                        tma_load_2d(st + kATile + kBTile / 2, &tm_b1, bars + BAR_FULL + s, kb * BK, nb * (BN / 2));
                    } else {
                        tma_load_2d(st + kATile, tb, bars + BAR_FULL + s, kb * BK, ncol);
                    }
                }
            }
            if (!ok) {
                // the loads already issued land before the CTA exits (bounded)
                for (int k = max(0, it - STAGES); k < it; ++k) {
                    const uint64_t t0 = globaltimer();
                    while (!mbar_try_wait(bars + BAR_FULL + k % STAGES, (uint32_t)(k / STAGES) & 1u) &&
                           globaltimer() - t0 < kTimeoutNs) {
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_bf16(BM, BN);
            int it = 0, i = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++i) {
                const int a = i & 1;
                if (i >= 2 && !(ok = lin_wait(bars + BAR_ACC_EMPTY + a, (uint32_t)((i >> 1) - 1) & 1u, p.hdr, 1)))
                    break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(a * BN);
                for (int kb = 0; kb < num_k; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (!(ok = lin_wait(bars + BAR_FULL + s, (uint32_t)(it / STAGES) & 1u, p.hdr, 2))) break;
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * kStage), sb = sa + kATile;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        umma_ss(d, umma_desc_sw128(sa + kk * 32), umma_desc_sw128(sb + kk * 32), idesc,
                                (kb | kk) != 0);
                    umma_commit(bars + BAR_EMPTY + s);
                }
                if (ok) umma_commit(bars + BAR_ACC_FULL + a);
            }
            if (!ok) {
                // the MMAs in flight finish before TMEM is freed (bounded wait)
                umma_commit(bars + BAR_DRAIN);
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(bars + BAR_DRAIN, 0) && globaltimer() - t0 < kTimeoutNs) {
                }
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;                       // TMEM lane quarter of this warp
        const int row_in_tile = q * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
        int i = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
            const int a = i & 1;
            if (!lin_warp_wait(bars + BAR_ACC_FULL + a, (uint32_t)(i >> 1) & 1u, p.hdr, 3)) break;
            tc_fence_after();
            const int nb = t % num_n, mb = t / num_n;
            const int row = mb * BM + row_in_tile;
            const bool live = row < p.M;
            if (p.epi == EPI_GEGLU) {
                // columns [0, 128): gate, [128, 256): up, for output columns nb * 128 + j
                const int oc0 = nb * (BN / 2);
                __nv_bfloat16 *orow = p.out0 + (size_t)row * p.ld_out + oc0;
#pragma unroll 1
                for (int c = 0; c < BN / 2; c += 32) {
                    uint32_t gv[32], uv[32];
                    tmem_ld32(lane_base + (uint32_t)(a * BN + c), gv);
                    tmem_ld32(lane_base + (uint32_t)(a * BN + BN / 2 + c), uv);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        const float g0 = __uint_as_float(gv[j]) + __ldg(p.bias0 + oc0 + c + j);
                        const float g1 = __uint_as_float(gv[j + 1]) + __ldg(p.bias0 + oc0 + c + j + 1);
                        const float u0 = __uint_as_float(uv[j]) + __ldg(p.bias1 + oc0 + c + j);
                        const float u1 = __uint_as_float(uv[j + 1]) + __ldg(p.bias1 + oc0 + c + j + 1);
                        pk[j >> 1] = pack_bf16(gelu_tanh_f(g0) * u0, gelu_tanh_f(g1) * u1);
                    }
                    if (live) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + c);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                    }
                }
            } else {
                const bool set1 = nb >= p.n_split;
                const int oc0 = (set1 ? nb - p.n_split : nb) * BN;
                const float *bias = set1 ? p.bias1 : p.bias0;
                __nv_bfloat16 *orow = (set1 ? p.out1 : p.out0) + (size_t)row * p.ld_out + oc0;
                const __nv_bfloat16 *rrow = p.epi == EPI_BIAS_RESIDUAL ? p.res0 + (size_t)row * p.ld_out + oc0 : nullptr;
#pragma unroll 1
                for (int c = 0; c < BN; c += 32) {
                    uint32_t v[32];
                    tmem_ld32(lane_base + (uint32_t)(a * BN + c), v);
                    tmem_wait_ld();
                    float f[32];
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const float4 b4 = bias ? __ldg(reinterpret_cast<const float4 *>(bias + oc0 + c + j))
                                               : make_float4(0.f, 0.f, 0.f, 0.f);
                        f[j] = __uint_as_float(v[j]) + b4.x;
                        f[j + 1] = __uint_as_float(v[j + 1]) + b4.y;
                        f[j + 2] = __uint_as_float(v[j + 2]) + b4.z;
                        f[j + 3] = __uint_as_float(v[j + 3]) + b4.w;
                    }
                    if (p.epi == EPI_BIAS_RESIDUAL && live) {
                        const uint4 *rs = reinterpret_cast<const uint4 *>(rrow + c);
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4) {
                            const uint4 r = __ldg(rs + v4);
                            const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                f[8 * v4 + 2 * e] += __uint_as_float(rw[e] << 16);
                                f[8 * v4 + 2 * e + 1] += __uint_as_float(rw[e] & 0xffff0000u);
                            }
                        }
                    }
                    if (live) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + c);
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4)
                            dst[v4] = make_uint4(pack_bf16(f[8 * v4], f[8 * v4 + 1]), pack_bf16(f[8 * v4 + 2], f[8 * v4 + 3]),
                                                 pack_bf16(f[8 * v4 + 4], f[8 * v4 + 5]), pack_bf16(f[8 * v4 + 6], f[8 * v4 + 7]));
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(bars + BAR_ACC_EMPTY + a);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace

size_t linear_workspace_bytes() { return kWsHeaderBytes; }

rglru_status linear_launch(const LinearArgs &a)
{
    if (a.M < 1 || a.K < BK || a.K % BK != 0 || a.n_out < 1) return RGLRU_ERR_INVALID_ARG;
    const bool geglu = a.epi == EPI_GEGLU;
    if (a.A == nullptr || a.W0 == nullptr || a.out0 == nullptr || a.ws == nullptr) return RGLRU_ERR_INVALID_ARG;
    if (geglu && (a.W1 == nullptr || a.bias0 == nullptr || a.bias1 == nullptr)) return RGLRU_ERR_INVALID_ARG;
    if (a.epi == EPI_BIAS_RESIDUAL && a.residual == nullptr) return RGLRU_ERR_INVALID_ARG;
    if (!geglu && a.W1 != nullptr && a.out1 == nullptr) return RGLRU_ERR_INVALID_ARG;
    // accumulator columns per set: the W rows a launch multiplies
    const int n0 = geglu ? 2 * a.n_out : a.n_out;
    if (geglu ? (a.n_out % (BN / 2) != 0) : (a.n_out % BN != 0)) return RGLRU_ERR_UNSUPPORTED;
    if ((size_t)a.M > 0x7fffffffull / 2) return RGLRU_ERR_UNSUPPORTED;
    auto encode = encode_fn();
    if (!encode) return RGLRU_ERR_CUDA;
    CUtensorMap tm_a, tm_b0, tm_b1;
    const cuuint64_t adim[2] = {(cuuint64_t)a.K, (cuuint64_t)a.M}, astride[1] = {(cuuint64_t)a.K * 2};
    const cuuint32_t abox[2] = {BK, BM};
    if (!encode_bf16(encode, &tm_a, a.A, 2, adim, astride, abox, CU_TENSOR_MAP_SWIZZLE_128B)) return RGLRU_ERR_CUDA;
    const cuuint64_t bdim[2] = {(cuuint64_t)a.K, (cuuint64_t)a.n_out}, bstride[1] = {(cuuint64_t)a.K * 2};
    const cuuint32_t bbox[2] = {BK, geglu ? (cuuint32_t)(BN / 2) : (cuuint32_t)BN};
    if (!encode_bf16(encode, &tm_b0, a.W0, 2, bdim, bstride, bbox, CU_TENSOR_MAP_SWIZZLE_128B)) return RGLRU_ERR_CUDA;
    if (!encode_bf16(encode, &tm_b1, a.W1 ? a.W1 : a.W0, 2, bdim, bstride, bbox, CU_TENSOR_MAP_SWIZZLE_128B))
        return RGLRU_ERR_CUDA;

    LinearParams p;
    p.M = a.M;
    p.K = a.K;
    p.epi = a.epi;
    p.bias0 = a.bias0;
    p.bias1 = a.bias1;
    p.res0 = static_cast<const __nv_bfloat16 *>(a.residual);
    p.out0 = static_cast<__nv_bfloat16 *>(a.out0);
    p.out1 = static_cast<__nv_bfloat16 *>(a.out1);
    p.ld_out = a.n_out;
    p.hdr = static_cast<WsHeader *>(a.ws);
    if (geglu) {
        p.N = n0;          // gate and up rows interleaved per tile of 256 accumulator columns
        p.n_split = 1 << 30;
    } else if (a.W1) {
        p.N = 2 * a.n_out;  // set 0 then set 1
        p.n_split = a.n_out / BN;
    } else {
        p.N = a.n_out;
        p.n_split = 1 << 30;
    }
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RGLRU_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return RGLRU_ERR_CUDA;
    static PerDeviceFlag smem_set;
    const rglru_status st = set_smem_limit_once((const void *)rglru_linear_kernel, kSmemBytes, smem_set);
    if (st != RGLRU_OK) return st;
    const long long tiles = (long long)((a.M + BM - 1) / BM) * (p.N / BN);
    const int grid = (int)(tiles < sms ? tiles : sms);
    rglru_linear_kernel<<<grid, kThreads, kSmemBytes, a.stream>>>(p, tm_a, tm_b0, tm_b1);
    return cuda_status(cudaGetLastError());
}

}  // namespace rglru
