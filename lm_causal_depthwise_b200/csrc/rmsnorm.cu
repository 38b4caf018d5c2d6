// rmsnorm.cu -- RMSNorm of bf16 rows on sm_100a: out = x * rsqrt(mean(x^2) + eps) * w.
//
// "Gemma explained: RecurrentGemma architecture", the RecurrentGemmaRMSNorm
// modules of the decoder-layer printout (temporal_pre_norm before the
// temporal block, channel_pre_norm before the MLP) and section "Residual
// block with recurrent block" (RMSNorm, then the block, the residual add,
// RMSNorm, the MLP).  The pages print the module names only; the
// normalisation is the standard root-mean-square one with a learned scale.
//
// One warp per row, the row read once into registers with 16-byte loads
// (8 bf16 per load), the sum of squares in fp32 reduced by shuffles, the
// scaled row written with 16-byte stores.  The kernel is bandwidth bound:
// 4 bytes per element (bf16 in, bf16 out).  Rows per CTA: 8 warps; the grid
// covers the rows once.
#include "internal.h"

namespace rglru {
namespace {

constexpr int kWarps = 8;
constexpr int kMaxVecPerLane = 16;  // rows of up to 16 * 8 * 32 = 4096 elements

template <int VPL>
__global__ void __launch_bounds__(kWarps * 32)
rglru_rmsnorm_kernel(int M, int N, const __nv_bfloat16 *__restrict__ x, const float *__restrict__ w, float eps,
                     __nv_bfloat16 *__restrict__ out)
{
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (row >= M) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + row * N);
    const int nvec = N / 8;
    uint4 v[VPL];
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        const int i = k * 32 + lane;
        v[k] = i < nvec ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
        const uint32_t q[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float lo = __uint_as_float(q[e] << 16), hi = __uint_as_float(q[e] & 0xffff0000u);
            ss = fmaf(lo, lo, ss);
            ss = fmaf(hi, hi, ss);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(ss / (float)N + eps);
    uint4 *dst = reinterpret_cast<uint4 *>(out + row * N);
    const float4 *w4 = reinterpret_cast<const float4 *>(w);
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        const int i = k * 32 + lane;
        if (i < nvec) {
            const float4 wa = __ldg(w4 + 2 * i), wb = __ldg(w4 + 2 * i + 1);
            const float ws[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
            const uint32_t q[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
            uint32_t r[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float lo = __uint_as_float(q[e] << 16) * inv * ws[2 * e];
                const float hi = __uint_as_float(q[e] & 0xffff0000u) * inv * ws[2 * e + 1];
                asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r[e]) : "f"(hi), "f"(lo));
            }
            dst[i] = make_uint4(r[0], r[1], r[2], r[3]);
        }
    }
}

}  // namespace

rglru_status rmsnorm_launch(int M, int N, const void *x, const float *w, float eps, void *out, cudaStream_t stream)
{
    if (M < 1 || N < 8 || N % 8 != 0 || N > kMaxVecPerLane * 8 * 32) return RGLRU_ERR_UNSUPPORTED;
    const unsigned grid = (unsigned)((M + kWarps - 1) / kWarps);
    const auto *xb = static_cast<const __nv_bfloat16 *>(x);
    auto *ob = static_cast<__nv_bfloat16 *>(out);
    const int vpl = (N / 8 + 31) / 32;
    if (vpl <= 4)
        rglru_rmsnorm_kernel<4><<<grid, kWarps * 32, 0, stream>>>(M, N, xb, w, eps, ob);
    else if (vpl <= 8)
        rglru_rmsnorm_kernel<8><<<grid, kWarps * 32, 0, stream>>>(M, N, xb, w, eps, ob);
    else
        rglru_rmsnorm_kernel<16><<<grid, kWarps * 32, 0, stream>>>(M, N, xb, w, eps, ob);
    return cuda_status(cudaGetLastError());
}

}  // namespace rglru
