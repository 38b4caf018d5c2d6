// simt_path.cu -- plain SIMT kernels of the RG-LRU block core (CUDA cores only).
//
// Two kernels, fp32 arithmetic with accurate transcendentals (no fast math):
//   1. simt_conv_gates: causal depthwise conv (k=4, document mask) and the two
//      block-diagonal gate pre-activations per (batch row, head, 32 tokens);
//   2. simt_scan: one thread per (batch row, channel), tokens in order:
//      sigmoid gates, a = sigmoid(Lambda)^(8 r), the sqrt(1-a^2) normalised
//      scan with resets, the tanh-GELU product, and the carried states.
// Structure of the block: "Gemma explained: RecurrentGemma architecture",
// RecurrentGemmaRecurrentBlock printout and section "Residual block with
// recurrent block"; RG-LRU equations of Griffin / RecurrentGemma (arXiv
// 2404.07839).  This path serves fp32 I/O (where the tensor-core path cannot
// meet a 1e-5 relative bar) and is a second, independent GPU implementation
// for cross-checks.
#include "internal.h"

namespace rglru {
namespace {

constexpr int kTT = 32;  // tokens per conv/gate block

template <typename IO> __device__ __forceinline__ float to_f(IO v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename IO> __device__ __forceinline__ IO from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

template <typename IO>
__global__ void __launch_bounds__(kHead)
simt_conv_gates(int T, int D, const IO *__restrict__ x, const float *__restrict__ conv_w,
                const float *__restrict__ conv_b, const IO *__restrict__ W_a,
                const float *__restrict__ b_a, const IO *__restrict__ W_x,
                const float *__restrict__ b_x, const int32_t *__restrict__ segpos,
                const IO *__restrict__ conv_state, float *__restrict__ xc_ws,
                float *__restrict__ pr_ws, float *__restrict__ pi_ws)
{
    __shared__ float sxc[kTT][kHead];
    const int j = threadIdx.x;
    const int hd = blockIdx.y;
    const int b = blockIdx.z;
    const int t0 = blockIdx.x * kTT;
    const int d = hd * kHead + j;
    const size_t rowB = (size_t)b * T;

    float w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = conv_w[(size_t)k * D + d];
    const float bias = conv_b[d];

    for (int tt = 0; tt < kTT; ++tt) {
        const int t = t0 + tt;
        float acc = 0.f;
        if (t < T) {
            const int pos = segpos[rowB + t];
            acc = bias;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int lag = 3 - k;
                if (lag <= pos) {
                    const int ts = t - lag;
                    const float xv = ts >= 0 ? to_f(x[(rowB + ts) * D + d])
                                             : to_f(conv_state[((size_t)b * 3 + 3 + ts) * D + d]);
                    acc = fmaf(w[k], xv, acc);
                }
            }
            xc_ws[(rowB + t) * D + d] = acc;
        }
        sxc[tt][j] = acc;
    }
    __syncthreads();

    float ar[kTT], ai[kTT];
    const float ba = b_a[d], bx = b_x[d];
#pragma unroll
    for (int tt = 0; tt < kTT; ++tt) { ar[tt] = ba; ai[tt] = bx; }
    const IO *wa = W_a + ((size_t)hd * kHead + j) * kHead;
    const IO *wx = W_x + ((size_t)hd * kHead + j) * kHead;
    for (int q = 0; q < kHead; ++q) {
        const float wav = to_f(wa[q]);
        const float wxv = to_f(wx[q]);
#pragma unroll
        for (int tt = 0; tt < kTT; ++tt) {
            const float v = sxc[tt][q];
            ar[tt] = fmaf(wav, v, ar[tt]);
            ai[tt] = fmaf(wxv, v, ai[tt]);
        }
    }
#pragma unroll
    for (int tt = 0; tt < kTT; ++tt) {
        const int t = t0 + tt;
        if (t < T) {
            pr_ws[(rowB + t) * D + d] = ar[tt];
            pi_ws[(rowB + t) * D + d] = ai[tt];
        }
    }
}

template <typename IO>
__global__ void __launch_bounds__(128)
simt_scan(int T, int D, const IO *__restrict__ x, const IO *__restrict__ g,
          const float *__restrict__ lambda, const int32_t *__restrict__ segpos,
          const float *__restrict__ xc_ws, const float *__restrict__ pr_ws,
          const float *__restrict__ pi_ws, IO *__restrict__ conv_state,
          float *__restrict__ h_state, IO *__restrict__ y)
{
    const int d = blockIdx.x * blockDim.x + threadIdx.x;
    const int b = blockIdx.y;
    if (d >= D) return;
    const size_t rowB = (size_t)b * T;
    const float lam = lambda[d];
    // log sigmoid(Lambda), in the branch that cannot overflow
    const float ls = lam >= 0.f ? -log1pf(expf(-lam)) : lam - log1pf(expf(lam));
    const float cls = kC * ls;
    float h = h_state[(size_t)b * D + d];
#pragma unroll 4
    for (int t = 0; t < T; ++t) {
        const size_t e = (rowB + t) * D + d;
        const int pos = segpos[rowB + t];
        const float r = 1.f / (1.f + expf(-pr_ws[e]));
        const float ig = 1.f / (1.f + expf(-pi_ws[e]));
        const float u = ig * xc_ws[e];
        if (pos == 0) {
            h = u;
        } else {
            const float ell = cls * r;
            const float a = expf(ell);
            const float m = sqrtf(-expm1f(2.f * ell));
            h = fmaf(a, h, m * u);
        }
        const float gv = to_f(g[e]);
        const float G = 0.5f * gv * (1.f + tanhf(0.7978845608028654f * (gv + 0.044715f * gv * gv * gv)));
        y[e] = from_f<IO>(G * h);
    }
    h_state[(size_t)b * D + d] = h;
    IO ncs[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        const int ts = T - 3 + k;
        ncs[k] = ts >= 0 ? x[(rowB + ts) * D + d] : conv_state[((size_t)b * 3 + 3 + ts) * D + d];
    }
#pragma unroll
    for (int k = 0; k < 3; ++k) conv_state[((size_t)b * 3 + k) * D + d] = ncs[k];
}

template <typename IO>
rglru_status launch(const PrefillArgs &a)
{
    const size_t n = (size_t)a.B * a.T * a.D;
    char *base = static_cast<char *>(a.ws) + kWsHeaderBytes;
    float *xc_ws = reinterpret_cast<float *>(base);
    float *pr_ws = xc_ws + n;
    float *pi_ws = pr_ws + n;
    const int H = a.D / kHead;
    dim3 g1((a.T + kTT - 1) / kTT, H, a.B);
    simt_conv_gates<IO><<<g1, kHead, 0, a.stream>>>(
        a.T, a.D, static_cast<const IO *>(a.x), a.conv_w, a.conv_b, static_cast<const IO *>(a.W_a),
        a.b_a, static_cast<const IO *>(a.W_x), a.b_x, a.segpos,
        static_cast<const IO *>(a.conv_state), xc_ws, pr_ws, pi_ws);
    if (cudaGetLastError() != cudaSuccess) return RGLRU_ERR_CUDA;
    dim3 g2((a.D + 127) / 128, a.B);
    simt_scan<IO><<<g2, 128, 0, a.stream>>>(
        a.T, a.D, static_cast<const IO *>(a.x), static_cast<const IO *>(a.g), a.lambda, a.segpos,
        xc_ws, pr_ws, pi_ws, static_cast<IO *>(a.conv_state), a.h_state, static_cast<IO *>(a.y));
    return cuda_status(cudaGetLastError());
}

}  // namespace

size_t simt_workspace_bytes(int B, int T, int D)
{
    return kWsHeaderBytes + align_up(3 * (size_t)B * T * D * sizeof(float), 256);
}

rglru_status simt_prefill(const PrefillArgs &a)
{
    return a.dt == RGLRU_IO_F32 ? launch<float>(a) : launch<__nv_bfloat16>(a);
}

}  // namespace rglru
