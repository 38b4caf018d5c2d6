// carry.cu -- the carried scan state across time shards of one long prefill.
//
// The RG-LRU recurrence h_t = a_t h_{t-1} + b_t ("RecurrentGemma: Moving Past
// Transformers for Efficient Open Language Models", the RG-LRU equations; a_t
// and b_t depend on the inputs only) is affine in the state a chunk starts
// from: a chunk that starts from h_in ends in
//     h_end = A h_in + H0   (per channel),
// A the product of the chunk's decays (0 when the chunk holds a document
// start) and H0 the end state from h_in = 0.  A rank that holds one time
// chunk of a long sequence runs its chunk from 0 and from 1, which gives H0
// and H1 = A + H0; after an all-gather of those pairs every rank folds them in
// rank order:
//     h_in_0 = h0,    h_in_{r+1} = (H1_r - H0_r) h_in_r + H0_r,
// and runs its chunk once more from its own h_in_r.  This kernel is the fold.
#include "internal.h"

namespace rglru {
namespace {

__global__ void __launch_bounds__(256)
rglru_carry_scan_kernel(int N, size_t BD, const float *__restrict__ H0, const float *__restrict__ H1,
                        const float *__restrict__ h0, float *__restrict__ h_in)
{
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < BD; e += (size_t)gridDim.x * blockDim.x) {
        float h = h0[e];
        for (int r = 0; r < N; ++r) {
            const size_t i = (size_t)r * BD + e;
            h_in[i] = h;
            h = fmaf(H1[i] - H0[i], h, H0[i]);
        }
    }
}

}  // namespace
}  // namespace rglru

using namespace rglru;

extern "C" RGLRU_API rglru_status rglru_carry_scan(int N, int B, int D, const float *H0, const float *H1,
                                                   const float *h0, float *h_in, cudaStream_t stream)
{
    if (N < 1 || B < 1 || D < 1 || (int64_t)B * D > (int64_t(1) << 40) / N) return RGLRU_ERR_INVALID_ARG;
    if (H0 == nullptr || H1 == nullptr || h0 == nullptr || h_in == nullptr) return RGLRU_ERR_INVALID_ARG;
    const size_t BD = (size_t)B * D, all = (size_t)N * BD * 4;
    const uintptr_t o0 = reinterpret_cast<uintptr_t>(h_in), o1 = o0 + all;
    const struct {
        const void *p;
        size_t n;
    } ins[] = {{H0, all}, {H1, all}, {h0, BD * 4}};
    for (const auto &s : ins) {
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(s.p), a1 = a0 + s.n;
        if (a0 < o1 && o0 < a1) return RGLRU_ERR_INVALID_ARG;
    }
    const size_t blocks = (BD + 255) / 256;
    rglru_carry_scan_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, stream>>>(N, BD, H0, H1, h0, h_in);
    return cuda_status(cudaGetLastError());
}
