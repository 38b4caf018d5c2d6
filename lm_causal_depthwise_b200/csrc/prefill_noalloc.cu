// prefill_noalloc.cu -- rglru_prefill_noalloc: the fused bf16 prefill with its
// scratch in a fixed device array, for callers that cannot allocate.
//
// Who needs it: code that must not call cudaMalloc (or any allocator) at the
// point where it runs the block -- a serving loop that planned all of its
// device memory at start-up and forbids allocation afterwards, a plug-in that
// is handed tensors but no allocator, or a caller that simply has no
// workspace buffer to pass.  Such a caller still owns and passes every input
// and output; only the kernel's scratch (ticket counters, per-tile flags and
// the cross-tile scan carry) lives here.
//
// The scratch is one file-scope __device__ array of kNoAllocScratchBytes.  Every
// GPU that loads the library holds it until the process exits.  All calls share
// it and it keeps the last call's contents, so each call first zeroes the words
// that must start at zero (status, test hook, tickets, flags).  Calls that can
// overlap on the GPU (two streams, or two host threads) race on it: callers
// must serialise them.
#include <mutex>

#include "internal.h"

namespace rglru {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB

static __device__ __align__(256) unsigned char g_prefill_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device; set up once per
// device index (the host symbol is only a stand-in and must never reach a
// kernel).  The cache assumes the device's context lives as long as the
// process: after a cudaDeviceReset the array may sit at another address, so
// a process that resets a device must not call this entry point on it again.
rglru_status scratch_address(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RGLRU_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return RGLRU_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_prefill_scratch) != cudaSuccess || ptr == nullptr)
            return RGLRU_ERR_CUDA;
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return RGLRU_OK;
}

}  // namespace
}  // namespace rglru

using namespace rglru;

extern "C" RGLRU_API rglru_status rglru_prefill_noalloc(int B, int T, int D, rglru_io_dtype dt, const void *x,
                                                        const void *gate_branch, const float *conv_w,
                                                        const float *conv_b, const void *W_a, const float *b_a,
                                                        const void *W_x, const float *b_x, const float *lambda,
                                                        const int32_t *segment_pos, void *conv_state,
                                                        float *h_state, void *y, cudaStream_t stream)
{
    if (dt != RGLRU_IO_BF16) return RGLRU_ERR_UNSUPPORTED;
    const size_t need = rglru_workspace_size(B, T, D, dt);
    if (need == 0) return RGLRU_ERR_INVALID_ARG;
    if (need > kNoAllocScratchBytes) return RGLRU_ERR_WORKSPACE;
    void *scratch = nullptr;
    const rglru_status st = scratch_address(&scratch);
    if (st != RGLRU_OK) return st;
    // status word, wait record and test hook from any earlier call back to zero
    // (the prefill itself zeroes the tickets and the tile flags)
    if (cudaMemsetAsync(scratch, 0, 4 * sizeof(int), stream) != cudaSuccess) return RGLRU_ERR_CUDA;
    return rglru_prefill(B, T, D, dt, x, gate_branch, conv_w, conv_b, W_a, b_a, W_x, b_x, lambda, segment_pos,
                         conv_state, h_state, y, scratch, kNoAllocScratchBytes, stream);
}
