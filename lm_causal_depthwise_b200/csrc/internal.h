// internal.h -- shared declarations of the librglru CUDA sources (not part of the ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <mutex>

#include "rglru.h"

namespace rglru {

constexpr int kHead = 256;      // channels per head (gate blocks are 256 x 256)
constexpr float kC = 8.0f;      // exponent scale in a = sigmoid(Lambda)^(c r)

// Workspace header.  A zero-filled header is the valid initial state.
struct WsHeader {
    int status;            // rglru_status recorded by device code (0 = OK)
    int detail;            // first wait that gave up: (CTA << 8) | (wait site + 1), 0 = none
    int debug_unit_plus1;  // test hook: chunk that skips publishing (+1), 0 = off
    int pad0;
    unsigned int ticket[1000];  // per-group work counters of the fused prefill kernel
};
constexpr size_t kWsHeaderBytes = 4096;
static_assert(sizeof(WsHeader) <= kWsHeaderBytes, "header too large");

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct PrefillArgs {
    int B, T, D;
    rglru_io_dtype dt;
    const void *x, *g;
    const float *conv_w, *conv_b;
    const void *W_a;
    const float *b_a;
    const void *W_x;
    const float *b_x;
    const float *lambda;
    const int32_t *segpos;
    void *conv_state;
    float *h_state;
    void *y;
    void *ws;
    size_t ws_bytes;
    cudaStream_t stream;
};

// Synchronous argument checks of a prefill or decode call (rglru_api.cu): io
// dtype, sizes, non-null 16-byte aligned pointers, no overlap between y, the
// inputs, the states and the workspace, and a workspace of `need` bytes.
rglru_status validate_prefill(const PrefillArgs &a, size_t need);

// SIMT path (simt_path.cu)
size_t simt_workspace_bytes(int B, int T, int D);
rglru_status simt_prefill(const PrefillArgs &a);

// Fused sm_100a prefill (prefill_fused.cu); returns RGLRU_ERR_UNSUPPORTED when
// the shape is outside what the kernel handles.
size_t fused_workspace_bytes(int B, int T, int D);
rglru_status fused_prefill(const PrefillArgs &a);

// Dense projections on the tensor cores (linear.cu).
struct LinearArgs {
    int M, n_out, K;         // A [M, K]; each W [n_out, K]; each out [M, n_out]
    int epi;                 // 0: bias, 1: bias + residual, 2: GELU_tanh(A W0^T + b0) * (A W1^T + b1)
    const void *A;
    const void *W0, *W1;     // W1: second projection of the same A (epi 0), or W_up (epi 2); else null
    const float *bias0, *bias1;
    const void *residual;    // [M, n_out] (epi 1)
    void *out0, *out1;
    void *ws;                // workspace header (device status)
    cudaStream_t stream;
};
size_t linear_workspace_bytes();
rglru_status linear_launch(const LinearArgs &a);

// RMSNorm of bf16 rows (rmsnorm.cu): out = x * rsqrt(mean(x^2) + eps) * w.
rglru_status rmsnorm_launch(int M, int N, const void *x, const float *w, float eps, void *out, cudaStream_t stream);

// Batched decode step (decode.cu)
size_t decode_workspace_bytes(int B, int D);
rglru_status decode_step(const PrefillArgs &a);

inline rglru_status cuda_status(cudaError_t e) { return e == cudaSuccess ? RGLRU_OK : RGLRU_ERR_CUDA; }

// Per-device record of a one-time kernel attribute: the dynamic shared-memory
// limit set by cudaFuncSetAttribute holds for the device that was current, so
// it is set once for each device index (below kMaxDevices) a process uses.
constexpr int kMaxDevices = 64;
struct PerDeviceFlag {
    bool done[kMaxDevices] = {};
};
// Sets `kernel`'s dynamic shared-memory limit to `bytes` on the current
// device unless `flag` records it as done there (rglru_api.cu).
rglru_status set_smem_limit_once(const void *kernel, int bytes, PerDeviceFlag &flag);

// cuTensorMapEncodeTiled from the driver (nullptr if unavailable), and a bf16
// tiled tensor map of `rank` dimensions (innermost first; strides in bytes of
// dimensions 1..rank-1) with zero fill out of bounds (rglru_api.cu).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();
bool encode_bf16(PFN_cuTensorMapEncodeTiled_v12000 encode, CUtensorMap *m, const void *base, int rank,
                 const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box, CUtensorMapSwizzle sw);

}  // namespace rglru
