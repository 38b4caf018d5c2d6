// internal.h -- shared declarations of the librglru CUDA sources (not part of the ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

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

// Batched decode step (decode.cu)
size_t decode_workspace_bytes(int B, int D);
rglru_status decode_step(const PrefillArgs &a);

inline rglru_status cuda_status(cudaError_t e) { return e == cudaSuccess ? RGLRU_OK : RGLRU_ERR_CUDA; }

}  // namespace rglru
