// block_api.cu -- C ABI of the dense projections, RMSNorm, the whole
// recurrent block (linear_x / linear_y -> conv + RG-LRU core -> linear_out)
// and the whole recurrent residual block (RMSNorm, recurrent block, residual,
// RMSNorm, GELU-gated MLP, residual).
//
// Structure: "Gemma explained: RecurrentGemma architecture", the
// RecurrentGemmaRecurrentBlock printout (linear_y, linear_x, linear_out, each
// Linear(2560, 2560, bias=True); conv_1d; rg_lru; GELU tanh) and section
// "Residual block with recurrent block" (the input feeds both branches; the
// GELU branch multiplies the conv + RG-LRU branch; linear_out follows).  The
// MLP entry point follows the RecurrentGemmaMlp printout (gate_proj, up_proj,
// down_proj, GELU tanh on the gate).
//
// Every entry point validates synchronously and enqueues work on `stream`;
// nothing here allocates or synchronises.
#include <cstdint>

#include "internal.h"

using namespace rglru;

namespace {

bool al16(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Span {
    uintptr_t lo, hi;
};
Span span(const void *p, size_t bytes)
{
    const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
    return {lo, lo + bytes};
}
bool meet(Span a, Span b) { return a.lo < b.hi && b.lo < a.hi; }

constexpr int64_t kMaxRows = int64_t(1) << 30;

bool linear_sizes_ok(int M, int N, int K, int n_multiple)
{
    return M >= 1 && M <= kMaxRows && N >= n_multiple && N % n_multiple == 0 && K >= 64 && K % 64 == 0 &&
           N <= (1 << 20) && K <= (1 << 20);
}

rglru_status check_ws(void *ws, size_t bytes, size_t need)
{
    if (ws == nullptr || !al16(ws) || bytes < need) return RGLRU_ERR_WORKSPACE;
    return RGLRU_OK;
}

// out must not overlap any input (out == residual exactly is allowed: each
// element is read and written by the same thread)
bool out_clear(Span out, std::initializer_list<Span> ins) {
    for (const Span &s : ins)
        if (meet(out, s)) return false;
    return true;
}

}  // namespace

extern "C" {

RGLRU_API size_t rglru_linear_workspace_size(void) { return linear_workspace_bytes(); }

RGLRU_API rglru_status rglru_linear(int M, int N, int K, const void *A, const void *W, const float *bias,
                                    void *out, void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    if (!linear_sizes_ok(M, N, K, 256)) return RGLRU_ERR_UNSUPPORTED;
    if (!al16(A) || !al16(W) || !al16(out) || (bias != nullptr && !al16(bias))) return RGLRU_ERR_INVALID_ARG;
    const size_t a_b = (size_t)M * K * 2, w_b = (size_t)N * K * 2, o_b = (size_t)M * N * 2;
    if (!out_clear(span(out, o_b), {span(A, a_b), span(W, w_b), span(bias, bias ? N * 4 : 0),
                                    span(workspace, workspace_bytes)}))
        return RGLRU_ERR_INVALID_ARG;
    const rglru_status st = check_ws(workspace, workspace_bytes, linear_workspace_bytes());
    if (st != RGLRU_OK) return st;
    LinearArgs a{};
    a.M = M; a.n_out = N; a.K = K; a.epi = 0;
    a.A = A; a.W0 = W; a.bias0 = bias; a.out0 = out; a.ws = workspace; a.stream = stream;
    return linear_launch(a);
}

RGLRU_API rglru_status rglru_linear_pair(int M, int N, int K, const void *A, const void *W0, const float *bias0,
                                         void *out0, const void *W1, const float *bias1, void *out1,
                                         void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    if (!linear_sizes_ok(M, N, K, 256)) return RGLRU_ERR_UNSUPPORTED;
    if (!al16(A) || !al16(W0) || !al16(W1) || !al16(out0) || !al16(out1) || (bias0 && !al16(bias0)) ||
        (bias1 && !al16(bias1)))
        return RGLRU_ERR_INVALID_ARG;
    const size_t a_b = (size_t)M * K * 2, w_b = (size_t)N * K * 2, o_b = (size_t)M * N * 2;
    const Span ins[] = {span(A, a_b), span(W0, w_b), span(W1, w_b), span(bias0, bias0 ? N * 4 : 0),
                        span(bias1, bias1 ? N * 4 : 0), span(workspace, workspace_bytes)};
    for (const Span &s : ins)
        if (meet(span(out0, o_b), s) || meet(span(out1, o_b), s)) return RGLRU_ERR_INVALID_ARG;
    if (meet(span(out0, o_b), span(out1, o_b))) return RGLRU_ERR_INVALID_ARG;
    const rglru_status st = check_ws(workspace, workspace_bytes, linear_workspace_bytes());
    if (st != RGLRU_OK) return st;
    LinearArgs a{};
    a.M = M; a.n_out = N; a.K = K; a.epi = 0;
    a.A = A; a.W0 = W0; a.W1 = W1; a.bias0 = bias0; a.bias1 = bias1; a.out0 = out0; a.out1 = out1;
    a.ws = workspace; a.stream = stream;
    return linear_launch(a);
}

RGLRU_API rglru_status rglru_linear_residual(int M, int N, int K, const void *A, const void *W, const float *bias,
                                             const void *residual, void *out, void *workspace,
                                             size_t workspace_bytes, cudaStream_t stream)
{
    if (!linear_sizes_ok(M, N, K, 256)) return RGLRU_ERR_UNSUPPORTED;
    if (!al16(A) || !al16(W) || !al16(residual) || !al16(out) || (bias && !al16(bias)))
        return RGLRU_ERR_INVALID_ARG;
    const size_t a_b = (size_t)M * K * 2, w_b = (size_t)N * K * 2, o_b = (size_t)M * N * 2;
    if (!out_clear(span(out, o_b), {span(A, a_b), span(W, w_b), span(bias, bias ? N * 4 : 0),
                                    span(workspace, workspace_bytes)}))
        return RGLRU_ERR_INVALID_ARG;
    if (residual != out && meet(span(out, o_b), span(residual, o_b))) return RGLRU_ERR_INVALID_ARG;
    const rglru_status st = check_ws(workspace, workspace_bytes, linear_workspace_bytes());
    if (st != RGLRU_OK) return st;
    LinearArgs a{};
    a.M = M; a.n_out = N; a.K = K; a.epi = 1;
    a.A = A; a.W0 = W; a.bias0 = bias; a.residual = residual; a.out0 = out; a.ws = workspace; a.stream = stream;
    return linear_launch(a);
}

RGLRU_API rglru_status rglru_linear_geglu(int M, int N, int K, const void *A, const void *W_gate,
                                          const float *b_gate, const void *W_up, const float *b_up, void *out,
                                          void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    if (!linear_sizes_ok(M, N, K, 128)) return RGLRU_ERR_UNSUPPORTED;
    if (!al16(A) || !al16(W_gate) || !al16(W_up) || !al16(b_gate) || !al16(b_up) || !al16(out))
        return RGLRU_ERR_INVALID_ARG;
    const size_t a_b = (size_t)M * K * 2, w_b = (size_t)N * K * 2, o_b = (size_t)M * N * 2;
    if (!out_clear(span(out, o_b), {span(A, a_b), span(W_gate, w_b), span(W_up, w_b), span(b_gate, N * 4),
                                    span(b_up, N * 4), span(workspace, workspace_bytes)}))
        return RGLRU_ERR_INVALID_ARG;
    const rglru_status st = check_ws(workspace, workspace_bytes, linear_workspace_bytes());
    if (st != RGLRU_OK) return st;
    LinearArgs a{};
    a.M = M; a.n_out = N; a.K = K; a.epi = 2;
    a.A = A; a.W0 = W_gate; a.W1 = W_up; a.bias0 = b_gate; a.bias1 = b_up; a.out0 = out;
    a.ws = workspace; a.stream = stream;
    return linear_launch(a);
}

// Workspace of the recurrent block: the fused core's workspace first (its
// header, status word included, is also the projections' header), then the
// bf16 intermediates x, gate branch and the core's output, [B, T, D] each.
RGLRU_API size_t rglru_recurrent_block_workspace_size(int B, int T, int D)
{
    const size_t core = rglru_workspace_size(B, T, D, RGLRU_IO_BF16);
    if (core == 0) return 0;
    return align_up(core, 256) + 3 * align_up((size_t)B * T * D * 2, 256);
}

RGLRU_API rglru_status rglru_recurrent_block_prefill(
    int B, int T, int D, const void *u, const void *W_lin_x, const float *b_lin_x, const void *W_lin_y,
    const float *b_lin_y, const float *conv_w, const float *conv_b, const void *W_a, const float *b_a,
    const void *W_x, const float *b_x, const float *lambda, const int32_t *segment_pos, void *conv_state,
    float *h_state, const void *W_out, const float *b_out, void *out, void *workspace, size_t workspace_bytes,
    cudaStream_t stream)
{
    const size_t need = rglru_recurrent_block_workspace_size(B, T, D);
    if (need == 0) return RGLRU_ERR_INVALID_ARG;
    if ((int64_t)B * T > kMaxRows) return RGLRU_ERR_UNSUPPORTED;
    if (workspace == nullptr || !al16(workspace) || workspace_bytes < need) return RGLRU_ERR_WORKSPACE;
    const size_t act = (size_t)B * T * D * 2;
    const size_t wsz = (size_t)D * D * 2;
    if (!al16(u) || !al16(W_lin_x) || !al16(W_lin_y) || !al16(W_out) || !al16(out) || !al16(b_lin_x) ||
        !al16(b_lin_y) || !al16(b_out))
        return RGLRU_ERR_INVALID_ARG;
    const Span ins[] = {span(u, act), span(W_lin_x, wsz), span(W_lin_y, wsz), span(W_out, wsz),
                        span(workspace, workspace_bytes), span(conv_state, (size_t)B * 3 * D * 2),
                        span(h_state, (size_t)B * D * 4)};
    for (const Span &s : ins)
        if (meet(span(out, act), s)) return RGLRU_ERR_INVALID_ARG;
    if (meet(span(u, act), span(workspace, workspace_bytes))) return RGLRU_ERR_INVALID_ARG;
    char *ws = static_cast<char *>(workspace);
    const size_t core = align_up(rglru_workspace_size(B, T, D, RGLRU_IO_BF16), 256);
    void *x = ws + core;
    void *g = ws + core + align_up(act, 256);
    void *y = ws + core + 2 * align_up(act, 256);
    const int M = B * T;
    rglru_status st = rglru_linear_pair(M, D, D, u, W_lin_x, b_lin_x, x, W_lin_y, b_lin_y, g, ws,
                                        kWsHeaderBytes, stream);
    if (st != RGLRU_OK) return st;
    st = rglru_prefill(B, T, D, RGLRU_IO_BF16, x, g, conv_w, conv_b, W_a, b_a, W_x, b_x, lambda, segment_pos,
                       conv_state, h_state, y, ws, core, stream);
    if (st != RGLRU_OK) return st;
    return rglru_linear(M, D, D, y, W_out, b_out, out, ws, kWsHeaderBytes, stream);
}

RGLRU_API rglru_status rglru_rmsnorm(int M, int N, const void *x, const float *weight, float eps, void *out,
                                     cudaStream_t stream)
{
    if (M < 1 || N < 8 || N % 8 != 0 || (int64_t)M > kMaxRows || !(eps > 0.f)) return RGLRU_ERR_UNSUPPORTED;
    if (!al16(x) || !al16(weight) || !al16(out)) return RGLRU_ERR_INVALID_ARG;
    const size_t bytes = (size_t)M * N * 2;
    if (out != x && meet(span(out, bytes), span(x, bytes))) return RGLRU_ERR_INVALID_ARG;
    if (meet(span(out, bytes), span(weight, (size_t)N * 4))) return RGLRU_ERR_INVALID_ARG;
    return rmsnorm_launch(M, N, x, weight, eps, out, stream);
}

// Workspace of the residual block: the fused core's workspace first (its
// header is shared by every launch), then x, the gate branch, the core's
// output, the normalised rows, h (the recurrent block's residual output),
// all [B, T, D] bf16, then the MLP's hidden rows [B, T, F] bf16.
RGLRU_API size_t rglru_residual_block_workspace_size(int B, int T, int D, int F)
{
    const size_t core = rglru_workspace_size(B, T, D, RGLRU_IO_BF16);
    if (core == 0 || F < 128 || F % 128 != 0 || F > (1 << 20)) return 0;
    return align_up(core, 256) + 5 * align_up((size_t)B * T * D * 2, 256) + align_up((size_t)B * T * F * 2, 256);
}

RGLRU_API rglru_status rglru_residual_block_prefill(
    int B, int T, int D, int F, const void *u, const float *w_temporal_norm, const void *W_lin_x,
    const float *b_lin_x, const void *W_lin_y, const float *b_lin_y, const float *conv_w, const float *conv_b,
    const void *W_a, const float *b_a, const void *W_x, const float *b_x, const float *lambda, const void *W_out,
    const float *b_out, const int32_t *segment_pos, void *conv_state, float *h_state, const float *w_channel_norm,
    const void *W_gate, const float *b_gate, const void *W_up, const float *b_up, const void *W_down,
    const float *b_down, float eps, void *out, void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    const size_t need = rglru_residual_block_workspace_size(B, T, D, F);
    if (need == 0) return RGLRU_ERR_INVALID_ARG;
    if ((int64_t)B * T > kMaxRows || !(eps > 0.f)) return RGLRU_ERR_UNSUPPORTED;
    if (workspace == nullptr || !al16(workspace) || workspace_bytes < need) return RGLRU_ERR_WORKSPACE;
    const size_t act = (size_t)B * T * D * 2;
    if (!al16(u) || !al16(out) || !al16(w_temporal_norm) || !al16(w_channel_norm)) return RGLRU_ERR_INVALID_ARG;
    // the operands of the steps after the core, checked before the core updates the states: a bad
    // argument leaves conv_state, h_state and out untouched
    if (!al16(W_lin_x) || !al16(W_lin_y) || !al16(W_out) || !al16(W_gate) || !al16(b_gate) || !al16(W_up) ||
        !al16(b_up) || !al16(W_down))
        return RGLRU_ERR_INVALID_ARG;
    for (const float *bias : {b_lin_x, b_lin_y, b_out, b_down})
        if (bias != nullptr && !al16(bias)) return RGLRU_ERR_INVALID_ARG;
    const Span ins[] = {span(u, act), span(workspace, workspace_bytes), span(conv_state, (size_t)B * 3 * D * 2),
                        span(h_state, (size_t)B * D * 4), span(W_lin_x, (size_t)D * D * 2),
                        span(W_lin_y, (size_t)D * D * 2), span(W_out, (size_t)D * D * 2),
                        span(W_gate, (size_t)F * D * 2), span(W_up, (size_t)F * D * 2),
                        span(W_down, (size_t)D * F * 2)};
    for (const Span &s : ins)
        if (meet(span(out, act), s)) return RGLRU_ERR_INVALID_ARG;
    if (meet(span(u, act), span(workspace, workspace_bytes))) return RGLRU_ERR_INVALID_ARG;
    char *ws = static_cast<char *>(workspace);
    const size_t core = align_up(rglru_workspace_size(B, T, D, RGLRU_IO_BF16), 256);
    const size_t a = align_up(act, 256);
    void *x = ws + core, *g = ws + core + a, *y = ws + core + 2 * a, *n = ws + core + 3 * a, *h = ws + core + 4 * a;
    void *m = ws + core + 5 * a;
    const int M = B * T;
    // temporal_pre_norm -> linear_x / linear_y -> conv + RG-LRU core -> linear_out + residual
    rglru_status st = rglru_rmsnorm(M, D, u, w_temporal_norm, eps, n, stream);
    if (st == RGLRU_OK)
        st = rglru_linear_pair(M, D, D, n, W_lin_x, b_lin_x, x, W_lin_y, b_lin_y, g, ws, kWsHeaderBytes, stream);
    if (st == RGLRU_OK)
        st = rglru_prefill(B, T, D, RGLRU_IO_BF16, x, g, conv_w, conv_b, W_a, b_a, W_x, b_x, lambda, segment_pos,
                           conv_state, h_state, y, ws, core, stream);
    if (st == RGLRU_OK) st = rglru_linear_residual(M, D, D, y, W_out, b_out, u, h, ws, kWsHeaderBytes, stream);
    // channel_pre_norm -> GELU-gated up projection -> down projection + residual
    if (st == RGLRU_OK) st = rglru_rmsnorm(M, D, h, w_channel_norm, eps, n, stream);
    if (st == RGLRU_OK)
        st = rglru_linear_geglu(M, F, D, n, W_gate, b_gate, W_up, b_up, m, ws, kWsHeaderBytes, stream);
    if (st == RGLRU_OK) st = rglru_linear_residual(M, D, F, m, W_down, b_down, h, out, ws, kWsHeaderBytes, stream);
    return st;
}

}  // extern "C"
