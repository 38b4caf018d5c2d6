/*
 * rglru.h -- C ABI of the B200 RG-LRU recurrent-block core (librglru.so).
 *
 * One call computes the core of a RecurrentGemma recurrent temporal block,
 * from the input of the causal depthwise conv to the product with the GELU
 * branch.  Structure: "Gemma explained: RecurrentGemma architecture"
 * (gemma.gh.miniasp.com), the RecurrentGemmaRecurrentBlock module printout
 * (Conv1d(D, D, kernel_size=4, padding=3, groups=D), RecurrentGemmaRglru,
 * PytorchGELUTanh) and the section "Residual block with recurrent block"
 * (conv then RG-LRU on one branch, GELU on the other, elementwise product).
 * The RG-LRU equations are those of Griffin / RecurrentGemma
 * ("RecurrentGemma: Moving Past Transformers for Efficient Open Language
 * Models", arXiv 2404.07839), which the pages name but do not print:
 *
 *   xc_t = conv_b + sum_{k=0..3} conv_w[k] * x_{t-3+k} * [3-k <= segpos_t]
 *   r_t  = sigmoid(W_a[h] xc_t + b_a),   i_t = sigmoid(W_x[h] xc_t + b_x)
 *   a_t  = sigmoid(Lambda)^(8 r_t)
 *   h_t  = a_t h_{t-1} + sqrt(1 - a_t^2) (i_t xc_t)      (segpos_t > 0)
 *   h_t  = i_t xc_t                                      (segpos_t == 0)
 *   y_t  = GELU_tanh(g_t) h_t
 *
 * Conventions for every call below
 *   - All tensor pointers are DEVICE pointers (cudaMalloc'd, or managed),
 *     except the *_host arguments of rglru_prefill_host,
 *     owned by the caller, 16-byte aligned.  The library allocates nothing,
 *     keeps no global state and never synchronises the stream (except
 *     rglru_get_device_status).  Work is enqueued on `stream`.
 *   - Layouts are row-major with the channel index fastest:
 *       x, gate_branch, y     [B, T, D]  io dtype
 *       conv_w [4, D] fp32    tap k multiplies the input 3-k steps back
 *       conv_b, b_a, b_x, lambda [D] fp32
 *       W_a, W_x [H, 256, 256] with H = D/256, index [head][out][in];
 *                 bf16 in RGLRU_IO_BF16 mode, fp32 in RGLRU_IO_F32 mode
 *       segment_pos [B, T] int32: position inside the current document;
 *                 0 marks a document start (resets h, masks conv taps);
 *                 values < 0 are not allowed; >= 3 means all taps valid
 *       conv_state [B, 3, D] io dtype, the last three raw inputs, oldest
 *                 first; read and overwritten in place
 *       h_state   [B, D] fp32; read and overwritten in place
 *   - D must be a multiple of 256 (heads of 256 channels).
 *   - y must not overlap any input.  The states are updated in place.
 *   - Argument errors are reported synchronously, before anything is
 *     enqueued.  A failed launch returns RGLRU_ERR_CUDA.  A device-side
 *     bounded wait that gave up is recorded in the workspace and read back
 *     by rglru_get_device_status.
 *   - The workspace is caller-owned device memory of at least the size the
 *     matching *_workspace_size call returns, zero-filled once before its
 *     first use (the calls leave it valid for the next one).  It may be
 *     reused across calls on the same stream but not shared by calls that
 *     can overlap on the GPU.
 */
#ifndef RGLRU_H
#define RGLRU_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define RGLRU_API __attribute__((visibility("default")))
#else
#define RGLRU_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RGLRU_OK = 0,
    RGLRU_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, overlap */
    RGLRU_ERR_UNSUPPORTED = 2,  /* shape or dtype the library does not handle */
    RGLRU_ERR_WORKSPACE = 3,    /* workspace missing or too small */
    RGLRU_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    RGLRU_ERR_TIMEOUT = 5       /* a device-side bounded wait gave up */
} rglru_status;

typedef enum {
    RGLRU_IO_F32 = 0,   /* x, gate_branch, y, conv_state, W_a, W_x in fp32 */
    RGLRU_IO_BF16 = 1   /* the same tensors in bf16 (the state h stays fp32) */
} rglru_io_dtype;

/* Library ABI version (major * 100 + minor). */
RGLRU_API int rglru_version(void);

/* Human-readable name of a status code (static storage, never NULL). */
RGLRU_API const char *rglru_status_string(rglru_status status);

/*
 * Workspace bytes rglru_prefill needs for these sizes (0 on bad sizes).
 * Holds the device status word and the cross-chunk scan carry (per chunk,
 * flags and (prod a, h) aggregates).
 */
RGLRU_API size_t rglru_workspace_size(int B, int T, int D, rglru_io_dtype dt);

/*
 * Prefill: runs the block core over T tokens of B sequences.
 * bf16 mode runs one fused kernel (conv, tensor-core gate projections,
 * chunked fp32 scan with a cross-chunk carry, GELU product); fp32 mode runs
 * the plain SIMT kernels of rglru_prefill_simt.
 * Outputs: y [B,T,D]; conv_state and h_state updated to their values after
 * token T-1.
 * Range (bf16 mode): the fused kernel keeps each token's GELU(g)*h_local
 * and GELU(g)*prod(a) between its two scan passes as f16, so it requires
 * |GELU(g)*h| and |GELU(g)| below 65504; beyond that y may be inf where the
 * recurrence is finite.  fp32 mode and rglru_prefill_simt have no such limit.
 */
RGLRU_API rglru_status rglru_prefill(int B, int T, int D, rglru_io_dtype dt,
                           const void *x, const void *gate_branch,
                           const float *conv_w, const float *conv_b,
                           const void *W_a, const float *b_a,
                           const void *W_x, const float *b_x,
                           const float *lambda, const int32_t *segment_pos,
                           void *conv_state, float *h_state, void *y,
                           void *workspace, size_t workspace_bytes,
                           cudaStream_t stream);

/*
 * Staging bytes rglru_prefill_host needs (0 on bad arguments): two slots,
 * each holding x, gate_branch and y for rows_per_chunk sequences
 * ([rows, T, D] io dtype) and their segment_pos ([rows, T] int32), every
 * piece 256-byte aligned.
 */
RGLRU_API size_t rglru_prefill_host_staging_size(int B, int T, int D, rglru_io_dtype dt,
                                                 int rows_per_chunk);

/*
 * rglru_prefill with the activations in HOST memory: x_host,
 * gate_branch_host ([B,T,D] io dtype) and segment_pos_host ([B,T] int32)
 * are read from host memory and y_host ([B,T,D]) is written there.
 * Page-locked host memory lets the copies run asynchronously; pageable
 * memory gives the same result without the overlap.  The parameters,
 * conv_state, h_state, the workspace and `staging` are device memory as for
 * rglru_prefill.
 *   rows_per_chunk  sequences per chunk (>= 1; values above B mean B).  The
 *                   batch is processed chunk by chunk: the upload of chunk
 *                   k + 1, the kernels of chunk k and the download of chunk
 *                   k - 1 run at once.
 *   staging         device memory of rglru_prefill_host_staging_size bytes,
 *                   256-byte aligned, not in use by other work.
 *   workspace       at least rglru_workspace_size(min(B, rows_per_chunk),
 *                   T, D, dt) bytes.
 * The result equals copying the inputs to the device, calling
 * rglru_prefill and copying y back (bit for bit in bf16 mode: the fused
 * kernel's results do not depend on how the batch is split).  Everything is
 * enqueued asynchronously: y_host, conv_state and h_state are complete for
 * work enqueued on `stream` after the call, and the host buffers must stay
 * valid until then.  The call creates two CUDA streams and a few events for
 * the copies and releases them before it returns (their work may still be
 * pending).  It synchronises nothing.
 */
RGLRU_API rglru_status rglru_prefill_host(int B, int T, int D, rglru_io_dtype dt,
                                const void *x_host, const void *gate_branch_host,
                                const float *conv_w, const float *conv_b,
                                const void *W_a, const float *b_a,
                                const void *W_x, const float *b_x,
                                const float *lambda, const int32_t *segment_pos_host,
                                void *conv_state, float *h_state, void *y_host,
                                int rows_per_chunk, void *staging, size_t staging_bytes,
                                void *workspace, size_t workspace_bytes,
                                cudaStream_t stream);

/*
 * Workspace bytes rglru_prefill_simt needs (0 on bad sizes): the device
 * status word plus three fp32 [B,T,D] intermediates (conv output and the
 * two gate pre-activations).
 */
RGLRU_API size_t rglru_simt_workspace_size(int B, int T, int D, rglru_io_dtype dt);

/*
 * The same computation as rglru_prefill on plain SIMT kernels (CUDA cores
 * only, fp32 arithmetic with accurate transcendentals), in either dtype.
 * It is the fp32-mode path and an independent second implementation for
 * cross-checks.  Same arguments and semantics as rglru_prefill.
 */
RGLRU_API rglru_status rglru_prefill_simt(int B, int T, int D, rglru_io_dtype dt,
                                const void *x, const void *gate_branch,
                                const float *conv_w, const float *conv_b,
                                const void *W_a, const float *b_a,
                                const void *W_x, const float *b_x,
                                const float *lambda, const int32_t *segment_pos,
                                void *conv_state, float *h_state, void *y,
                                void *workspace, size_t workspace_bytes,
                                cudaStream_t stream);

/* Workspace bytes rglru_decode_step needs for B sequences of width D. */
RGLRU_API size_t rglru_decode_workspace_size(int B, int D, rglru_io_dtype dt);

/*
 * Decode: one token for each of B sequences (the prefill recurrence with
 * T = 1).  x, gate_branch, y are [B, D]; segment_pos is [B]; conv_state and
 * h_state are updated in place.  Other arguments as rglru_prefill.
 * The bf16 kernel is launched with programmatic dependent launch: it may
 * start while the previous kernel on the stream finishes, and it reads
 * W_a, W_x and conv_w / conv_b before waiting for that kernel.  So these
 * parameters must not be written by a kernel that directly precedes the
 * call on the stream and releases its dependents early; every other input
 * is read only after the previous kernel has completed.
 */
RGLRU_API rglru_status rglru_decode_step(int B, int D, rglru_io_dtype dt,
                               const void *x, const void *gate_branch,
                               const float *conv_w, const float *conv_b,
                               const void *W_a, const float *b_a,
                               const void *W_x, const float *b_x,
                               const float *lambda, const int32_t *segment_pos,
                               void *conv_state, float *h_state, void *y,
                               void *workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/*
 * Synchronises `stream`, returns the device status recorded in `workspace`
 * by the calls enqueued so far (RGLRU_OK or RGLRU_ERR_TIMEOUT) and clears it.
 * RGLRU_ERR_CUDA if the synchronisation or the read fails.
 */
RGLRU_API rglru_status rglru_get_device_status(void *workspace, cudaStream_t stream);

/*
 * Test hook for the bounded waits (never used by a normal call): makes chunk
 * `unit` of the next rglru_prefill calls on this workspace skip publishing
 * its scan carry, so that its successor's wait runs out and records
 * RGLRU_ERR_TIMEOUT instead of hanging; on a decode workspace, CTA `unit` of
 * the next rglru_decode_step calls keeps its half of the gate GEMM's operand
 * from its peer CTA, whose wait runs out the same way (the call then takes a
 * few seconds).  unit = -1 turns it off.  The flag lives in the workspace
 * header and is enqueued on `stream`.
 */
RGLRU_API rglru_status rglru_debug_suppress_publish(void *workspace, int unit, cudaStream_t stream);

/*
 * rglru_prefill without a workspace argument, for callers that cannot
 * allocate device memory where they run the block (a serving loop whose
 * device memory is fixed at start-up, a plug-in handed tensors but no
 * allocator).  The pages have no counterpart to this call; it only changes
 * where the scratch lives.  It allocates nothing: the caller passes inputs
 * and outputs as for rglru_prefill, and the scratch is a library-owned device
 * array of 8 MiB per GPU, held from library load until the process exits.
 *   - bf16 only (RGLRU_ERR_UNSUPPORTED otherwise); shapes whose
 *     rglru_workspace_size exceeds 8 MiB are rejected with
 *     RGLRU_ERR_WORKSPACE before anything is enqueued.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *     The address is cached per device index for the life of the process, so
 *     a process that calls cudaDeviceReset on a device must not use this
 *     entry point on that device afterwards.
 *   - Every call shares the array and zeroes what must start at zero; calls
 *     that can overlap on the GPU (other streams, other host threads) race
 *     on it, so the caller must serialise them.
 *   - A device-side wait that runs out cannot be read back (there is no
 *     workspace handle); the next call clears the record.
 * Other arguments, layouts and semantics as rglru_prefill.
 */
RGLRU_API rglru_status rglru_prefill_noalloc(int B, int T, int D, rglru_io_dtype dt,
                                             const void *x, const void *gate_branch,
                                             const float *conv_w, const float *conv_b,
                                             const void *W_a, const float *b_a,
                                             const void *W_x, const float *b_x,
                                             const float *lambda, const int32_t *segment_pos,
                                             void *conv_state, float *h_state, void *y,
                                             cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Dense projections around the core and the whole recurrent block.
 *
 * "Gemma explained: RecurrentGemma architecture", the
 * RecurrentGemmaRecurrentBlock printout (linear_y, linear_x, linear_out:
 * Linear(2560, 2560, bias=True)) and section "Residual block with recurrent
 * block": the block input u feeds linear_x (then the conv and the RG-LRU)
 * and linear_y (the GELU branch); their product feeds linear_out.  The
 * RecurrentGemmaMlp printout gives gate_proj / up_proj (2560 -> 7680) with a
 * tanh GELU on the gate, and down_proj (7680 -> 2560).
 *
 * All of them: bf16 operands and outputs, fp32 bias, fp32 accumulation on
 * the tensor cores.  Weights use torch's Linear layout W [out, in] (row
 * = output feature, the input dimension contiguous).  Activations are
 * row-major [M, features] (M = B * T tokens).  Sizes: K (input features) a
 * multiple of 64, N (output features) a multiple of 256 (128 for
 * rglru_linear_geglu), M >= 1.  Pointers are device pointers, 16-byte
 * aligned; outputs must not overlap inputs (except out == residual).  The
 * workspace holds the device status word (rglru_linear_workspace_size bytes,
 * zero-filled once before first use); a bounded device wait that gave up is
 * read back with rglru_get_device_status.  Unsupported sizes return
 * RGLRU_ERR_UNSUPPORTED before anything is enqueued.
 * ------------------------------------------------------------------------ */

/* Workspace bytes of the rglru_linear* calls (the device status header). */
RGLRU_API size_t rglru_linear_workspace_size(void);

/* out[M, N] = A[M, K] W[N, K]^T + bias[N]   (bias may be NULL) */
RGLRU_API rglru_status rglru_linear(int M, int N, int K, const void *A, const void *W, const float *bias,
                                    void *out, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Two projections of the same input in one launch (linear_x and linear_y of
 * the block): out0 = A W0^T + bias0, out1 = A W1^T + bias1, each [M, N]. */
RGLRU_API rglru_status rglru_linear_pair(int M, int N, int K, const void *A, const void *W0, const float *bias0,
                                         void *out0, const void *W1, const float *bias1, void *out1,
                                         void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* out = A W^T + bias + residual  (residual [M, N]; out may equal residual) */
RGLRU_API rglru_status rglru_linear_residual(int M, int N, int K, const void *A, const void *W, const float *bias,
                                             const void *residual, void *out, void *workspace,
                                             size_t workspace_bytes, cudaStream_t stream);

/* MLP up-projection: out[M, N] = GELU_tanh(A W_gate^T + b_gate) * (A W_up^T + b_up),
 * W_gate, W_up [N, K]; biases required. */
RGLRU_API rglru_status rglru_linear_geglu(int M, int N, int K, const void *A, const void *W_gate,
                                          const float *b_gate, const void *W_up, const float *b_up, void *out,
                                          void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Workspace bytes of rglru_recurrent_block_prefill (0 on bad sizes): the
 * core's workspace plus the bf16 intermediates x, gate branch and core output. */
RGLRU_API size_t rglru_recurrent_block_workspace_size(int B, int T, int D);

/*
 * The recurrent block over T tokens of B sequences, bf16:
 *   x = u W_lin_x^T + b_lin_x,  g = u W_lin_y^T + b_lin_y      (one launch)
 *   y = rglru_prefill core (x, g, ...)                        (fused kernel)
 *   out = y W_out^T + b_out
 * u, out [B, T, D] bf16; W_lin_x, W_lin_y, W_out [D, D] bf16; their biases
 * [D] fp32; the core's parameters, segment_pos and states as rglru_prefill
 * (bf16 mode).  x, g and y are held in the workspace as bf16 [B, T, D], the
 * dtype of the core's inputs and output.  The workspace (zero-filled once)
 * carries one status word for all three launches.
 */
RGLRU_API rglru_status rglru_recurrent_block_prefill(
    int B, int T, int D, const void *u, const void *W_lin_x, const float *b_lin_x, const void *W_lin_y,
    const float *b_lin_y, const float *conv_w, const float *conv_b, const void *W_a, const float *b_a,
    const void *W_x, const float *b_x, const float *lambda, const int32_t *segment_pos, void *conv_state,
    float *h_state, const void *W_out, const float *b_out, void *out, void *workspace, size_t workspace_bytes,
    cudaStream_t stream);

/*
 * RMSNorm of bf16 rows: out[m, :] = x[m, :] * rsqrt(mean_n(x[m, n]^2) + eps) * weight
 * (x, out [M, N] bf16, weight [N] fp32, N a multiple of 8 up to 4096, eps > 0;
 * out may equal x).  The decoder layer's temporal_pre_norm and
 * channel_pre_norm (RecurrentGemmaRMSNorm in the printout; the pages give
 * no formula, so this is the standard root-mean-square normalisation with a
 * learned scale).
 */
RGLRU_API rglru_status rglru_rmsnorm(int M, int N, const void *x, const float *weight, float eps, void *out,
                                     cudaStream_t stream);

/* Workspace bytes of rglru_residual_block_prefill (0 on bad sizes). */
RGLRU_API size_t rglru_residual_block_workspace_size(int B, int T, int D, int F);

/*
 * The recurrent residual block ("Residual block with recurrent block" and
 * the decoder-layer printout) over T tokens of B sequences, bf16:
 *   n   = RMSNorm(u) (w_temporal_norm)
 *   h   = u + linear_out(GELU(linear_y(n)) * RG-LRU core(linear_x(n)))
 *   n'  = RMSNorm(h) (w_channel_norm)
 *   out = h + down_proj(GELU_tanh(gate_proj(n')) * up_proj(n'))
 * u, out [B, T, D]; W_gate, W_up [F, D], W_down [D, F] bf16 (F = 3 D in the
 * 2B model, MLP expansion factor 3); biases fp32; the recurrent block's
 * parameters, segment_pos and states as rglru_recurrent_block_prefill.
 * b_gate and b_up are required; b_lin_x, b_lin_y, b_out and b_down may be
 * NULL.  Every operand is checked before the first launch: on
 * RGLRU_ERR_INVALID_ARG nothing ran and the states and out are untouched.
 * Every intermediate is a bf16 tensor in the workspace (zero-filled once),
 * which carries one status word for all the launches.
 */
RGLRU_API rglru_status rglru_residual_block_prefill(
    int B, int T, int D, int F, const void *u, const float *w_temporal_norm, const void *W_lin_x,
    const float *b_lin_x, const void *W_lin_y, const float *b_lin_y, const float *conv_w, const float *conv_b,
    const void *W_a, const float *b_a, const void *W_x, const float *b_x, const float *lambda, const void *W_out,
    const float *b_out, const int32_t *segment_pos, void *conv_state, float *h_state, const float *w_channel_norm,
    const void *W_gate, const float *b_gate, const void *W_up, const float *b_up, const void *W_down,
    const float *b_down, float eps, void *out, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Local sliding-window MQA: the other temporal block.
 *
 * "Gemma explained: RecurrentGemma architecture", the
 * RecurrentGemmaSdpaAttention printout (q_proj D -> D and k_proj, v_proj
 * D -> 256 without bias, o_proj D -> D with bias, rotary_emb) and sections
 * "Residual block with local MQA" (H = D / 256 query heads of 256 share one
 * key/value head of 256; each position attends a fixed number of past tokens)
 * and "Local attention window size" (2048 tokens).  Readings where the pages
 * are silent: rotate-half RoPE over the whole head, the pairs (x[i],
 * x[i + 128]) turned by segment_pos * 10000^(-2i/256); scores scaled by 1/16;
 * query t attends key s when t - window < s <= t, s >= t - segment_pos[t]
 * (same document) and s >= 0 (a call sees the keys of its own tokens only).
 *
 * Layouts (bf16, row-major): qkv [B, T, (H + 2) * 256] holds the H query
 * heads, then k, then v of each token; v_t [B, 256, Tp] is v transposed,
 * Tp = T rounded up to a multiple of 8 (rglru_mqa_vt_size bytes);
 * segment_pos [B, T] int32 (>= 0); out [B, T, H * 256].  Every pointer is
 * device memory, 16-byte aligned; calls enqueue on `stream` and return after
 * synchronous argument checks (RGLRU_ERR_INVALID_ARG on null, misaligned or
 * overlapping arguments, RGLRU_ERR_UNSUPPORTED on sizes outside B <= 65535,
 * H <= 64, B * T <= 2^30).
 * ---------------------------------------------------------------------- */

/* Bytes of v_t for B sequences of T tokens (0 on bad sizes). */
RGLRU_API size_t rglru_mqa_vt_size(int B, int T);

/*
 * RoPE of the query heads and the key in place in qkv, at the positions
 * segment_pos, and v_t = the v columns of qkv transposed (its tokens past T
 * up to Tp are written as zeros).  qkv and v_t must not overlap.
 */
RGLRU_API rglru_status rglru_mqa_rope(int B, int T, int H, void *qkv, const int32_t *segment_pos, void *v_t,
                                      cudaStream_t stream);

/*
 * out[b, t, h] = sum_s softmax_s(q[b, t, h] . k[b, s] / 16) v[b, s] over the
 * keys s query t attends (see above), from qkv and v_t after rglru_mqa_rope.
 * fp32 scores and accumulation on the tensor cores, the probabilities rounded
 * to bf16 as the operand of the second product, out rounded to bf16.
 * window >= 1 (2048 in the 2B and 9B models).  The workspace (at least
 * rglru_linear_workspace_size() bytes, zero-filled once) carries the device
 * status: a wait inside the kernel that runs out (2 s) records
 * RGLRU_ERR_TIMEOUT there instead of hanging.  out must not overlap the inputs.
 */
RGLRU_API rglru_status rglru_mqa_attention(int B, int T, int H, int window, const void *qkv, const void *v_t,
                                           const int32_t *segment_pos, void *out, void *workspace,
                                           size_t workspace_bytes, cudaStream_t stream);

/* Workspace bytes of rglru_mqa_block_prefill (0 on bad sizes). */
RGLRU_API size_t rglru_mqa_block_workspace_size(int B, int T, int D);

/*
 * The local MQA temporal block over T tokens of B sequences, bf16:
 *   qkv = u W_qkv^T                       (q_proj, k_proj, v_proj in one launch)
 *   RoPE on q and k, v transposed          (rglru_mqa_rope)
 *   a   = local MQA(q, k, v)               (rglru_mqa_attention)
 *   out = a W_o^T + b_o                    (o_proj)
 * u, out [B, T, D]; W_qkv [D + 512, D] = the rows of W_q [D, D], then W_k
 * [256, D], then W_v [256, D]; W_o [D, D]; b_o [D] fp32 (may be NULL).  qkv,
 * v_t and a live in the workspace (zero-filled once), which carries one status
 * word for all four launches.
 */
RGLRU_API rglru_status rglru_mqa_block_prefill(int B, int T, int D, int window, const void *u, const void *W_qkv,
                                               const void *W_o, const float *b_o, const int32_t *segment_pos,
                                               void *out, void *workspace, size_t workspace_bytes,
                                               cudaStream_t stream);

/* Workspace bytes of rglru_mqa_decode_step (0 on unsupported sizes:
 * 1 <= B <= 65535, 1 <= H <= 16, window a multiple of 128 up to 2048). */
RGLRU_API size_t rglru_mqa_decode_workspace_size(int B, int H, int window);

/*
 * One decode step of the local MQA attention for B sequences (one token
 * each), after the QKV projection of that token:
 *   qkv         [B, (H + 2) * 256] bf16, read only: q heads, k, v of the token;
 *   segment_pos [B] int32 >= 0: the token's position in its document;
 *   k_cache     [B, window, 256] bf16, in/out: a ring per sequence, the rotated
 *               key of document position q at slot q % window;
 *   v_cache_t   [B, 256, window] bf16, in/out: the values, transposed (value
 *               of position q in column q % window);
 *   out         [B, H * 256] bf16.
 * The step writes this token's slot, then attends positions
 * max(0, p - window + 1) .. p (earlier steps of the same document must have
 * written them).  Every slot of both rings must hold finite values (zero-fill
 * them before first use): slots outside the attended range enter the
 * products with probability 0.  q and k are rotated (RoPE at segment_pos) and
 * rounded to bf16 as in rglru_mqa_rope; scores on the tensor cores in fp32,
 * probabilities as bf16 operands, sums in fp32, out rounded to bf16.  Two
 * kernels: per (sequence, block of 128 positions) partial maxima, sums and
 * outputs in the workspace, then their combination.  No buffer may overlap
 * another one that the step writes.
 */
RGLRU_API rglru_status rglru_mqa_decode_step(int B, int H, int window, const void *qkv, const int32_t *segment_pos,
                                             void *k_cache, void *v_cache_t, void *out, void *workspace,
                                             size_t workspace_bytes, cudaStream_t stream);

/* Workspace bytes of rglru_mqa_residual_block_prefill (0 on bad sizes). */
RGLRU_API size_t rglru_mqa_residual_block_workspace_size(int B, int T, int D, int F);

/*
 * The residual block with local MQA ("Residual block with local MQA" and the
 * decoder-layer printout: norm, temporal block, residual, norm, MLP,
 * residual) over T tokens of B sequences, bf16:
 *   n   = RMSNorm(u) (w_temporal_norm)
 *   h   = u + o_proj(local MQA(RoPE(q_proj n), RoPE(k_proj n), v_proj n))
 *   n'  = RMSNorm(h) (w_channel_norm)
 *   out = h + down_proj(GELU_tanh(gate_proj(n')) * up_proj(n'))
 * W_qkv, W_o, b_o as rglru_mqa_block_prefill; the MLP as
 * rglru_residual_block_prefill (W_gate, W_up [F, D], W_down [D, F]; b_gate
 * and b_up required, b_down may be NULL); every operand is checked before the
 * first launch.  Every intermediate is a bf16 tensor in the workspace
 * (zero-filled once), which carries one status word for all the launches.
 */
RGLRU_API rglru_status rglru_mqa_residual_block_prefill(
    int B, int T, int D, int F, int window, const void *u, const float *w_temporal_norm, const void *W_qkv,
    const void *W_o, const float *b_o, const int32_t *segment_pos, const float *w_channel_norm, const void *W_gate,
    const float *b_gate, const void *W_up, const float *b_up, const void *W_down, const float *b_down, float eps,
    void *out, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * The carried scan state of a long sequence split into N time chunks (one per
 * rank), from one exchange.  The recurrence is affine in the state a chunk
 * starts from: the chunk ends in A h_in + H0 per channel.  Each rank runs
 * rglru_prefill on its chunk from h_state = 0 and from h_state = 1, giving the
 * end states H0 and H1 (so A = H1 - H0); the ranks all-gather them; then
 *   h_in[0] = h0,   h_in[r + 1] = (H1[r] - H0[r]) h_in[r] + H0[r]
 * and each rank runs its chunk once more from h_in[rank], with conv_state =
 * the three raw inputs before its first token.
 *   H0, H1   [N, B, D] fp32, rank-major (the gathered end states);
 *   h0       [B, D] fp32: the state before the first chunk;
 *   h_in     [N, B, D] fp32 out: the state each chunk starts from.
 * Device pointers; h_in must not overlap the inputs.  In fp32 the subtraction
 * H1 - H0 carries the rounding of the end states (about 1e-7 of their size).
 */
RGLRU_API rglru_status rglru_carry_scan(int N, int B, int D, const float *H0, const float *H1, const float *h0,
                                        float *h_in, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* RGLRU_H */
