// rglru_api.cu -- the C ABI of librglru: argument checks, workspace sizing, dispatch.
//
// Every entry point validates its arguments synchronously and enqueues work
// on the caller's stream; nothing here allocates or synchronises (except
// rglru_get_device_status, which reads the device status word back).
#include <cstdint>
#include <cstring>

#include "internal.h"

using namespace rglru;

namespace {

constexpr int64_t kMaxElems = int64_t(1) << 40;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
    uintptr_t lo, hi;
};
bool overlaps(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }
Range range_of(const void *p, size_t bytes)
{
    const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
    return {lo, lo + bytes};
}

bool sizes_ok(int B, int T, int D)
{
    if (B < 1 || T < 1 || D < kHead || D % kHead != 0) return false;
    if (B > 65535) return false;
    return (int64_t)B * T * D <= kMaxElems;
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 rglru::encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

bool rglru::encode_bf16(PFN_cuTensorMapEncodeTiled_v12000 encode, CUtensorMap *m, const void *base, int rank,
                        const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box,
                        CUtensorMapSwizzle sw)
{
    if (encode == nullptr) return false;
    const cuuint32_t estride[5] = {1, 1, 1, 1, 1};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

rglru_status rglru::set_smem_limit_once(const void *kernel, int bytes, PerDeviceFlag &flag)
{
    static std::mutex m;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return RGLRU_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return RGLRU_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(m);
    if (!flag.done[dev]) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
            return RGLRU_ERR_CUDA;
        flag.done[dev] = true;
    }
    return RGLRU_OK;
}

rglru_status rglru::validate_prefill(const PrefillArgs &a, size_t need)
{
    if (a.dt != RGLRU_IO_F32 && a.dt != RGLRU_IO_BF16) return RGLRU_ERR_INVALID_ARG;
    if (!sizes_ok(a.B, a.T, a.D)) return RGLRU_ERR_INVALID_ARG;
    const void *ptrs[] = {a.x, a.g, a.conv_w, a.conv_b, a.W_a, a.b_a, a.W_x, a.b_x,
                          a.lambda, a.segpos, a.conv_state, a.h_state, a.y};
    for (const void *p : ptrs)
        if (p == nullptr || !aligned16(p)) return RGLRU_ERR_INVALID_ARG;
    if (a.ws == nullptr || !aligned16(a.ws)) return RGLRU_ERR_WORKSPACE;
    if (a.ws_bytes < need) return RGLRU_ERR_WORKSPACE;
    const size_t e = a.dt == RGLRU_IO_BF16 ? 2 : 4;
    const size_t act = (size_t)a.B * a.T * a.D * e;
    const Range ry = range_of(a.y, act);
    const Range rx = range_of(a.x, act), rg = range_of(a.g, act);
    const Range rcs = range_of(a.conv_state, (size_t)a.B * 3 * a.D * e);
    const Range rhs = range_of(a.h_state, (size_t)a.B * a.D * sizeof(float));
    const Range rws = range_of(a.ws, need);
    if (overlaps(ry, rx) || overlaps(ry, rg) || overlaps(ry, rcs) || overlaps(ry, rhs) ||
        overlaps(rcs, rhs) || overlaps(rcs, rx) || overlaps(rhs, rx) || overlaps(rws, ry) ||
        overlaps(rws, rx) || overlaps(rws, rg) || overlaps(rws, rcs) || overlaps(rws, rhs))
        return RGLRU_ERR_INVALID_ARG;
    return RGLRU_OK;
}

namespace {

PrefillArgs pack(int B, int T, int D, rglru_io_dtype dt, const void *x, const void *g,
                 const float *conv_w, const float *conv_b, const void *W_a, const float *b_a,
                 const void *W_x, const float *b_x, const float *lambda, const int32_t *segpos,
                 void *conv_state, float *h_state, void *y, void *ws, size_t ws_bytes,
                 cudaStream_t stream)
{
    PrefillArgs a;
    a.B = B; a.T = T; a.D = D; a.dt = dt;
    a.x = x; a.g = g; a.conv_w = conv_w; a.conv_b = conv_b;
    a.W_a = W_a; a.b_a = b_a; a.W_x = W_x; a.b_x = b_x;
    a.lambda = lambda; a.segpos = segpos; a.conv_state = conv_state; a.h_state = h_state;
    a.y = y; a.ws = ws; a.ws_bytes = ws_bytes; a.stream = stream;
    return a;
}

}  // namespace

extern "C" {

RGLRU_API int rglru_version(void) { return 100; }

RGLRU_API const char *rglru_status_string(rglru_status s)
{
    switch (s) {
    case RGLRU_OK: return "ok";
    case RGLRU_ERR_INVALID_ARG: return "invalid argument";
    case RGLRU_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case RGLRU_ERR_WORKSPACE: return "workspace missing or too small";
    case RGLRU_ERR_CUDA: return "CUDA error";
    case RGLRU_ERR_TIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

RGLRU_API size_t rglru_simt_workspace_size(int B, int T, int D, rglru_io_dtype dt)
{
    if (!sizes_ok(B, T, D) || (dt != RGLRU_IO_F32 && dt != RGLRU_IO_BF16)) return 0;
    return simt_workspace_bytes(B, T, D);
}

RGLRU_API size_t rglru_workspace_size(int B, int T, int D, rglru_io_dtype dt)
{
    if (!sizes_ok(B, T, D) || (dt != RGLRU_IO_F32 && dt != RGLRU_IO_BF16)) return 0;
    return dt == RGLRU_IO_BF16 ? fused_workspace_bytes(B, T, D) : simt_workspace_bytes(B, T, D);
}

RGLRU_API size_t rglru_decode_workspace_size(int B, int D, rglru_io_dtype dt)
{
    if (!sizes_ok(B, 1, D) || (dt != RGLRU_IO_F32 && dt != RGLRU_IO_BF16)) return 0;
    return dt == RGLRU_IO_BF16 ? decode_workspace_bytes(B, D) : simt_workspace_bytes(B, 1, D);
}

RGLRU_API rglru_status rglru_prefill_simt(int B, int T, int D, rglru_io_dtype dt, const void *x,
                                const void *gate_branch, const float *conv_w, const float *conv_b,
                                const void *W_a, const float *b_a, const void *W_x,
                                const float *b_x, const float *lambda, const int32_t *segment_pos,
                                void *conv_state, float *h_state, void *y, void *workspace,
                                size_t workspace_bytes, cudaStream_t stream)
{
    const PrefillArgs a = pack(B, T, D, dt, x, gate_branch, conv_w, conv_b, W_a, b_a, W_x, b_x,
                               lambda, segment_pos, conv_state, h_state, y, workspace,
                               workspace_bytes, stream);
    const size_t need = rglru_simt_workspace_size(B, T, D, dt);
    if (need == 0) return RGLRU_ERR_INVALID_ARG;
    const rglru_status v = validate_prefill(a, need);
    if (v != RGLRU_OK) return v;
    return simt_prefill(a);
}

RGLRU_API rglru_status rglru_prefill(int B, int T, int D, rglru_io_dtype dt, const void *x,
                           const void *gate_branch, const float *conv_w, const float *conv_b,
                           const void *W_a, const float *b_a, const void *W_x, const float *b_x,
                           const float *lambda, const int32_t *segment_pos, void *conv_state,
                           float *h_state, void *y, void *workspace, size_t workspace_bytes,
                           cudaStream_t stream)
{
    const PrefillArgs a = pack(B, T, D, dt, x, gate_branch, conv_w, conv_b, W_a, b_a, W_x, b_x,
                               lambda, segment_pos, conv_state, h_state, y, workspace,
                               workspace_bytes, stream);
    const size_t need = rglru_workspace_size(B, T, D, dt);
    if (need == 0) return RGLRU_ERR_INVALID_ARG;
    const rglru_status v = validate_prefill(a, need);
    if (v != RGLRU_OK) return v;
    return dt == RGLRU_IO_BF16 ? fused_prefill(a) : simt_prefill(a);
}

RGLRU_API rglru_status rglru_decode_step(int B, int D, rglru_io_dtype dt, const void *x,
                               const void *gate_branch, const float *conv_w, const float *conv_b,
                               const void *W_a, const float *b_a, const void *W_x,
                               const float *b_x, const float *lambda, const int32_t *segment_pos,
                               void *conv_state, float *h_state, void *y, void *workspace,
                               size_t workspace_bytes, cudaStream_t stream)
{
    const PrefillArgs a = pack(B, 1, D, dt, x, gate_branch, conv_w, conv_b, W_a, b_a, W_x, b_x,
                               lambda, segment_pos, conv_state, h_state, y, workspace,
                               workspace_bytes, stream);
    const size_t need = rglru_decode_workspace_size(B, D, dt);
    if (need == 0) return RGLRU_ERR_INVALID_ARG;
    const rglru_status v = validate_prefill(a, need);
    if (v != RGLRU_OK) return v;
    return dt == RGLRU_IO_BF16 ? decode_step(a) : simt_prefill(a);
}

RGLRU_API rglru_status rglru_get_device_status(void *workspace, cudaStream_t stream)
{
    if (workspace == nullptr || !aligned16(workspace)) return RGLRU_ERR_WORKSPACE;
    WsHeader h;
    if (cudaMemcpyAsync(&h, workspace, sizeof(int) * 2, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return RGLRU_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return RGLRU_ERR_CUDA;
    if (h.status != 0) {
        if (cudaMemsetAsync(workspace, 0, sizeof(int) * 2, stream) != cudaSuccess) return RGLRU_ERR_CUDA;
        if (cudaStreamSynchronize(stream) != cudaSuccess) return RGLRU_ERR_CUDA;
    }
    return static_cast<rglru_status>(h.status);
}

RGLRU_API rglru_status rglru_debug_suppress_publish(void *workspace, int unit, cudaStream_t stream)
{
    if (workspace == nullptr || !aligned16(workspace)) return RGLRU_ERR_WORKSPACE;
    if (unit < -1) return RGLRU_ERR_INVALID_ARG;
    // The value is copied from host memory that must outlive the async copy:
    // write it with a kernel-free memset pattern instead (4 bytes, little endian).
    const int v = unit + 1;
    char *dst = static_cast<char *>(workspace) + offsetof(WsHeader, debug_unit_plus1);
    for (int k = 0; k < 4; ++k)
        if (cudaMemsetAsync(dst + k, (v >> (8 * k)) & 0xff, 1, stream) != cudaSuccess)
            return RGLRU_ERR_CUDA;
    return RGLRU_OK;
}

}  // extern "C"
