// prefill_host.cu -- rglru_prefill_host: the prefill with its activations in
// host memory, the copies overlapped with the kernels.
//
// The batch is cut into chunks of rows_per_chunk sequences (sequences are
// independent, and the fused kernel's results do not depend on how tiles are
// split between launches, so the result is the one-call result bit for bit).
// Two device staging slots alternate between chunks.  Chunk k's upload runs
// on an upload stream, its kernel on the caller's stream and its download on
// a download stream, so the upload of chunk k + 1, the kernel of chunk k and
// the download of chunk k - 1 overlap.  Events order each slot's reuse:
//   upload k     waits for kernel k - 2 (which read the slot's inputs);
//   kernel k     waits for upload k and for download k - 2 (which read the
//                slot's y);
//   download k   waits for kernel k.
// The caller's stream finally waits for the last downloads, so everything the
// caller enqueues after the call sees y complete in host memory.
#include <cstdint>

#include "internal.h"

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return rglru::align_up(v, kAlign); }

struct Staging {
    size_t act, sp, slot;  // bytes of one chunk's x (= g = y), segment_pos, one slot
};

bool staging_layout(int B, int T, int D, rglru_io_dtype dt, int rows, Staging &s)
{
    if (B < 1 || T < 1 || D < rglru::kHead || D % rglru::kHead != 0 || rows < 1) return false;
    if (dt != RGLRU_IO_F32 && dt != RGLRU_IO_BF16) return false;
    const size_t r = (size_t)(rows < B ? rows : B);
    const size_t e = dt == RGLRU_IO_BF16 ? 2 : 4;
    s.act = align_up(r * T * D * e);
    s.sp = align_up(r * T * sizeof(int32_t));
    s.slot = 3 * s.act + s.sp;
    return true;
}

// Streams and events of one call, released on every exit path (the runtime
// defers the release of objects whose work is still pending).
struct CallObjects {
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t start = nullptr, h2d[2] = {}, comp[2] = {}, d2h[2] = {};
    ~CallObjects()
    {
        for (cudaEvent_t e : {start, h2d[0], h2d[1], comp[0], comp[1], d2h[0], d2h[1]})
            if (e) cudaEventDestroy(e);
        if (up) cudaStreamDestroy(up);
        if (down) cudaStreamDestroy(down);
    }
    bool create()
    {
        if (cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking) != cudaSuccess) return false;
        if (cudaStreamCreateWithFlags(&down, cudaStreamNonBlocking) != cudaSuccess) return false;
        for (cudaEvent_t *e : {&start, &h2d[0], &h2d[1], &comp[0], &comp[1], &d2h[0], &d2h[1]})
            if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return false;
        return true;
    }
};

}  // namespace

extern "C" {

RGLRU_API size_t rglru_prefill_host_staging_size(int B, int T, int D, rglru_io_dtype dt, int rows_per_chunk)
{
    Staging s;
    if (!staging_layout(B, T, D, dt, rows_per_chunk, s)) return 0;
    return 2 * s.slot;
}

RGLRU_API rglru_status rglru_prefill_host(int B, int T, int D, rglru_io_dtype dt, const void *x_host,
                                          const void *gate_branch_host, const float *conv_w,
                                          const float *conv_b, const void *W_a, const float *b_a,
                                          const void *W_x, const float *b_x, const float *lambda,
                                          const int32_t *segment_pos_host, void *conv_state, float *h_state,
                                          void *y_host, int rows_per_chunk, void *staging,
                                          size_t staging_bytes, void *workspace, size_t workspace_bytes,
                                          cudaStream_t stream)
{
    Staging s;
    if (!staging_layout(B, T, D, dt, rows_per_chunk, s)) return RGLRU_ERR_INVALID_ARG;
    if (x_host == nullptr || gate_branch_host == nullptr || segment_pos_host == nullptr || y_host == nullptr ||
        conv_state == nullptr || h_state == nullptr)
        return RGLRU_ERR_INVALID_ARG;
    if (staging == nullptr || (reinterpret_cast<uintptr_t>(staging) & (kAlign - 1)) != 0 ||
        staging_bytes < 2 * s.slot)
        return RGLRU_ERR_WORKSPACE;
    const int R = rows_per_chunk < B ? rows_per_chunk : B;
    if (workspace_bytes < rglru_workspace_size(R, T, D, dt)) return RGLRU_ERR_WORKSPACE;

    const size_t e = dt == RGLRU_IO_BF16 ? 2 : 4;
    const size_t row_act = (size_t)T * D * e, row_sp = (size_t)T * sizeof(int32_t);
    const char *xh = static_cast<const char *>(x_host), *gh = static_cast<const char *>(gate_branch_host);
    const char *sh = reinterpret_cast<const char *>(segment_pos_host);
    char *yh = static_cast<char *>(y_host);
    // y_host must not overlap the host inputs
    const uintptr_t y0 = reinterpret_cast<uintptr_t>(yh), y1 = y0 + (size_t)B * row_act;
    for (const char *in : {xh, gh, sh}) {
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(in);
        const uintptr_t a1 = a0 + (size_t)B * (in == sh ? row_sp : row_act);
        if (a0 < y1 && y0 < a1) return RGLRU_ERR_INVALID_ARG;
    }

    // the staging buffer must not overlap any device argument (an upload into
    // one slot runs while the other slot's kernel updates the states)
    {
        const uintptr_t s0 = reinterpret_cast<uintptr_t>(staging), s1 = s0 + 2 * s.slot;
        const size_t wbytes = (size_t)(D / rglru::kHead) * rglru::kHead * rglru::kHead * e;
        const struct {
            const void *p;
            size_t n;
        } dev[] = {{conv_state, (size_t)B * 3 * D * e}, {h_state, (size_t)B * D * sizeof(float)},
                   {workspace, workspace_bytes}, {conv_w, 4 * (size_t)D * sizeof(float)},
                   {conv_b, D * sizeof(float)}, {b_a, D * sizeof(float)}, {b_x, D * sizeof(float)},
                   {lambda, D * sizeof(float)}, {W_a, wbytes}, {W_x, wbytes}};
        for (const auto &b : dev) {
            const uintptr_t a0 = reinterpret_cast<uintptr_t>(b.p), a1 = a0 + b.n;
            if (b.p != nullptr && a0 < s1 && s0 < a1) return RGLRU_ERR_INVALID_ARG;
        }
    }

    // Each chunk's kernel call: rows [b0, b0 + rows) of the states, the
    // inputs and y in staging slot k % 2.
    char *st = static_cast<char *>(staging);
    auto chunk_call = [&](int k, int &b0, int &rows) {
        b0 = k * R;
        rows = B - b0 < R ? B - b0 : R;
        char *xs = st + (k & 1) * s.slot, *gs = xs + s.act, *ys = gs + s.act, *ss = ys + s.act;
        rglru::PrefillArgs a;
        a.B = rows; a.T = T; a.D = D; a.dt = dt;
        a.x = xs; a.g = gs; a.conv_w = conv_w; a.conv_b = conv_b;
        a.W_a = W_a; a.b_a = b_a; a.W_x = W_x; a.b_x = b_x; a.lambda = lambda;
        a.segpos = reinterpret_cast<const int32_t *>(ss);
        a.conv_state = static_cast<char *>(conv_state) + (size_t)b0 * 3 * D * e;
        a.h_state = h_state + (size_t)b0 * D;
        a.y = ys; a.ws = workspace; a.ws_bytes = workspace_bytes; a.stream = stream;
        return a;
    };
    // every chunk's arguments are checked before anything is enqueued
    const int chunks = (B + R - 1) / R;
    for (int k = 0; k < chunks; ++k) {
        int b0, rows;
        const rglru::PrefillArgs a = chunk_call(k, b0, rows);
        const rglru_status v = rglru::validate_prefill(a, rglru_workspace_size(rows, T, D, dt));
        if (v != RGLRU_OK) return v;
    }

    CallObjects o;
    if (!o.create()) return RGLRU_ERR_CUDA;
    // On a CUDA error part-way, `stream` still waits for what was enqueued
    // (events never recorded are complete), so later work on it does not race
    // with copies of this call.
    auto fail = [&]() {
        for (cudaEvent_t ev : {o.h2d[0], o.h2d[1], o.d2h[0], o.d2h[1]}) cudaStreamWaitEvent(stream, ev, 0);
        return RGLRU_ERR_CUDA;
    };
    // the upload may overwrite staging that work enqueued earlier on `stream` reads
    if (cudaEventRecord(o.start, stream) != cudaSuccess || cudaStreamWaitEvent(o.up, o.start, 0) != cudaSuccess)
        return RGLRU_ERR_CUDA;
    for (int k = 0; k < chunks; ++k) {
        int b0, rows;
        const rglru::PrefillArgs a = chunk_call(k, b0, rows);
        const int sl = k & 1;
        void *xs = const_cast<void *>(a.x), *gs = const_cast<void *>(a.g);
        void *ss = const_cast<int32_t *>(a.segpos);
        if (k >= 2 && cudaStreamWaitEvent(o.up, o.comp[sl], 0) != cudaSuccess) return fail();
        if (cudaMemcpyAsync(xs, xh + b0 * row_act, rows * row_act, cudaMemcpyHostToDevice, o.up) != cudaSuccess ||
            cudaMemcpyAsync(gs, gh + b0 * row_act, rows * row_act, cudaMemcpyHostToDevice, o.up) != cudaSuccess ||
            cudaMemcpyAsync(ss, sh + b0 * row_sp, rows * row_sp, cudaMemcpyHostToDevice, o.up) != cudaSuccess ||
            cudaEventRecord(o.h2d[sl], o.up) != cudaSuccess)
            return fail();
        if (cudaStreamWaitEvent(stream, o.h2d[sl], 0) != cudaSuccess) return fail();
        if (k >= 2 && cudaStreamWaitEvent(stream, o.d2h[sl], 0) != cudaSuccess) return fail();
        const rglru_status v = dt == RGLRU_IO_BF16 ? rglru::fused_prefill(a) : rglru::simt_prefill(a);
        if (v != RGLRU_OK) {
            fail();
            return v;
        }
        if (cudaEventRecord(o.comp[sl], stream) != cudaSuccess || cudaStreamWaitEvent(o.down, o.comp[sl], 0) != cudaSuccess)
            return fail();
        if (cudaMemcpyAsync(yh + b0 * row_act, a.y, rows * row_act, cudaMemcpyDeviceToHost, o.down) != cudaSuccess ||
            cudaEventRecord(o.d2h[sl], o.down) != cudaSuccess)
            return fail();
    }
    for (int sl = 0; sl < 2 && sl < chunks; ++sl)
        if (cudaStreamWaitEvent(stream, o.d2h[sl], 0) != cudaSuccess) return RGLRU_ERR_CUDA;
    return RGLRU_OK;
}

}  // extern "C"
