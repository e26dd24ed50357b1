// wkv7_forward_host: the forward with its inputs and outputs in host memory.
//
// The sequence is cut into time slices of whole 32-token chunks.  Slice k's
// inputs go up on one copy stream while slice k-1 computes on the caller's
// stream and slice k-2's y comes down on another copy stream; two device
// slots alternate.  The state stays on the device between slices (slice k
// starts from slice k-1's final state, in place), so the result is the
// forward over the whole sequence, cut at chunk boundaries.
//
//   copy-in  : | in 0 | in 1 | in 2 | in 3 | ...
//   compute  :        | fwd 0 | fwd 1 | fwd 2 | ...
//   copy-out :                | y 0  | y 1   | ...
//
// A slice of the [B, T, H, N] host tensors is B rows of t_k H N elements at
// a pitch of T H N elements: one 2D copy per tensor and slice.

namespace wkv7 {
namespace {

constexpr int kHostSlices = 8;     // target number of time slices

struct HostPlan {
    int t_slice = 0;               // tokens per slice (multiple of 32)
    int nslices = 0;
    size_t in_slot = 0, y_slot = 0, state = 0, fwd_ws = 0;   // bytes of each region
    size_t off_in[2] = {0, 0}, off_y[2] = {0, 0}, off_state = 0, off_fwd = 0, total = 0;
};

size_t dtype_bytes(wkv7_dtype d) { return d == WKV7_F32 ? 4 : 2; }

HostPlan host_plan(int B, int T, int H, wkv7_dtype in_dt, wkv7_dtype y_dt, wkv7_algo algo, int chunk_len) {
    HostPlan p;
    const int chunks = std::max(1, (T + 31) / 32);
    p.t_slice = 32 * ((chunks + kHostSlices - 1) / kHostSlices);
    p.nslices = T > 0 ? (T + p.t_slice - 1) / p.t_slice : 0;
    const size_t vec = (size_t)B * H * kN;                        // elements per token over B, H
    p.in_slot = round_up(6 * vec * p.t_slice * dtype_bytes(in_dt));
    p.y_slot = round_up(vec * p.t_slice * dtype_bytes(y_dt));
    p.state = round_up((size_t)B * H * kN * kN * sizeof(float));
    const int t_last = T - (p.nslices - 1) * p.t_slice;
    if (p.nslices > 0)
        p.fwd_ws = round_up(std::max(wkv7_forward_workspace_size(B, p.t_slice, H, kN, in_dt, algo, chunk_len),
                                     wkv7_forward_workspace_size(B, t_last, H, kN, in_dt, algo, chunk_len)));
    size_t o = 0;
    for (int s = 0; s < 2; ++s) { p.off_in[s] = o; o += p.in_slot; }
    for (int s = 0; s < 2; ++s) { p.off_y[s] = o; o += p.y_slot; }
    p.off_state = o; o += p.state;
    p.off_fwd = o; o += p.fwd_ws;
    p.total = o;
    return p;
}

// rows of `width` bytes, `height` of them, between two pitched buffers
cudaError_t copy_rows(void *dst, size_t dpitch, const void *src, size_t spitch, size_t width, size_t height,
                      cudaMemcpyKind kind, cudaStream_t st, size_t max_pitch) {
    if (height == 1 || (dpitch == width && spitch == width))
        return cudaMemcpyAsync(dst, src, width * height, kind, st);
    if (dpitch <= max_pitch && spitch <= max_pitch)
        return cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, height, kind, st);
    for (size_t r = 0; r < height; ++r) {
        cudaError_t e = cudaMemcpyAsync(static_cast<char *>(dst) + r * dpitch,
                                        static_cast<const char *>(src) + r * spitch, width, kind, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// Streams and events of one call; destroyed when the call returns (the
// driver releases them once the queued work that uses them has finished).
struct HostPipe {
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, end = nullptr, state_in = nullptr;
    cudaEvent_t loaded[2] = {nullptr, nullptr}, computed[2] = {nullptr, nullptr}, drained[2] = {nullptr, nullptr};
    cudaError_t err = cudaSuccess;

    void check(cudaError_t e) { if (err == cudaSuccess && e != cudaSuccess) err = e; }
    bool ok() const { return err == cudaSuccess; }
    HostPipe() {
        check(cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking));
        check(cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking));
        for (cudaEvent_t *e : {&start, &end, &state_in, &loaded[0], &loaded[1], &computed[0], &computed[1],
                               &drained[0], &drained[1]})
            check(cudaEventCreateWithFlags(e, cudaEventDisableTiming));
    }
    ~HostPipe() {
        for (cudaEvent_t e : {start, end, state_in, loaded[0], loaded[1], computed[0], computed[1], drained[0],
                              drained[1]})
            if (e) cudaEventDestroy(e);
        if (in) cudaStreamDestroy(in);
        if (out) cudaStreamDestroy(out);
    }
};

}  // namespace
}  // namespace wkv7

extern "C" {

size_t wkv7_forward_host_workspace_size(int B, int T, int H, int N, wkv7_dtype in_dtype, wkv7_dtype y_dtype,
                                        wkv7_algo algo, int chunk_len) {
    using namespace wkv7;
    if (B <= 0 || H <= 0 || T < 0 || N != kN || !dtype_ok(in_dtype) || !dtype_ok(y_dtype)) return 0;
    return host_plan(B, T, H, in_dtype, y_dtype, resolve_algo(T, in_dtype, algo), chunk_len).total;
}

wkv7_status wkv7_forward_host(int B, int T, int H, int N, wkv7_dtype in_dt, wkv7_dtype y_dt, const void *r,
                              const void *w, const void *k, const void *v, const void *a, const void *b,
                              const float *s0, void *y, float *sT, wkv7_algo algo, int chunk_len, void *workspace,
                              size_t workspace_bytes, cudaStream_t stream) {
    using namespace wkv7;
    wkv7_status s = check_dims(B, T, H, N);
    if (s != WKV7_OK) return s;
    if (!dtype_ok(in_dt) || !dtype_ok(y_dt)) return WKV7_ERR_INVALID_ARG;
    if (algo != WKV7_ALGO_AUTO && algo != WKV7_ALGO_SEQ && algo != WKV7_ALGO_CHUNK) return WKV7_ERR_INVALID_ARG;
    if (chunk_len != 0 && chunk_len != 32) return WKV7_ERR_UNSUPPORTED;
    if (!opt_ptr_ok(s0) || !opt_ptr_ok(sT)) return WKV7_ERR_INVALID_ARG;
    if ((size_t)B * H == 0) return WKV7_OK;
    if (T > 0)
        for (const void *p : {r, w, k, v, a, b, (const void *)y})
            if (!ptr_ok(p)) return WKV7_ERR_INVALID_ARG;
    // one algorithm for every slice: the one the whole sequence resolves to
    const wkv7_algo resolved = resolve_algo(T, in_dt, algo);
    if (resolved == WKV7_ALGO_CHUNK && in_dt != WKV7_BF16) return WKV7_ERR_UNSUPPORTED;
    const HostPlan p = host_plan(B, T, H, in_dt, y_dt, resolved, chunk_len);
    if (!ptr_ok(workspace) || workspace_bytes < p.total) return WKV7_ERR_INVALID_ARG;

    char *ws = static_cast<char *>(workspace);
    float *dstate = reinterpret_cast<float *>(ws + p.off_state);
    const size_t state_bytes = (size_t)B * H * kN * kN * sizeof(float);
    const size_t ib = dtype_bytes(in_dt), yb = dtype_bytes(y_dt);
    const size_t tok = (size_t)H * kN;                     // elements per (b, t)
    int dev = 0, max_pitch = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&max_pitch, cudaDevAttrMaxPitch, dev) != cudaSuccess)
        return WKV7_ERR_CUDA;

    HostPipe pipe;
    if (!pipe.ok()) return WKV7_ERR_CUDA;
    pipe.check(cudaEventRecord(pipe.start, stream));
    pipe.check(cudaStreamWaitEvent(pipe.in, pipe.start, 0));
    pipe.check(cudaStreamWaitEvent(pipe.out, pipe.start, 0));
    // entry state
    if (s0) {
        pipe.check(cudaMemcpyAsync(dstate, s0, state_bytes, cudaMemcpyHostToDevice, pipe.in));
        pipe.check(cudaEventRecord(pipe.state_in, pipe.in));
        pipe.check(cudaStreamWaitEvent(stream, pipe.state_in, 0));
    } else {
        pipe.check(cudaMemsetAsync(dstate, 0, state_bytes, stream));
    }
    const void *src[6] = {r, w, k, v, a, b};
    wkv7_status fwd_status = WKV7_OK;
    for (int sl = 0; sl < p.nslices && pipe.ok() && fwd_status == WKV7_OK; ++sl) {
        const int slot = sl & 1;
        const int t0 = sl * p.t_slice, tl = std::min(p.t_slice, T - t0);
        char *in = ws + p.off_in[slot];
        const size_t plane = (size_t)B * tl * tok * ib;    // one input tensor of this slice
        // inputs of slice sl, once slice sl-2 has finished reading the slot
        if (sl >= 2) pipe.check(cudaStreamWaitEvent(pipe.in, pipe.computed[slot], 0));
        for (int x = 0; x < 6; ++x)
            pipe.check(copy_rows(in + x * plane, tl * tok * ib, static_cast<const char *>(src[x]) + t0 * tok * ib,
                                 (size_t)T * tok * ib, tl * tok * ib, B, cudaMemcpyHostToDevice, pipe.in,
                                 (size_t)max_pitch));
        pipe.check(cudaEventRecord(pipe.loaded[slot], pipe.in));
        // the forward of slice sl, once its inputs are in and slice sl-2's y is out
        pipe.check(cudaStreamWaitEvent(stream, pipe.loaded[slot], 0));
        if (sl >= 2) pipe.check(cudaStreamWaitEvent(stream, pipe.drained[slot], 0));
        if (!pipe.ok()) break;
        void *yd = ws + p.off_y[slot];
        const void *d[6];
        for (int x = 0; x < 6; ++x) d[x] = in + x * plane;
        fwd_status = wkv7_forward(B, tl, H, N, in_dt, y_dt, d[0], d[1], d[2], d[3], d[4], d[5], dstate, yd, dstate,
                                  resolved, chunk_len, p.fwd_ws ? ws + p.off_fwd : nullptr, p.fwd_ws, stream);
        pipe.check(cudaEventRecord(pipe.computed[slot], stream));
        // y of slice sl back to the host
        pipe.check(cudaStreamWaitEvent(pipe.out, pipe.computed[slot], 0));
        pipe.check(copy_rows(static_cast<char *>(y) + t0 * tok * yb, (size_t)T * tok * yb, yd, tl * tok * yb,
                             tl * tok * yb, B, cudaMemcpyDeviceToHost, pipe.out, (size_t)max_pitch));
        pipe.check(cudaEventRecord(pipe.drained[slot], pipe.out));
    }
    // final state after the last slice's forward (stream order)
    if (sT && pipe.ok() && fwd_status == WKV7_OK) {
        pipe.check(cudaEventRecord(pipe.computed[0], stream));
        pipe.check(cudaStreamWaitEvent(pipe.out, pipe.computed[0], 0));
        pipe.check(cudaMemcpyAsync(sT, dstate, state_bytes, cudaMemcpyDeviceToHost, pipe.out));
    }
    // join both copy streams back into the caller's stream
    pipe.check(cudaEventRecord(pipe.end, pipe.out));
    pipe.check(cudaStreamWaitEvent(stream, pipe.end, 0));
    pipe.check(cudaEventRecord(pipe.end, pipe.in));
    pipe.check(cudaStreamWaitEvent(stream, pipe.end, 0));
    if (fwd_status != WKV7_OK) return fwd_status;
    return pipe.ok() ? WKV7_OK : WKV7_ERR_CUDA;
}

}  // extern "C"
