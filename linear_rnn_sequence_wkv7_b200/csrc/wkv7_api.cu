// extern "C" entry points of libwkv7.so: argument validation, workspace
// layout and kernel dispatch.  Every check happens on the host before any
// launch; nothing here allocates device memory or synchronizes (except
// wkv7_get_last_status / wkv7_get_device_status).
#include <stdint.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"

namespace wkv7 {

cudaError_t fwd_seq(int B, int T, int H, wkv7_dtype in_dt, wkv7_dtype y_dt, const void *r,
                    const void *w, const void *k, const void *v, const void *a, const void *b,
                    const float *s0, void *y, float *sT, long long wait_limit, cudaStream_t st);
cudaError_t fwd_checkpoints(int B, int T, int H, wkv7_dtype in_dt, const void *r, const void *w,
                            const void *k, const void *v, const void *a, const void *b, const float *s0,
                            float *ckpt, int CK, float *sT, long long wait_limit, cudaStream_t st);
cudaError_t step(int B, int H, wkv7_dtype in_dt, wkv7_dtype y_dt, const void *r, const void *w,
                 const void *k, const void *v, const void *a, const void *b, float *state, void *y,
                 cudaStream_t st);
cudaError_t bwd_chunked(int B, int T, int H, wkv7_dtype in_dt, wkv7_dtype g_dt, const void *r, const void *w,
                        const void *k, const void *v, const void *a, const void *b, const void *dy,
                        const float *dsT, const float *ckpt, const float *sfin, float *dS_out, void *dr,
                        void *dw, void *dk, void *dv, void *da, void *db, float *ds0, float *scratch,
                        size_t scratch_bytes, int sms, long long wait_limit, cudaStream_t st,
                        const uint4 *mq = nullptr);
size_t bwd_chunk_ckpt_bytes(int B, int T, int H);
size_t bwd_mq_bytes(int B, int T, int H);
bool bwd_use_dchain(int B, int T, int H, int sms, size_t scratch_cap);
cudaError_t bwd_dstate(int B, int T, int H, wkv7_dtype in_dt, const void *r, const void *w, const void *a,
                       const void *b, const void *dy, const float *dsT, float *dS_out, float *ds0, float *scratch,
                       size_t scratch_bytes, int sms, cudaStream_t st);
size_t dstate_scratch_for(int B, int T, int H, int sms, bool need_dS);
cudaError_t compose_adjoints(int B, int H, int nseg, const float *dsT, const float *summary, const float *F,
                             float *adj, cudaStream_t st);
cudaError_t fwd_chunk(int B, int T, int H, wkv7_dtype y_dt, const void *r, const void *w, const void *k,
                      const void *v, const void *a, const void *b, const float *s0, void *y, float *sT,
                      int nseg, void *workspace, long long wait_limit, cudaStream_t st, float *ckpt,
                      const EpiArgs &epi = EpiArgs{}, bool fixup = false, uint4 *mq = nullptr);
int chunk_segments_fixup(int B, int T, int H, int sm_count);
size_t chunk_fixup_workspace_bytes(int B, int T, int H, int nseg);
cudaError_t fwd_seq_train(int B, int T, int H, wkv7_dtype in_dt, wkv7_dtype y_dt, const void *r, const void *w,
                          const void *k, const void *v, const void *a, const void *b, const float *s0, void *y,
                          float *sT, float *ckpt, int CK, long long wait_limit, cudaStream_t st);
int chunk_segments(int B, int T, int H, int sm_count, bool summarize_last);
size_t chunk_workspace_bytes(int B, int T, int H, int nseg);
cudaError_t fwd_chunk_summary(int B, int T, int H, const void *r, const void *w, const void *k, const void *v,
                              const void *a, const void *b, float *summary, int nseg, void *workspace,
                              long long wait_limit, cudaStream_t st);
cudaError_t fwd_chunk_continue(int B, int T, int H, wkv7_dtype y_dt, const void *r, const void *w, const void *k,
                               const void *v, const void *a, const void *b, const float *s_in, void *y, float *sT,
                               int nseg, void *workspace, long long wait_limit, cudaStream_t st);
size_t summary_workspace_bytes(int B, int T, int H, int nseg);
cudaError_t compose_states(int B, int H, int nseg, const float *s0, const float *summary, float *out,
                           cudaStream_t st);

namespace {

constexpr int kBwdChunk = 32;        // backward chunk (= checkpoint interval, tokens)
constexpr long long kDefaultWaitCycles = 2000000000LL;   // ~1 s of SM clock
std::atomic<long long> g_wait_limit{0};                  // 0 = default
constexpr size_t kWsAlign = 256;

bool dtype_ok(wkv7_dtype d) { return d == WKV7_F32 || d == WKV7_BF16; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ptr_ok(const void *p) { return p != nullptr && aligned16(p); }
bool opt_ptr_ok(const void *p) { return p == nullptr || aligned16(p); }
size_t round_up(size_t x) { return (x + kWsAlign - 1) / kWsAlign * kWsAlign; }

wkv7_status from_cuda(cudaError_t e) { return e == cudaSuccess ? WKV7_OK : WKV7_ERR_CUDA; }

// Shape checks common to every entry point.  Returns OK, INVALID_ARG or UNSUPPORTED.
wkv7_status check_dims(int B, int T, int H, int N) {
    if (B < 0 || T < 0 || H < 0 || N <= 0) return WKV7_ERR_INVALID_ARG;
    if (B > 65535) return WKV7_ERR_UNSUPPORTED;             // grid.y limit of the scan kernels
    if ((int64_t)B * H > (int64_t)INT32_MAX / 64) return WKV7_ERR_UNSUPPORTED;
    if (N != kN) return WKV7_ERR_UNSUPPORTED;
    return WKV7_OK;
}

// sT (or ds0) := src, or zeros when src is NULL; used for T = 0.
wkv7_status copy_or_zero_state(float *dst, const float *src, int B, int H, cudaStream_t st) {
    if (!dst) return WKV7_OK;
    const size_t bytes = (size_t)B * H * kN * kN * sizeof(float);
    if (bytes == 0 || dst == src) return WKV7_OK;
    if (src) return from_cuda(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st));
    return from_cuda(cudaMemsetAsync(dst, 0, bytes, st));
}

// The algorithm AUTO resolves to: the chunked tensor-core form for bf16 inputs
// with at least two chunks of tokens, else the sequential scan (the only form
// for fp32 inputs, whose 1e-5 tolerance the bf16-split products cannot meet).
wkv7_algo resolve_algo(int T, wkv7_dtype in_dt, wkv7_algo algo) {
    if (algo != WKV7_ALGO_AUTO) return algo;
    return (in_dt == WKV7_BF16 && T >= 64) ? WKV7_ALGO_CHUNK : WKV7_ALGO_SEQ;
}

int current_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

// Segments of the summary / continue pair: the cost model's choice when the
// workspace holds their scratch, else 1 (both calls of a pair must get the
// same workspace size, so they agree).
int summary_segments(int B, int T, int H, const void *workspace, size_t workspace_bytes) {
    const int sms = current_sm_count();
    if (sms <= 0 || T <= 0 || workspace == nullptr || !aligned16(workspace)) return 1;
    const int want = chunk_segments(B, T, H, sms, true);
    return (want > 1 && workspace_bytes >= summary_workspace_bytes(B, T, H, want)) ? want : 1;
}

size_t bwd_ckpt_bytes(int B, int T, int H) { return bwd_chunk_ckpt_bytes(B, T, H); }

// Scratch shared by the backward's checkpoint pass (the segmented chunked
// forward, bf16 inputs) and then its state-gradient sweep (segments too).
int bwd_ckpt_segments(int B, int T, int H, int sms) { return sms > 0 ? chunk_segments(B, T, H, sms, false) : 1; }
size_t bwd_scratch_bytes(int B, int T, int H) {
    const int sms = current_sm_count();
    return std::max(round_up(chunk_workspace_bytes(B, T, H, bwd_ckpt_segments(B, T, H, sms))),
                    round_up(dstate_scratch_for(B, T, H, sms, true)));
}
size_t state_bytes(int B, int H) { return (size_t)B * H * kN * kN * sizeof(float); }

// wkv7_backward's workspace without the chunks' transition images: the state
// before every chunk, dL/dS at every chunk end, the final state and the
// segmented passes' scratch.  With the images too (wkv7_backward_workspace_size)
// dS can come from the transition chain.
size_t bwd_workspace_min(int B, int T, int H) {
    return 2 * round_up(bwd_ckpt_bytes(B, T, H)) + round_up(state_bytes(B, H)) + bwd_scratch_bytes(B, T, H);
}

}  // namespace
}  // namespace wkv7

using namespace wkv7;

extern "C" {

int wkv7_abi_version(void) { return WKV7_ABI_VERSION; }

const char *wkv7_status_string(wkv7_status s) {
    switch (s) {
        case WKV7_OK: return "ok";
        case WKV7_ERR_INVALID_ARG: return "invalid argument";
        case WKV7_ERR_UNSUPPORTED: return "unsupported";
        case WKV7_ERR_CUDA: return "CUDA error";
        case WKV7_ERR_TIMEOUT: return "device wait timed out";
        case WKV7_ERR_RANGE: return "input outside the chunked form's numeric domain";
        case WKV7_ERR_TOO_LARGE: return "problem exceeds the fixed scratch of wkv7_backward_noalloc";
    }
    return "unknown status";
}

size_t wkv7_forward_workspace_size(int B, int T, int H, int N, wkv7_dtype in_dtype, wkv7_algo algo,
                                   int chunk_len) {
    (void)chunk_len;
    if (B <= 0 || T <= 0 || H <= 0 || N != kN || !dtype_ok(in_dtype)) return 0;
    if (resolve_algo(T, in_dtype, algo) != WKV7_ALGO_CHUNK || in_dtype != WKV7_BF16) return 0;
    const int sms = current_sm_count();
    if (sms <= 0) return 0;
    // enough for either segmented form: the fix-up form (plain forward) or
    // the output-run form (with checkpoints or the time-mix epilogue)
    return std::max(chunk_workspace_bytes(B, T, H, chunk_segments(B, T, H, sms, false)),
                    chunk_fixup_workspace_bytes(B, T, H, chunk_segments_fixup(B, T, H, sms)));
}

}  // extern "C"

namespace wkv7 {
namespace {

// wkv7_forward, and with ckpt non-null the training forward that also keeps
// the state before every 32-token chunk; with epi.rho set (the chunked form
// only) the time-mix output epilogue replaces y
wkv7_status forward_impl(int B, int T, int H, int N, wkv7_dtype in_dt, wkv7_dtype y_dt, const void *r,
                         const void *w, const void *k, const void *v, const void *a, const void *b,
                         const float *s0, void *y, float *sT, wkv7_algo algo, int chunk_len, void *workspace,
                         size_t workspace_bytes, cudaStream_t stream, float *ckpt,
                         const EpiArgs &epi = EpiArgs{}, uint4 *mq = nullptr) {
    wkv7_status s = check_dims(B, T, H, N);
    if (s != WKV7_OK) return s;
    if (!dtype_ok(in_dt) || !dtype_ok(y_dt)) return WKV7_ERR_INVALID_ARG;
    if (algo != WKV7_ALGO_AUTO && algo != WKV7_ALGO_SEQ && algo != WKV7_ALGO_CHUNK) return WKV7_ERR_INVALID_ARG;
    if (chunk_len != 0 && chunk_len != 32) return WKV7_ERR_UNSUPPORTED;   // the chunked form's chunk
    if (!opt_ptr_ok(s0) || !opt_ptr_ok(sT)) return WKV7_ERR_INVALID_ARG;
    if ((size_t)B * H == 0) return WKV7_OK;
    if (T == 0) return copy_or_zero_state(sT, s0, B, H, stream);
    for (const void *p : {r, w, k, v, a, b, (const void *)y})
        if (!ptr_ok(p)) return WKV7_ERR_INVALID_ARG;
    if (resolve_algo(T, in_dt, algo) == WKV7_ALGO_CHUNK) {
        if (in_dt != WKV7_BF16) return WKV7_ERR_UNSUPPORTED;
        const long long lim = g_wait_limit.load();
        // sequence segments run in parallel when there are too few heads to
        // fill the GPU and the caller provided the workspace they need
        int nseg = 1;
        bool fixup = false;
        const int sms = current_sm_count();
        const bool ws_ok = workspace != nullptr && aligned16(workspace);
        if (sms > 0 && ws_ok && ckpt == nullptr && epi.rho == nullptr) {
            // plain forward: the fix-up form (one dual pass over every segment,
            // then y = y0 + S_in q) when its scratch is there
            const int want = chunk_segments_fixup(B, T, H, sms);
            if (want > 1 && workspace_bytes >= chunk_fixup_workspace_bytes(B, T, H, want)) {
                nseg = want;
                fixup = true;
            }
        }
        if (sms > 0 && ws_ok && !fixup) {
            const int want = chunk_segments(B, T, H, sms, false);
            if (want > 1 && workspace_bytes >= chunk_workspace_bytes(B, T, H, want)) nseg = want;
        }
        return from_cuda(fwd_chunk(B, T, H, y_dt, r, w, k, v, a, b, s0, y, sT, nseg, workspace,
                                   lim > 0 ? lim : kDefaultWaitCycles, stream, ckpt, epi, fixup, mq));
    }
    if (epi.rho) return WKV7_ERR_UNSUPPORTED;      // the scan's epilogue is a separate pass (timemix.cu)
    const long long lim = g_wait_limit.load() > 0 ? g_wait_limit.load() : kDefaultWaitCycles;
    if (ckpt)
        return from_cuda(fwd_seq_train(B, T, H, in_dt, y_dt, r, w, k, v, a, b, s0, y, sT, ckpt, kBwdChunk, lim, stream));
    return from_cuda(fwd_seq(B, T, H, in_dt, y_dt, r, w, k, v, a, b, s0, y, sT, lim, stream));
}

}  // namespace
}  // namespace wkv7

extern "C" {

wkv7_status wkv7_forward(int B, int T, int H, int N, wkv7_dtype in_dt, wkv7_dtype y_dt, const void *r,
                         const void *w, const void *k, const void *v, const void *a, const void *b,
                         const float *s0, void *y, float *sT, wkv7_algo algo, int chunk_len,
                         void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    return forward_impl(B, T, H, N, in_dt, y_dt, r, w, k, v, a, b, s0, y, sT, algo, chunk_len, workspace,
                        workspace_bytes, stream, nullptr);
}

size_t wkv7_saved_states_size(int B, int T, int H, int N) {
    if (B <= 0 || T <= 0 || H <= 0 || N != kN) return 0;
    // the state before every chunk, then every chunk's transition image
    return round_up(bwd_ckpt_bytes(B, T, H)) + round_up(bwd_mq_bytes(B, T, H));
}

wkv7_status wkv7_forward_train(int B, int T, int H, int N, wkv7_dtype in_dt, wkv7_dtype y_dt, const void *r,
                               const void *w, const void *k, const void *v, const void *a, const void *b,
                               const float *s0, void *y, float *sT, float *states, wkv7_algo algo, int chunk_len,
                               void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    wkv7_status s = check_dims(B, T, H, N);
    if (s != WKV7_OK) return s;
    if ((size_t)B * H > 0 && (!ptr_ok(sT) || (T > 0 && !ptr_ok(states)))) return WKV7_ERR_INVALID_ARG;
    if (in_dt != WKV7_BF16 || (size_t)B * H == 0 || T == 0)
        return forward_impl(B, T, H, N, in_dt, y_dt, r, w, k, v, a, b, s0, y, sT, algo, chunk_len, workspace,
                            workspace_bytes, stream, states);
    // bf16 inputs: the states and every chunk's transition come from the
    // chunked form (the backward's dS chain reads the transitions)
    uint4 *mq = reinterpret_cast<uint4 *>(reinterpret_cast<char *>(states) + round_up(bwd_ckpt_bytes(B, T, H)));
    if (resolve_algo(T, in_dt, algo) == WKV7_ALGO_CHUNK)
        return forward_impl(B, T, H, N, in_dt, y_dt, r, w, k, v, a, b, s0, y, sT, algo, chunk_len, workspace,
                            workspace_bytes, stream, states, EpiArgs{}, mq);
    // the scan for y and sT, then a chunked checkpoint pass (no y) for the states and transitions
    s = forward_impl(B, T, H, N, in_dt, y_dt, r, w, k, v, a, b, s0, y, sT, algo, chunk_len, workspace,
                     workspace_bytes, stream, nullptr);
    if (s != WKV7_OK) return s;
    const long long lim = g_wait_limit.load();
    return from_cuda(fwd_chunk(B, T, H, WKV7_BF16, r, w, k, v, a, b, s0, nullptr, nullptr, 1, nullptr,
                               lim > 0 ? lim : kDefaultWaitCycles, stream, states, EpiArgs{}, false, mq));
}

size_t wkv7_backward_from_states_workspace_size(int B, int T, int H, int N) {
    if (B <= 0 || T <= 0 || H <= 0 || N != kN) return 0;
    // dL/dS at every chunk end, the segmented sweep's scratch
    return round_up(bwd_ckpt_bytes(B, T, H)) + round_up(dstate_scratch_for(B, T, H, current_sm_count(), true));
}

wkv7_status wkv7_backward_from_states(int B, int T, int H, int N, wkv7_dtype in_dt, wkv7_dtype g_dt,
                                      const void *r, const void *w, const void *k, const void *v, const void *a,
                                      const void *b, const float *states, const float *sT, const void *dy,
                                      const float *dsT, void *dr, void *dw, void *dk, void *dv, void *da,
                                      void *db, float *ds0, void *workspace, size_t workspace_bytes,
                                      cudaStream_t stream) {
    wkv7_status s = check_dims(B, T, H, N);
    if (s != WKV7_OK) return s;
    if (!dtype_ok(in_dt) || !dtype_ok(g_dt)) return WKV7_ERR_INVALID_ARG;
    if (!opt_ptr_ok(dsT) || !ptr_ok(ds0)) return WKV7_ERR_INVALID_ARG;
    if ((size_t)B * H == 0) return WKV7_OK;
    if (T == 0) return copy_or_zero_state(ds0, dsT, B, H, stream);
    for (const void *p : {r, w, k, v, a, b, dy, (const void *)states, (const void *)sT, (const void *)dr,
                          (const void *)dw, (const void *)dk, (const void *)dv, (const void *)da, (const void *)db})
        if (!ptr_ok(p)) return WKV7_ERR_INVALID_ARG;
    if (workspace_bytes < wkv7_backward_from_states_workspace_size(B, T, H, N) || !ptr_ok(workspace))
        return WKV7_ERR_INVALID_ARG;
    const long long lim = g_wait_limit.load();
    const size_t ds_bytes = round_up(bwd_ckpt_bytes(B, T, H));
    char *ws = static_cast<char *>(workspace);
    // bf16 inputs: dS by the transition chain from the transitions the
    // training forward saved after the states; fp32: the per-token sweep
    const uint4 *mq = in_dt == WKV7_BF16
                          ? reinterpret_cast<const uint4 *>(reinterpret_cast<const char *>(states) +
                                                            round_up(bwd_ckpt_bytes(B, T, H)))
                          : nullptr;
    return from_cuda(bwd_chunked(B, T, H, in_dt, g_dt, r, w, k, v, a, b, dy, dsT, states, sT,
                                 reinterpret_cast<float *>(ws), dr, dw, dk, dv, da, db, ds0,
                                 reinterpret_cast<float *>(ws + ds_bytes), workspace_bytes - ds_bytes,
                                 current_sm_count(), lim > 0 ? lim : kDefaultWaitCycles, stream, mq));
}

size_t wkv7_forward_summary_workspace_size(int B, int T, int H, int N) {
    if (B <= 0 || T <= 0 || H <= 0 || N != kN) return 0;
    const int sms = current_sm_count();
    if (sms <= 0) return 0;
    return summary_workspace_bytes(B, T, H, chunk_segments(B, T, H, sms, true));
}

wkv7_status wkv7_forward_summary(int B, int T, int H, int N, wkv7_dtype in_dt, const void *r, const void *w,
                                 const void *k, const void *v, const void *a, const void *b, float *summary,
                                 void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    wkv7_status s = check_dims(B, T, H, N);
    if (s != WKV7_OK) return s;
    if (!dtype_ok(in_dt)) return WKV7_ERR_INVALID_ARG;
    if (in_dt != WKV7_BF16) return WKV7_ERR_UNSUPPORTED;                // computed by the chunked form
    if (!opt_ptr_ok(workspace)) return WKV7_ERR_INVALID_ARG;
    if ((size_t)B * H == 0) return WKV7_OK;
    if (!ptr_ok(summary)) return WKV7_ERR_INVALID_ARG;
    if (T > 0)
        for (const void *p : {r, w, k, v, a, b})
            if (!ptr_ok(p)) return WKV7_ERR_INVALID_ARG;
    const long long lim = g_wait_limit.load();
    const int nseg = summary_segments(B, T, H, workspace, workspace_bytes);
    return from_cuda(fwd_chunk_summary(B, T, H, r, w, k, v, a, b, summary, nseg, workspace,
                                       lim > 0 ? lim : kDefaultWaitCycles, stream));
}

wkv7_status wkv7_forward_continue(int B, int T, int H, int N, wkv7_dtype in_dt, wkv7_dtype y_dt, const void *r,
                                  const void *w, const void *k, const void *v, const void *a, const void *b,
                                  const float *s_in, void *y, float *sT, void *workspace, size_t workspace_bytes,
                                  cudaStream_t stream) {
    wkv7_status s = check_dims(B, T, H, N);
    if (s != WKV7_OK) return s;
    if (!dtype_ok(in_dt) || !dtype_ok(y_dt)) return WKV7_ERR_INVALID_ARG;
    if (in_dt != WKV7_BF16) return WKV7_ERR_UNSUPPORTED;
    if (!opt_ptr_ok(s_in) || !opt_ptr_ok(sT) || !opt_ptr_ok(workspace)) return WKV7_ERR_INVALID_ARG;
    if ((size_t)B * H == 0) return WKV7_OK;
    if (T == 0) return copy_or_zero_state(sT, s_in, B, H, stream);
    for (const void *p : {r, w, k, v, a, b, (const void *)y})
        if (!ptr_ok(p)) return WKV7_ERR_INVALID_ARG;
    const long long lim = g_wait_limit.load();
    const int nseg = summary_segments(B, T, H, workspace, workspace_bytes);
    return from_cuda(fwd_chunk_continue(B, T, H, y_dt, r, w, k, v, a, b, s_in, y, sT, nseg, workspace,
                                        lim > 0 ? lim : kDefaultWaitCycles, stream));
}

wkv7_status wkv7_compose_states(int nseg, int B, int H, int N, const float *s0, const float *summaries,
                                float *states, cudaStream_t stream) {
    wkv7_status s = check_dims(B, 0, H, N);
    if (s != WKV7_OK) return s;
    if (nseg < 0 || !opt_ptr_ok(s0)) return WKV7_ERR_INVALID_ARG;
    if ((size_t)B * H == 0) return WKV7_OK;
    if (!ptr_ok(states) || (nseg > 0 && !ptr_ok(summaries))) return WKV7_ERR_INVALID_ARG;
    return from_cuda(compose_states(B, H, nseg, s0, summaries, states, stream));
}

int wkv7_forward_resolve_algo(int T, wkv7_dtype in_dtype, wkv7_algo algo) {
    if (!dtype_ok(in_dtype) || T < 0) return -1;
    if (algo != WKV7_ALGO_AUTO && algo != WKV7_ALGO_SEQ && algo != WKV7_ALGO_CHUNK) return -1;
    return (int)resolve_algo(T, in_dtype, algo);
}

wkv7_status wkv7_step(int B, int H, int N, wkv7_dtype in_dt, wkv7_dtype y_dt, const void *r,
                      const void *w, const void *k, const void *v, const void *a, const void *b,
                      float *state, void *y, cudaStream_t stream) {
    wkv7_status s = check_dims(B, 1, H, N);
    if (s != WKV7_OK) return s;
    if (!dtype_ok(in_dt) || !dtype_ok(y_dt)) return WKV7_ERR_INVALID_ARG;
    if ((size_t)B * H == 0) return WKV7_OK;
    for (const void *p : {r, w, k, v, a, b, (const void *)state, (const void *)y})
        if (!ptr_ok(p)) return WKV7_ERR_INVALID_ARG;
    return from_cuda(wkv7::step(B, H, in_dt, y_dt, r, w, k, v, a, b, state, y, stream));
}

size_t wkv7_backward_workspace_size(int B, int T, int H, int N) {
    if (B <= 0 || T <= 0 || H <= 0 || N != kN) return 0;
    // state before every chunk, dL/dS at every chunk end, the final state, the
    // segmented passes' scratch, the chunks' transition images
    return bwd_workspace_min(B, T, H) + round_up(bwd_mq_bytes(B, T, H));
}

wkv7_status wkv7_backward(int B, int T, int H, int N, wkv7_dtype in_dt, wkv7_dtype g_dt, const void *r,
                          const void *w, const void *k, const void *v, const void *a, const void *b,
                          const float *s0, const void *dy, const float *dsT, void *dr, void *dw, void *dk,
                          void *dv, void *da, void *db, float *ds0, void *workspace,
                          size_t workspace_bytes, cudaStream_t stream) {
    wkv7_status s = check_dims(B, T, H, N);
    if (s != WKV7_OK) return s;
    if (!dtype_ok(in_dt) || !dtype_ok(g_dt)) return WKV7_ERR_INVALID_ARG;
    if (!opt_ptr_ok(s0) || !opt_ptr_ok(dsT) || !ptr_ok(ds0)) return WKV7_ERR_INVALID_ARG;
    if ((size_t)B * H == 0) return WKV7_OK;
    if (T == 0) return copy_or_zero_state(ds0, dsT, B, H, stream);
    for (const void *p : {r, w, k, v, a, b, dy, (const void *)dr, (const void *)dw, (const void *)dk,
                          (const void *)dv, (const void *)da, (const void *)db})
        if (!ptr_ok(p)) return WKV7_ERR_INVALID_ARG;
    if (workspace_bytes < bwd_workspace_min(B, T, H) || !ptr_ok(workspace)) return WKV7_ERR_INVALID_ARG;
    char *ws = static_cast<char *>(workspace);
    float *ckpt = reinterpret_cast<float *>(ws);
    float *dSo = reinterpret_cast<float *>(ws + round_up(bwd_ckpt_bytes(B, T, H)));
    float *sfin = reinterpret_cast<float *>(ws + 2 * round_up(bwd_ckpt_bytes(B, T, H)));
    size_t used = 2 * round_up(bwd_ckpt_bytes(B, T, H)) + round_up(state_bytes(B, H));
    const int sms = current_sm_count();
    // the chunks' transitions for the dS chain: bf16 inputs, room for them
    // next to the scratch, and the chain estimated faster than the sweep
    uint4 *mq = nullptr;
    if (in_dt == WKV7_BF16 && workspace_bytes >= bwd_workspace_min(B, T, H) + round_up(bwd_mq_bytes(B, T, H)) &&
        bwd_use_dchain(B, T, H, sms, workspace_bytes - used - round_up(bwd_mq_bytes(B, T, H)))) {
        mq = reinterpret_cast<uint4 *>(ws + used);
        used += round_up(bwd_mq_bytes(B, T, H));
    }
    char *scratch = ws + used;
    const size_t scratch_bytes = workspace_bytes - used;
    // checkpoints: the chunked tensor-core forward without y for bf16 inputs
    // (its chunk is the backward's; sequence segments side by side when the
    // heads are few), the sequential scan for fp32 inputs
    const long long lim = g_wait_limit.load();
    cudaError_t e;
    if (in_dt == WKV7_BF16) {
        const int want = bwd_ckpt_segments(B, T, H, sms);
        const int nseg = (want > 1 && scratch_bytes >= chunk_workspace_bytes(B, T, H, want)) ? want : 1;
        e = fwd_chunk(B, T, H, WKV7_BF16, r, w, k, v, a, b, s0, nullptr, sfin, nseg, scratch,
                      lim > 0 ? lim : kDefaultWaitCycles, stream, ckpt, EpiArgs{}, false, mq);
    } else {
        e = fwd_checkpoints(B, T, H, in_dt, r, w, k, v, a, b, s0, ckpt, kBwdChunk, sfin,
                            lim > 0 ? lim : kDefaultWaitCycles, stream);
    }
    if (e != cudaSuccess) return WKV7_ERR_CUDA;
    return from_cuda(bwd_chunked(B, T, H, in_dt, g_dt, r, w, k, v, a, b, dy, dsT, ckpt, sfin, dSo, dr, dw, dk,
                                 dv, da, db, ds0, reinterpret_cast<float *>(scratch), scratch_bytes, sms,
                                 lim > 0 ? lim : kDefaultWaitCycles, stream, mq));
}

size_t wkv7_state_gradient_workspace_size(int B, int T, int H, int N) {
    if (B <= 0 || T <= 0 || H <= 0 || N != kN) return 0;
    return dstate_scratch_for(B, T, H, current_sm_count(), false);
}

wkv7_status wkv7_state_gradient(int B, int T, int H, int N, wkv7_dtype in_dt, const void *r, const void *w,
                                const void *a, const void *b, const void *dy, const float *dsT, float *ds0,
                                void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    wkv7_status s = check_dims(B, T, H, N);
    if (s != WKV7_OK) return s;
    if (!dtype_ok(in_dt)) return WKV7_ERR_INVALID_ARG;
    if (!opt_ptr_ok(dsT) || !ptr_ok(ds0) || !opt_ptr_ok(workspace)) return WKV7_ERR_INVALID_ARG;
    if ((size_t)B * H == 0) return WKV7_OK;
    if (T == 0) return copy_or_zero_state(ds0, dsT, B, H, stream);
    for (const void *p : {r, w, a, b, dy})
        if (!ptr_ok(p)) return WKV7_ERR_INVALID_ARG;
    return from_cuda(bwd_dstate(B, T, H, in_dt, r, w, a, b, dy, dsT, nullptr, ds0, static_cast<float *>(workspace),
                                workspace ? workspace_bytes : 0, current_sm_count(), stream));
}

wkv7_status wkv7_compose_adjoints(int nseg, int B, int H, int N, const float *dsT, const float *summaries,
                                  const float *F, float *adj, cudaStream_t stream) {
    wkv7_status s = check_dims(B, 0, H, N);
    if (s != WKV7_OK) return s;
    if (nseg < 0 || !opt_ptr_ok(dsT)) return WKV7_ERR_INVALID_ARG;
    if ((size_t)B * H == 0) return WKV7_OK;
    if (!ptr_ok(adj) || (nseg > 0 && (!ptr_ok(summaries) || !ptr_ok(F)))) return WKV7_ERR_INVALID_ARG;
    return from_cuda(compose_adjoints(B, H, nseg, dsT, summaries, F, adj, stream));
}

void wkv7_set_wait_limit(long long cycles) { g_wait_limit.store(cycles > 0 ? cycles : 0); }

wkv7_status wkv7_get_last_status(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return WKV7_ERR_CUDA;
    int h = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&h, g_device_status, sizeof(int)) != cudaSuccess) return WKV7_ERR_CUDA;
    if (h != 0 && cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return WKV7_ERR_CUDA;
    return static_cast<wkv7_status>(h);
}

wkv7_status wkv7_get_device_status(cudaStream_t stream) { return wkv7_get_last_status(stream); }

}  // extern "C"
