// si_host_io.cu -- si_indexer_topk on host buffers: the copies in and out are
// overlapped with the computation by row windows.
//
// Every query row selects its keys on its own (StreamIndex: Memory-Bounded
// Compressed Sparse Attention via Streaming Top-k, Abstract), so the rows can
// be computed in windows with si_indexer_topk_rows.  While one window runs on
// the caller's stream, the q and w rows of the next are copied in on one copy
// stream and the results of the previous one copied out on another.  Windows
// run last rows first: under the causal mask they are the most work, so the
// first copy-in (small) and the last copy-out (the shortest rows' results)
// are what stays exposed.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>
#include <utility>
#include <vector>

#include "si.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kWindowAlign = 256;  // si_indexer_topk_rows' row alignment

// The two copy streams of each device, created on first use and kept for the
// life of the process (non-blocking, so they never wait on the legacy stream).
struct CopyStreams {
    cudaStream_t in = nullptr, out = nullptr;
};
std::mutex g_streams_mu;
CopyStreams g_streams[kMaxDevices];

si_status copy_streams(CopyStreams* cs) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SI_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_streams_mu);
    CopyStreams& s = g_streams[dev];
    if (!s.in && cudaStreamCreateWithFlags(&s.in, cudaStreamNonBlocking) != cudaSuccess) return SI_ERR_CUDA;
    if (!s.out && cudaStreamCreateWithFlags(&s.out, cudaStreamNonBlocking) != cudaSuccess) return SI_ERR_CUDA;
    *cs = s;
    return SI_OK;
}

// Events of one call: recorded, waited on, then released; cudaEventDestroy
// on an event still pending frees it once the device has passed it.
struct Events {
    std::vector<cudaEvent_t> ev;
    ~Events() {
        for (cudaEvent_t e : ev) cudaEventDestroy(e);
    }
    cudaEvent_t make() {
        cudaEvent_t e = nullptr;
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
        ev.push_back(e);
        return e;
    }
};

// Rows [t0, t1) of every batch of a [B, S, row_bytes] tensor: one strided copy.
cudaError_t copy_rows(void* dst, const void* src, int64_t B, int64_t S, size_t row_bytes, int64_t t0, int64_t t1,
                      cudaMemcpyKind kind, cudaStream_t s) {
    const size_t pitch = static_cast<size_t>(S) * row_bytes;
    const size_t off = static_cast<size_t>(t0) * row_bytes;
    return cudaMemcpy2DAsync(static_cast<char*>(dst) + off, pitch, static_cast<const char*>(src) + off, pitch,
                             static_cast<size_t>(t1 - t0) * row_bytes, static_cast<size_t>(B), kind, s);
}

}  // namespace

extern "C" int64_t si_host_window_rows(int64_t S, int chunks) {
    if (S <= 0) return 0;
    if (chunks < 1) chunks = 1;
    int64_t step = (S + chunks - 1) / chunks / kWindowAlign * kWindowAlign;
    return step < kWindowAlign ? kWindowAlign : step;
}

extern "C" si_status si_indexer_topk_host(const void* q_h, const float* w_h, const void* kc_h, int64_t B, int64_t S,
                                          int64_t T, int H_I, int d_I, int m, int k, int32_t* idx_h, float* score_h,
                                          void* q_d, float* w_d, void* kc_d, int32_t* idx_d, float* score_d,
                                          void* workspace, size_t workspace_bytes, int chunks, si_stream_t stream) {
    if (!q_h || !w_h || (T > 0 && !kc_h) || !idx_h || !score_h || chunks < 0) return SI_ERR_INVALID_ARG;
    // The device-side checks (shapes, alignment, workspace size) are those of
    // si_indexer_topk_rows: an empty window runs them all and enqueues nothing.
    si_status st = si_indexer_topk_rows(q_d, w_d, kc_d, B, S, T, H_I, d_I, m, k, 0, 0, idx_d, score_d, workspace,
                                        workspace_bytes, stream);
    if (st != SI_OK) return st;
    if (chunks == 0) {  // measured at S=262,144: 8 -> 947, 16 -> 975, 32 -> 985 TFLOP/s end to end
        const int64_t c = S / 2048;
        chunks = static_cast<int>(c < 1 ? 1 : (c > 32 ? 32 : c));
    }
    const int64_t step = si_host_window_rows(S, chunks);
    std::vector<std::pair<int64_t, int64_t>> win;
    for (int64_t t0 = 0; t0 < S; t0 += step) win.emplace_back(t0, t0 + step < S ? t0 + step : S);
    std::reverse(win.begin(), win.end());

    CopyStreams cs;
    st = copy_streams(&cs);
    if (st != SI_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Events evs;
    auto fail = [](cudaError_t e) { return e == cudaSuccess ? SI_OK : SI_ERR_CUDA; };

    // The copy-in stream starts after everything already queued on `stream`
    // (the previous call's reads of these buffers included).
    cudaEvent_t start = evs.make();
    if (!start) return SI_ERR_CUDA;
    if ((st = fail(cudaEventRecord(start, s))) != SI_OK) return st;
    if ((st = fail(cudaStreamWaitEvent(cs.in, start, 0))) != SI_OK) return st;
    const size_t q_row = static_cast<size_t>(H_I) * d_I * 2, w_row = static_cast<size_t>(H_I) * 4;
    const size_t o_row = static_cast<size_t>(k) * 4;
    if (T > 0 && (st = fail(cudaMemcpyAsync(kc_d, kc_h, static_cast<size_t>(B * T) * d_I * 2, cudaMemcpyHostToDevice,
                                            cs.in))) != SI_OK)
        return st;
    std::vector<cudaEvent_t> in_done, out_ready;
    for (const auto& [t0, t1] : win) {
        if ((st = fail(copy_rows(q_d, q_h, B, S, q_row, t0, t1, cudaMemcpyHostToDevice, cs.in))) != SI_OK) return st;
        if ((st = fail(copy_rows(w_d, w_h, B, S, w_row, t0, t1, cudaMemcpyHostToDevice, cs.in))) != SI_OK) return st;
        cudaEvent_t e = evs.make();
        if (!e || (st = fail(cudaEventRecord(e, cs.in))) != SI_OK) return e ? st : SI_ERR_CUDA;
        in_done.push_back(e);
    }
    if ((st = si_reset_device_status(workspace, stream)) != SI_OK) return st;
    for (size_t i = 0; i < win.size(); ++i) {
        if ((st = fail(cudaStreamWaitEvent(s, in_done[i], 0))) != SI_OK) return st;
        st = si_indexer_topk_rows(q_d, w_d, kc_d, B, S, T, H_I, d_I, m, k, win[i].first, win[i].second, idx_d,
                                  score_d, workspace, workspace_bytes, stream);
        if (st != SI_OK) return st;
        cudaEvent_t e = evs.make();
        if (!e || (st = fail(cudaEventRecord(e, s))) != SI_OK) return e ? st : SI_ERR_CUDA;
        out_ready.push_back(e);
    }
    for (size_t i = 0; i < win.size(); ++i) {
        const auto [t0, t1] = win[i];
        if ((st = fail(cudaStreamWaitEvent(cs.out, out_ready[i], 0))) != SI_OK) return st;
        if ((st = fail(copy_rows(idx_h, idx_d, B, S, o_row, t0, t1, cudaMemcpyDeviceToHost, cs.out))) != SI_OK)
            return st;
        if ((st = fail(copy_rows(score_h, score_d, B, S, o_row, t0, t1, cudaMemcpyDeviceToHost, cs.out))) != SI_OK)
            return st;
    }
    // `stream` completes after the last copy out.
    cudaEvent_t end = evs.make();
    if (!end) return SI_ERR_CUDA;
    if ((st = fail(cudaEventRecord(end, cs.out))) != SI_OK) return st;
    return fail(cudaStreamWaitEvent(s, end, 0));
}
