// si_lib.cu -- host side of the C ABI (include/si.h): argument checks,
// workspace sizing, TMA descriptors and kernel launches on the caller's
// stream.  No allocation, no host synchronisation (except in
// si_check_device_status, which is documented to synchronise).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "si.h"
#include "si_host.cuh"
#include "si_keys.cuh"
#include "si_sort.cuh"

namespace si_host {

// With SI_DEBUG set in the environment, CUDA failures are also printed to stderr.
si_status cuda_fail(const char* where, cudaError_t e) {
    static const bool verbose = std::getenv("SI_DEBUG") != nullptr;
    if (verbose) std::fprintf(stderr, "streaming_top_indexer: %s: %s\n", where, cudaGetErrorString(e));
    return SI_ERR_CUDA;
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}
}  // namespace

bool encode_3d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
               uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1,
               CUtensorMapSwizzle sw) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    cuuint32_t box[3] = {box0, box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    std::memset(map, 0, sizeof(*map));
    CUresult r = enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
               uint64_t stride1_bytes, uint32_t box0, uint32_t box1, CUtensorMapSwizzle sw) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {d0, d1};
    cuuint64_t strides[1] = {stride1_bytes};
    cuuint32_t box[2] = {box0, box1};
    cuuint32_t estr[2] = {1, 1};
    std::memset(map, 0, sizeof(*map));
    CUresult r = enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {
std::mutex g_dev_mu;
int g_dev_sms[64] = {};
}  // namespace

int device_sms(int dev) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (dev < 0 || dev >= 64) return 0;
    if (g_dev_sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        g_dev_sms[dev] = n;
    }
    return g_dev_sms[dev];
}

}  // namespace si_host

namespace {
std::atomic<uint64_t> g_timeout_ns{2000000000ull};
}  // namespace

uint64_t si_host::timeout_ns() { return g_timeout_ns.load(); }

namespace {

using si_host::cuda_fail;
using si_host::kHeaderBytes;
using si_host::kMaxCtas;
using si_host::kMaxDynSmem;
// Row windows of si_indexer_topk_rows start (and, except at S, end) on
// multiples of this, a multiple of every unit's query count (256/H_I).
constexpr int64_t kRowAlign = 256;
// Whether the select kernel sorts each row at unit end (default) or leaves the
// rows unordered for the separate row sort.
std::atomic<bool> g_sort_in_select{true};
// Design parameters set by si_set_tuning (0: the default).
std::atomic<int> g_pool_entries{0}, g_cut_slack{0}, g_check_tiles{0};

uint32_t check_tiles_in_use() {
    const int c = g_check_tiles.load();
    return c > 0 ? static_cast<uint32_t>(c) : si::kCheckTiles;
}
uint32_t cut_slack_in_use() {
    const int c = g_cut_slack.load();
    return c > 0 ? static_cast<uint32_t>(c) : si::kCompactSlack;
}

bool supported_h(int h) { return h == 8 || h == 16 || h == 32 || h == 64; }
bool supported_d(int d) { return d == 64 || d == 128; }

// Shared-memory bytes (dynamic + static) of the select kernel.
uint32_t select_smem(int H, int D, bool pool_in_smem, int P) {
#define SI_CASE(HH, DD) \
    if (H == HH && D == DD) return si::SelCfg<HH, DD>::smem_bytes(pool_in_smem, P);
    SI_CASE(8, 64) SI_CASE(8, 128) SI_CASE(16, 64) SI_CASE(16, 128)
    SI_CASE(32, 64) SI_CASE(32, 128) SI_CASE(64, 64) SI_CASE(64, 128)
#undef SI_CASE
    return 0;
}

// Where the per-query candidate pools live and how large they are.  A pool
// in shared memory takes all the room left (fewer pool cuts) and must hold
// at least max(k + 288, min(2k, k + 768)) entries: room for k + 28 survivors
// of a cut plus two tiles of appends in each warp's sub-range, and enough
// spare room that cuts stay rare (measured: at k = 1024, H_I = 64 a 1856-entry
// shared-memory pool beats a 4096-entry workspace pool by 15-23 %).
// Otherwise the pools take max(4k, k + 288) entries in the workspace, and the
// shared memory they leave holds the exact-cut candidate buffers.
struct PoolPlan {
    bool smem;
    int P;
};

PoolPlan pool_plan(int H, int D, int k) {
    auto r32 = [](int x) { return (x + 31) / 32 * 32; };
    const uint32_t qt = 256u / static_cast<uint32_t>(H);
    const uint32_t fixed = select_smem(H, D, true, 0);  // everything but the pools
    // room the appends need between two pool checks, plus survivors of a cut
    const int need = k + static_cast<int>(4 * (32 * check_tiles_in_use() + 1)) + 28;
    const int forced = g_pool_entries.load();
    if (forced > 0) {  // si_set_tuning: a given capacity (at least `need`), in shared memory if it fits
        const int p = r32(forced > need ? forced : need);
        if (fixed + qt * static_cast<uint32_t>(p) * 8u <= kMaxDynSmem && p <= 65504) return {true, p};
        return {false, p};
    }
    const int spare = 2 * k < k + 768 ? 2 * k : k + 768;
    int min_p = r32(spare > k + 288 ? spare : k + 288);
    if (min_p < need) min_p = r32(need);
    if (fixed + qt * static_cast<uint32_t>(min_p) * 8u <= kMaxDynSmem) {
        int p = static_cast<int>((kMaxDynSmem - fixed) / (qt * 8u)) / 32 * 32;
        if (p > 65504) p = 65504;  // pool counts are 16-bit fields
        return {true, p};
    }
    return {false, r32(4 * k > min_p ? 4 * k : min_p)};
}

// Keys per thread of the unit-end row sort inside the select kernel (the
// half's 128 threads sort 128 * E >= k keys), or 0 when rows are left
// unordered for the separate row-sort kernel:
//  - k > 1024 (E = 16): the network no longer unrolls into registers, and
//    measured at k = 2048 (B=4, S=131,072) the select kernel then took 407 ms
//    against 205 ms + 22.5 ms for the separate sort;
//  - the sort's exchange buffer (the query's own shared-memory pool, or the
//    half's STREAM_CAND-key buffer with workspace pools) holds fewer than
//    128 * E keys.
// At k = 512 (S=262,144) the two designs measured within 0.5 % of each other.
int row_sort_e(int H, int D, int k) {
    if (k > 1024) return 0;
    int e = 1;
    while (128 * e < k) e <<= 1;
    const PoolPlan pp = pool_plan(H, D, k);
    int cap = 0;
#define SI_CASE(HH, DD) \
    if (H == HH && D == DD) cap = pp.smem ? pp.P : si::SelCfg<HH, DD>::STREAM_CAND;
    SI_CASE(8, 64) SI_CASE(8, 128) SI_CASE(16, 64) SI_CASE(16, 128)
    SI_CASE(32, 64) SI_CASE(32, 128) SI_CASE(64, 64) SI_CASE(64, 128)
#undef SI_CASE
    return 128 * e <= cap ? e : 0;
}

size_t global_pool_bytes(int H, int D, int k) {
    const PoolPlan pp = pool_plan(H, D, k);
    if (pp.smem) return 0;
    const size_t QT = 256 / H;
    return static_cast<size_t>(kMaxCtas) * QT * pp.P * sizeof(uint64_t);
}

si_status check_common(const void* q, const float* w, const void* kc, int64_t B, int64_t S, int64_t T,
                       int H, int D, int m) {
    if (B < 1 || S < 1 || T < 0 || m < 1) return SI_ERR_INVALID_ARG;
    if (!q || !w || (T > 0 && !kc)) return SI_ERR_INVALID_ARG;
    if (!supported_h(H) || !supported_d(D)) return SI_ERR_UNSUPPORTED;
    if (S * H >= (int64_t{1} << 31) || T >= (int64_t{1} << 31) || B >= (int64_t{1} << 31))
        return SI_ERR_UNSUPPORTED;
    auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!a16(q) || !a16(w) || (T > 0 && !a16(kc))) return SI_ERR_MISALIGNED;
    return SI_OK;
}

si_status check_topk(const void* q, const float* w, const void* kc, int64_t B, int64_t S, int64_t T, int H,
                     int D, int m, int k, const int32_t* out_idx, const float* out_score, const void* ws,
                     size_t ws_bytes) {
    si_status st = check_common(q, w, kc, B, S, T, H, D, m);
    if (st != SI_OK) return st;
    if (k < 1 || k > 2048) return SI_ERR_UNSUPPORTED;
    if (!out_idx || !out_score || !ws) return SI_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(out_idx) & 3u) || (reinterpret_cast<uintptr_t>(out_score) & 3u) ||
        (reinterpret_cast<uintptr_t>(ws) & 15u))
        return SI_ERR_MISALIGNED;
    if (ws_bytes < si_workspace_bytes(B, S, T, H, D, m, k)) return SI_ERR_WORKSPACE_TOO_SMALL;
    return SI_OK;
}

// Query rows [t_lo, t_hi) of every batch; the whole problem is [0, S).  The
// select kernel's instantiations live in one translation unit per H_I
// (si_select_h*.cu); this picks the pools and the row sort and dispatches.
si_status launch_select(const void* q, const float* w, const void* kc, int64_t B, int64_t S, int64_t T, int H, int D,
                        int m, int k, int32_t* out_idx, float* out_score, float* dense, void* ws,
                        cudaStream_t stream, int64_t t_lo = 0, int64_t t_hi = -1) {
    si_host::SelectLaunch a{};
    a.q = q;
    a.w = w;
    a.kc = kc;
    a.B = B;
    a.S = S;
    a.T = T;
    a.H = H;
    a.D = D;
    a.m = m;
    a.k = dense ? 1 : k;
    a.out_idx = out_idx;
    a.out_score = out_score;
    a.dense = dense;
    a.ws = ws;
    a.stream = stream;
    a.t_lo = t_lo;
    a.t_hi = t_hi < 0 ? S : t_hi;
    const PoolPlan pp = dense ? PoolPlan{true, 0} : pool_plan(H, D, a.k);
    a.smem_pool = pp.smem;
    a.P = pp.P;
    a.sort_e = (dense || !g_sort_in_select.load()) ? 0 : row_sort_e(H, D, k);
    a.check_tiles = check_tiles_in_use();
    a.cut_slack = cut_slack_in_use();
    a.timeout_ns = g_timeout_ns.load();
    a.gpool = pp.smem ? nullptr : reinterpret_cast<uint64_t*>(static_cast<uint8_t*>(ws) + kHeaderBytes);
#ifdef SI_TRACE
    // Tracing builds: per-warp cycle counters after the pools; the caller adds
    // kMaxCtas * kTraceWarps * kTraceSlots * 8 bytes to the workspace.
    a.trace = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(ws) + kHeaderBytes +
                                                    (pp.smem ? 0 : global_pool_bytes(H, D, a.k)));
#endif
    switch (H) {
        case 8: return si_host::launch_select_h8(a);
        case 16: return si_host::launch_select_h16(a);
        case 32: return si_host::launch_select_h32(a);
        case 64: return si_host::launch_select_h64(a);
        default: return SI_ERR_UNSUPPORTED;
    }
}

// Whether the select kernel leaves rows in their final order for these sizes.
bool select_sorts_rows(int H, int D, int k) { return g_sort_in_select.load() && row_sort_e(H, D, k) > 0; }

si_status launch_pad(int32_t* out_idx, float* out_score, int64_t n, cudaStream_t stream) {
    if (n <= 0) return SI_OK;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    si::pad_rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(out_idx, out_score, n);
    return cudaGetLastError() == cudaSuccess ? SI_OK : SI_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t si_workspace_bytes(int64_t B, int64_t S, int64_t T, int H_I, int d_I, int m, int k) {
    if (B < 1 || S < 1 || T < 0 || m < 1 || k < 1 || k > 2048 || !supported_h(H_I) || !supported_d(d_I)) return 0;
    return kHeaderBytes + global_pool_bytes(H_I, d_I, k);
}

si_status si_select_topk(const void* q, const float* w, const void* kc, int64_t B, int64_t S, int64_t T, int H_I,
                         int d_I, int m, int k, int32_t* out_idx, float* out_score, void* workspace,
                         size_t workspace_bytes, si_stream_t stream) {
    si_status st = check_topk(q, w, kc, B, S, T, H_I, d_I, m, k, out_idx, out_score, workspace, workspace_bytes);
    if (st != SI_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) return launch_pad(out_idx, out_score, B * S * k, s);
    return launch_select(q, w, kc, B, S, T, H_I, d_I, m, k, out_idx, out_score, nullptr, workspace, s);
}

si_status si_sort_topk(int32_t* out_idx, float* out_score, int64_t rows, int k, si_stream_t stream) {
    if (!out_idx || !out_score || rows < 0) return SI_ERR_INVALID_ARG;
    if (k < 1 || k > 2048) return SI_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(out_idx) & 3u) || (reinterpret_cast<uintptr_t>(out_score) & 3u))
        return SI_ERR_MISALIGNED;
    if (rows == 0) return SI_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t blocks64 = (rows + si::kSortWarps - 1) / si::kSortWarps;
    if (blocks64 > 0x7FFFFFFF) return SI_ERR_UNSUPPORTED;
    const unsigned blocks = static_cast<unsigned>(blocks64);
    const unsigned threads = 32 * si::kSortWarps;
    int k2 = 32;
    while (k2 < k) k2 <<= 1;
    if (rows > 0x7FFFFFFF) return SI_ERR_UNSUPPORTED;
    const unsigned rows_grid = static_cast<unsigned>(rows);  // one block per row (long rows)
    switch (k2 / 32) {
        case 1: si::sort_rows_kernel<1><<<blocks, threads, 0, s>>>(out_idx, out_score, rows, k); break;
        case 2: si::sort_rows_kernel<2><<<blocks, threads, 0, s>>>(out_idx, out_score, rows, k); break;
        case 4: si::sort_rows_lane_kernel<4><<<blocks, threads, 0, s>>>(out_idx, out_score, rows, k); break;
        case 8: si::sort_rows_lane_kernel<8><<<blocks, threads, 0, s>>>(out_idx, out_score, rows, k); break;
        case 16: si::sort_rows_lane_kernel<16><<<blocks, threads, 0, s>>>(out_idx, out_score, rows, k); break;
        case 32: si::sort_rows_block_kernel<1024><<<rows_grid, 128, 0, s>>>(out_idx, out_score, rows, k); break;
        case 64: si::sort_rows_block_kernel<2048><<<rows_grid, 256, 0, s>>>(out_idx, out_score, rows, k); break;
        default: return SI_ERR_UNSUPPORTED;
    }
    return cudaGetLastError() == cudaSuccess ? SI_OK : SI_ERR_CUDA;
}

si_status si_indexer_topk(const void* q, const float* w, const void* kc, int64_t B, int64_t S, int64_t T, int H_I,
                          int d_I, int m, int k, int32_t* out_idx, float* out_score, void* workspace,
                          size_t workspace_bytes, si_stream_t stream) {
    si_status st = check_topk(q, w, kc, B, S, T, H_I, d_I, m, k, out_idx, out_score, workspace, workspace_bytes);
    if (st != SI_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, kHeaderBytes, s) != cudaSuccess) return SI_ERR_CUDA;
    if (T == 0) return launch_pad(out_idx, out_score, B * S * k, s);
    st = launch_select(q, w, kc, B, S, T, H_I, d_I, m, k, out_idx, out_score, nullptr, workspace, s);
    if (st != SI_OK) return st;
    if (select_sorts_rows(H_I, d_I, k)) return SI_OK;
    return si_sort_topk(out_idx, out_score, B * S, k, stream);
}

si_status si_indexer_topk_rows(const void* q, const float* w, const void* kc, int64_t B, int64_t S, int64_t T,
                               int H_I, int d_I, int m, int k, int64_t t_begin, int64_t t_end, int32_t* out_idx,
                               float* out_score, void* workspace, size_t workspace_bytes, si_stream_t stream) {
    si_status st = check_topk(q, w, kc, B, S, T, H_I, d_I, m, k, out_idx, out_score, workspace, workspace_bytes);
    if (st != SI_OK) return st;
    if (t_begin < 0 || t_end > S || t_begin > t_end) return SI_ERR_INVALID_ARG;
    if (t_begin % kRowAlign != 0 || (t_end % kRowAlign != 0 && t_end != S)) return SI_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (t_begin == t_end) return SI_OK;
    const int64_t n = t_end - t_begin;
    if (T == 0) {
        for (int64_t b = 0; b < B; ++b) {
            const int64_t off = (b * S + t_begin) * k;
            st = launch_pad(out_idx + off, out_score + off, n * k, s);
            if (st != SI_OK) return st;
        }
        return SI_OK;
    }
    st = launch_select(q, w, kc, B, S, T, H_I, d_I, m, k, out_idx, out_score, nullptr, workspace, s, t_begin, t_end);
    if (st != SI_OK) return st;
    if (select_sorts_rows(H_I, d_I, k)) return SI_OK;
    for (int64_t b = 0; b < B; ++b) {
        const int64_t off = (b * S + t_begin) * k;
        st = si_sort_topk(out_idx + off, out_score + off, n, k, stream);
        if (st != SI_OK) return st;
    }
    return SI_OK;
}

si_status si_indexer_scores(const void* q, const float* w, const void* kc, int64_t B, int64_t S, int64_t T, int H_I,
                            int d_I, int m, float* out_scores, void* workspace, size_t workspace_bytes,
                            si_stream_t stream) {
    si_status st = check_common(q, w, kc, B, S, T, H_I, d_I, m);
    if (st != SI_OK) return st;
    if (!out_scores || !workspace) return SI_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(out_scores) & 3u) || (reinterpret_cast<uintptr_t>(workspace) & 15u))
        return SI_ERR_MISALIGNED;
    if (workspace_bytes < kHeaderBytes) return SI_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, kHeaderBytes, s) != cudaSuccess) return SI_ERR_CUDA;
    if (T == 0) return SI_OK;
    return launch_select(q, w, kc, B, S, T, H_I, d_I, m, 1, nullptr, nullptr, out_scores, workspace, s);
}

si_status si_reset_device_status(void* workspace, si_stream_t stream) {
    if (!workspace) return SI_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 15u) return SI_ERR_MISALIGNED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return cudaMemsetAsync(workspace, 0, kHeaderBytes, s) == cudaSuccess ? SI_OK : SI_ERR_CUDA;
}

si_status si_check_device_status(const void* workspace, si_stream_t stream) {
    if (!workspace) return SI_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return SI_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SI_ERR_CUDA;
    if (word == 0) return SI_OK;
    if (word == si::kErrTimeout) return SI_ERR_TIMEOUT;
    return SI_ERR_CUDA;
}

si_status si_selftest_timeout(void* workspace, size_t workspace_bytes, uint64_t limit_ns, si_stream_t stream) {
    if (!workspace) return SI_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 15u) return SI_ERR_MISALIGNED;
    if (workspace_bytes < kHeaderBytes) return SI_ERR_WORKSPACE_TOO_SMALL;
    if (limit_ns == 0 || limit_ns > 10000000000ull) return SI_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, kHeaderBytes, s) != cudaSuccess) return SI_ERR_CUDA;
    si::timeout_selftest_kernel<<<1, 32, 0, s>>>(static_cast<uint32_t*>(workspace), limit_ns);
    return cudaGetLastError() == cudaSuccess ? SI_OK : SI_ERR_CUDA;
}

int si_select_sorts_rows(int H_I, int d_I, int k) {
    if (!supported_h(H_I) || !supported_d(d_I) || k < 1 || k > 2048) return 0;
    return select_sorts_rows(H_I, d_I, k) ? 1 : 0;
}

void si_set_sort_in_select(int enable) { g_sort_in_select.store(enable != 0); }

si_status si_set_tuning(int pool_entries, int cut_slack, int check_tiles) {
    if (pool_entries < 0 || pool_entries > 65504 || cut_slack < 0 || cut_slack > 4096 || check_tiles < 0 ||
        check_tiles > 16)
        return SI_ERR_INVALID_ARG;
    g_pool_entries.store(pool_entries);
    g_cut_slack.store(cut_slack);
    g_check_tiles.store(check_tiles);
    return SI_OK;
}

void si_set_timeout_ns(uint64_t ns) {
    if (ns > 0) g_timeout_ns.store(ns);
}

const char* si_status_string(si_status s) {
    switch (s) {
        case SI_OK: return "SI_OK";
        case SI_ERR_INVALID_ARG: return "SI_ERR_INVALID_ARG";
        case SI_ERR_UNSUPPORTED: return "SI_ERR_UNSUPPORTED";
        case SI_ERR_MISALIGNED: return "SI_ERR_MISALIGNED";
        case SI_ERR_WORKSPACE_TOO_SMALL: return "SI_ERR_WORKSPACE_TOO_SMALL";
        case SI_ERR_CUDA: return "SI_ERR_CUDA";
        case SI_ERR_TIMEOUT: return "SI_ERR_TIMEOUT";
    }
    return "SI_ERR_UNKNOWN";
}

const char* si_version(void) { return "streaming_top_indexer_b200 0.1.0 (sm_100a)"; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Variant that needs no caller-allocated workspace.
//
// Some callers cannot hand the library a device buffer: a plugin running
// inside a host application that owns every byte of device memory and gives
// plugins no allocator, or a serving loop whose memory plan is frozen after
// start-up.  For them the scratch that si_indexer_topk keeps in the caller's
// workspace (the device error word, plus candidate pools when they do not fit
// in shared memory) lives instead in the fixed array below, one per device.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t{1} << 20;  // 1 MiB on every device that loads the library

// Device-side storage.  In host code this name only stands for the symbol;
// its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[64] = {};

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (with that device current) and remembered.
si_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SI_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return SI_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return SI_OK;
}

}  // namespace

extern "C" si_status si_indexer_topk_noalloc(const void* q, const float* w, const void* kc, int64_t B, int64_t S,
                                             int64_t T, int H_I, int d_I, int m, int k, int32_t* out_idx,
                                             float* out_score, uint32_t* out_status, si_stream_t stream) {
    si_status st = check_common(q, w, kc, B, S, T, H_I, d_I, m);
    if (st != SI_OK) return st;
    if (k < 1 || k > 2048) return SI_ERR_UNSUPPORTED;
    if (!out_idx || !out_score) return SI_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(out_idx) & 3u) || (reinterpret_cast<uintptr_t>(out_score) & 3u) ||
        (reinterpret_cast<uintptr_t>(out_status) & 3u))
        return SI_ERR_MISALIGNED;
    const size_t need = si_workspace_bytes(B, S, T, H_I, d_I, m, k);
    if (need == 0) return SI_ERR_UNSUPPORTED;
    if (need > kNoAllocScratchBytes) return SI_ERR_WORKSPACE_TOO_SMALL;  // beyond the built-in scratch
    void* ws = nullptr;
    st = noalloc_scratch(&ws);
    if (st != SI_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // The array keeps the previous call's contents: clear the error word.
    if (cudaMemsetAsync(ws, 0, kHeaderBytes, s) != cudaSuccess) return SI_ERR_CUDA;
    if (T == 0) {
        st = launch_pad(out_idx, out_score, B * S * k, s);
    } else {
        st = launch_select(q, w, kc, B, S, T, H_I, d_I, m, k, out_idx, out_score, nullptr, ws, s);
        if (st == SI_OK && !select_sorts_rows(H_I, d_I, k)) st = si_sort_topk(out_idx, out_score, B * S, k, stream);
    }
    if (st != SI_OK) return st;
    if (out_status && cudaMemcpyAsync(out_status, ws, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return SI_ERR_CUDA;
    return SI_OK;
}
