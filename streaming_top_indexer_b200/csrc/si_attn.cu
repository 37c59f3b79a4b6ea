// si_attn.cu -- C ABI of the sparse attention stage (include/si.h):
// argument checks, TMA descriptors and the launch of sparse_attn_kernel.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "si.h"
#include "si_attn.cuh"
#include "si_host.cuh"

#ifdef SI_ATTN_TRACE
// Tracing builds only: the timeline buffer and a reader for it.
static __device__ unsigned long long g_attn_trace[4 * si::kATraceItems * 4];
extern "C" __attribute__((visibility("default"))) int si_attn_trace_read(unsigned long long* host_out) {
    return cudaMemcpyFromSymbol(host_out, g_attn_trace, sizeof(g_attn_trace)) == cudaSuccess ? 0 : 1;
}
#endif

namespace {

template <int D, int DV>
si_status launch_attn_t(const void* q, const void* kcache, const void* vcache, const int32_t* idx, int64_t B,
                        int64_t S, int64_t T, int k, float scale, void* out, float* lse, uint32_t* status,
                        cudaStream_t stream) {
    using C = si::AttnCfg<D, DV>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SI_ERR_CUDA;
    const int sms = si_host::device_sms(dev);
    if (sms <= 0) return SI_ERR_CUDA;
    si::AttnParams p{};
    p.rows = B * S;
    p.S = S;
    p.T = T;
    p.k = k;
    p.nchunks = (k + C::NK - 1) / C::NK;
    p.idx = idx;
    p.kcache = static_cast<const uint16_t*>(kcache);
    p.vcache = static_cast<const uint16_t*>(vcache);
    p.out = static_cast<uint16_t*>(out);
    p.lse = lse;
    p.c2 = scale * 1.4426950408889634f;
    p.err = status;
    p.timeout_ns = si_host::timeout_ns();
#ifdef SI_ATTN_TRACE
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p.trace), g_attn_trace) != cudaSuccess) return SI_ERR_CUDA;
#endif

    CUtensorMap tq;
    const uint64_t rows = static_cast<uint64_t>(B * S);
    // q as [B*S*128 rows, d]: one row's heads are one 128-row box per 64 columns
    if (!si_host::encode_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, D, rows * C::HA, D * 2ull, 64, C::HA,
                            CU_TENSOR_MAP_SWIZZLE_128B))
        return SI_ERR_CUDA;

    const uint32_t smem = C::DYN_BYTES;
    auto kern = si::sparse_attn_kernel<D, DV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return si_host::cuda_fail("attention kernel shared-memory attribute", e);
    int64_t grid = sms < si_host::kMaxCtas ? sms : si_host::kMaxCtas;
    if (grid > p.rows) grid = p.rows;
    kern<<<static_cast<unsigned>(grid), C::THREADS, smem, stream>>>(tq, p);
    e = cudaGetLastError();
    return e == cudaSuccess ? SI_OK : si_host::cuda_fail("attention kernel launch", e);
}

}  // namespace

extern "C" si_status si_sparse_attention(const void* q, const void* kcache, const void* vcache, const int32_t* idx,
                                         int64_t B, int64_t S, int64_t T, int H_a, int d, int d_v, int k,
                                         float scale, void* out, float* lse, uint32_t* status, si_stream_t stream) {
    if (B < 1 || S < 1 || T < 0 || k < 1) return SI_ERR_INVALID_ARG;
    if (!q || !idx || !out || !lse || !status || (T > 0 && (!kcache || !vcache))) return SI_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return SI_ERR_INVALID_ARG;
    if (H_a != 128 || (d != 64 && d != 128) || (d_v != 64 && d_v != 128) || k > 2048) return SI_ERR_UNSUPPORTED;
    if (B * S * 128 >= (int64_t{1} << 31) || B * T >= (int64_t{1} << 31)) return SI_ERR_UNSUPPORTED;
    auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    auto a4 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; };
    if (!a16(q) || !a16(out) || (T > 0 && (!a16(kcache) || !a16(vcache))) || !a4(idx) || !a4(lse) || !a4(status))
        return SI_ERR_MISALIGNED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(status, 0, sizeof(uint32_t), s) != cudaSuccess) return SI_ERR_CUDA;
    if (T == 0) {
        const int64_t n_lse = B * S * 128;
        int64_t blocks = (n_lse * d_v + 255) / 256;
        if (blocks > 4096) blocks = 4096;
        si::attn_empty_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(static_cast<uint16_t*>(out), lse,
                                                                           n_lse * d_v, n_lse);
        return cudaGetLastError() == cudaSuccess ? SI_OK : SI_ERR_CUDA;
    }
    if (d == 128 && d_v == 128) return launch_attn_t<128, 128>(q, kcache, vcache, idx, B, S, T, k, scale, out, lse, status, s);
    if (d == 128 && d_v == 64) return launch_attn_t<128, 64>(q, kcache, vcache, idx, B, S, T, k, scale, out, lse, status, s);
    if (d == 64 && d_v == 128) return launch_attn_t<64, 128>(q, kcache, vcache, idx, B, S, T, k, scale, out, lse, status, s);
    return launch_attn_t<64, 64>(q, kcache, vcache, idx, B, S, T, k, scale, out, lse, status, s);
}
