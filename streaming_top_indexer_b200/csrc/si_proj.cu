// si_proj.cu -- C ABI of the indexer's upstream producers (include/si.h):
// argument checks, TMA descriptors and the three launches of gemm_kernel.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "si.h"
#include "si_gemm.cuh"
#include "si_host.cuh"

namespace {

// A: rows of K bf16 at a_row (elements) apart, batches a_batch apart; W: [N, KB] bf16.
template <int BN, bool F32>
si_status launch_gemm(const void* A, int64_t K, int64_t R, int64_t batches, int64_t a_row, int64_t a_batch,
                      const void* W, int64_t N, int64_t KB, float alpha, void* C, uint32_t* status,
                      cudaStream_t stream) {
    using G = si::GemmCfg<BN>;
    if (R == 0 || N == 0) return SI_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SI_ERR_CUDA;
    const int sms = si_host::device_sms(dev);
    if (sms <= 0) return SI_ERR_CUDA;
    CUtensorMap ta, tb;
    if (!si_host::encode_3d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, static_cast<uint64_t>(K),
                            static_cast<uint64_t>(R), static_cast<uint64_t>(batches), static_cast<uint64_t>(a_row) * 2,
                            static_cast<uint64_t>(a_batch) * 2, 64, G::BM, CU_TENSOR_MAP_SWIZZLE_128B))
        return SI_ERR_CUDA;
    if (!si_host::encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, static_cast<uint64_t>(KB),
                            static_cast<uint64_t>(N), static_cast<uint64_t>(KB) * 2, 64, BN,
                            CU_TENSOR_MAP_SWIZZLE_128B))
        return SI_ERR_CUDA;
    si::GemmParams p{};
    p.R = R;
    p.batches = batches;
    p.N = N;
    p.K = K;
    p.KB = KB;
    p.alpha = alpha;
    p.C = C;
    p.tiles_m = (R + G::BM - 1) / G::BM;
    p.tiles_n = (N + BN - 1) / BN;
    p.err = status;
    p.timeout_ns = si_host::timeout_ns();
    auto kern = si::gemm_kernel<BN, F32>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(G::DYN_BYTES));
    if (e != cudaSuccess) return si_host::cuda_fail("producer GEMM shared-memory attribute", e);
    const int64_t tiles = batches * p.tiles_m * p.tiles_n;
    int64_t grid = sms < si_host::kMaxCtas ? sms : si_host::kMaxCtas;
    if (grid > tiles) grid = tiles;
    kern<<<static_cast<unsigned>(grid), G::THREADS, G::DYN_BYTES, stream>>>(ta, tb, p);
    e = cudaGetLastError();
    return e == cudaSuccess ? SI_OK : si_host::cuda_fail("producer GEMM launch", e);
}

// Column tile by output width: 256 (q), 128 (kc), 64 (w and small widths).
template <bool F32>
si_status launch_gemm_n(const void* A, int64_t K, int64_t R, int64_t batches, int64_t a_row, int64_t a_batch,
                        const void* W, int64_t N, int64_t KB, float alpha, void* C, uint32_t* status,
                        cudaStream_t s) {
    if (N >= 256) return launch_gemm<256, F32>(A, K, R, batches, a_row, a_batch, W, N, KB, alpha, C, status, s);
    if (N >= 128) return launch_gemm<128, F32>(A, K, R, batches, a_row, a_batch, W, N, KB, alpha, C, status, s);
    return launch_gemm<64, F32>(A, K, R, batches, a_row, a_batch, W, N, KB, alpha, C, status, s);
}

}  // namespace

extern "C" si_status si_indexer_inputs(const void* x, const void* w_q, const void* w_w, const void* w_k,
                                       int64_t B, int64_t S, int d_model, int H_I, int d_I, int m, void* q,
                                       float* w, void* kc, uint32_t* status, si_stream_t stream) {
    if (B < 1 || S < 1 || m < 1 || d_model < 64 || H_I < 1 || d_I < 1) return SI_ERR_INVALID_ARG;
    if (!x || !w_q || !w_w || !w_k || !q || !w || !kc || !status) return SI_ERR_INVALID_ARG;
    if (d_model % 64 != 0 || (static_cast<int64_t>(H_I) * d_I) % 8 != 0 || H_I % 4 != 0 || d_I % 8 != 0)
        return SI_ERR_UNSUPPORTED;
    const int64_t T = S / m;
    if (B * S >= (int64_t{1} << 31) || static_cast<int64_t>(m) * d_model >= (int64_t{1} << 31)) return SI_ERR_UNSUPPORTED;
    auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!a16(x) || !a16(w_q) || !a16(w_w) || !a16(w_k) || !a16(q) || !a16(w) || !a16(kc) ||
        (reinterpret_cast<uintptr_t>(status) & 3u))
        return SI_ERR_MISALIGNED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(status, 0, sizeof(uint32_t), s) != cudaSuccess) return SI_ERR_CUDA;
    const int64_t D = d_model;
    // q = x W_q^T: rows are tokens
    si_status st = launch_gemm_n<false>(x, D, S, B, D, S * D, w_q, static_cast<int64_t>(H_I) * d_I, D, 1.0f, q,
                                        status, s);
    if (st != SI_OK) return st;
    // w = x W_w^T (fp32)
    st = launch_gemm_n<true>(x, D, S, B, D, S * D, w_w, H_I, D, 1.0f, w, status, s);
    if (st != SI_OK) return st;
    // kc: a row is m consecutive tokens (K = m * d_model); W_k wraps every d_model columns; alpha = 1/m
    if (T > 0)
        st = launch_gemm_n<false>(x, static_cast<int64_t>(m) * D, T, B, static_cast<int64_t>(m) * D, S * D, w_k, d_I,
                                  D, 1.0f / static_cast<float>(m), kc, status, s);
    return st;
}
