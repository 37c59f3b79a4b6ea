// si_cut_bench.cu -- microbenchmark of one pool cut and one unit-end emit of
// the select kernel (cut_pool / emit_best), outside the kernel: each 128-thread
// half of 148 CTAs runs the call on a synthetic pool, timed with clock64.
// Development tool only; the library does not use it.
//
// Build: python -m streaming_top_indexer_b200.build --cut-bench
// Run:   streaming_top_indexer_b200/_build/si_cut_bench SMEM P KEPT CNT K SLACK MODE TIES [SORT_E]
//   SMEM   1: the pool in shared memory; 0: in global memory, with the
//          3072-key shared-memory buffer the select kernel gives workspace pools
//   P      pool capacity; KEPT survivors of an earlier cut at the pool front;
//          CNT appended keys in each of the four warps' sub-ranges
//   K      k; SLACK the entries above k an intermediate cut may keep
//   MODE   0: cut_pool; 1: emit_best (SORT_E: keys per thread of the row sort, 0 = unsorted)
//   TIES   1: 16 score levels (many equal scores), 0: distinct random scores
// Prints the mean cycles per call over the halves.
#include <cuda.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "si_select.cuh"

using namespace si;

namespace {

__device__ __forceinline__ uint32_t mix32(uint32_t x) {
    x ^= x >> 16;
    x *= 0x7feb352du;
    x ^= x >> 15;
    x *= 0x846ca68bu;
    x ^= x >> 16;
    return x;
}

// distinct keys (distinct key index i), positive scores
__device__ __forceinline__ uint64_t make_key(uint32_t seed, uint32_t i, int ties) {
    uint32_t h = mix32(seed * 0x9E3779B9u + i);
    if (ties) h &= 0xF0000000u;
    return (static_cast<uint64_t>(0x80000000u | (h >> 1)) << 32) | static_cast<uint64_t>(~i);
}

constexpr int kBig = 3072;  // the select kernel's per-half buffer for workspace pools

template <bool SMEM_POOL>
__global__ void __launch_bounds__(256, 1) cut_bench(uint64_t* gpool, int P, int kept0, int cnt, int k, int slack,
                                                    int mode, int iters, int ties, int sort_e, int32_t* oidx,
                                                    float* osc, long long* out) {
    extern __shared__ __align__(1024) uint8_t dsm[];
    __shared__ CutScratch cs_s[2];
    const int half = threadIdx.x >> 7, htid = threadIdx.x & 127;
    const uint32_t bar_id = 1 + half;
    CutScratch& cs = cs_s[half];
    uint64_t* big = SMEM_POOL ? nullptr : reinterpret_cast<uint64_t*>(dsm) + half * kBig;
    uint64_t* pq = SMEM_POOL ? reinterpret_cast<uint64_t*>(dsm) + half * P
                             : gpool + (static_cast<size_t>(blockIdx.x) * 2 + half) * P;
    const uint32_t F = (P - kept0) / 4;
    const uint32_t c4[4] = {static_cast<uint32_t>(cnt), static_cast<uint32_t>(cnt), static_cast<uint32_t>(cnt),
                            static_cast<uint32_t>(cnt)};
    uint32_t phase = 0;
    long long tot = 0;
    const uint32_t seed = blockIdx.x * 2 + half;
    for (int it = 0; it < iters; ++it) {
        // refill: survivors [0, kept0), warp w's sub-range [kept0 + w*F, + cnt)
        for (int i = htid; i < kept0 + 4 * static_cast<int>(F); i += 128) {
            const int r = i < kept0 ? -1 : (i - kept0) / static_cast<int>(F);
            const int o = i < kept0 ? 0 : (i - kept0) % static_cast<int>(F);
            if (r < 0 || o < cnt) pq[i] = make_key(seed + it * 977, i, ties);
        }
        __threadfence_block();
        bar_sync(bar_id, 128);
        const long long t0 = clock64();
        const PoolRegions rg = pool_regions(kept0, F, c4);
        if (mode == 0) {
            uint32_t kept = 0;
            cut_pool(pq, rg, k, k + slack, 0ull, cs, htid, bar_id, phase, kept, big, kBig);
        } else {
            const size_t row = (static_cast<size_t>(blockIdx.x) * 2 + half) * k;
            emit_best(pq, rg, k, cs, htid, bar_id, phase, oidx + row, osc + row, big, kBig, sort_e);
        }
        bar_sync(bar_id, 128);
        tot += clock64() - t0;
    }
    if (htid == 0) out[blockIdx.x * 2 + half] = tot / iters;
}

}  // namespace

int main(int argc, char** argv) {
    if (argc < 9) {
        std::fprintf(stderr, "usage: %s SMEM P KEPT CNT K SLACK MODE TIES [SORT_E]\n", argv[0]);
        return 2;
    }
    const int sm = std::atoi(argv[1]), P = std::atoi(argv[2]), kept0 = std::atoi(argv[3]), cnt = std::atoi(argv[4]);
    const int k = std::atoi(argv[5]), slack = std::atoi(argv[6]), mode = std::atoi(argv[7]), ties = std::atoi(argv[8]);
    const int sort_e = argc > 9 ? std::atoi(argv[9]) : 0;
    // argument checks that keep every access in bounds
    if (P < 64 || P % 32 || kept0 < 0 || kept0 >= P || cnt < 0 || cnt > (P - kept0) / 4 || k < 1 || k > 2048 ||
        slack < 0 || (sm && 2 * static_cast<size_t>(P) * 8 > 200 * 1024) || (sort_e && 128 * sort_e < k) ||
        (mode == 1 && sort_e && sm && 128 * sort_e > P)) {
        std::fprintf(stderr, "arguments out of range\n");
        return 2;
    }
    const int G = 148, iters = 20;
    uint64_t* gpool = nullptr;
    int32_t* oidx = nullptr;
    float* osc = nullptr;
    long long* out = nullptr;
    cudaMalloc(&gpool, static_cast<size_t>(G) * 2 * P * 8);
    cudaMalloc(&oidx, static_cast<size_t>(G) * 2 * k * 4);
    cudaMalloc(&osc, static_cast<size_t>(G) * 2 * k * 4);
    cudaMalloc(&out, G * 2 * sizeof(long long));
    const size_t dyn = sm ? 2 * static_cast<size_t>(P) * 8 : 2 * kBig * 8;
    auto kern = sm ? cut_bench<true> : cut_bench<false>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dyn));
    kern<<<G, 256, dyn>>>(gpool, P, kept0, cnt, k, slack, mode, iters, ties, sort_e, oidx, osc, out);
    const cudaError_t e = cudaDeviceSynchronize();
    std::vector<long long> h(G * 2);
    cudaMemcpy(h.data(), out, h.size() * sizeof(long long), cudaMemcpyDeviceToHost);
    double s = 0;
    for (long long v : h) s += static_cast<double>(v);
    std::printf("smem=%d P=%d kept=%d cnt=%d k=%d slack=%d mode=%s ties=%d sort_e=%d: %s, cycles per call %.0f\n", sm, P,
                kept0, cnt, k, slack, mode ? "emit" : "cut", ties, sort_e, cudaGetErrorString(e), s / h.size());
    cudaFree(gpool);
    cudaFree(oidx);
    cudaFree(osc);
    cudaFree(out);
    return e == cudaSuccess ? 0 : 1;
}
