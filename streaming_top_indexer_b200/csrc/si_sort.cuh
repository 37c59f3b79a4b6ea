// si_sort.cuh -- final ordering of each query row's top-k, and padding fill.
//
// The select kernel leaves every row's k entries in pool order.  Here one
// warp sorts one row in registers with a bitonic network on the packed
// 64-bit keys (score descending, index ascending; padding last).  Element i
// of the row lives in lane i%32, slot i/32, so loads and stores are
// coalesced; partner distances below 32 are lane shuffles, larger ones are
// register swaps.
#pragma once
#include <cstdint>

#include "si_keys.cuh"

namespace si {

constexpr int kSortWarps = 8;

template <int E>  // slots per lane; the network sorts 32*E >= k keys
__global__ void __launch_bounds__(32 * kSortWarps) sort_rows_kernel(int32_t* __restrict__ idx,
                                                                    float* __restrict__ score,
                                                                    int64_t rows, int k) {
    constexpr int K2 = 32 * E;
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kSortWarps + (threadIdx.x >> 5);
    if (row >= rows) return;
    int32_t* ri = idx + row * k;
    float* rs = score + row * k;
    uint64_t v[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int i = e * 32 + lane;
        v[e] = (i < k) ? pack_key(rs[i], static_cast<uint32_t>(ri[i])) : 0ull;
    }
#pragma unroll
    for (int size = 2; size <= K2; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            if (stride >= 32) {
                const int es = stride >> 5;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int pe = e ^ es;
                    if (pe > e) {
                        const bool desc = ((e * 32) & size) == 0;
                        const uint64_t a = v[e], b = v[pe];
                        const bool swap = desc ? (a < b) : (a > b);
                        v[e] = swap ? b : a;
                        v[pe] = swap ? a : b;
                    }
                }
            } else {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int i = e * 32 + lane;
                    const uint64_t other = __shfl_xor_sync(0xffffffffu, v[e], stride);
                    const bool lower = (lane & stride) == 0;
                    const bool desc = (i & size) == 0;
                    const bool take_max = (lower == desc);
                    v[e] = take_max ? (v[e] > other ? v[e] : other) : (v[e] < other ? v[e] : other);
                }
            }
        }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int i = e * 32 + lane;
        if (i < k) {
            ri[i] = key_index(v[e]);
            rs[i] = key_score(v[e]);
        }
    }
}

// Same ordering for long rows (32*E > 512): one block of K2/2 threads per row
// runs the bitonic network in shared memory, one compare-exchange per thread
// and stage, instead of holding 64 keys per lane in registers.
template <int K2>
__global__ void __launch_bounds__(K2 / 2) sort_rows_smem_kernel(int32_t* __restrict__ idx, float* __restrict__ score,
                                                                 int64_t rows, int k) {
    __shared__ uint64_t v[K2];
    const int tid = threadIdx.x;
    const int64_t row = blockIdx.x;
    if (row >= rows) return;
    int32_t* ri = idx + row * k;
    float* rs = score + row * k;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int i = tid + h * (K2 / 2);
        v[i] = (i < k) ? pack_key(rs[i], static_cast<uint32_t>(ri[i])) : 0ull;
    }
    __syncthreads();
    for (int size = 2; size <= K2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const int i = ((tid / stride) * 2 * stride) + (tid % stride);  // lower index of this thread's pair
            const int j = i + stride;
            const bool desc = (i & size) == 0;
            const uint64_t a = v[i], b = v[j];
            if (desc ? (a < b) : (a > b)) {
                v[i] = b;
                v[j] = a;
            }
            __syncthreads();
        }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int i = tid + h * (K2 / 2);
        if (i < k) {
            ri[i] = key_index(v[i]);
            rs[i] = key_score(v[i]);
        }
    }
}

// Every row all padding (no key is visible to any query).
__global__ void pad_rows_kernel(int32_t* __restrict__ idx, float* __restrict__ score, int64_t n) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
        idx[i] = -1;
        score[i] = -__int_as_float(0x7f800000);
    }
}

// Self-test of the bounded wait: waits on an mbarrier that nothing arrives
// on; the wait must give up after limit_ns and record a timeout.
__global__ void timeout_selftest_kernel(uint32_t* err, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, err, limit_ns);
    __syncthreads();
}

}  // namespace si
