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
                        const bool swap = (a < b) == desc;  // keys distinct, or equal padding
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
                    v[e] = ((v[e] > other) == take_max) ? v[e] : other;
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

// Same ordering with E consecutive entries per lane (element i is slot i%E
// of lane i/E), one warp per row, for E = 4, 8, 16: partner distances below E
// are register swaps and the rest lane shuffles, fewer shuffle stages than
// the interleaved layout above, and each lane moves its entries with 16-byte
// accesses when the row is aligned.
template <int E>
__global__ void __launch_bounds__(32 * kSortWarps) sort_rows_lane_kernel(int32_t* __restrict__ idx,
                                                                         float* __restrict__ score, int64_t rows,
                                                                         int k) {
    static_assert(E % 4 == 0 && E <= 16, "four-entry vectors per lane");
    constexpr int K2 = 32 * E;
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kSortWarps + (threadIdx.x >> 5);
    if (row >= rows) return;
    int32_t* ri = idx + row * k + lane * E;
    float* rs = score + row * k + lane * E;
    const bool vec = ((reinterpret_cast<uintptr_t>(ri) | reinterpret_cast<uintptr_t>(rs)) & 15u) == 0 &&
                     lane * E + E <= k;
    uint64_t v[E];
    if (vec) {
#pragma unroll
        for (int c = 0; c < E / 4; ++c) {
            const int4 i4 = reinterpret_cast<const int4*>(ri)[c];
            const float4 s4 = reinterpret_cast<const float4*>(rs)[c];
            v[4 * c + 0] = pack_key(s4.x, static_cast<uint32_t>(i4.x));
            v[4 * c + 1] = pack_key(s4.y, static_cast<uint32_t>(i4.y));
            v[4 * c + 2] = pack_key(s4.z, static_cast<uint32_t>(i4.z));
            v[4 * c + 3] = pack_key(s4.w, static_cast<uint32_t>(i4.w));
        }
    } else {
#pragma unroll
        for (int e = 0; e < E; ++e)
            v[e] = (lane * E + e < k) ? pack_key(rs[e], static_cast<uint32_t>(ri[e])) : 0ull;
    }
#pragma unroll
    for (int size = 2; size <= K2; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            if (stride < E) {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int pe = e ^ stride;
                    if (pe > e) {
                        // keys are distinct (padding zeros are equal, and swapping
                        // them changes nothing), so one compare decides
                        const bool desc = ((lane * E + e) & size) == 0;
                        const uint64_t a = v[e], b = v[pe];
                        const bool sw = (a < b) == desc;
                        v[e] = sw ? b : a;
                        v[pe] = sw ? a : b;
                    }
                }
            } else {
                const int pl = stride / E;  // partner lane distance
                const bool lower = (lane & pl) == 0;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const uint64_t o = __shfl_xor_sync(0xffffffffu, v[e], pl);
                    const bool desc = ((lane * E + e) & size) == 0;
                    const bool take_max = (lower == desc);
                    v[e] = ((v[e] > o) == take_max) ? v[e] : o;
                }
            }
        }
    }
    if (vec) {
#pragma unroll
        for (int c = 0; c < E / 4; ++c) {
            reinterpret_cast<int4*>(ri)[c] = make_int4(key_index(v[4 * c]), key_index(v[4 * c + 1]),
                                                       key_index(v[4 * c + 2]), key_index(v[4 * c + 3]));
            reinterpret_cast<float4*>(rs)[c] = make_float4(key_score(v[4 * c]), key_score(v[4 * c + 1]),
                                                           key_score(v[4 * c + 2]), key_score(v[4 * c + 3]));
        }
    } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
            if (lane * E + e < k) {
                ri[e] = key_index(v[e]);
                rs[e] = key_score(v[e]);
            }
        }
    }
}

// Same ordering for long rows (K2 = 1024 or 2048 keys): one block of K2/8
// threads per row, eight keys per thread; element i is slot i%8 of thread
// i/8, so each thread loads and stores 8 consecutive entries.  Partner
// distances below 8 are register swaps, those below 256 lane shuffles inside
// the warp, and only the stages at 256 and above (3 for 1024, 6 for 2048)
// exchange through shared memory, double-buffered with one barrier each.
template <int K2>
__global__ void __launch_bounds__(K2 / 8) sort_rows_block_kernel(int32_t* __restrict__ idx,
                                                                 float* __restrict__ score, int64_t rows, int k) {
    constexpr int E = 8;
    __shared__ uint64_t xs[2][K2];
    const int tid = threadIdx.x;
    const int64_t row = blockIdx.x;
    if (row >= rows) return;
    int32_t* ri = idx + row * k;
    float* rs = score + row * k;
    // A thread's eight entries are 32 contiguous bytes of each array: two
    // 16-byte accesses when the row is 16-byte aligned and complete.
    const bool vec = ((reinterpret_cast<uintptr_t>(ri) | reinterpret_cast<uintptr_t>(rs)) & 15u) == 0 &&
                     tid * E + E <= k;
    uint64_t v[E];
    if (vec) {
        const int4 i0 = reinterpret_cast<const int4*>(ri + tid * E)[0];
        const int4 i1 = reinterpret_cast<const int4*>(ri + tid * E)[1];
        const float4 s0 = reinterpret_cast<const float4*>(rs + tid * E)[0];
        const float4 s1 = reinterpret_cast<const float4*>(rs + tid * E)[1];
        const int iv[E] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
        const float sv[E] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = pack_key(sv[e], static_cast<uint32_t>(iv[e]));
    } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int i = tid * E + e;
            v[e] = (i < k) ? pack_key(rs[i], static_cast<uint32_t>(ri[i])) : 0ull;
        }
    }
    int buf = 0;
#pragma unroll
    for (int size = 2; size <= K2; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            if (stride < E) {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int pe = e ^ stride;
                    if (pe > e) {
                        const bool desc = ((tid * E + e) & size) == 0;
                        const uint64_t a = v[e], b = v[pe];
                        const bool sw = (a < b) == desc;  // keys distinct, or equal padding
                        v[e] = sw ? b : a;
                        v[pe] = sw ? a : b;
                    }
                }
            } else {
                const int pt = stride / E;  // partner thread distance
                const bool lower = (tid & pt) == 0;
                uint64_t o[E];
                if (stride < 32 * E) {
#pragma unroll
                    for (int e = 0; e < E; ++e) o[e] = __shfl_xor_sync(0xffffffffu, v[e], pt);
                } else {
#pragma unroll
                    for (int e = 0; e < E; ++e) xs[buf][tid * E + e] = v[e];
                    __syncthreads();
#pragma unroll
                    for (int e = 0; e < E; ++e) o[e] = xs[buf][(tid ^ pt) * E + e];
                    buf ^= 1;
                }
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const bool desc = ((tid * E + e) & size) == 0;
                    const bool take_max = (lower == desc);
                    v[e] = ((v[e] > o[e]) == take_max) ? v[e] : o[e];
                }
            }
        }
    }
    if (vec) {
        reinterpret_cast<int4*>(ri + tid * E)[0] =
            make_int4(key_index(v[0]), key_index(v[1]), key_index(v[2]), key_index(v[3]));
        reinterpret_cast<int4*>(ri + tid * E)[1] =
            make_int4(key_index(v[4]), key_index(v[5]), key_index(v[6]), key_index(v[7]));
        reinterpret_cast<float4*>(rs + tid * E)[0] =
            make_float4(key_score(v[0]), key_score(v[1]), key_score(v[2]), key_score(v[3]));
        reinterpret_cast<float4*>(rs + tid * E)[1] =
            make_float4(key_score(v[4]), key_score(v[5]), key_score(v[6]), key_score(v[7]));
    } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int i = tid * E + e;
            if (i < k) {
                ri[i] = key_index(v[e]);
                rs[i] = key_score(v[e]);
            }
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
