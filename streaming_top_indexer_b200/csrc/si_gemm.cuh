// si_gemm.cuh -- the indexer's upstream producers as one bf16 tcgen05 GEMM, sm_100a.
//
// The lightning indexer scores queries against keys compressed at ratio m
// (StreamIndex: Memory-Bounded Compressed Sparse Attention via Streaming
// Top-k, Abstract); the Abstract gives neither the projections nor the
// compressor.  Reading of this library, weights in [out, in] layout:
//     q  = x W_q^T  (bf16)     w = x W_w^T  (fp32)
//     kc[s] = (1/m) sum_{j<m} x[s*m + j] W_k^T  (bf16)
// All three are one kernel shape:
//     C[b, r, n] = alpha * sum_{k < K} A[b, r, k] * Bw[n, k mod KB]
// with A read through a 3-D tensor map {K, R, batches} (for the compressor
// a row is m consecutive tokens, K = m * d_model, and the weight operand
// wraps every KB = d_model columns, so no stacked copy of W_k exists) and
// the weights through a 2-D map {KB, N}.
//
// One persistent CTA per SM walks output tiles of 128 rows x BN columns:
//   warp 0     TMA producer: A and weight k-blocks of 64 (128-byte rows,
//              128-byte swizzle) into an NSTAGE ring;
//   warp 1     TMEM allocation; one thread issues tcgen05.mma (M=128,
//              N=BN, K=16) into two BN-column fp32 accumulators;
//   warps 2-5  epilogue: tcgen05.ld, scale, convert, store (the TMEM lane
//              quarter of warp w is w % 4).
#pragma once
#include <cuda.h>

#include <cstdint>

#include "si_ptx.cuh"

namespace si {

struct GemmParams {
    int64_t R;          // rows per batch
    int64_t batches;
    int64_t N, K, KB;   // K: reduction length; KB: period of the weight columns (K when it does not wrap)
    float alpha;
    void* C;            // [batches, R, N], bf16 or fp32
    int64_t tiles_m;    // ceil(R / 128)
    int64_t tiles_n;    // ceil(N / BN)
    uint32_t* err;
    uint64_t timeout_ns;
};

template <int BN>
struct GemmCfg {
    static_assert(BN == 64 || BN == 128 || BN == 256, "BN");
    static constexpr int BM = 128, BK = 64;
    static constexpr uint32_t A_BYTES = BM * 128u;      // 128 rows x 64 bf16
    static constexpr uint32_t B_BYTES = BN * 128u;
    static constexpr int NSTAGE = BN == 256 ? 4 : 6;
    static constexpr uint32_t OFF_A = 0;
    static constexpr uint32_t OFF_B = NSTAGE * A_BYTES;
    static constexpr uint32_t DYN_BYTES = OFF_B + NSTAGE * B_BYTES + 1024;
    static constexpr int THREADS = 192;
    static constexpr uint32_t TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;
};

enum : int { kGFull = 0, kGEmpty = 6, kGAccFull = 12, kGAccEmpty = 14, kGDrain = 16, kGNumBars = 17 };

__device__ __forceinline__ bool gemm_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < limit_ns)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

template <int BN, bool OUT_F32>
__global__ void __launch_bounds__(GemmCfg<BN>::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const GemmParams p) {
    using C = GemmCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[kGNumBars];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag_s;
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar0 = smem_u32(bars);
    auto bar = [bar0](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = &abort_flag_s;
    const uint64_t lim = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(bar(kGFull + s), 1);
            mbar_init(bar(kGEmpty + s), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(kGAccFull + i), 1);
            mbar_init(bar(kGAccEmpty + i), 4);
        }
        mbar_init(bar(kGDrain), 1);
        abort_flag_s = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tm_a);
        prefetch_tmap(&tm_b);
    }
    if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;

    const int64_t G = gridDim.x;
    const int64_t tiles = p.batches * p.tiles_m * p.tiles_n;
    const int nkb = static_cast<int>(p.K / C::BK);
    // tile t: column tile fastest (CTAs next to each other share the rows of A)
    auto tile_of = [&](int64_t t, int64_t& b, int64_t& r0, int64_t& n0) {
        n0 = (t % p.tiles_n) * BN;
        const int64_t mt = t / p.tiles_n;
        r0 = (mt % p.tiles_m) * C::BM;
        b = mt / p.tiles_m;
    };

    if (warp == 0) {
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < tiles; t += G) {
                int64_t b, r0, n0;
                tile_of(t, b, r0, n0);
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const uint32_t st = it % C::NSTAGE, u = it / C::NSTAGE;
                    if (u >= 1 && !(ok = mbar_wait(bar(kGEmpty + st), (u - 1) & 1u, abort_flag, p.err, lim))) break;
                    mbar_arrive_expect_tx(bar(kGFull + st), C::A_BYTES + C::B_BYTES);
                    tma_load_3d(sbase + C::OFF_A + st * C::A_BYTES, &tm_a, bar(kGFull + st), kb * C::BK,
                                static_cast<int>(r0), static_cast<int>(b));
                    tma_load_2d(sbase + C::OFF_B + st * C::B_BYTES, &tm_b, bar(kGFull + st),
                                static_cast<int>((static_cast<int64_t>(kb) * C::BK) % p.KB), static_cast<int>(n0));
                }
            }
            if (!ok) {  // let the loads already issued land
                const uint32_t n = it < C::NSTAGE ? it : C::NSTAGE;
                for (uint32_t i = it - n; i < it; ++i)
                    gemm_wait_bounded(bar(kGFull + i % C::NSTAGE), (i / C::NSTAGE) & 1u, 100000000ull);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(C::BM, BN);
            uint32_t it = 0, tile_it = 0;
            bool ok = true, issued = false;
            for (int64_t t = blockIdx.x; ok && t < tiles; t += G, ++tile_it) {
                const uint32_t ab = tile_it & 1u, au = tile_it >> 1;
                if (au >= 1 && !(ok = mbar_wait(bar(kGAccEmpty + ab), (au - 1) & 1u, abort_flag, p.err, lim))) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + ab * BN;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const uint32_t st = it % C::NSTAGE, u = it / C::NSTAGE;
                    if (!(ok = mbar_wait(bar(kGFull + st), u & 1u, abort_flag, p.err, lim))) break;
                    tc_fence_after();
                    const uint64_t da = smem_desc_sw128(sbase + C::OFF_A + st * C::A_BYTES);
                    const uint64_t db = smem_desc_sw128(sbase + C::OFF_B + st * C::B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < C::BK / 16; ++kk)  // 32 bytes = 2 descriptor units per K step
                        umma_bf16(d_tmem, da + kk * 2, db + kk * 2, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(bar(kGEmpty + st));
                    issued = true;
                }
                if (!ok) break;
                umma_commit(bar(kGAccFull + ab));
            }
            if (issued) {
                umma_commit(bar(kGDrain));
                gemm_wait_bounded(bar(kGDrain), 0, 100000000ull);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 2-5)
        const int quarter = warp & 3;
        const int row_in_tile = quarter * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        uint32_t tile_it = 0;
        for (int64_t t = blockIdx.x; t < tiles; t += G, ++tile_it) {
            int64_t b, r0, n0;
            tile_of(t, b, r0, n0);
            const uint32_t ab = tile_it & 1u, au = tile_it >> 1;
            bool ok = mbar_wait(bar(kGAccFull + ab), au & 1u, abort_flag, p.err, lim);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const int64_t r = r0 + row_in_tile;
            const bool row_ok = r < p.R;
            const int64_t crow = (b * p.R + r) * p.N;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem_base + ab * BN + c0 + lane_off, v);
                tmem_wait_ld(v);
                const int64_t n = n0 + c0;
                if (!row_ok || n >= p.N) continue;
                const bool full = n + 32 <= p.N;
                if constexpr (OUT_F32) {
                    float* dst = static_cast<float*>(p.C) + crow + n;
                    if (full) {
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            reinterpret_cast<float4*>(dst)[e] =
                                make_float4(__uint_as_float(v[4 * e]) * p.alpha, __uint_as_float(v[4 * e + 1]) * p.alpha,
                                            __uint_as_float(v[4 * e + 2]) * p.alpha,
                                            __uint_as_float(v[4 * e + 3]) * p.alpha);
                    } else {
                        for (int e = 0; e < 32 && n + e < p.N; ++e) dst[e] = __uint_as_float(v[e]) * p.alpha;
                    }
                } else {
                    uint16_t* dst = static_cast<uint16_t*>(p.C) + crow + n;
                    uint32_t w16[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        uint32_t r2;
                        asm("cvt.rn.bf16x2.f32 %0, %1, %2;"
                            : "=r"(r2)
                            : "f"(__uint_as_float(v[2 * e + 1]) * p.alpha), "f"(__uint_as_float(v[2 * e]) * p.alpha));
                        w16[e] = r2;
                    }
                    if (full) {
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            reinterpret_cast<uint4*>(dst)[e] = make_uint4(w16[4 * e], w16[4 * e + 1], w16[4 * e + 2],
                                                                          w16[4 * e + 3]);
                    } else {
                        for (int e = 0; e < 32 && n + e < p.N; ++e)
                            dst[e] = static_cast<uint16_t>((w16[e >> 1] >> (16 * (e & 1))) & 0xFFFFu);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kGAccEmpty + ab));
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace si
