// si_attn.cuh -- CSA sparse attention over the indexer's selected keys, sm_100a.
//
// After the lightning indexer has picked the top-k compressed keys of each
// query, the sparse attention reads only those keys (StreamIndex:
// Memory-Bounded Compressed Sparse Attention via Streaming Top-k, Abstract).
// Reading of this library: for query row t, head h,
//     out[t,h,:] = sum_{j in J_t} softmax_j(scale * q[t,h,:] . K[j,:]) V[j,:]
//     lse[t,h]   = log sum_{j in J_t} exp(scale * q[t,h,:] . K[j,:])
// over the entries J_t of idx[t, 0..k) that lie in [0, T) (others are
// padding).  K and V are the compressed key/value entries shared by all heads.
//
// One CTA per SM, a persistent loop over query rows (all rows cost the same:
// ceil(k/64) key chunks).  Per row the 128 heads are the MMA's M (one TMEM
// lane each); per chunk of 64 selected keys:
//   S   = Q K^T      tcgen05.mma M=128 N=64  K=d    (fp32 in TMEM)
//   P   = softmax    one thread per head, online, bf16 into shared memory
//   O  += P V        tcgen05.mma M=128 N=dv K=64    (V as an MN-major operand)
// Roles (192 threads): warp 0 loads q by TMA (double-buffered) and gathers
// the chunk's K and V rows with TMA gather4 (four rows per instruction, no
// multicast) into a 4-stage ring; warp 1 allocates TMEM and issues the MMAs
// (S of chunk g+1 before O of chunk g, across rows); warps 2-5 compute the
// softmax.  The running max is kept in base-2 units; O in TMEM is rescaled
// only when a chunk's max exceeds the running max by more than 8 (so every
// p <= 2^8 before normalisation).  At the end of a row, out = O / l in bf16
// and lse = ln 2 * (m + log2 l); a row with no valid entry gives 0 and -inf.
#pragma once
#include <cuda.h>

#include <cstdint>

#include "si_ptx.cuh"

namespace si {

struct AttnParams {
    int64_t rows;         // B * S query rows
    int64_t S, T;
    int k;                // entries per idx row
    int nchunks;          // ceil(k / 64)
    const int32_t* idx;   // [B*S, k]
    uint16_t* out;        // bf16 [B*S, 128, DV]
    float* lse;           // [B*S, 128]
    float c2;             // scale * log2(e)
    uint32_t* err;        // device status word
    uint64_t timeout_ns;
};

template <int D, int DV>
struct AttnCfg {
    static_assert(D == 64 || D == 128, "d");
    static_assert(DV == 64 || DV == 128, "d_v");
    static constexpr int HA = 128;                     // heads: MMA M, TMEM lanes
    static constexpr int NK = 64;                      // keys per chunk
    static constexpr int NST = 4;                      // K/V ring stages
    static constexpr uint32_t Q_SUB = HA * 128u;       // 64 columns of q: 16 KB
    static constexpr uint32_t Q_BYTES = (D / 64) * Q_SUB;
    static constexpr uint32_t KV_SUB = NK * 128u;      // 64 columns of 64 keys: 8 KB
    static constexpr uint32_t K_BYTES = (D / 64) * KV_SUB;
    static constexpr uint32_t V_BYTES = (DV / 64) * KV_SUB;
    static constexpr uint32_t P_BYTES = HA * 128u;     // [128 heads x 64 keys] bf16
    static constexpr uint32_t OFF_Q = 0;               // 2 buffers
    static constexpr uint32_t OFF_K = OFF_Q + 2 * Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + NST * K_BYTES;
    static constexpr uint32_t OFF_P = OFF_V + NST * V_BYTES;  // 2 buffers
    static constexpr uint32_t DYN_BYTES = OFF_P + 2 * P_BYTES + 1024;  // + alignment slack
    static constexpr int THREADS = 192;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TM_S = 0;                // S[2]: columns 0 and 64
    static constexpr uint32_t TM_O = 128;              // O[2]: columns 128 and 128 + DV
    static_assert(TM_O + 2 * DV <= TMEM_COLS, "TMEM budget");
    // Rescale threshold of the running max, base-2 units.
    static constexpr float RESCALE = 8.0f;
};

enum : int {
    kAQFull = 0,       // [2]
    kAQEmpty = 2,      // [2]
    kAKFull = 4,       // [4]
    kAVFull = 8,       // [4]
    kAKVEmpty = 12,    // [4]
    kASFull = 16,      // [2]
    kASFree = 18,      // [2]
    kAPFull = 20,      // [2]
    kAPEmpty = 22,     // [2]
    kAOFull = 24,      // [2]
    kAOFree = 26,      // [2]
    kADrain = 28,
    kANumBars = 29
};

__device__ __forceinline__ bool attn_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < limit_ns)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

template <int D, int DV>
__global__ void __launch_bounds__(AttnCfg<D, DV>::THREADS, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
    using C = AttnCfg<D, DV>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[kANumBars];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag_s;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t bar0 = smem_u32(bars);
    auto bar = [bar0](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = &abort_flag_s;
    const uint64_t lim = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(kAQFull + i), 1);
            mbar_init(bar(kAQEmpty + i), 1);
            mbar_init(bar(kASFull + i), 1);
            mbar_init(bar(kASFree + i), 4);
            mbar_init(bar(kAPFull + i), 4);
            mbar_init(bar(kAPEmpty + i), 1);
            mbar_init(bar(kAOFull + i), 1);
            mbar_init(bar(kAOFree + i), 4);
        }
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(bar(kAKFull + s), 1);
            mbar_init(bar(kAVFull + s), 1);
            mbar_init(bar(kAKVEmpty + s), 1);
        }
        mbar_init(bar(kADrain), 1);
        abort_flag_s = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;

    const int64_t G = gridDim.x;
    const int64_t nrows = (p.rows - blockIdx.x + G - 1) / G;  // rows blockIdx.x + i*G
    const int NC = p.nchunks;
    const int64_t total = nrows * NC;                           // chunks of this CTA

    if (warp == 0) {
        // ------------------------------------------------ TMA: q tiles, K/V gathers
        // Lane l gathers rows 4*(l%16) .. +3 of the chunk; lanes 0-15 the first
        // 64 columns, lanes 16-31 the second (d or d_v = 128).
        const int gg = lane & 15, cc = lane >> 4;
        uint32_t kv_it = 0;
        int64_t q_it = 0;
        bool ok = true;
        for (int64_t i = 0; ok && i < nrows; ++i) {
            const int64_t row = blockIdx.x + i * G;
            const int64_t b = row / p.S;
            const uint32_t qb = static_cast<uint32_t>(i & 1);
            if (i >= 2) ok = mbar_wait(bar(kAQEmpty + qb), static_cast<uint32_t>((i >> 1) - 1) & 1u, abort_flag, p.err,
                                       lim);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(kAQFull + qb), C::Q_BYTES);
#pragma unroll
                for (int c = 0; c < D / 64; ++c)
                    tma_load_2d(sbase + C::OFF_Q + qb * C::Q_BYTES + c * C::Q_SUB, &tm_q, bar(kAQFull + qb), c * 64,
                                static_cast<int>(row * C::HA));
            }
            ++q_it;
            const int32_t* irow = p.idx + row * p.k;
            for (int c = 0; c < NC; ++c) {
                const uint32_t st = kv_it % C::NST, u = kv_it / C::NST;
                if (u >= 1) ok = mbar_wait(bar(kAKVEmpty + st), (u - 1) & 1u, abort_flag, p.err, lim);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                int r[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = c * C::NK + 4 * gg + e;
                    const int v = j < p.k ? irow[j] : -1;
                    // padding and out-of-range entries read key 0 (masked by the softmax)
                    r[e] = static_cast<int>(b * p.T) + ((v >= 0 && v < p.T) ? v : 0);
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(kAKFull + st), C::K_BYTES);
                    mbar_arrive_expect_tx(bar(kAVFull + st), C::V_BYTES);
                }
                __syncwarp();
                if (cc < D / 64)
                    tma_gather4(sbase + C::OFF_K + st * C::K_BYTES + cc * C::KV_SUB + gg * 512u, &tm_k,
                                bar(kAKFull + st), cc * 64, r[0], r[1], r[2], r[3]);
                if (cc < DV / 64)
                    tma_gather4(sbase + C::OFF_V + st * C::V_BYTES + cc * C::KV_SUB + gg * 512u, &tm_v,
                                bar(kAVFull + st), cc * 64, r[0], r[1], r[2], r[3]);
                ++kv_it;
            }
        }
        if (!ok && lane == 0) {
            // let every load already issued land before the CTA exits
            const uint64_t drain = 100000000ull;
            const uint32_t n = kv_it < C::NST ? kv_it : C::NST;
            for (uint32_t it = kv_it - n; it < kv_it; ++it) {
                attn_wait_bounded(bar(kAKFull + it % C::NST), (it / C::NST) & 1u, drain);
                attn_wait_bounded(bar(kAVFull + it % C::NST), (it / C::NST) & 1u, drain);
            }
            for (int64_t i = q_it - 2 < 0 ? 0 : q_it - 2; i < q_it; ++i)
                attn_wait_bounded(bar(kAQFull + (i & 1)), static_cast<uint32_t>(i >> 1) & 1u, drain);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(C::HA, C::NK);
            constexpr uint32_t idesc_o = idesc_bf16_f32_bmn(C::HA, DV);
            bool ok = true, issued = false;
            // O += P V for chunk h (of row h / NC)
            auto issue_pv = [&](int64_t h) -> bool {
                const int64_t i = h / NC;
                const int c = static_cast<int>(h % NC);
                const uint32_t pb = static_cast<uint32_t>(h & 1);
                const uint32_t st = static_cast<uint32_t>(h % C::NST), u = static_cast<uint32_t>(h / C::NST);
                const uint32_t ob = static_cast<uint32_t>(i & 1);
                if (!mbar_wait(bar(kAPFull + pb), static_cast<uint32_t>(h >> 1) & 1u, abort_flag, p.err, lim))
                    return false;
                if (!mbar_wait(bar(kAVFull + st), u & 1u, abort_flag, p.err, lim)) return false;
                if (c == 0 && i >= 2 &&
                    !mbar_wait(bar(kAOFree + ob), static_cast<uint32_t>((i >> 1) - 1) & 1u, abort_flag, p.err, lim))
                    return false;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + C::TM_O + ob * DV;
                const uint32_t a_base = sbase + C::OFF_P + pb * C::P_BYTES;
                const uint32_t b_base = sbase + C::OFF_V + st * C::V_BYTES;
#pragma unroll
                for (int kk = 0; kk < C::NK / 16; ++kk)
                    umma_bf16(d_tmem, smem_desc_sw128(a_base + kk * 32),
                              smem_desc_sw128_mn(b_base + kk * 2048, C::KV_SUB, 1024), idesc_o,
                              (c > 0 || kk > 0) ? 1u : 0u);
                umma_commit(bar(kAPEmpty + pb));
                umma_commit(bar(kAKVEmpty + st));
                if (c == NC - 1) umma_commit(bar(kAOFull + ob));
                return true;
            };
            int64_t g = 0;
            for (; g < total; ++g) {
                const int64_t i = g / NC;
                const int c = static_cast<int>(g % NC);
                const uint32_t qb = static_cast<uint32_t>(i & 1);
                if (c == 0) ok = mbar_wait(bar(kAQFull + qb), static_cast<uint32_t>(i >> 1) & 1u, abort_flag, p.err,
                                           lim);
                const uint32_t st = static_cast<uint32_t>(g % C::NST), u = static_cast<uint32_t>(g / C::NST);
                ok = ok && mbar_wait(bar(kAKFull + st), u & 1u, abort_flag, p.err, lim);
                const uint32_t sb = static_cast<uint32_t>(g & 1), us = static_cast<uint32_t>(g >> 1);
                if (us >= 1) ok = ok && mbar_wait(bar(kASFree + sb), (us - 1) & 1u, abort_flag, p.err, lim);
                if (!ok) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + C::TM_S + sb * C::NK;
                const uint32_t a_base = sbase + C::OFF_Q + qb * C::Q_BYTES;
                const uint32_t b_base = sbase + C::OFF_K + st * C::K_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t sub = kk / 4, off = (kk % 4) * 32;
                    umma_bf16(d_tmem, smem_desc_sw128(a_base + sub * C::Q_SUB + off),
                              smem_desc_sw128(b_base + sub * C::KV_SUB + off), idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(bar(kASFull + sb));
                if (c == NC - 1) umma_commit(bar(kAQEmpty + qb));
                issued = true;
                if (g >= 1 && !(ok = issue_pv(g - 1))) break;
            }
            if (ok && total > 0) issue_pv(total - 1);
            if (issued) {
                umma_commit(bar(kADrain));
                attn_wait_bounded(bar(kADrain), 0, 100000000ull);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ softmax (warps 2-5)
        const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
        const int h = quarter * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t p_row = static_cast<uint32_t>(h >> 3) * 1024u + static_cast<uint32_t>(h & 7) * 128u;
        const float LN2 = 0.6931471805599453f;
        int64_t g = 0;
        bool ok = true;
        for (int64_t i = 0; ok && i < nrows; ++i) {
            const int64_t row = blockIdx.x + i * G;
            const int32_t* irow = p.idx + row * p.k;
            float m_run = -__int_as_float(0x7f800000), l_run = 0.0f;
            for (int c = 0; c < NC; ++c, ++g) {
                const uint32_t sb = static_cast<uint32_t>(g & 1), us = static_cast<uint32_t>(g >> 1);
                // validity of the chunk's 64 entries
                const int j0 = c * C::NK + lane, j1 = j0 + 32;
                const int v0 = j0 < p.k ? irow[j0] : -1, v1 = j1 < p.k ? irow[j1] : -1;
                const uint32_t mw0 = __ballot_sync(0xffffffffu, v0 >= 0 && v0 < p.T);
                const uint32_t mw1 = __ballot_sync(0xffffffffu, v1 >= 0 && v1 < p.T);
                ok = mbar_wait(bar(kASFull + sb), us & 1u, abort_flag, p.err, lim);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
                uint32_t sr[64];
                tmem_ld32(tmem_base + C::TM_S + sb * C::NK + lane_off, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                tmem_ld32(tmem_base + C::TM_S + sb * C::NK + 32 + lane_off,
                          *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kASFree + sb));
                // scores in base-2 units; invalid entries -inf
                float x[64];
                float m_c = -__int_as_float(0x7f800000);
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    const bool valid = ((j < 32 ? mw0 >> j : mw1 >> (j - 32)) & 1u) != 0;
                    x[j] = valid ? __uint_as_float(sr[j]) * p.c2 : -__int_as_float(0x7f800000);
                    m_c = fmaxf(m_c, x[j]);
                }
                const uint32_t ob = static_cast<uint32_t>(i & 1);
                const uint32_t o_addr = tmem_base + C::TM_O + ob * DV + lane_off;
                if (c == 0) {
                    m_run = m_c;
                } else if (m_c > m_run + C::RESCALE) {
                    // O (chunks up to g-1) and l to the new max: wait for the
                    // previous chunk's P V, then scale O in TMEM.
                    const uint32_t pprev = static_cast<uint32_t>((g - 1) & 1);
                    ok = mbar_wait(bar(kAPEmpty + pprev), static_cast<uint32_t>((g - 1) >> 1) & 1u, abort_flag, p.err,
                                   lim);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    tc_fence_after();
                    const float f = ex2_approx(m_run - m_c);
                    l_run *= f;
#pragma unroll
                    for (int cb = 0; cb < DV / 32; ++cb) {
                        uint32_t o[32];
                        tmem_ld32(o_addr + cb * 32, o);
                        tmem_wait_ld(o);
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
                        tmem_st32(o_addr + cb * 32, o);
                    }
                    tmem_wait_st();
                    m_run = m_c;
                }
                // the P buffer is free once the P V of chunk g-2 is done
                if (us >= 1) {
                    ok = mbar_wait(bar(kAPEmpty + sb), (us - 1) & 1u, abort_flag, p.err, lim);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                }
                // p = 2^(x - m), bf16, into P[sb] (row h, 128-byte swizzle)
                uint8_t* prow = smem + C::OFF_P + sb * C::P_BYTES + p_row;
                float sum = 0.0f;
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = c8 * 8 + 2 * e;
                        const float pa = x[j] == -__int_as_float(0x7f800000) ? 0.0f : ex2_approx(x[j] - m_run);
                        const float pb2 =
                            x[j + 1] == -__int_as_float(0x7f800000) ? 0.0f : ex2_approx(x[j + 1] - m_run);
                        sum += pa + pb2;
                        w4[e] = pack_bf16x2(pa, pb2);
                    }
                    *reinterpret_cast<uint4*>(prow + ((c8 ^ (h & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
                l_run += sum;
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kAPFull + sb));
                if (c == NC - 1) {
                    // end of the row: out = O / l (bf16), lse
                    ok = mbar_wait(bar(kAOFull + ob), static_cast<uint32_t>(i >> 1) & 1u, abort_flag, p.err, lim);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    tc_fence_after();
                    const float inv = l_run > 0.0f ? 1.0f / l_run : 0.0f;
                    uint16_t* orow = p.out + (row * C::HA + h) * DV;
#pragma unroll
                    for (int cb = 0; cb < DV / 32; ++cb) {
                        uint32_t o[32];
                        tmem_ld32(o_addr + cb * 32, o);
                        tmem_wait_ld(o);
                        uint32_t w[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
                        uint4* dst = reinterpret_cast<uint4*>(orow + cb * 32);
#pragma unroll
                        for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                    }
                    p.lse[row * C::HA + h] = l_run > 0.0f ? (m_run + lg2_approx(l_run)) * LN2 : -__int_as_float(0x7f800000);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(kAOFree + ob));
                }
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// Every output row of a problem without keys: out = 0, lse = -inf.
__global__ void attn_empty_kernel(uint16_t* __restrict__ out, float* __restrict__ lse, int64_t n_out, int64_t n_lse) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_out; i += stride) out[i] = 0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_lse; i += stride)
        lse[i] = -__int_as_float(0x7f800000);
}

}  // namespace si
