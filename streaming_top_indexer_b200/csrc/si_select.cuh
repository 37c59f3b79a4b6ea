// si_select.cuh -- fused CSA indexer scoring + streaming top-k for sm_100a.
//
// One persistent CTA per SM.  A work unit is one block of QT = 256/H_I
// consecutive queries of one batch; the CTA streams the unit's causally
// visible compressed keys through in tiles of 128 and keeps a running top-k
// per query, so the [B,S,H_I,T] score tensor never exists (StreamIndex:
// Memory-Bounded Compressed Sparse Attention via Streaming Top-k, Abstract:
// the indexer step without materialising the intermediate, with a
// partition-merge of per-chunk candidates into the running top-k).
//
// Per key tile j of a unit:
//   acc[s, (q,h)] = sum_d kc[b, 128j+s, d] * q[b, t0+q, h, d]
// is one 128 x 256 x d_I tcgen05 MMA (bf16 in, fp32 in TMEM): keys are the
// MMA's M (TMEM lanes) and (query, head) pairs its N (TMEM columns), so each
// epilogue thread owns one key and reduces the heads of a query in registers:
//   score[t, s] = sum_h w[b,t,h] * max(acc[s,(t,h)], 0)      (h ascending)
// followed by the causal mask (s+1)*m <= t+1, i.e. s < min(T, (t+1)/m).
//
// Roles (320 threads): warp 0 issues TMA loads (w, q once per unit; kc per
// tile into a ring of smem stages), warp 1 allocates TMEM and issues the
// MMAs into two 256-column accumulators, warps 2..9 are the epilogue: two
// halves of four warps, half h owning queries [h*QT/2, (h+1)*QT/2) and each
// warp of a half one 32-lane quarter of TMEM.
//
// Running top-k: every (score, key) pair is packed into a 64-bit key whose
// unsigned order is the selection order (score descending, key index
// ascending).  A candidate enters a per-query pool only if it beats the
// query's threshold (the current k-th best).  When a pool nears its capacity
// P, one warp finds the k-th best pool entry by a most-significant-digit-first
// radix select, keeps exactly the k best entries and raises the threshold.
// At the end of a unit the pool is cut to k and written, unsorted, to the
// outputs; a separate kernel sorts each row.
#pragma once
#include <cuda.h>

#include <cstdint>

#include "si_keys.cuh"
#include "si_ptx.cuh"

namespace si {

struct SelectParams {
    int64_t B, S, T;
    int m, k;
    int P;              // pool capacity per query (multiple of 32, >= k + 256)
    int64_t nblk;       // query blocks per batch
    int64_t units;      // B * nblk
    int32_t* out_idx;   // [B,S,k]
    float* out_score;   // [B,S,k]
    float* dense;       // dense-score mode: [B,S,T] fp32, else nullptr
    uint64_t* gpool;    // pools in global memory (per CTA QT*P), or nullptr
    uint32_t* err;      // device error word
    uint64_t timeout_ns;
};

template <int H, int D>
struct SelCfg {
    static_assert(H == 8 || H == 16 || H == 32 || H == 64, "H_I");
    static_assert(D == 64 || D == 128, "d_I");
    static constexpr int N = 256;               // MMA N: queries x heads per unit
    static constexpr int QT = N / H;            // queries per unit
    static constexpr int QH = QT / 2;           // queries per epilogue half
    static constexpr int BM = 128;              // keys per tile (MMA M)
    static constexpr int KCH = D / 64;          // 128-byte K chunks
    static constexpr int STAGES = (D == 64) ? 4 : 3;
    static constexpr uint32_t Q_CHUNK = N * 128u;
    static constexpr uint32_t KC_CHUNK = BM * 128u;
    static constexpr uint32_t Q_BYTES = KCH * Q_CHUNK;
    static constexpr uint32_t KC_BYTES = KCH * KC_CHUNK;
    static constexpr uint32_t W_BYTES = QT * H * 4u;
    static constexpr int EPI_WARPS = 8;
    static constexpr int THREADS = 64 + 32 * EPI_WARPS;
    static constexpr uint32_t TMEM_COLS = 512;  // two 256-column accumulators
    // shared memory map, relative to a 1024-byte aligned base
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_KC = OFF_Q + Q_BYTES;
    static constexpr uint32_t OFF_W = OFF_KC + STAGES * KC_BYTES;
    static constexpr uint32_t OFF_HIST = OFF_W + 2 * W_BYTES;
    static constexpr uint32_t OFF_CTRL = OFF_HIST + EPI_WARPS * 256 * 4;
    static constexpr uint32_t CTRL_BYTES = 1024;
    static constexpr uint32_t OFF_POOL = OFF_CTRL + CTRL_BYTES;
    static constexpr uint32_t ALIGN_SLACK = 1024;
    static constexpr uint32_t smem_bytes(bool pool_in_smem, int P) {
        return OFF_POOL + (pool_in_smem ? static_cast<uint32_t>(QT) * P * 8u : 0u) + ALIGN_SLACK;
    }
};

// Control block (inside OFF_CTRL): mbarriers then scalars.
enum : int {
    kBarKcFull = 0,    // [4]
    kBarKcEmpty = 4,   // [4]
    kBarQFull = 8,
    kBarQEmpty = 9,
    kBarWFull = 10,    // [2]
    kBarWEmpty = 12,   // [2]
    kBarAccFull = 14,  // [2]
    kBarAccEmpty = 16, // [2]
    kBarDrain = 18,
    kNumBars = 19
};
constexpr uint32_t kCtrlTmemSlot = 256;
constexpr uint32_t kCtrlAbort = 260;
constexpr uint32_t kCtrlCount = 320;   // u32 [<=32]
constexpr uint32_t kCtrlTheta = 512;   // u64 [<=32]

struct UnitInfo {
    int64_t b, t0;
    int ntiles;
};

// Units are ordered longest first: unit u is query block nblk-1-u/B of batch u%B.
__device__ __forceinline__ UnitInfo decode_unit(int64_t u, const SelectParams& p, int QT) {
    UnitInfo ui;
    const int64_t blk = p.nblk - 1 - u / p.B;
    ui.b = u % p.B;
    ui.t0 = blk * QT;
    const int64_t tend = (ui.t0 + QT < p.S) ? ui.t0 + QT : p.S;
    int64_t vmax = tend / p.m;  // keys visible to query tend-1
    if (vmax > p.T) vmax = p.T;
    ui.ntiles = static_cast<int>((vmax + 127) / 128);
    return ui;
}

// Zig-zag static schedule: round r gives CTA c unit r*G+c (r even) or
// r*G+G-1-c (r odd), which balances the longest-first cost ramp.
__device__ __forceinline__ int64_t unit_of_round(int64_t r, int64_t G, int64_t c) {
    return r * G + ((r & 1) ? (G - 1 - c) : c);
}

__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < limit_ns)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// ------------------------------------------------------------------ epilogue
// Scores of this thread's key for the QH queries of its half.  `taddr` points
// at the half's first column in this warp's lane quarter; `wq` at the half's
// w values [QH][H] in shared memory.
template <int H, int QH>
__device__ __forceinline__ void half_scores(uint32_t taddr, const float* wq, float (&sc)[QH]) {
#pragma unroll
    for (int q = 0; q < QH; ++q) sc[q] = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + c * 32, r);
        tmem_wait_ld(r);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int col = c * 32 + i;
            const int q = col / H;
            const int h = col % H;
            sc[q] = fmaf(wq[q * H + h], fmaxf(__uint_as_float(r[i]), 0.0f), sc[q]);
        }
    }
}

// k-th largest of the n (> k, distinct) keys of `pool`, by one warp.
// Radix select from the most significant bit in which the pool's keys differ,
// 8 bits per pass; stops as soon as the digit bucket holding the k-th key has
// a single member.
__device__ __noinline__ uint64_t warp_kth_largest(const uint64_t* pool, int n, int k, uint32_t* hist,
                                                  int lane) {
    uint64_t kmin = ~0ull, kmax = 0ull;
    for (int i = lane; i < n; i += 32) {
        const uint64_t x = pool[i];
        kmin = x < kmin ? x : kmin;
        kmax = x > kmax ? x : kmax;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t a = __shfl_xor_sync(0xffffffffu, kmin, o);
        const uint64_t b = __shfl_xor_sync(0xffffffffu, kmax, o);
        kmin = a < kmin ? a : kmin;
        kmax = b > kmax ? b : kmax;
    }
    const int hb = 63 - __clzll(static_cast<long long>(kmin ^ kmax));
    uint64_t dmask = (hb >= 63) ? 0ull : ~((2ull << hb) - 1ull);  // decided bits
    uint64_t prefix = kmin & dmask;
    int lo = hb + 1;  // bits >= lo are decided
    uint32_t need = static_cast<uint32_t>(k);
    uint32_t bucket = 0;
    while (true) {
        const int shift = lo > 8 ? lo - 8 : 0;
        const int width = lo - shift;
        const uint64_t dig_mask = (1ull << width) - 1ull;
        for (int i = lane; i < 256; i += 32) hist[i] = 0;
        __syncwarp();
        for (int i = lane; i < n; i += 32) {
            const uint64_t x = pool[i];
            if ((x & dmask) == prefix) atomicAdd(&hist[(x >> shift) & dig_mask], 1u);
        }
        __syncwarp();
        // Scan the 256 bins from the top: lane l owns bins 255-8l .. 248-8l.
        uint32_t c[8];
        uint32_t sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            c[j] = hist[255 - lane * 8 - j];
            sum += c[j];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const uint32_t excl = incl - sum;
        const bool mine = excl < need && need <= incl;
        const uint32_t bal = __ballot_sync(0xffffffffu, mine);
        const int src = __ffs(bal) - 1;
        uint32_t digit = 0, above = 0, cnt = 0;
        if (lane == src) {
            uint32_t cum = excl;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (cnt == 0 && cum + c[j] >= need) {
                    digit = 255u - lane * 8u - j;
                    above = cum;
                    cnt = c[j];
                }
                cum += c[j];
            }
        }
        digit = __shfl_sync(0xffffffffu, digit, src);
        above = __shfl_sync(0xffffffffu, above, src);
        cnt = __shfl_sync(0xffffffffu, cnt, src);
        __syncwarp();
        need -= above;
        prefix |= static_cast<uint64_t>(digit) << shift;
        dmask |= dig_mask << shift;
        lo = shift;
        bucket = cnt;
        if (bucket == 1 || lo == 0) break;
    }
    if (lo == 0) return prefix;
    uint64_t found = 0;
    for (int i = lane; i < n; i += 32) {
        const uint64_t x = pool[i];
        if ((x & dmask) == prefix) found = x;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t v = __shfl_xor_sync(0xffffffffu, found, o);
        found = v > found ? v : found;
    }
    return found;
}

// Keep the pool entries >= kth (exactly k of them), in place, by one warp.
__device__ __forceinline__ void warp_keep_at_least(uint64_t* pool, int n, uint64_t kth, int lane) {
    uint32_t out = 0;
    for (int base = 0; base < n; base += 32) {
        const int i = base + lane;
        const uint64_t x = i < n ? pool[i] : 0ull;
        const bool keep = i < n && x >= kth;
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        __syncwarp();
        if (keep) pool[out + __popc(bal & lanemask_lt())] = x;
        out += __popc(bal);
        __syncwarp();
    }
}

// ------------------------------------------------------------------ kernel
template <int H, int D>
__global__ void __launch_bounds__(SelCfg<H, D>::THREADS, 1)
    select_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                  const __grid_constant__ CUtensorMap tm_w, const SelectParams p) {
    using C = SelCfg<H, D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    uint8_t* ctrl = smem + C::OFF_CTRL;
    const uint32_t bar0 = sbase + C::OFF_CTRL;
    auto bar = [bar0](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl + kCtrlTmemSlot);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl + kCtrlAbort);
    uint32_t* cnt = reinterpret_cast<uint32_t*>(ctrl + kCtrlCount);
    uint64_t* theta = reinterpret_cast<uint64_t*>(ctrl + kCtrlTheta);
    const int P = p.P;
    uint64_t* pool = p.gpool ? p.gpool + static_cast<size_t>(blockIdx.x) * C::QT * P
                             : reinterpret_cast<uint64_t*>(smem + C::OFF_POOL);
    const uint64_t lim = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(bar(kBarKcFull + s), 1);
            mbar_init(bar(kBarKcEmpty + s), 1);
        }
        mbar_init(bar(kBarQFull), 1);
        mbar_init(bar(kBarQEmpty), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(kBarWFull + i), 1);
            mbar_init(bar(kBarWEmpty + i), C::EPI_WARPS);
            mbar_init(bar(kBarAccFull + i), 1);
            mbar_init(bar(kBarAccEmpty + i), C::EPI_WARPS);
        }
        mbar_init(bar(kBarDrain), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_kc);
        prefetch_tmap(&tm_w);
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int64_t G = gridDim.x;
    const int64_t cta = blockIdx.x;
    const int64_t U = p.units;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t kc_it = 0, q_it = 0, w_it = 0;
            bool ok = true;
            for (int64_t r = 0; ok && r * G < U; ++r) {
                const int64_t u = unit_of_round(r, G, cta);
                if (u >= U) continue;
                const UnitInfo ui = decode_unit(u, p, C::QT);
                if (ui.ntiles == 0) continue;
                const uint32_t ws = w_it & 1u;
                if (!(ok = mbar_wait(bar(kBarWEmpty + ws), ((w_it >> 1) & 1u) ^ 1u, abort_flag, p.err, lim)))
                    break;
                mbar_arrive_expect_tx(bar(kBarWFull + ws), C::W_BYTES);
                tma_load_3d(sbase + C::OFF_W + ws * C::W_BYTES, &tm_w, bar(kBarWFull + ws), 0,
                            static_cast<int>(ui.t0), static_cast<int>(ui.b));
                ++w_it;
                if (!(ok = mbar_wait(bar(kBarQEmpty), (q_it & 1u) ^ 1u, abort_flag, p.err, lim))) break;
                mbar_arrive_expect_tx(bar(kBarQFull), C::Q_BYTES);
#pragma unroll
                for (int c = 0; c < C::KCH; ++c)
                    tma_load_3d(sbase + C::OFF_Q + c * C::Q_CHUNK, &tm_q, bar(kBarQFull), c * 64,
                                static_cast<int>(ui.t0 * H), static_cast<int>(ui.b));
                ++q_it;
                for (int j = 0; j < ui.ntiles; ++j) {
                    const uint32_t st = kc_it % C::STAGES;
                    if (!(ok = mbar_wait(bar(kBarKcEmpty + st), ((kc_it / C::STAGES) & 1u) ^ 1u, abort_flag,
                                         p.err, lim)))
                        break;
                    mbar_arrive_expect_tx(bar(kBarKcFull + st), C::KC_BYTES);
#pragma unroll
                    for (int c = 0; c < C::KCH; ++c)
                        tma_load_3d(sbase + C::OFF_KC + st * C::KC_BYTES + c * C::KC_CHUNK, &tm_kc,
                                    bar(kBarKcFull + st), c * 64, j * C::BM, static_cast<int>(ui.b));
                    ++kc_it;
                }
            }
            if (!ok) {
                // Let every load already issued land before the CTA exits.
                const uint64_t drain = 100000000ull;
                const uint32_t n = kc_it < C::STAGES ? kc_it : C::STAGES;
                for (uint32_t i = kc_it - n; i < kc_it; ++i)
                    mbar_wait_bounded(bar(kBarKcFull + i % C::STAGES), (i / C::STAGES) & 1u, drain);
                if (q_it) mbar_wait_bounded(bar(kBarQFull), (q_it - 1) & 1u, drain);
                if (w_it) mbar_wait_bounded(bar(kBarWFull + ((w_it - 1) & 1u)), ((w_it - 1) >> 1) & 1u, drain);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(C::BM, C::N);
            uint32_t kc_it = 0, q_it = 0, acc_it = 0;
            bool ok = true, issued = false;
            for (int64_t r = 0; ok && r * G < U; ++r) {
                const int64_t u = unit_of_round(r, G, cta);
                if (u >= U) continue;
                const UnitInfo ui = decode_unit(u, p, C::QT);
                if (ui.ntiles == 0) continue;
                if (!(ok = mbar_wait(bar(kBarQFull), q_it & 1u, abort_flag, p.err, lim))) break;
                for (int j = 0; j < ui.ntiles; ++j) {
                    const uint32_t st = kc_it % C::STAGES;
                    if (!(ok = mbar_wait(bar(kBarKcFull + st), (kc_it / C::STAGES) & 1u, abort_flag, p.err, lim)))
                        break;
                    const uint32_t buf = acc_it & 1u;
                    if (!(ok = mbar_wait(bar(kBarAccEmpty + buf), ((acc_it >> 1) & 1u) ^ 1u, abort_flag, p.err,
                                         lim)))
                        break;
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + buf * C::N;
                    const uint32_t a_base = sbase + C::OFF_KC + st * C::KC_BYTES;
                    const uint32_t b_base = sbase + C::OFF_Q;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t c = kk / 4, off = (kk % 4) * 32;
                        umma_bf16(d_tmem, smem_desc_sw128(a_base + c * C::KC_CHUNK + off),
                                  smem_desc_sw128(b_base + c * C::Q_CHUNK + off), idesc, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(bar(kBarKcEmpty + st));
                    umma_commit(bar(kBarAccFull + buf));
                    issued = true;
                    ++kc_it;
                    ++acc_it;
                }
                if (!ok) break;
                umma_commit(bar(kBarQEmpty));
                ++q_it;
            }
            if (issued) {
                umma_commit(bar(kBarDrain));
                mbar_wait_bounded(bar(kBarDrain), 0, 100000000ull);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue
        const int e = warp - 2;
        const int quarter = warp & 3;
        const int half = e >> 2;
        const int wih = e & 3;
        const uint32_t bar_id = 1u + static_cast<uint32_t>(half);
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        uint32_t* hist = reinterpret_cast<uint32_t*>(smem + C::OFF_HIST) + e * 256;
        const bool dense = p.dense != nullptr;
        const int k = p.k;
        const uint32_t trigger = static_cast<uint32_t>(P - C::BM);
        uint32_t acc_it = 0, w_it = 0;
        bool bad = false;
        for (int64_t r = 0; r * G < U; ++r) {
            const int64_t u = unit_of_round(r, G, cta);
            if (u >= U) continue;
            const UnitInfo ui = decode_unit(u, p, C::QT);
            if (wih == 0 && lane < C::QH) {
                cnt[half * C::QH + lane] = 0;
                theta[half * C::QH + lane] = 0ull;
            }
            int32_t vis[C::QH];  // visible keys of each query of the half (0 past S)
#pragma unroll
            for (int q = 0; q < C::QH; ++q) {
                const int64_t t = ui.t0 + half * C::QH + q;
                int64_t v = (t < p.S) ? (t + 1) / p.m : 0;
                vis[q] = static_cast<int32_t>(v < p.T ? v : p.T);
            }
            bar_sync(bar_id, 128);
            uint32_t wslot = 0;
            bool wok = true;
            if (ui.ntiles > 0) {
                wslot = w_it & 1u;
                wok = mbar_wait(bar(kBarWFull + wslot), (w_it >> 1) & 1u, abort_flag, p.err, lim);
                wok = __all_sync(0xffffffffu, wok);
                ++w_it;
            }
            const float* wq =
                reinterpret_cast<const float*>(smem + C::OFF_W + wslot * C::W_BYTES) + half * C::QH * H;
            for (int j = 0; j < ui.ntiles; ++j) {
                const uint32_t buf = acc_it & 1u;
                bool ok = wok && mbar_wait(bar(kBarAccFull + buf), (acc_it >> 1) & 1u, abort_flag, p.err, lim);
                ok = __all_sync(0xffffffffu, ok);  // warp-uniform; also reconverges before tcgen05.ld
                ++acc_it;
                tc_fence_after();
                float sc[C::QH];
                half_scores<H, C::QH>(tmem_base + buf * C::N + half * 128 + lane_off, wq, sc);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarAccEmpty + buf));
                const int32_t s = j * C::BM + quarter * 32 + lane;
                if (ok) {
                    if (dense) {
#pragma unroll
                        for (int q = 0; q < C::QH; ++q) {
                            if (s < vis[q]) {
                                const int64_t t = ui.t0 + half * C::QH + q;
                                p.dense[(ui.b * p.S + t) * p.T + s] = canonical_score(sc[q]);
                            }
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < C::QH; ++q) {
                            const int qi = half * C::QH + q;
                            const uint64_t key = pack_key(sc[q], static_cast<uint32_t>(s));
                            const bool pass = s < vis[q] && key > theta[qi];
                            const uint32_t bal = __ballot_sync(0xffffffffu, pass);
                            if (bal) {
                                const int leader = __ffs(bal) - 1;
                                uint32_t base = 0;
                                if (lane == leader) base = atomicAdd(&cnt[qi], static_cast<uint32_t>(__popc(bal)));
                                base = __shfl_sync(0xffffffffu, base, leader);
                                if (pass) pool[qi * P + base + __popc(bal & lanemask_lt())] = key;
                            }
                        }
                    }
                }
                if (bar_red_or(bar_id, 128, !ok || *abort_flag)) {
                    bad = true;
                    break;
                }
                if (!dense) {
                    bool need = false;
#pragma unroll
                    for (int q = 0; q < C::QH; ++q) need |= cnt[half * C::QH + q] > trigger;
                    if (bar_red_or(bar_id, 128, need)) {
                        for (int q = wih; q < C::QH; q += 4) {
                            const int qi = half * C::QH + q;
                            const uint32_t n = cnt[qi];
                            if (n > trigger) {
                                uint64_t* pq = pool + qi * P;
                                const uint64_t kth = warp_kth_largest(pq, n, k, hist, lane);
                                warp_keep_at_least(pq, n, kth, lane);
                                if (lane == 0) {
                                    cnt[qi] = static_cast<uint32_t>(k);
                                    theta[qi] = kth;
                                }
                            }
                        }
                        bar_sync(bar_id, 128);
                    }
                }
            }
            if (bad) break;
            if (ui.ntiles > 0) {
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarWEmpty + wslot));
            }
            if (!dense) {
                for (int q = wih; q < C::QH; q += 4) {
                    const int qi = half * C::QH + q;
                    const int64_t t = ui.t0 + qi;
                    if (t >= p.S) continue;
                    uint64_t* pq = pool + qi * P;
                    uint32_t n = cnt[qi];
                    if (n > static_cast<uint32_t>(k)) {
                        const uint64_t kth = warp_kth_largest(pq, n, k, hist, lane);
                        warp_keep_at_least(pq, n, kth, lane);
                        n = static_cast<uint32_t>(k);
                    }
                    const int64_t row = (ui.b * p.S + t) * static_cast<int64_t>(k);
                    for (int i = lane; i < k; i += 32) {
                        int32_t oi = -1;
                        float os = -__int_as_float(0x7f800000);
                        if (i < static_cast<int>(n)) {
                            const uint64_t x = pq[i];
                            oi = key_index(x);
                            os = key_score(x);
                        }
                        p.out_idx[row + i] = oi;
                        p.out_score[row + i] = os;
                    }
                }
            }
            bar_sync(bar_id, 128);
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace si
