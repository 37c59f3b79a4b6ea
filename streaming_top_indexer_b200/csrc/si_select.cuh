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

// Optional cycle tracing (build flag SI_TRACE; off in the product library).
// Every thread accumulates cycle counts in registers; lane 0 of each warp
// writes them to SelectParams::trace[(cta * 10 + warp) * kTraceSlots + slot].
constexpr int kTraceSlots = 16;
constexpr int kTraceWarps = 10;
enum : int {
    kTrMmaKcFull = 0, kTrMmaAccEmpty, kTrMmaQFull, kTrProdKcEmpty, kTrProdQEmpty, kTrEpiAccFull,
    kTrEpiScores, kTrEpiArrive, kTrEpiFilter, kTrEpiBarrier, kTrEpiCompact, kTrCompactions, kTrTiles,
    kTrTotal, kTrEpiWFull, kTrEpiFinal
};
#ifdef SI_TRACE
__device__ __forceinline__ long long tr_clock() {
    long long c;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(c)::"memory");
    return c;
}
#define SI_TR_DECL unsigned long long tr_acc[kTraceSlots] = {}
#define SI_TR_T0(v) const long long v = tr_clock()
#define SI_TR_ADD(slot, v, cond) (tr_acc[slot] += static_cast<unsigned long long>(tr_clock() - (v)))
#define SI_TR_INC(slot, cond) (tr_acc[slot] += (cond) ? 1ull : 0ull)
#define SI_TR_DEPF(x) asm volatile("" ::"f"(x))
#define SI_TR_DEPI(x) asm volatile("" ::"r"(x))
#else
#define SI_TR_DECL (void)0
#define SI_TR_T0(v) (void)0
#define SI_TR_ADD(slot, v, cond) (void)0
#define SI_TR_INC(slot, cond) (void)0
#define SI_TR_DEPF(x) (void)0
#define SI_TR_DEPI(x) (void)0
#endif

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
    unsigned long long* trace;  // SI_TRACE builds only: [grid][kTraceWarps][kTraceSlots]
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
    // dynamic shared memory map, relative to a 1024-byte aligned base
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_KC = OFF_Q + Q_BYTES;
    static constexpr uint32_t OFF_W = OFF_KC + STAGES * KC_BYTES;
    static constexpr uint32_t OFF_POOL = OFF_W + 2 * W_BYTES;
    static constexpr uint32_t ALIGN_SLACK = 1024;
    // static shared memory: barriers, counters, thresholds, histograms
    static constexpr uint32_t STATIC_BYTES = 10240;  // >= actual static use
    static constexpr uint32_t dyn_bytes(bool pool_in_smem, int P) {
        return OFF_POOL + (pool_in_smem ? static_cast<uint32_t>(QT) * P * 8u : 0u) + ALIGN_SLACK;
    }
    static constexpr uint32_t smem_bytes(bool pool_in_smem, int P) {
        return dyn_bytes(pool_in_smem, P) + STATIC_BYTES;
    }
    // Epilogue accumulators: NP float2 partial sums per query, so that every
    // dependent FMA chain is at most 8 long (4 for H_I=8).
    static constexpr int NP = (8 / QH) < 1 ? 1 : ((8 / QH) > 4 ? 4 : 8 / QH);
};

// Extra entries an intermediate pool cut may keep above k (the cut at the end
// of a unit is exact).
constexpr uint32_t kCompactSlack = 256;

// Mbarrier slots.
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
// Accumulates 32 TMEM columns (chunk c of the half) into the partial sums.
// Column j of the half is head (j % H) of query (j / H); consecutive heads
// are paired into one packed f32x2 FMA, pair p of a query goes to partial
// sum p % NP.
template <int H, int QH, int NP>
__device__ __forceinline__ void accumulate_chunk(const uint32_t (&r)[32], int c, const float* wq,
                                                 float2 (&acc)[QH][NP]) {
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
        const int col = c * 32 + i;
        const int q = col / H;
        const int h = col % H;
        const float4 w4 = *reinterpret_cast<const float4*>(wq + q * H + h);
        const float2 x01 = make_float2(fmaxf(__uint_as_float(r[i]), 0.0f), fmaxf(__uint_as_float(r[i + 1]), 0.0f));
        const float2 x23 = make_float2(fmaxf(__uint_as_float(r[i + 2]), 0.0f), fmaxf(__uint_as_float(r[i + 3]), 0.0f));
        const int p0 = (h / 2) % NP, p1 = (h / 2 + 1) % NP;
        acc[q][p0] = __ffma2_rn(make_float2(w4.x, w4.y), x01, acc[q][p0]);
        acc[q][p1] = __ffma2_rn(make_float2(w4.z, w4.w), x23, acc[q][p1]);
    }
}

// Scores of this thread's key for the QH queries of its half:
// score = sum_h w[h] * max(acc[h], 0), summed in a fixed order (partial sums
// by head pair, then a fixed tree), so equal inputs give equal scores
// whatever the key's position in the tile.  `taddr` points at the half's
// first column in this warp's lane quarter; `wq` at the half's w [QH][H].
// TMEM loads are software-pipelined two chunks deep.
template <int H, int QH, int NP>
__device__ __forceinline__ void half_scores(uint32_t taddr, const float* wq, float (&sc)[QH]) {
    float2 acc[QH][NP];
#pragma unroll
    for (int q = 0; q < QH; ++q)
#pragma unroll
        for (int a = 0; a < NP; ++a) acc[q][a] = make_float2(0.0f, 0.0f);
    uint32_t ra[32], rb[32];
    tmem_ld32(taddr, ra);
    tmem_wait_ld(ra);
    tmem_ld32(taddr + 32, rb);
    accumulate_chunk<H, QH, NP>(ra, 0, wq, acc);
    tmem_wait_ld(rb);
    tmem_ld32(taddr + 64, ra);
    accumulate_chunk<H, QH, NP>(rb, 1, wq, acc);
    tmem_wait_ld(ra);
    tmem_ld32(taddr + 96, rb);
    accumulate_chunk<H, QH, NP>(ra, 2, wq, acc);
    tmem_wait_ld(rb);
    accumulate_chunk<H, QH, NP>(rb, 3, wq, acc);
#pragma unroll
    for (int q = 0; q < QH; ++q) {
        float part[NP];
#pragma unroll
        for (int a = 0; a < NP; ++a) part[a] = acc[q][a].x + acc[q][a].y;
#pragma unroll
        for (int w = 1; w < NP; w *= 2)
#pragma unroll
            for (int a = 0; a + w < NP; a += 2 * w) part[a] = part[a] + part[a + w];
        sc[q] = part[0];
    }
}

// A query's pool is a list of up to five address-ordered regions: the
// survivors of the last cut, [0, kept), then one append sub-range per
// epilogue warp of the half, [kept + w*F, kept + w*F + count_w).
struct PoolRegions {
    int start[5];
    int len[5];
    __device__ __forceinline__ int total() const { return len[0] + len[1] + len[2] + len[3] + len[4]; }
};

// Calls f(x) for every key of the regions that thread `tid` of the half owns
// (virtual positions tid, tid+128, ...), four loads in flight at a time.
template <typename F>
__device__ __forceinline__ void half_for_each(const uint64_t* pool, const PoolRegions& rg, int tid, F f) {
#pragma unroll 1
    for (int r = 0; r < 5; ++r) {
        const uint64_t* base = pool + rg.start[r];
        const int len = rg.len[r];
        int i = tid;
        for (; i + 384 < len; i += 512) {
            const uint64_t x0 = base[i], x1 = base[i + 128], x2 = base[i + 256], x3 = base[i + 384];
            f(x0);
            f(x1);
            f(x2);
            f(x3);
        }
        for (; i < len; i += 128) f(base[i]);
    }
}

// Lower bound L of the k best of the n (> k, distinct) keys in the regions,
// computed by the 128 threads of one epilogue half (tid 0..127, named
// barrier bar_id): at least k and at most k + slack keys are >= L (exactly k
// when slack == 0).  Radix select from the most significant bit in which the
// keys differ, 8 bits per pass; each warp fills its own 256-bin histogram
// (hist[4][256]) and every warp scans the sum itself, so all threads reach
// the same decision without a broadcast.  It stops at the first pass whose
// bucket holding the k-th key leaves at most `slack` extra keys above L.
__device__ __forceinline__ uint64_t half_select_bound(const uint64_t* pool, const PoolRegions& rg, int k,
                                                      uint32_t slack, uint32_t (*hist)[256],
                                                      unsigned long long* xch, int tid, uint32_t bar_id) {
    const int lane = tid & 31, wq = tid >> 5;
    uint32_t* my_hist = hist[wq];
    uint64_t kmin = ~0ull, kmax = 0ull;
    half_for_each(pool, rg, tid, [&](uint64_t x) {
        kmin = x < kmin ? x : kmin;
        kmax = x > kmax ? x : kmax;
    });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t a = __shfl_xor_sync(0xffffffffu, kmin, o);
        const uint64_t b = __shfl_xor_sync(0xffffffffu, kmax, o);
        kmin = a < kmin ? a : kmin;
        kmax = b > kmax ? b : kmax;
    }
    if (lane == 0) {
        xch[wq] = kmin;
        xch[4 + wq] = kmax;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) my_hist[lane + 32 * j] = 0;
    bar_sync(bar_id, 128);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        kmin = xch[w] < kmin ? xch[w] : kmin;
        kmax = xch[4 + w] > kmax ? xch[4 + w] : kmax;
    }
    const int hb = 63 - __clzll(static_cast<long long>(kmin ^ kmax));
    uint64_t dmask = (hb >= 63) ? 0ull : ~((2ull << hb) - 1ull);  // decided bits
    uint64_t prefix = kmin & dmask;
    int lo = hb + 1;  // bits >= lo are decided
    uint32_t need = static_cast<uint32_t>(k);
    while (true) {
        const int shift = lo > 8 ? lo - 8 : 0;
        const int width = lo - shift;
        const uint64_t dig_mask = (1ull << width) - 1ull;
        half_for_each(pool, rg, tid, [&](uint64_t x) {
            if ((x & dmask) == prefix) atomicAdd(&my_hist[(x >> shift) & dig_mask], 1u);
        });
        bar_sync(bar_id, 128);
        // Scan the 256 bins from the top: lane l owns bins 255-8l .. 248-8l.
        uint32_t c[8];
        uint32_t sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int bin = 255 - lane * 8 - j;
            c[j] = hist[0][bin] + hist[1][bin] + hist[2][bin] + hist[3][bin];
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
        need -= above;  // keys still needed from the chosen bucket (1..cnt)
        prefix |= static_cast<uint64_t>(digit) << shift;
        dmask |= dig_mask << shift;
        lo = shift;
        // every thread has read the histograms before anyone clears them again
        bar_sync(bar_id, 128);
        if (cnt - need <= slack || lo == 0) break;
#pragma unroll
        for (int j = 0; j < 8; ++j) my_hist[lane + 32 * j] = 0;
        __syncwarp();
    }
    return prefix;  // decided bits of the bucket, zeros below: its lowest key
}

// Walks the region entries >= L in address order, 512 at a time (four per
// thread), and hands each kept entry with its output position to `emit`; the
// 128 threads of the half cooperate (per-warp counts exchanged through
// rcnt[2][4], double-buffered by round parity).  Returns the number kept.
template <typename Emit>
__device__ __forceinline__ uint32_t half_walk_kept(const uint64_t* pool, const PoolRegions& rg, uint64_t L,
                                                   uint32_t* rcnt, int tid, uint32_t bar_id, Emit emit) {
    const int lane = tid & 31, wq = tid >> 5;
    const uint32_t lt = lanemask_lt();
    uint32_t out = 0, round = 0;
#pragma unroll 1
    for (int r = 0; r < 5; ++r) {
        const uint64_t* base = pool + rg.start[r];
        const int len = rg.len[r];
        for (int b0 = 0; b0 < len; b0 += 512) {
            // this warp's 128 consecutive entries: four groups of 32
            uint64_t x[4];
            uint32_t bal[4];
            uint32_t mine = 0;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const int i = b0 + wq * 128 + g * 32 + lane;
                const bool in = i < len;
                x[g] = in ? base[i] : 0ull;
                bal[g] = __ballot_sync(0xffffffffu, in && x[g] >= L);
                mine += static_cast<uint32_t>(__popc(bal[g]));
            }
            uint32_t* rc = rcnt + (round & 1u) * 4u;
            if (lane == 0) rc[wq] = mine;
            bar_sync(bar_id, 128);
            uint32_t pos = out, total = 0;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const uint32_t cw = rc[w];
                pos += (w < wq) ? cw : 0u;
                total += cw;
            }
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                if ((bal[g] >> lane) & 1u) emit(x[g], pos + static_cast<uint32_t>(__popc(bal[g] & lt)));
                pos += static_cast<uint32_t>(__popc(bal[g]));
            }
            out += total;
            ++round;
        }
    }
    return out;
}

// Regions of query slot `qi` from the published survivor count and the four
// warps' append counts.
__device__ __forceinline__ PoolRegions pool_regions(uint32_t kept, uint32_t F, const uint32_t* cnt4) {
    PoolRegions rg;
    rg.start[0] = 0;
    rg.len[0] = static_cast<int>(kept);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        rg.start[w + 1] = static_cast<int>(kept + w * F);
        rg.len[w + 1] = static_cast<int>(cnt4[w]);
    }
    return rg;
}

// ------------------------------------------------------------------ kernel
template <int H, int D, bool SMEM_POOL>
__global__ void __launch_bounds__(SelCfg<H, D>::THREADS, 1)
    select_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                  const __grid_constant__ CUtensorMap tm_w, const SelectParams p) {
    using C = SelCfg<H, D>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[kNumBars];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag_s;
    // Pool bookkeeping published at cuts, [half][query of the half]: append
    // counts of the four warps, survivors of the cut and the lower bound.
    __shared__ uint32_t cntw[2][16][4];
    __shared__ uint32_t hist_s[2][4][256];          // per half and warp: radix histograms
    __shared__ unsigned long long xch_s[2][8];      // per half: min/max exchange
    __shared__ uint32_t rcnt_s[2][8];               // per half: warp counts of a walk round
    SI_TR_DECL;
    SI_TR_T0(t_kernel0);

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t bar0 = smem_u32(bars);
    auto bar = [bar0](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    volatile int* abort_flag = &abort_flag_s;
    const int P = p.P;
    uint64_t* pool = SMEM_POOL ? reinterpret_cast<uint64_t*>(smem + C::OFF_POOL)
                               : p.gpool + static_cast<size_t>(blockIdx.x) * C::QT * P;
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
        abort_flag_s = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_kc);
        prefetch_tmap(&tm_w);
    }
    if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;

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
                SI_TR_T0(tq0);
                ok = mbar_wait(bar(kBarQEmpty), (q_it & 1u) ^ 1u, abort_flag, p.err, lim);
                SI_TR_ADD(kTrProdQEmpty, tq0, true);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(kBarQFull), C::Q_BYTES);
#pragma unroll
                for (int c = 0; c < C::KCH; ++c)
                    tma_load_3d(sbase + C::OFF_Q + c * C::Q_CHUNK, &tm_q, bar(kBarQFull), c * 64,
                                static_cast<int>(ui.t0 * H), static_cast<int>(ui.b));
                ++q_it;
                for (int j = 0; j < ui.ntiles; ++j) {
                    const uint32_t st = kc_it % C::STAGES;
                    SI_TR_T0(tk0);
                    ok = mbar_wait(bar(kBarKcEmpty + st), ((kc_it / C::STAGES) & 1u) ^ 1u, abort_flag, p.err, lim);
                    SI_TR_ADD(kTrProdKcEmpty, tk0, true);
                    if (!ok) break;
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
                SI_TR_T0(tq0);
                ok = mbar_wait(bar(kBarQFull), q_it & 1u, abort_flag, p.err, lim);
                SI_TR_ADD(kTrMmaQFull, tq0, true);
                if (!ok) break;
                for (int j = 0; j < ui.ntiles; ++j) {
                    const uint32_t st = kc_it % C::STAGES;
                    SI_TR_T0(tk0);
                    ok = mbar_wait(bar(kBarKcFull + st), (kc_it / C::STAGES) & 1u, abort_flag, p.err, lim);
                    SI_TR_ADD(kTrMmaKcFull, tk0, true);
                    if (!ok) break;
                    const uint32_t buf = acc_it & 1u;
                    SI_TR_T0(ta0);
                    ok = mbar_wait(bar(kBarAccEmpty + buf), ((acc_it >> 1) & 1u) ^ 1u, abort_flag, p.err, lim);
                    SI_TR_ADD(kTrMmaAccEmpty, ta0, true);
                    if (!ok) break;
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
        const int htid = wih * 32 + lane;  // thread index within the half
        uint32_t(*hist)[256] = hist_s[half];
        unsigned long long* xch = xch_s[half];
        uint32_t* rcnt = rcnt_s[half];
        const bool dense = p.dense != nullptr;
        const int k = p.k;
        const uint32_t Pu = static_cast<uint32_t>(P);
        // An intermediate cut keeps at most k + cut_slack entries, which leaves
        // every warp's sub-range at least 33 free slots (P >= k + 256).
        const uint32_t cut_slack =
            Pu > static_cast<uint32_t>(k) + 132u + kCompactSlack ? kCompactSlack : Pu - static_cast<uint32_t>(k) - 132u;
        uint32_t acc_it = 0, w_it = 0;
        bool bad = false;
        for (int64_t r = 0; r * G < U; ++r) {
            const int64_t u = unit_of_round(r, G, cta);
            if (u >= U) continue;
            const UnitInfo ui = decode_unit(u, p, C::QT);
            // Pool state of each query of the half, identical in the four warps
            // except the append sub-range: survivors [0, kp), this warp's
            // sub-range [bw, bw + fw) holding cw appended keys, lower bound lb.
            uint64_t lb[C::QH];
            uint32_t kp[C::QH], cw[C::QH];
            // free room after the survivors, split four ways: this warp's sub-range
            auto fw = [&](int q) { return (Pu - kp[q]) / 4u; };
            auto bw = [&](int q) { return kp[q] + wih * fw(q); };
            int32_t vis[C::QH];  // visible keys of each query of the half (0 past S)
#pragma unroll
            for (int q = 0; q < C::QH; ++q) {
                lb[q] = 0ull;
                kp[q] = 0u;
                cw[q] = 0u;
                const int64_t t = ui.t0 + half * C::QH + q;
                int64_t v = (t < p.S) ? (t + 1) / p.m : 0;
                vis[q] = static_cast<int32_t>(v < p.T ? v : p.T);
            }
            const bool tr_lead = true;
            (void)tr_lead;
            bar_sync(bar_id, 128);
            uint32_t wslot = 0;
            bool wok = true;
            if (ui.ntiles > 0) {
                wslot = w_it & 1u;
                SI_TR_T0(tw0);
                wok = mbar_wait(bar(kBarWFull + wslot), (w_it >> 1) & 1u, abort_flag, p.err, lim);
                wok = __all_sync(0xffffffffu, wok);
                SI_TR_ADD(kTrEpiWFull, tw0, tr_lead);
                ++w_it;
            }
            const float* wq =
                reinterpret_cast<const float*>(smem + C::OFF_W + wslot * C::W_BYTES) + half * C::QH * H;
            for (int j = 0; j < ui.ntiles; ++j) {
                const uint32_t buf = acc_it & 1u;
                SI_TR_T0(tf0);
                bool ok = wok && mbar_wait(bar(kBarAccFull + buf), (acc_it >> 1) & 1u, abort_flag, p.err, lim);
                ok = __all_sync(0xffffffffu, ok);  // warp-uniform; also reconverges before tcgen05.ld
                SI_TR_ADD(kTrEpiAccFull, tf0, tr_lead);
                SI_TR_INC(kTrTiles, tr_lead);
                ++acc_it;
                tc_fence_after();
                SI_TR_T0(ts0);
                float sc[C::QH];
                half_scores<H, C::QH, C::NP>(tmem_base + buf * C::N + half * 128 + lane_off, wq, sc);
#pragma unroll
                for (int q = 0; q < C::QH; ++q) SI_TR_DEPF(sc[q]);
                SI_TR_ADD(kTrEpiScores, ts0, tr_lead);
                SI_TR_T0(tar0);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarAccEmpty + buf));
                SI_TR_ADD(kTrEpiArrive, tar0, tr_lead);
                SI_TR_T0(tfl0);
                const int32_t s = j * C::BM + quarter * 32 + lane;
                bool need = false;
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
                        // Append to this warp's own sub-range: no atomics, no
                        // shuffles; at most 32 keys per query and tile.
#pragma unroll
                        for (int q = 0; q < C::QH; ++q) {
                            const uint64_t key = pack_key(sc[q], static_cast<uint32_t>(s));
                            const bool pass = s < vis[q] && key >= lb[q];
                            const uint32_t bal = __ballot_sync(0xffffffffu, pass);
                            if (pass) pool[(half * C::QH + q) * P + bw(q) + cw[q] + __popc(bal & lanemask_lt())] = key;
                            cw[q] += static_cast<uint32_t>(__popc(bal));
                            need |= cw[q] + 32u > fw(q);
                        }
                    }
                }
                // One barrier per tile (abort and cut requests are OR-reduced);
                // two more only when some sub-range is nearly full or a wait failed.
                const bool bad_here = !ok || *abort_flag;
                SI_TR_DEPI(static_cast<int>(need));
                SI_TR_ADD(kTrEpiFilter, tfl0, tr_lead);
                SI_TR_T0(tb0);
                const bool any_flag = bar_red_or(bar_id, 128, bad_here || need);
                SI_TR_ADD(kTrEpiBarrier, tb0, tr_lead);
                if (any_flag) {
                    SI_TR_T0(tc0);
                    if (lane == 0)
#pragma unroll
                        for (int q = 0; q < C::QH; ++q) cntw[half][q][wih] = cw[q];
                    if (bar_red_or(bar_id, 128, bad_here)) {
                        bad = true;
                        break;
                    }
                    // Cut every pool with a nearly full sub-range, one query at a
                    // time, all 128 threads of the half together.
#pragma unroll
                    for (int q = 0; q < C::QH; ++q) {
                        const uint32_t* c4 = cntw[half][q];
                        const uint32_t f = fw(q);
                        const bool cut = c4[0] + 32u > f || c4[1] + 32u > f || c4[2] + 32u > f || c4[3] + 32u > f;
                        if (!cut) continue;  // uniform over the half
                        uint64_t* pq = pool + (half * C::QH + q) * P;
                        const PoolRegions rg = pool_regions(kp[q], f, c4);
                        uint64_t L = lb[q];
                        SI_TR_T0(tsel0);
                        if (rg.total() > k) L = half_select_bound(pq, rg, k, cut_slack, hist, xch, htid, bar_id);
                        SI_TR_ADD(0, tsel0, true);
                        SI_TR_T0(twk0);
                        const uint32_t kept = half_walk_kept(pq, rg, L, rcnt, htid, bar_id,
                                                             [&](uint64_t x, uint32_t pos) { pq[pos] = x; });
                        SI_TR_ADD(1, twk0, true);
#ifdef SI_TRACE
                        tr_acc[3] += static_cast<unsigned long long>(rg.total());
                        tr_acc[4] += kept;
#endif
                        SI_TR_INC(kTrCompactions, true);
                        kp[q] = kept;
                        lb[q] = L;
                        cw[q] = 0u;
                        bar_sync(bar_id, 128);
                    }
                    SI_TR_ADD(kTrEpiCompact, tc0, tr_lead);
                }
            }
            if (bad) break;
            if (ui.ntiles > 0) {
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarWEmpty + wslot));
            }
            SI_TR_T0(tfin0);
            if (!dense) {
                if (lane == 0)
#pragma unroll
                    for (int q = 0; q < C::QH; ++q) cntw[half][q][wih] = cw[q];
                bar_sync(bar_id, 128);
#pragma unroll
                for (int q = 0; q < C::QH; ++q) {
                    const int qi = half * C::QH + q;
                    const int64_t t = ui.t0 + qi;
                    if (t >= p.S) continue;  // uniform over the half
                    const uint64_t* pq = pool + qi * P;
                    const PoolRegions rg = pool_regions(kp[q], fw(q), cntw[half][q]);
                    const uint64_t L =
                        rg.total() > k ? half_select_bound(pq, rg, k, 0u, hist, xch, htid, bar_id) : 0ull;
                    const int64_t row = (ui.b * p.S + t) * static_cast<int64_t>(k);
                    // The k best (or all, when fewer), unordered, then padding.
                    const uint32_t out = half_walk_kept(pq, rg, L, rcnt, htid, bar_id, [&](uint64_t x, uint32_t pos) {
                        p.out_idx[row + pos] = key_index(x);
                        p.out_score[row + pos] = key_score(x);
                    });
                    for (int i = static_cast<int>(out) + htid; i < k; i += 128) {
                        p.out_idx[row + i] = -1;
                        p.out_score[row + i] = -__int_as_float(0x7f800000);
                    }
                    bar_sync(bar_id, 128);
                }
            }
            bar_sync(bar_id, 128);
            SI_TR_ADD(kTrEpiFinal, tfin0, tr_lead);
        }
    }

    __syncthreads();
#ifdef SI_TRACE
    SI_TR_ADD(kTrTotal, t_kernel0, true);
    if (lane == 0 && p.trace)
        for (int i = 0; i < kTraceSlots; ++i)
            p.trace[(static_cast<size_t>(blockIdx.x) * kTraceWarps + warp) * kTraceSlots + i] = tr_acc[i];
#endif
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace si
