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
// At the end of a unit the pool is cut to exactly its k best keys, which the
// half sorts in shared memory and registers and writes in their final order
// (a separate row sort remains for the few shapes whose sort does not fit).
#pragma once
#include <cuda.h>

#include <cstdint>

#include "si_keys.cuh"
#include "si_ptx.cuh"

namespace si {

// Optional cycle tracing (build flag SI_TRACE; off in the product library).
// Every thread accumulates cycle counts in registers; lane 0 of each warp
// writes them to SelectParams::trace[(cta * kTraceWarps + warp) * kTraceSlots + slot].
constexpr int kTraceSlots = 20;
constexpr int kTraceWarps = 12;  // warps per CTA (checked against SelCfg::THREADS)
enum : int {
    kTrMmaKcFull = 0, kTrMmaAccEmpty, kTrMmaQFull, kTrProdKcEmpty, kTrProdQEmpty, kTrEpiAccFull,
    kTrEpiScores, kTrEpiArrive, kTrEpiFilter, kTrEpiBarrier, kTrEpiCompact, kTrCompactions, kTrTiles,
    kTrTotal, kTrEpiWFull, kTrEpiFinal, kTrEpiAppend, kTrEpiUnit
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
    int P;              // pool capacity per query (multiple of 32, >= k + 288)
    int64_t t_lo, t_hi; // query rows [t_lo, t_hi) of every batch are computed
    int64_t nblk;       // query blocks per batch in [t_lo, t_hi)
    int64_t units;      // B * nblk
    int32_t* out_idx;   // [B,S,k]
    float* out_score;   // [B,S,k]
    float* dense;       // dense-score mode: [B,S,T] fp32, else nullptr
    uint64_t* gpool;    // pools in global memory (per CTA QT*P), or nullptr
    uint32_t* err;      // device error word
    int sort_e;         // > 0: rows are written sorted, 128 * sort_e >= k keys per row; 0: unordered
    uint32_t check_tiles;   // key tiles between two checks of the pools' fill (kCheckTiles by default)
    uint32_t cut_slack;     // most entries above k an intermediate cut keeps (kCompactSlack by default)
    uint64_t timeout_ns;
    unsigned long long* trace;  // SI_TRACE builds only: [grid][kTraceWarps][kTraceSlots]
};

template <int H, int D>
struct SelCfg {
    static_assert(H == 8 || H == 16 || H == 32 || H == 64, "H_I");
    static_assert(D == 64 || D == 128, "d_I");
    static constexpr int N = 256;               // MMA N: queries x heads per unit
    static constexpr int QT = N / H;            // queries per unit
    static constexpr int NGROUPS = 2;           // epilogue groups of four warps
    static constexpr int QH = QT / NGROUPS;     // queries per epilogue group
    static constexpr int CG = N / NGROUPS;      // TMEM columns per epilogue group
    static constexpr int BM = 128;              // keys per tile (MMA M)
    static constexpr int KCH = D / 64;          // 128-byte K chunks
    static constexpr int STAGES = (D == 64) ? 4 : 3;
    static constexpr uint32_t Q_CHUNK = N * 128u;
    static constexpr uint32_t KC_CHUNK = BM * 128u;
    static constexpr uint32_t Q_BYTES = KCH * Q_CHUNK;
    static constexpr uint32_t KC_BYTES = KCH * KC_CHUNK;
    static constexpr uint32_t W_BYTES = QT * H * 4u;
    static constexpr int EPI_WARPS = 4 * NGROUPS;
    static constexpr int EPI_WARP0 = 4;         // warps 0-3: TMA producer, MMA issuer, two idle
    static constexpr int THREADS = 32 * EPI_WARP0 + 32 * EPI_WARPS;
    // Registers: launched at 168 per thread; the control warpgroup then gives
    // up all but the minimum (24) so that each epilogue thread can hold its
    // 128 head weights and two TMEM chunks in flight (240).
    static constexpr uint32_t REGS_LAUNCH = 168, REGS_CTRL = 24, REGS_EPI = 240;
    static_assert(NGROUPS == 2, "register split assumes two epilogue warpgroups");
    static_assert(THREADS / 32 == kTraceWarps, "trace layout holds one slot row per warp");
    static_assert(REGS_CTRL * 128 + REGS_EPI * 32 * EPI_WARPS == REGS_LAUNCH * THREADS,
                  "the register split must add up to the launch allocation");
    static constexpr uint32_t TMEM_COLS = 512;  // two 256-column accumulators
    // dynamic shared memory map, relative to a 1024-byte aligned base
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_KC = OFF_Q + Q_BYTES;
    static constexpr uint32_t OFF_W = OFF_KC + STAGES * KC_BYTES;
    static constexpr uint32_t OFF_POOL = OFF_W + 2 * W_BYTES;
    static constexpr uint32_t ALIGN_SLACK = 1024;
    // static shared memory: barriers, counters, thresholds, histograms
    // Upper bound of the kernel's static shared memory (the host checks the
    // real figure at launch; pools in shared memory are sized with this).
    static constexpr uint32_t STATIC_BYTES = 6144;
    // With the pools in the workspace, each epilogue group gets a buffer of
    // STREAM_CAND keys in shared memory for the exact cut of its large pools.
    static constexpr int STREAM_CAND = 3072;
    static_assert(STREAM_CAND >= 2048, "final selections (k <= 2048) of workspace pools are packed into it");
    static constexpr uint32_t dyn_bytes(bool pool_in_smem, int P) {
        return OFF_POOL +
               (pool_in_smem ? static_cast<uint32_t>(QT) * P * 8u : static_cast<uint32_t>(NGROUPS * STREAM_CAND) * 8u) +
               ALIGN_SLACK;
    }
    static constexpr uint32_t smem_bytes(bool pool_in_smem, int P) {
        return dyn_bytes(pool_in_smem, P) + STATIC_BYTES;
    }
    // Epilogue accumulators: NP float2 partial sums per query (two at H_I=64,
    // one otherwise).  More partial sums shorten the dependent FMA chains but
    // cost registers that the epilogue, holding 128 head weights per thread,
    // does not have: measured, two beat four at H_I=64.
    static constexpr int NP = (4 / QH) < 1 ? 1 : ((4 / QH) > 2 ? 2 : 4 / QH);
};

// Defaults of two design parameters (SelectParams::cut_slack, check_tiles):
// extra entries an intermediate pool cut may keep above k (the cut at the end
// of a unit is exact), and key tiles between two checks of the pools' fill
// (each check is a named barrier over the epilogue half).
constexpr uint32_t kCompactSlack = 256;
constexpr uint32_t kCheckTiles = 2;

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

// Units are ordered longest first: unit u is query block nblk-1-u/B (of the
// rows [t_lo, t_hi)) of batch u%B.
__device__ __forceinline__ UnitInfo decode_unit(int64_t u, const SelectParams& p, int QT) {
    UnitInfo ui;
    const int64_t blk = p.nblk - 1 - u / p.B;
    ui.b = u % p.B;
    ui.t0 = p.t_lo + blk * QT;
    const int64_t tend = (ui.t0 + QT < p.t_hi) ? ui.t0 + QT : p.t_hi;
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
// sum p % NP.  The ReLU of a head pair is one packed add, x + |x| =
// 2*max(x, 0) (exact in binary floating point), so the partial sums hold
// twice the weighted sums and are halved at the end, also exact unless a
// partial sum is subnormal or beyond half the fp32 range: the scores equal
// sum_h w_h * max(x_h, 0) summed in the same order.  Measured against a mix
// of max() on the ALU pipe and scalar adds: equal or up to 2 % faster.
template <int H, int QH, int NP, int CG>
__device__ __forceinline__ void accumulate_chunk(const uint32_t (&r)[32], int c, const float (&wr)[CG],
                                                 float2 (&acc)[QH][NP]) {
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
        const int col = c * 32 + i;
        const int q = col / H;
        const int h = col % H;
        const float4 w4 = make_float4(wr[col], wr[col + 1], wr[col + 2], wr[col + 3]);
        const int p0 = (h / 2) % NP, p1 = (h / 2 + 1) % NP;
        const float a0 = __uint_as_float(r[i]), a1 = __uint_as_float(r[i + 1]);
        const float a2 = __uint_as_float(r[i + 2]), a3 = __uint_as_float(r[i + 3]);
        const float2 x01 = __fadd2_rn(make_float2(a0, a1), make_float2(fabsf(a0), fabsf(a1)));
        const float2 x23 = __fadd2_rn(make_float2(a2, a3), make_float2(fabsf(a2), fabsf(a3)));
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
template <int H, int QH, int NP, int NCH>
__device__ __forceinline__ void half_scores(uint32_t taddr, const float (&wr)[32 * NCH], float (&sc)[QH]) {
    float2 acc[QH][NP];
#pragma unroll
    for (int q = 0; q < QH; ++q)
#pragma unroll
        for (int a = 0; a < NP; ++a) acc[q][a] = make_float2(0.0f, 0.0f);
    uint32_t ra[32], rb[32];
    tmem_ld32(taddr, ra);
    tmem_wait_ld(ra);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        uint32_t(&cur)[32] = (c & 1) ? rb : ra;
        uint32_t(&nxt)[32] = (c & 1) ? ra : rb;
        if (c + 1 < NCH) tmem_ld32(taddr + (c + 1) * 32, nxt);
        accumulate_chunk<H, QH, NP, 32 * NCH>(cur, c, wr, acc);
        if (c + 1 < NCH) tmem_wait_ld(nxt);
    }
#pragma unroll
    for (int q = 0; q < QH; ++q) {
        float part[NP];
#pragma unroll
        for (int a = 0; a < NP; ++a) part[a] = (acc[q][a].x + acc[q][a].y) * 0.5f;  // undo x + |x| = 2 relu(x)
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

// The regions of a plain buffer of m keys (one region, [0, m)).
__device__ __forceinline__ PoolRegions single_region(int m) {
    PoolRegions one;
    one.start[0] = 0;
    one.len[0] = m;
#pragma unroll
    for (int r = 1; r < 5; ++r) {
        one.start[r] = m;
        one.len[r] = 0;
    }
    return one;
}

// Most keys an exact cut gathers between two adjacent samples.
constexpr int kCandCap = 256;

// Per-half scratch of a pool cut, in shared memory.
struct CutScratch {
    unsigned long long srt[32];  // 32 samples sorted descending; 0 (below any key) past the last
    union {
        unsigned long long cand[kCandCap];  // staged samples, then the keys of the bracket (exact cut)
        uint32_t hist[256];                 // radix fallback histogram
    };
    unsigned long long xch[8];   // cross-warp exchange
    uint32_t rcnt[2][4];         // per-warp counts, double-buffered by call parity
    uint32_t ncand;
};

// Calls f(x) for every key of the regions that thread `tid` of the half owns
// (virtual positions tid, tid+128, ...).
template <typename F>
__device__ __forceinline__ void half_for_each(const uint64_t* pool, const PoolRegions& rg, int tid, F f) {
#pragma unroll
    for (int r = 0; r < 5; ++r) {
        const uint64_t* base = pool + rg.start[r];
        const int len = rg.len[r];
#pragma unroll 2
        for (int i = tid; i < len; i += 128) f(base[i]);
    }
}

// Address of virtual position v of the address-ordered regions (v < total):
// region r holds positions [e_r, e_r + len_r) with e_r the sum of the
// earlier lengths, and the last region whose e_r <= v holds v (an empty
// region ends where it starts).  The e_r are the same for every v, so a run
// of calls shares them and each call is four independent compare-selects.
__device__ __forceinline__ int region_addr(const PoolRegions& rg, int v) {
    int a = rg.start[0] + v;
    int e = rg.len[0];
#pragma unroll
    for (int r = 1; r < 5; ++r) {
        a = v >= e ? rg.start[r] + (v - e) : a;
        e += rg.len[r];
    }
    return a;
}

// Exclusive prefix over the warp of per-lane counts below 32, and the warp's
// total: bit b of every lane's count is one ballot, so the five ballots and
// population counts are independent of one another.
__device__ __forceinline__ uint32_t warp_prefix_small(uint32_t v, int lane, uint32_t& total) {
    const uint32_t below = (1u << lane) - 1u;
    uint32_t pre = 0, tot = 0;
#pragma unroll
    for (int b = 0; b < 5; ++b) {
        const uint32_t m = __ballot_sync(0xffffffffu, (v >> b) & 1u);
        pre += static_cast<uint32_t>(__popc(m & below)) << b;
        tot += static_cast<uint32_t>(__popc(m)) << b;
    }
    total = tot;
    return pre;
}

// Sum over the 128 threads of the half, with one barrier; `phase` selects the
// exchange buffer and must advance identically in every thread.
__device__ __forceinline__ uint32_t half_sum(uint32_t c, CutScratch& cs, int tid, uint32_t bar_id, uint32_t& phase) {
    const int lane = tid & 31, wq = tid >> 5;
    c = __reduce_add_sync(0xffffffffu, c);
    uint32_t* rc = cs.rcnt[phase & 1u];
    ++phase;
    if (lane == 0) rc[wq] = c;
    bar_sync(bar_id, 128);
    return rc[0] + rc[1] + rc[2] + rc[3];
}

// Key sources of a cut: the pool read from memory on every pass, or the
// pool's keys held in registers (kRegKeys per thread, pools up to 2048).
struct StreamKeys {
    const uint64_t* pool;
    PoolRegions rg;
    // Eight loads in flight per thread: these pools live in global memory.
    template <typename F>
    __device__ __forceinline__ void for_each(int tid, F f) const {
#pragma unroll 1
        for (int r = 0; r < 5; ++r) {
            const uint64_t* base = pool + rg.start[r];
            const int len = rg.len[r];
            int i = tid;
            for (; i + 7 * 128 < len; i += 8 * 128) {
                uint64_t x[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) x[u] = base[i + u * 128];
#pragma unroll
                for (int u = 0; u < 8; ++u) f(x[u]);
            }
            for (; i < len; i += 128) f(base[i]);
        }
    }
};

constexpr int kRegKeys = 16;
static_assert(kRegKeys < 32, "walk prefix counts fit in five bits");

struct RegKeys {
    uint64_t x[kRegKeys];
    int n;
    __device__ __forceinline__ void load(const uint64_t* pool, const PoolRegions& rg, int tid) {
        n = rg.total();
#pragma unroll
        for (int j = 0; j < kRegKeys; ++j) {
            const int v = j * 128 + tid;
            x[j] = v < n ? pool[region_addr(rg, v)] : 0ull;
        }
    }
    template <typename F>
    __device__ __forceinline__ void for_each(int tid, F f) const {
#pragma unroll
        for (int j = 0; j < kRegKeys; ++j)
            if (j * 128 + tid < n) f(x[j]);
    }
};

// Number of keys >= L (every thread of the half gets it).
template <typename Keys>
__device__ __forceinline__ uint32_t half_count_ge(const Keys& keys, uint64_t L, CutScratch& cs, int tid,
                                                  uint32_t bar_id, uint32_t& phase) {
    uint32_t c = 0;
    keys.for_each(tid, [&](uint64_t x) { c += x >= L ? 1u : 0u; });
    return half_sum(c, cs, tid, bar_id, phase);
}

// Radix select (fallback): lower bound L with k <= #(keys >= L) <= k + slack,
// by the 128 threads of the half.  8 bits per pass from the most significant
// bit in which the keys differ, on a shared 256-bin histogram; every warp
// scans the histogram itself, so all threads reach the same decision.
static __device__ __noinline__ uint64_t half_radix_bound(const uint64_t* pool, const PoolRegions& rg, int k, uint32_t slack,
                                                  CutScratch& cs, int tid, uint32_t bar_id) {
    const int lane = tid & 31, wq = tid >> 5;
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
        cs.xch[wq] = kmin;
        cs.xch[4 + wq] = kmax;
    }
    cs.hist[tid] = 0;
    cs.hist[tid + 128] = 0;
    bar_sync(bar_id, 128);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        kmin = cs.xch[w] < kmin ? cs.xch[w] : kmin;
        kmax = cs.xch[4 + w] > kmax ? cs.xch[4 + w] : kmax;
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
            if ((x & dmask) == prefix) atomicAdd(&cs.hist[(x >> shift) & dig_mask], 1u);
        });
        bar_sync(bar_id, 128);
        uint32_t c[8];
        uint32_t sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            c[j] = cs.hist[255 - lane * 8 - j];
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
        bar_sync(bar_id, 128);  // every thread has read the histogram
        if (cnt - need <= slack || lo == 0) break;
        cs.hist[tid] = 0;
        cs.hist[tid + 128] = 0;
        bar_sync(bar_id, 128);
    }
    return prefix;  // decided bits of the bucket, zeros below: its lowest key
}

// Warp 0 draws min(n, 32) keys at evenly spaced virtual positions and places
// each at its rank among them (keys are distinct): cs.srt[0..ns) sorted
// descending, 0 past the last.  Also clears cs.ncand.  Ends with a barrier of
// the half; returns ns.
__device__ __forceinline__ int half_samples(const uint64_t* pool, const PoolRegions& rg, CutScratch& cs, int tid,
                                            uint32_t bar_id) {
    const int lane = tid & 31;
    const int n = rg.total();
    const int ns = n < 32 ? n : 32;
    if (tid < 32) {
        const uint64_t me = lane < ns ? pool[region_addr(rg, n >= 32 ? (lane * n) >> 5 : lane)] : 0ull;
        cs.cand[lane] = me;
        __syncwarp();
        int r = lane;
        if (lane < ns) {
            r = 0;
#pragma unroll 8
            for (int i = 0; i < 32; ++i) r += cs.cand[i] > me ? 1 : 0;
        }
        cs.srt[r] = me;
    }
    if (tid == 0) cs.ncand = 0;
    bar_sync(bar_id, 128);
    return ns;
}

// Lower bound L of the best keys in the regions, by the 128 threads of one
// epilogue half: k <= #(keys >= L) <= max_keep (max_keep == k: exactly the k
// best).  Needs n > k.
//  1. Warp 0 draws 32 evenly spaced keys and places each at its rank among
//     them (keys are distinct), which sorts them.
//  2. Counting passes (one barrier each) test samples near the rank that
//     predicts the target count, stepping one sample at a time, until a
//     sample qualifies or two adjacent samples bracket the k-th key.
//  3. Exact cut: the keys between the bracketing samples (about n/16 for the
//     bracket that holds a given rank) are gathered, and each is ranked
//     against the others by the whole half to pick the k-th.
//  4. With BIG (pools in the workspace), a bracket of more than kCandCap
//     keys is gathered into `big` (up to big_cap keys, shared memory) and
//     the same select picks the k-th key among them.  Any larger bracket
//     falls back to the radix select.
//  When a sample qualifies directly, `counts_out` (if given) gets the
//  per-warp counts of keys at or above it, which that counting pass left in
//  shared memory (they stay valid until the half's next exchange).
template <bool BIG = false, typename Keys>
__device__ __forceinline__ uint64_t half_select_bound(const Keys& keys, const uint64_t* pool, const PoolRegions& rg,
                                                      int k, uint32_t max_keep, CutScratch& cs, int tid,
                                                      uint32_t bar_id, uint32_t& phase, uint64_t* big = nullptr,
                                                      int big_cap = 0, const uint32_t** counts_out = nullptr) {
    const int n = rg.total();
    const int ns = half_samples(pool, rg, cs, tid, bar_id);
    // c(r) = #(keys >= srt[r]) grows with r; c(-1) = 0 (no bound), c(ns) = n (bound 0)
    const uint32_t ku = static_cast<uint32_t>(k);
    const uint32_t target = max_keep > ku ? (ku + max_keep) / 2u : ku;
    int r = static_cast<int>((static_cast<long long>(target) * ns + n - 1) / n) - 1;
    r = r < 0 ? 0 : (r > ns - 1 ? ns - 1 : r);
    int lo_r = -1, hi_r = ns;
    uint32_t c_lo = 0, c_hi = static_cast<uint32_t>(n);
    for (int it = 0; it < 8; ++it) {
        const uint32_t c = half_count_ge(keys, cs.srt[r], cs, tid, bar_id, phase);
        if (c >= ku && c <= max_keep) {
            if (counts_out) *counts_out = cs.rcnt[(phase - 1u) & 1u];  // the buffer half_sum just used
            return cs.srt[r];
        }
        if (c < ku) {
            lo_r = r;
            c_lo = c;
            ++r;
        } else {
            hi_r = r;
            c_hi = c;
            --r;
        }
        if (r <= lo_r || r >= hi_r) break;
    }
    const uint32_t m = c_hi - c_lo;  // keys in [lower, upper)
    const bool small = m <= static_cast<uint32_t>(kCandCap);
    bool use_big = false;
    if constexpr (BIG) use_big = !small && m <= static_cast<uint32_t>(big_cap);
    if (hi_r - lo_r != 1 || !(small || use_big)) {
        bar_sync(bar_id, 128);
        return half_radix_bound(pool, rg, k, max_keep - ku, cs, tid, bar_id);
    }
    const uint64_t upper = lo_r >= 0 ? cs.srt[lo_r] : ~0ull;
    const uint64_t lower = hi_r < ns ? cs.srt[hi_r] : 0ull;
    uint64_t* dst = use_big ? big : reinterpret_cast<uint64_t*>(cs.cand);
    keys.for_each(tid, [&](uint64_t x) {
        if (x >= lower && x < upper) dst[atomicAdd(&cs.ncand, 1u)] = x;
    });
    bar_sync(bar_id, 128);
    if constexpr (BIG) {
        if (use_big) {
            // The k-th key is the (k - c_lo)-th of the bracket (fewer than m,
            // since no sample qualified): the same select over the buffer.
            const PoolRegions one = single_region(static_cast<int>(m));
            const int kb = static_cast<int>(ku - c_lo);
            if (m <= 128u * kRegKeys) {
                RegKeys rk;
                rk.load(big, one, tid);
                return half_select_bound(rk, big, one, kb, static_cast<uint32_t>(kb), cs, tid, bar_id, phase);
            }
            const StreamKeys sk{big, one};
            return half_select_bound(sk, big, one, kb, static_cast<uint32_t>(kb), cs, tid, bar_id, phase);
        }
    }
    // The bracket's keys are distinct: the one with exactly `want` keys of the
    // bracket above it is the k-th key.
    const int want = static_cast<int>(ku - c_lo) - 1;  // 0-based rank inside the bracket
    const int mi = static_cast<int>(m);
    for (int c = tid; c < mi; c += 128) {
        const uint64_t x = cs.cand[c];
        int r = 0;
#pragma unroll 8
        for (int i = 0; i < mi; ++i) r += cs.cand[i] > x ? 1 : 0;
        if (r == want) cs.xch[0] = x;
    }
    bar_sync(bar_id, 128);
    return cs.xch[0];
}

// The exact k-th key of a large pool (workspace pools, which get a shared-
// memory buffer `big`) in one pass over the keys: after the samples, the keys
// above a window of samples around the predicted rank of the k-th key are
// counted and the keys inside the window gathered into `big` (sized to fill
// about half of it); when the k-th key falls inside, the sample select runs
// on the gathered keys.  Returns false, with nothing decided, when it does
// not or the window overflowed the buffer.  Needs n > k.
template <typename Keys>
__device__ __forceinline__ bool half_window_bound(const Keys& keys, const uint64_t* pool, const PoolRegions& rg, int k,
                                                  CutScratch& cs, int tid, uint32_t bar_id, uint32_t& phase,
                                                  uint64_t* big, int big_cap, uint64_t& L) {
    const int n = rg.total();
    const int ns = half_samples(pool, rg, cs, tid, bar_id);
    const uint32_t ku = static_cast<uint32_t>(k);
    // sample r has about (r + 1) * n / (ns + 1) keys at or above it
    const int per_gap = n / (ns + 1) + 1;
    int w = (big_cap / 2) / per_gap;  // sample gaps in the window
    w = w < 2 ? 2 : w;
    const int r0 = static_cast<int>((static_cast<long long>(ku) * (ns + 1) + n - 1) / n) - 1;
    int a = r0 - w / 2;  // window [srt[b], srt[a]); a = -1: no upper end
    a = a < -1 ? -1 : (a > ns - 1 ? ns - 1 : a);
    const int b = a + w > ns ? ns : a + w;  // b = ns: no lower end
    const uint64_t upper = a >= 0 ? cs.srt[a] : ~0ull;
    const uint64_t lower = b < ns ? cs.srt[b] : 0ull;
    const uint32_t cap = static_cast<uint32_t>(big_cap);
    uint32_t above = 0;
    keys.for_each(tid, [&](uint64_t x) {
        if (x >= upper) {
            ++above;
        } else if (x >= lower) {
            const uint32_t slot = atomicAdd(&cs.ncand, 1u);
            if (slot < cap) big[slot] = x;
        }
    });
    above = half_sum(above, cs, tid, bar_id, phase);  // its barrier also completes the gather
    const uint32_t m = cs.ncand;
    if (m > cap || above >= ku || above + m < ku) return false;  // uniform over the half
    const uint32_t kb = ku - above;  // the k-th key is the kb-th of the window
    if (kb == m) {
        L = lower;  // the window's smallest key (b < ns here, since n > k)
        return true;
    }
    const PoolRegions one = single_region(static_cast<int>(m));
    if (m <= 128u * kRegKeys) {
        RegKeys rk;
        rk.load(big, one, tid);
        L = half_select_bound(rk, big, one, static_cast<int>(kb), kb, cs, tid, bar_id, phase);
    } else {
        const StreamKeys sk{big, one};
        L = half_select_bound(sk, big, one, static_cast<int>(kb), kb, cs, tid, bar_id, phase);
    }
    return true;
}

// One pass over a large pool (workspace pools): every key at or above a bound
// is gathered into the shared-memory buffer `big`.  A pool of at most big_cap
// keys is gathered whole.  For a larger one the bound is the sample whose
// predicted count of keys at or above it is (k + big_cap) / 2, from 256
// samples at evenly spaced positions (two per thread, each ranked against
// all).  Returns true, with m keys in big[0, m), when k <= m <= big_cap:
// then big holds every key of the pool's k best, and an intermediate cut
// finishes in shared memory (one pass over the pool instead of two:
// measured, 38k -> 28k cycles for an 8K-key pool at k = 2048).  Returns false
// when the bound fell outside (the pool is only read, so the caller then
// takes the other path).  `lower_out` gets the bound (0 for a whole pool).
// Needs n > k and big_cap >= k.
template <typename Keys>
__device__ __forceinline__ bool half_gather_top(const Keys& keys, const uint64_t* pool, const PoolRegions& rg, int k,
                                                CutScratch& cs, int tid, uint32_t bar_id, uint64_t* big,
                                                int big_cap, uint32_t& m_out, uint64_t& lower_out) {
    static_assert(kCandCap == 256, "two samples per thread of the half");
    const int n = rg.total();
    uint64_t lower = 0ull;  // every key
    if (tid == 0) cs.ncand = 0;
    if (n > big_cap) {
        const uint64_t s0 = pool[region_addr(rg, static_cast<int>((static_cast<long long>(tid) * n) >> 8))];
        const uint64_t s1 = pool[region_addr(rg, static_cast<int>((static_cast<long long>(tid + 128) * n) >> 8))];
        cs.cand[tid] = s0;
        cs.cand[tid + 128] = s1;
        bar_sync(bar_id, 128);
        // sample at rank r (0 = largest) has about (r + 1) * n / 257 keys at or above it
        const long long target = (static_cast<long long>(k) + big_cap) / 2;
        int want = static_cast<int>((target * 257 + n / 2) / n) - 1;
        want = want < 0 ? 0 : (want > 255 ? 255 : want);
        int r0 = 0, r1 = 0;
#pragma unroll 8
        for (int i = 0; i < 256; ++i) {
            const uint64_t c = cs.cand[i];
            r0 += c > s0 ? 1 : 0;
            r1 += c > s1 ? 1 : 0;
        }
        // the samples are distinct keys (distinct positions), so one thread has rank `want`
        if (r0 == want) cs.xch[0] = s0;
        if (r1 == want) cs.xch[0] = s1;
        bar_sync(bar_id, 128);
        lower = cs.xch[0];
    } else {
        bar_sync(bar_id, 128);  // the count is cleared before any thread gathers
    }
    const uint32_t cap = static_cast<uint32_t>(big_cap);
    keys.for_each(tid, [&](uint64_t x) {
        if (x >= lower) {
            const uint32_t slot = atomicAdd(&cs.ncand, 1u);
            if (slot < cap) big[slot] = x;
        }
    });
    bar_sync(bar_id, 128);
    const uint32_t m = cs.ncand;
    bar_sync(bar_id, 128);  // every thread has read the count before the scratch is reused
    m_out = m;
    lower_out = lower;
    return m >= static_cast<uint32_t>(k) && m <= cap;
}

// Hands every region entry >= L, with a distinct output position in
// [0, kept), to `emit`, by the 128 threads of the half; returns kept.
// Positions are assigned per warp in blocks (entry order is not kept).  Each
// chunk of 2048 entries is loaded into registers before one barrier and
// written after it, so packing the pool into its own front is safe in place:
// a chunk's writes never reach past its own entries.
template <typename Emit>
__device__ __forceinline__ uint32_t half_walk_kept(const uint64_t* pool, const PoolRegions& rg, uint64_t L,
                                                   CutScratch& cs, int tid, uint32_t bar_id, uint32_t& phase,
                                                   Emit emit) {
    constexpr int EP = 16;  // entries per thread per chunk (the walk prefix needs EP < 32)
    const int lane = tid & 31, wq = tid >> 5;
    const int n = rg.total();
    uint32_t out = 0;
    for (int c0 = 0; c0 < n; c0 += 128 * EP) {
        uint64_t x[EP];
        uint32_t keep = 0, mine = 0;
#pragma unroll
        for (int j = 0; j < EP; ++j) {
            const int v = c0 + j * 128 + tid;
            x[j] = v < n ? pool[region_addr(rg, v)] : 0ull;
            const bool kp = v < n && x[j] >= L;
            keep |= (kp ? 1u : 0u) << j;
            mine += kp ? 1u : 0u;
        }
        // exclusive prefix of `mine` (at most EP < 32) over the warp, and per-warp totals
        uint32_t wtot;
        const uint32_t excl = warp_prefix_small(mine, lane, wtot);
        uint32_t* rc = cs.rcnt[phase & 1u];
        ++phase;
        if (lane == 0) rc[wq] = wtot;
        bar_sync(bar_id, 128);
        uint32_t pos = out + excl, total = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const uint32_t cw = rc[w];
            pos += (w < wq) ? cw : 0u;
            total += cw;
        }
#pragma unroll
        for (int j = 0; j < EP; ++j)
            if ((keep >> j) & 1u) emit(x[j], pos++);
        out += total;
    }
    return out;
}

// half_walk_kept for keys held in registers: one barrier, then each thread
// emits its kept keys (safe in place: every key was read before).  With
// `known` (the per-warp counts of keys >= L, from the counting pass that
// chose L), the exchange and its barrier are skipped.
template <typename Emit>
__device__ __forceinline__ uint32_t half_walk_reg(const RegKeys& rk, uint64_t L, CutScratch& cs, int tid,
                                                  uint32_t bar_id, uint32_t& phase, Emit emit,
                                                  const uint32_t* known = nullptr) {
    const int lane = tid & 31, wq = tid >> 5;
    uint32_t keep = 0, mine = 0;
#pragma unroll
    for (int j = 0; j < kRegKeys; ++j) {
        const bool kp = j * 128 + tid < rk.n && rk.x[j] >= L;
        keep |= (kp ? 1u : 0u) << j;
        mine += kp ? 1u : 0u;
    }
    uint32_t wtot;
    const uint32_t excl = warp_prefix_small(mine, lane, wtot);  // mine <= kRegKeys < 32
    const uint32_t* rc = known;
    if (!known) {
        uint32_t* mine_rc = cs.rcnt[phase & 1u];
        ++phase;
        if (lane == 0) mine_rc[wq] = wtot;
        bar_sync(bar_id, 128);
        rc = mine_rc;
    }
    uint32_t pos = excl, total = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t cw = rc[w];
        pos += (w < wq) ? cw : 0u;
        total += cw;
    }
#pragma unroll
    for (int j = 0; j < kRegKeys; ++j)
        if ((keep >> j) & 1u) emit(rk.x[j], pos++);
    return total;
}

// Cuts one query's pool to its best keys -- between k and max_keep of them,
// or all when there are at most k -- packed at the front of the pool, by the
// 128 threads of the half.  Returns the new lower bound; `kept` gets the count.
// A large workspace pool is first gathered above a sampled bound into `big`
// (half_gather_top), so the select and the pack read shared memory.
// `big`: the group's shared-memory candidate buffer (STREAM_CAND keys) when
// the pools are in the workspace, else null.
static __device__ __noinline__ uint64_t cut_pool(uint64_t* pq, PoolRegions rg, int k, uint32_t max_keep, uint64_t lb,
                                          CutScratch& cs, int tid, uint32_t bar_id, uint32_t& phase,
                                          uint32_t& kept, uint64_t* big, int big_cap) {
    uint64_t L = lb;
    auto pack = [&](uint64_t x, uint32_t pos) { pq[pos] = x; };
    if (rg.total() <= 128 * kRegKeys) {
        RegKeys rk;
        rk.load(pq, rg, tid);
        // when a sample qualifies, its counting pass already has the per-warp
        // counts the pack needs (and every key is in registers: safe in place)
        const uint32_t* known = nullptr;
        if (rk.n > k)
            L = big ? half_select_bound<true>(rk, pq, rg, k, max_keep, cs, tid, bar_id, phase, big, big_cap, &known)
                    : half_select_bound(rk, pq, rg, k, max_keep, cs, tid, bar_id, phase, nullptr, 0, &known);
        kept = half_walk_reg(rk, L, cs, tid, bar_id, phase, pack, known);
    } else {
        const StreamKeys sk{pq, rg};
        uint32_t m = 0;
        uint64_t lower = 0ull;
        if (big && half_gather_top(sk, pq, rg, k, cs, tid, bar_id, big, big_cap, m, lower)) {
            // the pool's best keys are all in big[0, m): select and pack from shared memory
            const PoolRegions one = single_region(static_cast<int>(m));
            if (m > static_cast<uint32_t>(k)) {
                if (m <= 128u * kRegKeys) {
                    RegKeys rk;
                    rk.load(big, one, tid);
                    L = half_select_bound(rk, big, one, k, max_keep, cs, tid, bar_id, phase);
                } else {
                    const StreamKeys bk{big, one};
                    L = half_select_bound(bk, big, one, k, max_keep, cs, tid, bar_id, phase);
                }
            } else {
                L = lower;  // exactly k keys at or above the bound: all kept, and it is the new bound
            }
            kept = half_walk_kept(big, one, L, cs, tid, bar_id, phase, pack);
            return L;
        }
        if (rg.total() > k) {
            if (!(big && half_window_bound(sk, pq, rg, k, cs, tid, bar_id, phase, big, big_cap, L)))
                L = big ? half_select_bound<true>(sk, pq, rg, k, max_keep, cs, tid, bar_id, phase, big, big_cap)
                        : half_select_bound(sk, pq, rg, k, max_keep, cs, tid, bar_id, phase);
        }
        kept = half_walk_kept(pq, rg, L, cs, tid, bar_id, phase, pack);
    }
    return L;
}

// Sorts the n packed keys buf[0, n) of one query (n <= k <= 128*E) in
// descending key order -- score descending, then key index ascending -- and
// writes the row's k entries, padding (-1, -inf) past n; by the 128 threads
// of the half.  A bitonic network over 128*E keys: element i is slot i%E of
// thread i/E (zero keys, below every real key, fill [n, 128*E)).  Partner
// distances below E are register swaps, those below 32*E lane shuffles, and
// the rest (the last three stages' worth) exchange through buf itself, which
// must hold 128*E keys.  Each thread then writes E consecutive row entries.
template <int E>
__device__ __noinline__ void half_sort_emit(uint64_t* buf, int n, int k, int tid, uint32_t bar_id, int32_t* out_idx,
                                            float* out_score) {
    constexpr int K2 = 128 * E;
    uint64_t v[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int i = tid * E + e;
        v[e] = i < n ? buf[i] : 0ull;
    }
    bar_sync(bar_id, 128);  // every key is in registers before buf serves the exchanges
#pragma unroll
    for (int size = 2; size <= K2; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            if (stride < E) {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int pe = e ^ stride;
                    if (pe > e) {
                        // keys are distinct (zero fill keys are equal, and swapping
                        // them changes nothing), so one compare decides
                        const bool desc = ((tid * E + e) & size) == 0;
                        const uint64_t a = v[e], b = v[pe];
                        const bool sw = (a < b) == desc;
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
                    for (int e = 0; e < E; ++e) buf[tid * E + e] = v[e];
                    bar_sync(bar_id, 128);
#pragma unroll
                    for (int e = 0; e < E; ++e) o[e] = buf[(tid ^ pt) * E + e];
                    bar_sync(bar_id, 128);  // read before the next exchange overwrites
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
    const int i0 = tid * E;
    if constexpr (E >= 4) {
        const bool vec = ((reinterpret_cast<uintptr_t>(out_idx + i0) | reinterpret_cast<uintptr_t>(out_score + i0)) &
                          15u) == 0 && i0 + E <= k;
        if (vec) {
#pragma unroll
            for (int c = 0; c < E / 4; ++c) {
                int32_t ix[4];
                float sc[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const bool real = i0 + 4 * c + u < n;
                    ix[u] = real ? key_index(v[4 * c + u]) : -1;
                    sc[u] = real ? key_score(v[4 * c + u]) : -__int_as_float(0x7f800000);
                }
                reinterpret_cast<int4*>(out_idx + i0)[c] = make_int4(ix[0], ix[1], ix[2], ix[3]);
                reinterpret_cast<float4*>(out_score + i0)[c] = make_float4(sc[0], sc[1], sc[2], sc[3]);
            }
            return;
        }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int i = i0 + e;
        if (i < k) {
            const bool real = i < n;
            out_idx[i] = real ? key_index(v[e]) : -1;
            out_score[i] = real ? key_score(v[e]) : -__int_as_float(0x7f800000);
        }
    }
}

// Writes the k best keys of one query's pool (or all, when fewer) to its
// output row, then pads the row with (-1, -inf); by the half.  The kept keys
// are packed first -- into the shared-memory buffer `big` when the pool is in
// the workspace (k <= 2048 < STREAM_CAND), else to the front of the shared-
// memory pool.  With sort_e > 0 they are then sorted (half_sort_emit) and the
// row is final; otherwise the row is written in pool order, unsorted.
static __device__ __noinline__ void emit_best(uint64_t* pq, PoolRegions rg, int k, CutScratch& cs, int tid,
                                       uint32_t bar_id, uint32_t& phase, int32_t* out_idx, float* out_score,
                                       uint64_t* big, int big_cap, int sort_e) {
    uint64_t* dst = big ? big : pq;
    auto pack = [&](uint64_t x, uint32_t pos) { dst[pos] = x; };
    const uint32_t ku = static_cast<uint32_t>(k);
    uint32_t out;
    if (rg.total() <= 128 * kRegKeys) {
        RegKeys rk;
        rk.load(pq, rg, tid);
        const uint64_t L =
            rk.n <= k ? 0ull
            : big     ? half_select_bound<true>(rk, pq, rg, k, ku, cs, tid, bar_id, phase, big, big_cap)
                      : half_select_bound(rk, pq, rg, k, ku, cs, tid, bar_id, phase);
        out = half_walk_reg(rk, L, cs, tid, bar_id, phase, pack);
    } else {
        const StreamKeys sk{pq, rg};
        uint64_t L = 0ull;
        if (rg.total() > k) {
            // (gathering the keys above a sampled bound first, as cut_pool does,
            // measured slower here: the exact select over the gathered keys
            // costs more than the window select)
            if (!(big && half_window_bound(sk, pq, rg, k, cs, tid, bar_id, phase, big, big_cap, L)))
                L = big ? half_select_bound<true>(sk, pq, rg, k, ku, cs, tid, bar_id, phase, big, big_cap)
                        : half_select_bound(sk, pq, rg, k, ku, cs, tid, bar_id, phase);
        }
        out = half_walk_kept(pq, rg, L, cs, tid, bar_id, phase, pack);
    }
    bar_sync(bar_id, 128);  // the packed keys are visible to the whole half
    // With sort_e set, the row is written in its final order; the packed keys'
    // buffer (the pool, or `big`) holds at least 128 * sort_e keys.
    switch (sort_e) {
        case 1: half_sort_emit<1>(dst, static_cast<int>(out), k, tid, bar_id, out_idx, out_score); return;
        case 2: half_sort_emit<2>(dst, static_cast<int>(out), k, tid, bar_id, out_idx, out_score); return;
        case 4: half_sort_emit<4>(dst, static_cast<int>(out), k, tid, bar_id, out_idx, out_score); return;
        case 8: half_sort_emit<8>(dst, static_cast<int>(out), k, tid, bar_id, out_idx, out_score); return;
        case 16: half_sort_emit<16>(dst, static_cast<int>(out), k, tid, bar_id, out_idx, out_score); return;
        default: break;
    }
    for (int i = tid; i < k; i += 128) {
        if (i < static_cast<int>(out)) {
            const uint64_t x = dst[i];
            out_idx[i] = key_index(x);
            out_score[i] = key_score(x);
        } else {
            out_idx[i] = -1;
            out_score[i] = -__int_as_float(0x7f800000);
        }
    }
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
    __shared__ uint32_t cntw[C::NGROUPS][C::QH][4];
    __shared__ CutScratch cut_s[C::NGROUPS];        // per group: pool-cut scratch
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

    if (warp < C::EPI_WARP0) {
    // The control warpgroup hands registers to the epilogue warpgroups.
    regs_shrink_to<C::REGS_CTRL>();
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
#ifdef SI_FAULT_TEST
                    // Test builds only (never the product library): CTA 0 does not
                    // signal its third accumulator.  The epilogue's bounded wait on it
                    // runs out, which exercises the abort path end to end: error word,
                    // abort flag, drain of issued loads and MMAs, TMEM release.
                    if (!(cta == 0 && acc_it == 2)) umma_commit(bar(kBarAccFull + buf));
#else
                    umma_commit(bar(kBarAccFull + buf));
#endif
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
    }
    } else {
        // ------------------------------------------------ epilogue
        regs_grow_to<C::REGS_EPI>();
        const int e = warp - C::EPI_WARP0;
        const int quarter = warp & 3;
        const int half = e >> 2;  // epilogue group
        const int wih = e & 3;
        const uint32_t bar_id = 1u + static_cast<uint32_t>(half);
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const int htid = wih * 32 + lane;  // thread index within the half
        CutScratch& cs = cut_s[half];
        // workspace pools: the group's exact-cut buffer takes the room of the shared-memory pools
        uint64_t* big = SMEM_POOL ? nullptr : reinterpret_cast<uint64_t*>(smem + C::OFF_POOL) + half * C::STREAM_CAND;
        uint32_t cphase = 0;  // exchange-buffer parity of the half's cut helpers
        const bool dense = p.dense != nullptr;
        const int k = p.k;
        const uint32_t Pu = static_cast<uint32_t>(P);
        // An intermediate cut keeps at most k + cut_slack entries, which leaves
        // every warp's sub-range more than check_tiles*32 free slots (the host
        // ensures P >= k + 4 * (32 * check_tiles + 1) + 28).
        const uint32_t ct = p.check_tiles;
        const uint32_t room = 4u * (32u * ct + 1u);
        const uint32_t cut_slack =
            Pu > static_cast<uint32_t>(k) + room + p.cut_slack ? p.cut_slack : Pu - static_cast<uint32_t>(k) - room;
        uint32_t acc_it = 0, w_it = 0;
        bool bad = false;
        for (int64_t r = 0; r * G < U; ++r) {
            const int64_t u = unit_of_round(r, G, cta);
            if (u >= U) continue;
            const UnitInfo ui = decode_unit(u, p, C::QT);
            SI_TR_T0(tun0);
            // Pool state of each query of the half, identical in the four warps
            // except the append sub-range: survivors [0, kp), this warp's
            // sub-range [bw, bw + fw) holding cw appended keys, lower bound lb.
            uint64_t lb[C::QH];
            uint32_t kp[C::QH] = {}, cw[C::QH] = {};
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
                int64_t v = (t < p.t_hi) ? (t + 1) / p.m : 0;
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
            // The half's head weights stay in registers for the whole unit
            // (reloaded after a pool cut, whose call does not preserve them).
            float wr[C::CG];
            auto load_w = [&]() {
#pragma unroll
                for (int i = 0; i < C::CG; i += 4) {
                    const float4 v = *reinterpret_cast<const float4*>(wq + i);
                    wr[i] = v.x;
                    wr[i + 1] = v.y;
                    wr[i + 2] = v.z;
                    wr[i + 3] = v.w;
                }
            };
            if (ui.ntiles > 0) load_w();
            SI_TR_ADD(kTrEpiUnit, tun0, tr_lead);
            bool need_acc = false, bad_acc = false;
            uint32_t check_cd = ct;  // tiles until the next pool check
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
                half_scores<H, C::QH, C::NP, C::CG / 32>(tmem_base + buf * C::N + half * C::CG + lane_off, wr, sc);
#pragma unroll
                for (int q = 0; q < C::QH; ++q) SI_TR_DEPF(sc[q]);
                SI_TR_ADD(kTrEpiScores, ts0, tr_lead);
                SI_TR_T0(tar0);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarAccEmpty + buf));
                SI_TR_ADD(kTrEpiArrive, tar0, tr_lead);
                SI_TR_T0(tap0);
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
                            need |= cw[q] + 32u * ct > fw(q);
                        }
                    }
                }
                SI_TR_ADD(kTrEpiAppend, tap0, tr_lead);
                SI_TR_T0(tfl0);
                // One barrier every check_tiles tiles (abort and cut requests are
                // OR-reduced; sub-ranges keep room for check_tiles tiles of
                // appends); two more only when some sub-range is nearly full or
                // a wait failed.
                need_acc |= need;
                bad_acc |= !ok;
                if (--check_cd != 0 && j + 1 != ui.ntiles) continue;
                check_cd = ct;
                const bool bad_here = bad_acc || *abort_flag;
                SI_TR_DEPI(static_cast<int>(need_acc));
                SI_TR_ADD(kTrEpiFilter, tfl0, tr_lead);
                SI_TR_T0(tb0);
                const bool any_flag = bar_red_or(bar_id, 128, bad_here || need_acc);
                need_acc = false;
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
                        const uint32_t mg = 32u * ct;
                        const bool cut = c4[0] + mg > f || c4[1] + mg > f || c4[2] + mg > f || c4[3] + mg > f;
                        if (!cut) continue;  // uniform over the half
                        uint64_t* pq = pool + (half * C::QH + q) * P;
                        uint32_t kept = 0;
                        const uint64_t L = cut_pool(pq, pool_regions(kp[q], f, c4), k,
                                                    static_cast<uint32_t>(k) + cut_slack, lb[q], cs, htid, bar_id,
                                                    cphase, kept, big, C::STREAM_CAND);
                        SI_TR_INC(kTrCompactions, true);
                        kp[q] = kept;
                        lb[q] = L;
                        cw[q] = 0u;
                        bar_sync(bar_id, 128);
                    }
                    load_w();
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
                    if (t >= p.t_hi) continue;  // uniform over the half
                    const int64_t row = (ui.b * p.S + t) * static_cast<int64_t>(k);
                    emit_best(pool + qi * P, pool_regions(kp[q], fw(q), cntw[half][q]), k, cs, htid, bar_id, cphase,
                              p.out_idx + row, p.out_score + row, big, C::STREAM_CAND, p.sort_e);
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
