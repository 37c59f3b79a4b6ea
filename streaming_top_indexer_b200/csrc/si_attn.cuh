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
// One CTA per SM, a persistent loop over query rows; every row costs the same
// (ceil(k/64) key chunks).  Per row the 128 heads are the MMA's M (one TMEM
// lane each); per pair of chunks of 64 selected keys (per chunk when the
// count is odd):
//   S   = Q K^T      tcgen05.mma M=128 N=128 K=d    (fp32 in TMEM; N=64 alone)
// and per chunk:
//   P   = softmax    one thread per head, online, bf16 into shared memory
//   O  += P V        tcgen05.mma M=128 N=dv K=64    (V as an MN-major operand)
// Each tcgen05.mma instruction costs the issuing thread about 100 cycles
// whatever its N, so S over two chunks at once halves the S issue time
// (16 instructions per 128 keys in all, against 24 one chunk at a time).
// Roles (384 threads):
//   warp 0      TMA: q tiles (one buffer per softmax group);
//   warp 1      TMEM allocation and the MMA issuer (an event loop: S and,
//               per softmax group, P V are each issued as soon as their
//               inputs are ready);
//   warps 2-3   the chunks' K and V rows, gathered by index with 16-byte
//               cp.async copies into an NST-stage ring (NST even; K is laid
//               out sub-tile-major so that stages 2j and 2j+1 form one
//               128-row operand), half of each chunk's
//               rows per warp (the selected rows are scattered 128- or 256-byte rows:
//               measured, TMA gather4 moved them at about 10 GB/s per SM, one
//               128-byte row segment every ~12 ns, which bounded the kernel);
//               they also publish each chunk's validity mask with the stage's
//               barrier;
//   warps 4-11  two softmax groups of four warps.  Group w takes the CTA's
//               rows with w = (row ordinal) & 1; the two groups' chunks are
//               interleaved, so one group's softmax overlaps the other's MMAs.
// The running max is in base-2 units; O in TMEM is rescaled only when a
// chunk's max exceeds the running max by more than 8 (every p <= 2^8 before
// normalisation).  At the end of a row, out = O / l in bf16 and
// lse = ln 2 * (m + log2 l); a row with no valid entry gives 0 and -inf.
#pragma once
#include <cuda.h>

#include <cstdint>

#include "si_ptx.cuh"

namespace si {

// Optional timeline tracing (build flag SI_ATTN_TRACE; off in the product
// library): CTA 0 records clock64() at each role's hand-offs for its first
// kATraceItems work items in trace[(role * kATraceItems + item) * 4 + event].
// Roles: 0 gather warp 2, 1 MMA issuer, 2 and 3 the softmax groups (lane 0 of
// their first warp).
constexpr int kATraceItems = 256;
#ifdef SI_ATTN_TRACE
#define SI_AT(role, item, ev)                                                                              \
    do {                                                                                                   \
        if (blockIdx.x == 0 && (item) < kATraceItems && p.trace)                                           \
            p.trace[((role) * kATraceItems + (item)) * 4 + (ev)] = static_cast<unsigned long long>(clock64()); \
    } while (0)
#else
#define SI_AT(role, item, ev) (void)0
#endif

struct AttnParams {
    int64_t rows;         // B * S query rows
    int64_t S, T;
    int k;                // entries per idx row
    int nchunks;          // ceil(k / 64)
    const int32_t* idx;   // [B*S, k]
    const uint16_t* kcache;  // bf16 [B*T, D]
    const uint16_t* vcache;  // bf16 [B*T, DV]
    uint16_t* out;        // bf16 [B*S, 128, DV]
    float* lse;           // [B*S, 128]
    float c2;             // scale * log2(e)
    uint32_t* err;        // device status word
    uint64_t timeout_ns;
    unsigned long long* trace;  // SI_ATTN_TRACE builds only
};

template <int D, int DV>
struct AttnCfg {
    static_assert(D == 64 || D == 128, "d");
    static_assert(DV == 64 || DV == 128, "d_v");
    static constexpr int HA = 128;                     // heads: MMA M, TMEM lanes
    static constexpr int NK = 64;                      // keys per chunk
    static constexpr uint32_t Q_SUB = HA * 128u;       // 64 columns of q: 16 KB
    static constexpr uint32_t Q_BYTES = (D / 64) * Q_SUB;
    static constexpr uint32_t KV_SUB = NK * 128u;      // 64 columns of 64 keys: 8 KB
    static constexpr uint32_t K_BYTES = (D / 64) * KV_SUB;
    static constexpr uint32_t V_BYTES = (DV / 64) * KV_SUB;
    static constexpr uint32_t P_BYTES = HA * 128u;     // [128 heads x 64 keys] bf16
    static constexpr uint32_t STATIC_MAX = 2048;       // bound of the kernel's static shared memory
    static constexpr uint32_t SMEM_LIMIT = 232448;     // per block, opt-in
    // everything but the K/V ring: two q buffers, one P buffer per group, alignment slack
    static constexpr uint32_t FIXED = 2 * Q_BYTES + 2 * P_BYTES + 1024 + STATIC_MAX;
    static constexpr int NST_FIT = static_cast<int>((SMEM_LIMIT - FIXED) / (K_BYTES + V_BYTES));
    // K/V ring stages, even: a chunk pair takes stages 2j, 2j+1
    static constexpr int NST = (NST_FIT > 6 ? 6 : NST_FIT) & ~1;
    static_assert(NST >= 2, "shared memory budget");
    static constexpr uint32_t OFF_Q = 0;                // [2] by softmax group
    static constexpr uint32_t OFF_P = OFF_Q + 2 * Q_BYTES;   // [group]
    // K ring: [d/64 sub-tiles][NST stages][64 keys x 128 bytes], so that two
    // adjacent stages of one sub-tile are 128 consecutive rows
    static constexpr uint32_t OFF_K = OFF_P + 2 * P_BYTES;
    static constexpr uint32_t K_SUB_STRIDE = NST * KV_SUB;
    static constexpr uint32_t OFF_V = OFF_K + NST * K_BYTES;
    static constexpr uint32_t DYN_BYTES = OFF_V + NST * V_BYTES + 1024;
    static constexpr int THREADS = 384;
    // Registers: every role runs in the launch allocation (168 per thread;
    // ptxas -v reports about 56 bytes of spill stores); a setmaxnreg re-split
    // between the control and softmax warpgroups made ptxas spill much more
    // around it, so there is none.
    static constexpr uint32_t TMEM_COLS = 512;
    // TMEM: group w: S[w][2] at columns 128w + {0, 64}; O[w] at 256 + w*DV
    static constexpr uint32_t TM_O = 256;
    static_assert(TM_O + 2 * DV <= TMEM_COLS, "TMEM budget");
    static constexpr float RESCALE = 8.0f;              // base-2 units
};

enum : int {
    kAQFull = 0,       // [2] by group
    kAQEmpty = 2,      // [2]
    kASFull = 4,       // [group][2]
    kASFree = 8,       // [group][2]
    kAPFull = 12,      // [group]
    kAPEmpty = 14,     // [group]
    kAOFull = 16,      // [2]
    kAOFree = 18,      // [2]
    kADrain = 20,
    kAKFull = 21,      // [NST] K and V rows of the stage landed (with its mask)
    kAKVEmpty = 27,    // [NST]
    kANumBars = 33
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

// The CTA's work items (one 64-key chunk each) in issue order: its rows
// i = 0 .. nrows-1 (query row blockIdx.x + i * gridDim.x) go in pairs
// (2p, 2p+1), one per softmax group, and the two rows' chunks alternate by
// chunk pairs: (2p, 0), (2p, 1), (2p+1, 0), (2p+1, 1), (2p, 2), (2p, 3), ...;
// with an odd chunk count the last chunks follow alone, (2p, NC-1),
// (2p+1, NC-1).  An odd last row runs alone, its chunks in order.  Every
// chunk pair starts at an even item, so its two ring stages are adjacent.
struct AttnItem {
    int64_t i;   // row ordinal in the CTA
    int c;       // chunk of the row
    int w;       // softmax group (= i & 1)
    int64_t lc;  // the group's own chunk ordinal
};

__device__ __forceinline__ AttnItem attn_item(int64_t g, int64_t nrows, int NC) {
    AttnItem it;
    const int64_t pair_items = 2 * static_cast<int64_t>(NC);
    const int64_t base = (nrows >> 1) * pair_items;
    if (g < base) {
        const int64_t p = g / pair_items;
        const int r = static_cast<int>(g % pair_items);
        const int full = (NC >> 1) * 4;  // items of the two rows' complete chunk pairs
        if (r < full) {
            it.w = (r >> 1) & 1;
            it.c = (r >> 2) * 2 + (r & 1);
        } else {
            it.w = r - full;
            it.c = NC - 1;
        }
        it.i = 2 * p + it.w;
    } else {
        it.i = nrows - 1;
        it.c = static_cast<int>(g - base);
        it.w = 0;
    }
    it.lc = (it.i >> 1) * NC + it.c;
    return it;
}

// Item index of chunk c of row ordinal i (the inverse of attn_item).
__device__ __forceinline__ int64_t attn_item_of(int64_t i, int c, int64_t nrows, int NC) {
    const int64_t pair = i >> 1;
    if (pair == (nrows >> 1)) return (nrows >> 1) * 2 * NC + c;  // the odd last row, alone
    const int w = static_cast<int>(i & 1);
    const int64_t base = pair * 2 * NC;
    if (c < (NC & ~1)) return base + (c >> 1) * 4 + w * 2 + (c & 1);
    return base + (NC >> 1) * 4 + w;
}

template <int D, int DV>
__global__ void __launch_bounds__(AttnCfg<D, DV>::THREADS, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const AttnParams p) {
    using C = AttnCfg<D, DV>;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[kANumBars];
    __shared__ uint32_t masks[C::NST][2];   // validity of the 64 entries of each ring stage
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
            mbar_init(bar(kAOFull + i), 1);
            mbar_init(bar(kAOFree + i), 4);
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(bar(kASFull + i), 1);
            mbar_init(bar(kASFree + i), 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(kAPFull + i), 4);
            mbar_init(bar(kAPEmpty + i), 1);
        }
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(bar(kAKFull + s), 2);  // K and V rows of the stage: one arrival per gatherer warp
            mbar_init(bar(kAKVEmpty + s), 1);
        }
        mbar_init(bar(kADrain), 1);
        abort_flag_s = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) prefetch_tmap(&tm_q);
    if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;

    const int64_t G = gridDim.x;
    const int64_t nrows = (p.rows - blockIdx.x + G - 1) / G;  // rows blockIdx.x + i*G
    const int NC = p.nchunks;
    const int64_t total = nrows * NC;                           // work items of this CTA

    if (warp < 4) {
        if (warp == 0) {
            // -------------------------------------------- TMA: q tiles
            // One [128 heads x d] tile per row, in the CTA's row order, into the
            // buffer of the row's softmax group once its previous row's S MMAs
            // are done.
            if (lane == 0) {
                bool ok = true;
                int64_t i = 0;
                for (; i < nrows; ++i) {
                    const int w = static_cast<int>(i & 1);
                    const int64_t use = i >> 1;
                    if (use >= 1 &&
                        !(ok = mbar_wait(bar(kAQEmpty + w), static_cast<uint32_t>(use - 1) & 1u, abort_flag, p.err, lim)))
                        break;
                    const int64_t row = blockIdx.x + i * G;
                    mbar_arrive_expect_tx(bar(kAQFull + w), C::Q_BYTES);
#pragma unroll
                    for (int c = 0; c < D / 64; ++c)
                        tma_load_2d(sbase + C::OFF_Q + w * C::Q_BYTES + c * C::Q_SUB, &tm_q, bar(kAQFull + w), c * 64,
                                    static_cast<int>(row * C::HA));
                }
                if (!ok)  // let the tiles already issued land before the CTA exits
                    for (int64_t j = i - 2 < 0 ? 0 : i - 2; j < i; ++j)
                        attn_wait_bounded(bar(kAQFull + (j & 1)), static_cast<uint32_t>(j >> 1) & 1u, 100000000ull);
            }
            __syncwarp();
        } else if (warp >= 2) {
            // -------------------------------------------- K/V gathers (warps 2-3)
            // Warp 2 copies rows 0-31 of each 64-key chunk, warp 3 rows 32-63,
            // both at once, with 16-byte cp.async copies into the 128-byte-
            // swizzled layout of the MMA operands (a row of d columns is d/8
            // pieces; consecutive lanes take consecutive pieces of one row, so
            // loads coalesce).  A warp signals its half of a chunk once its
            // copies have landed (wait_group) and been made visible to the
            // tensor cores (proxy fence).  When the next chunk's stage is
            // already free, its copies are issued before that wait, keeping
            // the loads in flight.
            const int half = warp - 2;
            const int64_t S = p.S, T = p.T;
            auto entry = [&](int64_t g) -> int {
                const AttnItem it = attn_item(g, nrows, NC);
                const int j = it.c * C::NK + half * 32 + lane;
                return j < p.k ? p.idx[(blockIdx.x + it.i * G) * p.k + j] : -1;
            };
            // copies of one operand (DD = d for K, d_v for V) of the warp's 32 rows;
            // 64-column sub-tile cc of the stage starts at dst_stage + cc * sub_stride
            auto copy_rows = [&](const uint16_t* cache, uint32_t dst_stage, uint32_t sub_stride, int key, int64_t kbase,
                                 int dd) {
                const int ppr = dd / 8;              // 16-byte pieces per row
                const int rpi = 32 / ppr;            // rows per warp instruction
                const int pc = lane % ppr, cc = pc >> 3, c16 = pc & 7;
                for (int it2 = 0; it2 < 32 / rpi; ++it2) {
                    const int lr = it2 * rpi + lane / ppr;          // row within the warp's 32
                    const int r = half * 32 + lr;                   // row within the chunk
                    const int kr = __shfl_sync(0xffffffffu, key, lr);
                    const uint32_t dst = dst_stage + cc * sub_stride + static_cast<uint32_t>(r >> 3) * 1024u +
                                         static_cast<uint32_t>(r & 7) * 128u +
                                         (static_cast<uint32_t>(c16 ^ (r & 7)) << 4);
                    cp_async_16(dst, cache + (kbase + kr) * dd + pc * 8);
                }
            };
            // issue the copies of item g (its stage is free), with its mask
            auto issue = [&](int64_t g, int ent) {
                const AttnItem it = attn_item(g, nrows, NC);
                const int64_t kbase = (blockIdx.x + it.i * G) / S * T;
                const uint32_t st = static_cast<uint32_t>(g % C::NST);
                const bool valid = ent >= 0 && ent < T;
                const int key = valid ? ent : 0;  // padding reads key 0, masked in the softmax
                const uint32_t m = __ballot_sync(0xffffffffu, valid);
                if (lane == 0) masks[st][half] = m;  // published by the release of this warp's arrive
                copy_rows(p.kcache, sbase + C::OFF_K + st * C::KV_SUB, C::K_SUB_STRIDE, key, kbase, D);
                copy_rows(p.vcache, sbase + C::OFF_V + st * C::V_BYTES, C::KV_SUB, key, kbase, DV);
                cp_async_commit();
                if (half == 0 && lane == 0) SI_AT(0, g, 3);
            };
            auto signal = [&](int64_t g) {
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kAKFull + static_cast<uint32_t>(g % C::NST)));
                if (half == 0 && lane == 0) SI_AT(0, g, 2);
            };
            auto stage_free = [&](int64_t g) -> bool {  // non-blocking
                const uint32_t u = static_cast<uint32_t>(g / C::NST);
                return u == 0 || mbar_test_wait(bar(kAKVEmpty + static_cast<uint32_t>(g % C::NST)), (u - 1) & 1u);
            };
            bool ok = true;
            int64_t g = 0;           // oldest chunk issued and not yet signalled
            bool pending = false;
            if (total > 0) {
                if (half == 0 && lane == 0) SI_AT(0, 0, 0);
                issue(0, entry(0));
                pending = true;
            }
            int nxt_ent = total > 1 ? entry(1) : -1;
            while (pending) {
                const int64_t gn = g + 1;
                bool early = false;
                if (gn < total) {
                    early = __all_sync(0xffffffffu, stage_free(gn));
                    if (early) {
                        if (half == 0 && lane == 0) SI_AT(0, gn, 0);
                        issue(gn, nxt_ent);
                        nxt_ent = gn + 1 < total ? entry(gn + 1) : -1;
                        cp_async_wait<1>();  // chunk g landed
                    }
                }
                if (!early) cp_async_wait<0>();
                signal(g);
                g = gn;
                pending = early;
                if (!pending && g < total) {
                    // the next chunk's stage was busy: wait for it, then issue
                    if (half == 0 && lane == 0) SI_AT(0, g, 0);
                    const uint32_t u = static_cast<uint32_t>(g / C::NST);
                    ok = mbar_wait(bar(kAKVEmpty + static_cast<uint32_t>(g % C::NST)), (u - 1) & 1u, abort_flag, p.err,
                                   lim);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    if (half == 0 && lane == 0) SI_AT(0, g, 1);
                    issue(g, nxt_ent);
                    nxt_ent = g + 1 < total ? entry(g + 1) : -1;
                    pending = true;
                }
            }
            cp_async_wait<0>();
            __syncwarp();
        } else if (warp == 1) {
            // -------------------------------------------- MMA issuer
            // An event loop: S of the next chunk pair (or lone chunk, in issue
            // order) and, for each softmax group, P V of its next chunk are
            // issued as soon as their inputs are ready (tested without
            // blocking).  The groups' O accumulations are independent, so
            // neither waits for the other.
            if (lane == 0) {
                constexpr uint32_t idesc_s = idesc_bf16_f32(C::HA, C::NK);
                constexpr uint32_t idesc_s2 = idesc_bf16_f32(C::HA, 2 * C::NK);
                constexpr uint32_t idesc_o = idesc_bf16_f32_bmn(C::HA, DV);
                // descriptors of the operand tiles' first K step; a K step of 16
                // adds 32 bytes (K-major) or 2048 bytes (MN-major V) to the start
                // address, i.e. 2 or 128 to the descriptor's low field
                const uint64_t dq0 = smem_desc_sw128(sbase + C::OFF_Q);
                const uint64_t dk0 = smem_desc_sw128(sbase + C::OFF_K);
                const uint64_t dp0 = smem_desc_sw128(sbase + C::OFF_P);
                const uint64_t dv0 = smem_desc_sw128_mn(sbase + C::OFF_V, C::KV_SUB, 1024);
                bool issued = false;
                int64_t gs = 0;
                AttnItem is = attn_item(0, nrows, NC);
                // per group: its next chunk for P V, as (row ordinal, chunk)
                int64_t pr[2] = {0, 1};
                int pc[2] = {0, 0};
                uint64_t t_progress = global_timer_ns();
                uint32_t spins = 0;
                auto group_done = [&](int w) { return pr[w] >= nrows; };
                while (!(group_done(0) && group_done(1))) {
                    bool progress = false;
                    if (gs < total) {
                        const uint32_t st = static_cast<uint32_t>(gs % C::NST), u = static_cast<uint32_t>(gs / C::NST);
                        // chunks c and c+1 of the row at items gs, gs+1 (stages st, st+1).
                        // Pairs need an even chunk count: then a pair's first chunk has an
                        // even group ordinal lc and takes the first of the group's two S
                        // halves, so the pair's 128 columns are the group's S region.
                        const bool two = (NC & 1) == 0 && (is.c & 1) == 0;
                        const int sb = is.w * 2 + static_cast<int>(is.lc & 1);
                        const int64_t su = is.lc >> 1;  // uses of the S half (both halves for a pair)
                        const bool ready =
                            (is.c != 0 || mbar_test_wait(bar(kAQFull + is.w), static_cast<uint32_t>(is.i >> 1) & 1u)) &&
                            mbar_test_wait(bar(kAKFull + st), u & 1u) &&
                            (!two || mbar_test_wait(bar(kAKFull + st + 1), u & 1u)) &&
                            (su == 0 || (mbar_test_wait(bar(kASFree + sb), static_cast<uint32_t>(su - 1) & 1u) &&
                                         (!two || mbar_test_wait(bar(kASFree + sb + 1),
                                                                 static_cast<uint32_t>(su - 1) & 1u))));
                        if (ready) {
                            SI_AT(1, gs, 0);
                            tc_fence_after();
                            const uint32_t d_tmem = tmem_base + is.w * 128 + static_cast<uint32_t>(is.lc & 1) * C::NK;
                            const uint64_t da = dq0 + ((is.w * C::Q_BYTES) >> 4);
                            const uint64_t db = dk0 + ((st * C::KV_SUB) >> 4);
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint32_t off = ((kk / 4) * C::Q_SUB + (kk % 4) * 32) >> 4;
                                const uint32_t offk = ((kk / 4) * C::K_SUB_STRIDE + (kk % 4) * 32) >> 4;
                                umma_bf16(d_tmem, da + off, db + offk, two ? idesc_s2 : idesc_s, kk > 0 ? 1u : 0u);
                            }
                            umma_commit(bar(kASFull + sb));
                            if (two) umma_commit(bar(kASFull + sb + 1));
                            if (is.c + (two ? 1 : 0) == NC - 1) umma_commit(bar(kAQEmpty + is.w));
                            SI_AT(1, gs, 1);
                            issued = progress = true;
                            gs += two ? 2 : 1;
                            if (gs < total) is = attn_item(gs, nrows, NC);
                        }
                    }
#pragma unroll
                    for (int w = 0; w < 2; ++w) {
                        if (group_done(w)) continue;
                        const int64_t i = pr[w];
                        const int c = pc[w];
                        // the chunk's place in issue order, and the group's own ordinal
                        const int64_t g = attn_item_of(i, c, nrows, NC);
                        if (g >= gs) continue;  // its S is not issued yet
                        const int64_t lc = (i >> 1) * NC + c, ouse = i >> 1;
                        const bool ready = mbar_test_wait(bar(kAPFull + w), static_cast<uint32_t>(lc) & 1u) &&
                                           (c != 0 || ouse == 0 ||
                                            mbar_test_wait(bar(kAOFree + w), static_cast<uint32_t>(ouse - 1) & 1u));
                        if (!ready) continue;
                        SI_AT(1, g, 2);
                        tc_fence_after();
                        const uint32_t st = static_cast<uint32_t>(g % C::NST);
                        const uint32_t d_tmem = tmem_base + C::TM_O + w * DV;
                        const uint64_t da = dp0 + ((w * C::P_BYTES) >> 4);
                        const uint64_t db = dv0 + ((st * C::V_BYTES) >> 4);
#pragma unroll
                        for (int kk = 0; kk < C::NK / 16; ++kk)
                            umma_bf16(d_tmem, da + kk * 2, db + kk * 128, idesc_o, (c > 0 || kk > 0) ? 1u : 0u);
                        umma_commit(bar(kAPEmpty + w));
                        umma_commit(bar(kAKVEmpty + st));
                        if (c == NC - 1) umma_commit(bar(kAOFull + w));
                        SI_AT(1, g, 3);
                        progress = true;
                        if (++pc[w] == NC) {
                            pc[w] = 0;
                            pr[w] += 2;
                        }
                    }
                    if (progress) {
                        t_progress = global_timer_ns();
                        spins = 0;
                    } else if ((++spins & 63u) == 0) {
                        if (*abort_flag) break;
                        if (global_timer_ns() - t_progress > lim) {
                            atomicCAS(p.err, 0u, kErrTimeout);
                            *abort_flag = 1;
                            break;
                        }
                    }
                }
                if (issued) {
                    umma_commit(bar(kADrain));
                    attn_wait_bounded(bar(kADrain), 0, 100000000ull);
                }
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------ softmax groups (warps 4-11)
        const int w = (warp - 4) >> 2;      // group
        const int quarter = warp & 3;       // TMEM lanes 32*quarter .. +31
        const int h = quarter * 32 + lane;  // head
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t p_row = static_cast<uint32_t>(h >> 3) * 1024u + static_cast<uint32_t>(h & 7) * 128u;
        const float NEG_INF = -__int_as_float(0x7f800000);
        const float LN2 = 0.6931471805599453f;
        const uint32_t o_addr = tmem_base + C::TM_O + w * DV + lane_off;
        bool ok = true;
        // this group's rows are the CTA's row ordinals w, w+2, ...
        for (int64_t i = w; ok && i < nrows; i += 2) {
            const int64_t row = blockIdx.x + i * G;
            float m_run = NEG_INF, l_run = 0.0f;
            for (int c = 0; c < NC; ++c) {
                // global item index of (i, c)
                const int64_t g = attn_item_of(i, c, nrows, NC);
                const int64_t lc = (i >> 1) * NC + c;
                const int sb = w * 2 + static_cast<int>(lc & 1);
                const uint32_t su = static_cast<uint32_t>(lc >> 1);
                const uint32_t st = static_cast<uint32_t>(g % C::NST), ku = static_cast<uint32_t>(g / C::NST);
                // the K barrier also publishes the stage's validity mask
                if (quarter == 0 && lane == 0) SI_AT(2 + w, g, 0);
                ok = mbar_wait(bar(kAKFull + st), ku & 1u, abort_flag, p.err, lim);
                ok = ok && mbar_wait(bar(kASFull + sb), su & 1u, abort_flag, p.err, lim);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                const uint64_t mask = static_cast<uint64_t>(masks[st][0]) | (static_cast<uint64_t>(masks[st][1]) << 32);
                tc_fence_after();
                // scores, then in place their base-2 values (invalid entries -inf)
                uint32_t xr[64];
                const uint32_t s_addr = tmem_base + w * 128 + static_cast<uint32_t>(lc & 1) * C::NK + lane_off;
                tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&xr[0]));
                tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&xr[32]));
                tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(&xr[0]));
                tmem_wait_ld(*reinterpret_cast<uint32_t(*)[32]>(&xr[32]));
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kASFree + sb));
                if (quarter == 0 && lane == 0) SI_AT(2 + w, g, 1);
                if (mask == ~0ull) {
#pragma unroll
                    for (int j = 0; j < 64; ++j) xr[j] = __float_as_uint(__uint_as_float(xr[j]) * p.c2);
                } else {
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        xr[j] = ((mask >> j) & 1ull) ? __float_as_uint(__uint_as_float(xr[j]) * p.c2)
                                                     : __float_as_uint(NEG_INF);
                }
                const float* x = reinterpret_cast<const float*>(xr);
                float mx[8];
#pragma unroll
                for (int a = 0; a < 8; ++a) mx[a] = x[a];
#pragma unroll
                for (int j = 8; j < 64; ++j) mx[j & 7] = fmaxf(mx[j & 7], x[j]);
#pragma unroll
                for (int s = 4; s > 0; s >>= 1)
#pragma unroll
                    for (int a = 0; a < s; ++a) mx[a] = fmaxf(mx[a], mx[a + s]);
                const float m_c = mx[0];
                if (c == 0) {
                    m_run = m_c;
                } else if (m_c > m_run + C::RESCALE) {
                    // O (chunks so far) and l to the new max: wait for the group's
                    // previous P V, then scale O in TMEM.
                    ok = mbar_wait(bar(kAPEmpty + w), static_cast<uint32_t>(lc - 1) & 1u, abort_flag, p.err, lim);
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
                // the group's P buffer is free once its previous chunk's P V is done
                if (lc >= 1) {
                    ok = mbar_wait(bar(kAPEmpty + w), static_cast<uint32_t>(lc - 1) & 1u, abort_flag, p.err, lim);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                }
                // p = 2^(x - m) (0 for invalid entries), bf16 into P (row h, 128-byte
                // swizzle); l by eight partial sums
                uint8_t* prow = smem + C::OFF_P + w * C::P_BYTES + p_row;
                if (m_run == NEG_INF) {
                    // no valid entry in the row so far: every p is 0
#pragma unroll
                    for (int c8 = 0; c8 < 8; ++c8) *reinterpret_cast<uint4*>(prow + (c8 << 4)) = make_uint4(0, 0, 0, 0);
                } else {
                    const float2 negm = make_float2(-m_run, -m_run);
                    float2 part[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                      make_float2(0.f, 0.f)};
#pragma unroll
                    for (int c8 = 0; c8 < 8; ++c8) {
                        uint32_t w4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int j = c8 * 8 + 2 * e;
                            // invalid entries: ex2(-inf - m) = 0
                            const float2 d2 = __fadd2_rn(make_float2(x[j], x[j + 1]), negm);
                            const float pa = ex2_approx(d2.x), pb2 = ex2_approx(d2.y);
                            part[e] = __fadd2_rn(part[e], make_float2(pa, pb2));
                            w4[e] = pack_bf16x2(pa, pb2);
                        }
                        *reinterpret_cast<uint4*>(prow + ((c8 ^ (h & 7)) << 4)) =
                            make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                    const float2 s01 = __fadd2_rn(part[0], part[1]), s23 = __fadd2_rn(part[2], part[3]);
                    const float2 s4 = __fadd2_rn(s01, s23);
                    l_run += s4.x + s4.y;
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kAPFull + w));
                if (quarter == 0 && lane == 0) SI_AT(2 + w, g, 2);
                if (c == NC - 1) {
                    // end of the row: out = O / l (bf16), lse
                    const int64_t ouse = i >> 1;
                    ok = mbar_wait(bar(kAOFull + w), static_cast<uint32_t>(ouse) & 1u, abort_flag, p.err, lim);
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
                        uint32_t wv[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            wv[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
                        uint4* dst = reinterpret_cast<uint4*>(orow + cb * 32);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dst[e] = make_uint4(wv[4 * e], wv[4 * e + 1], wv[4 * e + 2], wv[4 * e + 3]);
                    }
                    p.lse[row * C::HA + h] = l_run > 0.0f ? (m_run + lg2_approx(l_run)) * LN2 : NEG_INF;
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(kAOFree + w));
                    if (quarter == 0 && lane == 0) SI_AT(2 + w, g, 3);
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
