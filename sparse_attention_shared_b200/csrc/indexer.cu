// Full / Reindex indexer: exact top-P pool and top-k list per query.
//
// "CED: Continuing Context with a Causal Encoder and Decoder":
//   "Selecting Positions and Reading Values with Attention" (Fig. 4) -- the
//   indexer scores cached positions with Indexer Q and Indexer K and returns a
//   list of positions; "What Full, Reindex, and Reuse Share" (Fig. 5) -- Full
//   scores every position and keeps a candidate pool wider than top-k; Reindex
//   rescores only that pool; "One Token Sequence and Causal Access" (Fig. 2) --
//   only positions <= t are candidates.
// Score (a reading of the pages): sum_h w[h] * max(0, qi[h] . ki[s]), exact in
// int32. Ranking: score descending, then position ascending.
//
// Design (B200): one cooperative launch. A "unit" is one query; a group of G
// co-resident CTAs handles one unit at a time (persistent loop when there are
// more units than groups). Each CTA scores a contiguous chunk of the unit's
// candidates into shared memory:
//   * Full mode with 32/64/128-byte keys: warp-specialised tensor-core scan.
//     A TMA warp streams key tiles of up to 256 rows into an 8-stage ring
//     (kStages), an MMA warp issues tcgen05.mma kind::i8 (keys as M = 128
//     rows, the index query's heads as N = 16) into 4 TMEM buffers, and 16
//     epilogue warps (kSel threads, two groups of 8 warps that take alternate
//     tiles) apply the ReLU and head weights to the int32 accumulators.
//     mbarriers link the roles, so the scan runs at the rate of its slowest
//     role.
//   * Reindex mode and other key widths: rows are gathered (or TMA-staged)
//     and scored with dp4a.
// Then the group finds the exact cut with a distributed radix select on a
// 36-bit order-preserving key of the score: a 12-bit log-scale digit first,
// then two 12-bit digits of the remaining bits. Each round costs one group
// barrier (an atomic counter with a bounded spin). Once the threshold digit
// holds at most kCandCap elements, they are gathered and every CTA finds the
// exact threshold score T among them with a local radix select; exact ties at
// T are cut by position through per-CTA counts. Every CTA then writes its
// selected positions at its offset, in ascending order, with no further sync.
//
// Calls with many queries take other kernels below: Full calls whose queries share
// keys (index_mq_score_kernel, index_mq_estimate_kernel, index_mq_select_kernel:
// sampled estimates, candidate bits, a tensor-core rescoring cut, the cooperative
// kernel for the queries left over), and Reindex calls with more queries than SMs
// (index_mq_select_kernel over the pool).
#include <cuda.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cstdlib>
#include <cstring>

#include "csa2_common.cuh"

namespace csa2 {

constexpr int kSel = 512;                    // threads that run the scan epilogue and the select phase
constexpr int kSelWarps = kSel / 32;
constexpr int kBpt = 4096 / kSel;            // level-0 bins per select thread
constexpr int kTcThreads = kSel + 64;        // + one TMA warp and one MMA warp
constexpr int kBins = 4096;
constexpr int kG0Stride = kBins + 32;        // a level-0 histogram buffer and its element count (word kBins)
constexpr int kCandCap = 4096;
constexpr int kStageBytes = 16384;
constexpr int kStages = 8;
constexpr int kTmemBufs = 4;
constexpr int kSmemScores = 16384;                  // scores kept in shared memory
constexpr int kCtrlInts = 32;
constexpr int kMaxG = 64;

// per-group-slot control words (persistent in the workspace; zero at first use)
enum { CTRL_BAR = 0, CTRL_EPOCH = 1, CTRL_BAR_BASE = 2, CTRL_CAND0 = 3, CTRL_CAND1 = 4 };

struct IdxParams {
    int mode;  // CSA2_FULL or CSA2_REINDEX
    int B, Tq, N, Hi, Di;
    int r[2];            // track sizes: pool P (0 = off), top-k
    int32_t* out[2];     // pool_out, topk_out
    const int32_t* q_pos;
    const int8_t* qi;
    int32_t w[16];
    const int8_t* ki;
    int64_t ki_seq_stride;
    const int32_t* pool_in;
    int P_in;
    int units, G, groups, chunk;
    int32_t* spill;      // [groups*G][chunk] scores when chunk > kSmemScores
    int local_sel;       // Reindex: every CTA of the group cuts over all of the unit's scores
    int keys_ready;      // keys and positions were complete before the previous kernel began
    // Full with queries that share keys: the sampled tiles' scores, the estimates, the
    // candidate words (one bit per position) and the units the cut leaves to the Full
    // kernel ([0] count, [1 ..] units)
    const int32_t* mq_sample;
    int64_t mq_sstride;
    int mq_tstep;
    int4* mq_est;
    const int32_t* mq_words;
    int64_t mq_wstride;
    int32_t* fb_list;
    const int32_t* unit_list;   // Full kernel: the units to take ([0] count, [1 ..] units), nullptr: all
    int rstride;         // per-unit stride of rscore
    int32_t* rscore;     // [units][rstride] published scores (local_sel)
    // L2 prefetch of the global cache rows each top-k list selects (pf_fp4 nullptr: off)
    const uint8_t* pf_fp4;
    const uint8_t* pf_scale;
    int pf_N, pf_code_bytes, pf_scale_bytes;
    int m;                   // sequence compression rate of the global entries (<= 1: one per position)
    long long wait_budget;   // SM cycles a CTA waits at a group barrier before it reports a timeout
    int skip_arrival;        // fault injection: the last CTA of a group never arrives at its first barrier
    int* ctrl;           // [slots][kCtrlInts]
    int* g0;             // [slots][3][kG0Stride]: histogram, then the element count
    int* gl;             // [slots][2 tracks][2 levels][kBins]
    int2* cand;          // [slots][2 tracks][kCandCap]
    int* pub;            // [slots][2 tracks][3][kMaxG]
    int32_t* status;
};

struct __align__(1024) IdxSmem {
    // key tiles; after a unit's scan: candidate buffers [0, 64 KB), radix histograms [64 KB, 96 KB)
    uint8_t stage[kStages][kStageBytes];
    uint8_t qtc[16 * 128];                 // index query as a tensor-core operand (16 rows)
    int sc[kSmemScores];                   // scores of this CTA's chunk, by element index
    int hist0[kBins];
    int8_t q[16 * 128];
    uint64_t full_bar[kStages];
    uint64_t empty_bar[kStages];
    uint64_t tfull_bar[kTmemBufs];
    uint64_t tempty_bar[kTmemBufs];
    uint32_t tmem_base;
    int abort;
    alignas(16) int red[8 * kSelWarps];
    alignas(16) int info[64];
    alignas(16) int wsum[4 * kSelWarps];
    int wlist_n[kSelWarps];   // entries in each warp's ordered list
    int wlist_ovf;            // some warp's list overflowed
};
constexpr int kHistlOff = 2 * (int)sizeof(int2) * kCandCap;   // byte offset of the radix histograms
constexpr int kListOff = kHistlOff + 2 * kBins * 4;            // byte offset of the per-warp ordered lists
constexpr int kListCap = 512;                                  // entries per warp
static_assert(kListOff + kSelWarps * kListCap * 4 <= (int)sizeof(((IdxSmem*)0)->stage), "select buffers");
// (a Reindex pool cut in one select per group has at most kSmemScores entries over G >= 2 CTAs)
static_assert(kSelWarps * kListCap >= kSmemScores / 2, "a Reindex chunk's positions fit the list region");
static_assert(kStages * kStageBytes % 1024 == 0, "tensor-core operand alignment");
static_assert(sizeof(IdxSmem) + 1024 <= 232448, "shared memory per block");

struct Slot {
    int* ctrl;
    int* g0;
    int* gl;
    int2* cand;
    int* pub;
};

// Radix histogram of track tr (select phase only: it overlays the key stages).
__device__ __forceinline__ int* histl(IdxSmem& S, int tr) {
    return reinterpret_cast<int*>(&S.stage[0][0] + kHistlOff) + tr * kBins;
}

// Per-warp ordered lists of the write phase (select phase only: they overlay the key stages).
__device__ __forceinline__ int* wlists(IdxSmem& S) { return reinterpret_cast<int*>(&S.stage[0][0] + kListOff); }

__device__ __forceinline__ Slot slot_of(const IdxParams& p, int group) {
    Slot s;
    s.ctrl = p.ctrl + (size_t)group * kCtrlInts;
    s.g0 = p.g0 + (size_t)group * 3 * kG0Stride;
    s.gl = p.gl + (size_t)group * 4 * kBins;
    s.cand = p.cand + (size_t)group * 2 * kCandCap;
    s.pub = p.pub + (size_t)group * 6 * kMaxG;
    return s;
}

// ------------------------------------------------------------ order key
// 12-bit log-scale bin of a non-negative magnitude: exact below 64, then 64 bins
// per octave (6 mantissa bits after the leading one).
__device__ __forceinline__ uint32_t mag_bin(uint32_t y) {
    if (y < 64u) return y;
    const int e = 31 - __clz(y);
    return 64u + (uint32_t)(e - 6) * 64u + ((y >> (e - 6)) & 63u);
}

// Strictly increasing map of an int32 score to a 36-bit key: the top 12 bits are
// the log-scale bin (2048 +- bin of the magnitude), the low 24 bits the rest of
// the magnitude, left-aligned (complemented for negative scores).
__device__ __forceinline__ uint64_t ext_key(int32_t x) {
    const uint32_t y = x >= 0 ? (uint32_t)x : (uint32_t)(-1 - x);
    const uint32_t mb = mag_bin(y);
    uint32_t sub = 0;
    if (y >= 64u) {
        const int nbits = (31 - __clz(y)) - 6;
        const uint32_t mask = (nbits > 0) ? ((1u << nbits) - 1u) : 0u;
        uint32_t low = y & mask;
        if (x < 0) low = mask - low;
        sub = (nbits > 0) ? (low << (24 - nbits)) : 0u;
    }
    const uint32_t d0 = x >= 0 ? 2048u + mb : 2047u - mb;
    return ((uint64_t)d0 << 24) | sub;
}

__device__ __forceinline__ uint32_t digit_at(uint64_t ext, int level) {
    return (uint32_t)(ext >> (24 - 12 * level)) & 4095u;
}

// Level-0 digit only (the 12-bit log-scale bin of the score).
__device__ __forceinline__ uint32_t bin0(int32_t x) {
    return x >= 0 ? 2048u + mag_bin((uint32_t)x) : 2047u - mag_bin((uint32_t)(-1 - x));
}

// The score interval [lo, hi] that maps to level-0 bin d.
__device__ __forceinline__ void bin0_interval(uint32_t d, int& lo, int& hi) {
    const bool pos = d >= 2048u;
    const uint32_t f = pos ? d - 2048u : 2047u - d;
    long long ylo, yhi;
    if (f < 64u) {
        ylo = yhi = f;
    } else {
        const int e = (int)((f - 64u) / 64u) + 6;
        const long long m = (f - 64u) % 64u;
        ylo = (64 + m) << (e - 6);
        yhi = ((64 + m + 1) << (e - 6)) - 1;
    }
    if (pos) { lo = (int)ylo; hi = (int)yhi; }
    else     { lo = (int)(-1 - yhi); hi = (int)(-1 - ylo); }
}

// ------------------------------------------------------------ select-group sync
// The select phase runs on threads [0, kSel) and synchronises on named barrier 1,
// so extra warps of the CTA (the TMA and MMA warps) need not take part.
#define CSA2_STR2(x) #x
#define CSA2_STR(x) CSA2_STR2(x)
#define CSA2_SEL_THREADS 512
static_assert(CSA2_SEL_THREADS == kSel, "named-barrier thread count");
__device__ __forceinline__ void sel_sync() { asm volatile("bar.sync 1, " CSA2_STR(CSA2_SEL_THREADS) ";" ::: "memory"); }

__device__ __forceinline__ int sel_and(int v) {
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.s32 q, %1, 0;\n\t"
        "bar.red.and.pred p, 1, " CSA2_STR(CSA2_SEL_THREADS) ", q;\n\t"
        "selp.s32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"(v)
        : "memory");
    return r;
}

// Exclusive scan over the select threads; returns the total in `total`.
__device__ __forceinline__ int sel_scan_excl(int v, int* red, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    sel_sync();
    if (lane == 31) red[warp] = x;
    sel_sync();
    if (warp == 0) {
        int s = lane < (kSel / 32) ? red[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < kSel / 32) red[32 + lane] = s;
    }
    sel_sync();
    const int warp_excl = warp ? red[32 + warp - 1] : 0;
    total = red[32 + kSel / 32 - 1];
    return warp_excl + x - v;
}

__device__ __forceinline__ int sel_sum(int v, int* red) {
    int total;
    sel_scan_excl(v, red, total);
    return total;
}

__device__ __forceinline__ int sel_min(int v, int* red) {
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    sel_sync();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    sel_sync();
    int m = red[0];
    for (int w = 1; w < kSel / 32; ++w) m = min(m, red[w]);
    return m;
}

// Group barrier over the G CTAs of a slot: the counter grows by one per CTA.
// The arrival is a release add (it publishes this CTA's earlier writes, which the
// named barrier has ordered before it) and the poll an acquire load. The wait
// ends with a failure after `budget` SM cycles (this CTA reports the timeout) or
// as soon as the status word shows a timeout another CTA reported, so one
// missing CTA costs the group one budget, not one per CTA. `skip` (fault
// injection, set from the host) makes this CTA leave without arriving.
__device__ bool group_barrier(int* counter, int target, int32_t* st, long long budget, bool skip = false) {
    sel_sync();
    int ok = 1;
    if (threadIdx.x == 0) {
        if (skip) {
            ok = 0;
        } else {
            asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(counter) : "memory");
            if (ld_acquire_gpu(counter) < target) {
                const long long t0 = clock64();
                while (ld_acquire_gpu(counter) < target) {
                    if (st != nullptr && ld_relaxed_gpu(st) == CSA2_ERR_TIMEOUT) {
                        ok = 0;
                        break;
                    }
                    if (clock64() - t0 > budget) {
                        report(st, CSA2_ERR_TIMEOUT, 1);
                        ok = 0;
                        break;
                    }
                    __nanosleep(20);
                }
            }
        }
    }
    return sel_and(ok) != 0;
}

// In a global 4096-bin histogram, find the bin holding the r-th
// largest element (1-based). Writes {bin, count above the bin, count in it}.
__device__ void find_rank_bin_global(const int* hist, int r, int* red, int* out) {
    const int t = threadIdx.x;
    int h[kBpt];
    const int4* src = reinterpret_cast<const int4*>(hist + kBpt * t);
#pragma unroll
    for (int i = 0; i < kBpt / 4; ++i) {
        int4 v = __ldcg(src + i);
        h[4 * i] = v.x; h[4 * i + 1] = v.y; h[4 * i + 2] = v.z; h[4 * i + 3] = v.w;
    }
    int s = 0;
#pragma unroll
    for (int i = 0; i < kBpt; ++i) s += h[i];
    int total;
    const int excl = sel_scan_excl(s, red, total);
    int above = total - excl - s;    // elements in bins above this thread's range
    if (above < r && r <= above + s) {
#pragma unroll
        for (int i = kBpt - 1; i >= 0; --i) {
            if (above < r && r <= above + h[i]) {
                out[0] = kBpt * t + i;
                out[1] = above;
                out[2] = h[i];
            }
            above += h[i];
        }
    }
    sel_sync();
}

// Both tracks' rank bins in one pass over a global 4096-bin histogram: for rank
// r[k] > 0 writes {bin, count above, count in bin} to out[8k..8k+2].
__device__ void find_rank_bins2(const int* hist, const int* r, int* red, int* out) {
    const int t = threadIdx.x;
    int h[kBpt];
    const int4* src = reinterpret_cast<const int4*>(hist + kBpt * t);
#pragma unroll
    for (int i = 0; i < kBpt / 4; ++i) {
        int4 v = __ldcg(src + i);
        h[4 * i] = v.x; h[4 * i + 1] = v.y; h[4 * i + 2] = v.z; h[4 * i + 3] = v.w;
    }
    int s = 0;
#pragma unroll
    for (int i = 0; i < kBpt; ++i) s += h[i];
    int total;
    const int excl = sel_scan_excl(s, red, total);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int rk = r[k];
        int above = total - excl - s;
        if (rk > 0 && above < rk && rk <= above + s) {
#pragma unroll
            for (int i = kBpt - 1; i >= 0; --i) {
                if (above < rk && rk <= above + h[i]) {
                    out[8 * k + 0] = kBpt * t + i;
                    out[8 * k + 1] = above;
                    out[8 * k + 2] = h[i];
                }
                above += h[i];
            }
        }
    }
    sel_sync();
}

// Push the non-zero bins of a shared histogram into a global one.
__device__ __forceinline__ void push_hist(const int* sh, int* gh) {
    for (int i = threadIdx.x; i < kBins; i += kSel) {
        const int v = sh[i];
        if (v) atomicAdd(gh + i, v);
    }
}

__device__ __forceinline__ int sum_above(const int* sh, int bin) {
    int s = 0;
    for (int i = threadIdx.x; i < kBins; i += kSel) s += (i > bin) ? sh[i] : 0;
    return s;
}

// Two exclusive scans at once over the select threads; totals in `total`.
__device__ __forceinline__ int2 sel_scan_excl2(int2 v, int* red, int2& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int2 x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y0 = __shfl_up_sync(0xffffffffu, x.x, o), y1 = __shfl_up_sync(0xffffffffu, x.y, o);
        if (lane >= o) { x.x += y0; x.y += y1; }
    }
    sel_sync();
    if (lane == 31) { red[2 * warp] = x.x; red[2 * warp + 1] = x.y; }
    sel_sync();
    if (warp == 0) {
        int s0 = lane < kSelWarps ? red[2 * lane] : 0, s1 = lane < kSelWarps ? red[2 * lane + 1] : 0;
#pragma unroll
        for (int o = 1; o < kSelWarps; o <<= 1) {
            const int y0 = __shfl_up_sync(0xffffffffu, s0, o), y1 = __shfl_up_sync(0xffffffffu, s1, o);
            if (lane >= o) { s0 += y0; s1 += y1; }
        }
        if (lane < kSelWarps) { red[2 * kSelWarps + 2 * lane] = s0; red[2 * kSelWarps + 2 * lane + 1] = s1; }
    }
    sel_sync();
    const int e0 = warp ? red[2 * kSelWarps + 2 * (warp - 1)] : 0, e1 = warp ? red[2 * kSelWarps + 2 * (warp - 1) + 1] : 0;
    total = make_int2(red[4 * kSelWarps - 2], red[4 * kSelWarps - 1]);
    return make_int2(e0 + x.x - v.x, e1 + x.y - v.y);
}

// The thresholds of both tracks at once. For track k (skipped when Ck = 0): the
// rk-th largest value (1-based, with multiplicity) among the values xk[0..Ck) in
// shared memory that lie in [lok, hik] (others are ignored). Radix passes of up to 8
// bits over x - lok, from the top: the select threads count the values that share the
// digits fixed so far into a 256-bin histogram per track, then warp k alone finds the
// bin holding rank rk (eight bins per lane and one suffix scan across the lanes). A
// pass costs two barriers; the histograms are double-buffered so the next pass's
// buffer is cleared during this one. A track whose chosen bin holds at most 32 values
// with bits still to resolve ranks those values directly instead.
// hist: 1088 ints ([2 buffers][2 tracks][256] and [2][32] values). The two tracks
// share every barrier. Returns {T0, need0, T1, need1}: need = how many elements
// equal to T are ranked within the first r.
static_assert(kSel == 2 * 256, "local_select2: one histogram bin of one track per select thread");
__device__ __noinline__ int4 local_select2(const int* x0, int C0, int r0, int lo0, int hi0, const int* x1, int C1,
                                           int r1, int lo1, int hi1, int* hist, int* red, int* info) {
    (void)red;
    const int t = threadIdx.x, lane = t & 31, wk = t >> 5;
    auto nbits = [](int lo, int hi) {
        const uint32_t w = (uint32_t)((long long)hi - (long long)lo);
        return w == 0u ? 0 : 32 - __clz(w);
    };
    int rem0 = C0 > 0 ? nbits(lo0, hi0) : 0, rem1 = C1 > 0 ? nbits(lo1, hi1) : 0;
    uint32_t pf0 = 0, pf1 = 0;
    int T0 = 0, T1 = 0;
    bool fin0 = false, fin1 = false;   // threshold found by ranking the last few values directly
    int* bv = hist + 1024;             // the last few values of each track
    hist[t] = 0;                       // buffer 0 (kSel = 2 tracks x 256 bins)
    sel_sync();
    int buf = 0;
#pragma unroll 1
    while (rem0 > 0 || rem1 > 0) {
        int* hb = hist + buf * 512;
        const int tk0 = min(rem0, 8), sh0 = rem0 - tk0;
        const int tk1 = min(rem1, 8), sh1 = rem1 - tk1;
        hist[(buf ^ 1) * 512 + t] = 0;   // last read before the barrier that ended the previous pass
        if (rem0 > 0) {
#pragma unroll 1
            for (int i = t; i < C0; i += kSel) {
                const int x = x0[i];
                const uint32_t v = (uint32_t)((long long)x - (long long)lo0);
                if (x >= lo0 && x <= hi0 && (uint32_t)(((uint64_t)v) >> (sh0 + tk0)) == pf0)
                    atomicAdd(&hb[(v >> sh0) & ((1u << tk0) - 1u)], 1);
            }
        }
        if (rem1 > 0) {
#pragma unroll 1
            for (int i = t; i < C1; i += kSel) {
                const int x = x1[i];
                const uint32_t v = (uint32_t)((long long)x - (long long)lo1);
                if (x >= lo1 && x <= hi1 && (uint32_t)(((uint64_t)v) >> (sh1 + tk1)) == pf1)
                    atomicAdd(&hb[256 + ((v >> sh1) & ((1u << tk1) - 1u))], 1);
            }
        }
        sel_sync();
        if (wk < 2 && (wk == 0 ? rem0 : rem1) > 0) {
            // warp wk: lane l holds bins 8l .. 8l + 7; the bin with (count above) < r <= (count above) + its count
            const int r = wk == 0 ? r0 : r1;
            const int4* h4 = reinterpret_cast<const int4*>(hb + wk * 256 + 8 * lane);
            const int4 ha = h4[0], hb4 = h4[1];
            const int hv[8] = {ha.x, ha.y, ha.z, ha.w, hb4.x, hb4.y, hb4.z, hb4.w};
            int sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) sum += hv[i];
            int incl = sum;   // this lane's bins and every higher lane's
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_down_sync(0xffffffffu, incl, o);
                if (lane + o < 32) incl += y;
            }
            int above = incl - sum;
            if (above < r && r <= incl) {
#pragma unroll
                for (int i = 7; i >= 0; --i) {
                    if (r <= above + hv[i]) {
                        info[3 * wk] = 8 * lane + i;
                        info[3 * wk + 1] = above;
                        info[3 * wk + 2] = hv[i];
                        break;
                    }
                    above += hv[i];
                }
            }
        }
        if (t == 0) { info[6] = 0; info[7] = 0; }
        sel_sync();
        if (rem0 > 0) { r0 -= info[1]; pf0 = (pf0 << tk0) | (uint32_t)info[0]; rem0 = sh0; }
        if (rem1 > 0) { r1 -= info[4]; pf1 = (pf1 << tk1) | (uint32_t)info[3]; rem1 = sh1; }
        const bool bf0 = rem0 > 0 && info[2] <= 32, bf1 = rem1 > 0 && info[5] <= 32;
        if (bf0 || bf1) {
            if (bf0) {
#pragma unroll 1
                for (int i = t; i < C0; i += kSel) {
                    const int x = x0[i];
                    const uint32_t v = (uint32_t)((long long)x - (long long)lo0);
                    if (x >= lo0 && x <= hi0 && (uint32_t)(((uint64_t)v) >> rem0) == pf0) bv[atomicAdd(&info[6], 1) & 31] = x;
                }
            }
            if (bf1) {
#pragma unroll 1
                for (int i = t; i < C1; i += kSel) {
                    const int x = x1[i];
                    const uint32_t v = (uint32_t)((long long)x - (long long)lo1);
                    if (x >= lo1 && x <= hi1 && (uint32_t)(((uint64_t)v) >> rem1) == pf1)
                        bv[32 + (atomicAdd(&info[7], 1) & 31)] = x;
                }
            }
            sel_sync();
            // warp 0 ranks track 0's values, warp 1 track 1's: the value with
            // (#larger) < r <= (#larger or equal) is the threshold
            if ((wk == 0 && bf0) || (wk == 1 && bf1)) {
                const int m = min(info[6 + wk], 32);
                const int r = wk == 0 ? r0 : r1;
                const int vi = lane < m ? bv[32 * wk + lane] : 0;
                int gt = 0, ge = 0;
#pragma unroll 1
                for (int j = 0; j < m; ++j) {
                    const int vj = __shfl_sync(0xffffffffu, vi, j);
                    gt += vj > vi;
                    ge += vj >= vi;
                }
                if (lane < m && gt < r && r <= ge) { info[8 + 2 * wk] = vi; info[9 + 2 * wk] = r - gt; }
            }
            sel_sync();
            if (bf0) { T0 = info[8]; r0 = info[9]; fin0 = true; rem0 = 0; }
            if (bf1) { T1 = info[10]; r1 = info[11]; fin1 = true; rem1 = 0; }
        }
        buf ^= 1;
    }
    return make_int4(fin0 ? T0 : (int)((long long)lo0 + (long long)pf0), r0,
                     fin1 ? T1 : (int)((long long)lo1 + (long long)pf1), r1);
}

// ------------------------------------------------------------ select + write
// The select code runs once per unit, straight after a scan that has streamed the
// keys through L2, so its instructions are fetched cold: it is kept small. Each
// pass over the chunk's scores is one out-of-line loop, the per-track bookkeeping
// runs in plain loops, and every digit prefix is turned into the interval of
// scores it covers, so the common passes only compare scores with bounds.

// Track states (identical in every CTA of a group).
enum { TS_OFF = 0, TS_ALL = 1, TS_RADIX = 2, TS_CAND = 3, TS_EQ = 4, TS_FIN_CAND = 5, TS_FIN_EQ = 6 };

struct UnitCtx {
    int u, t, lo, my_n, n_all, cta, j, epoch;
    const int32_t* pool;   // Reindex: the unit's pool (positions of the elements)
};

// Select state of one track (pool or top-k); the same in every CTA of a group.
struct Track {
    int state;        // TS_*
    int rrem;         // rank still to find inside the current prefix
    int C;            // elements of the whole group inside the current prefix
    int level;        // index of the last fixed digit (0: the level-0 bin)
    int above;        // this CTA's elements above the current prefix
    int lo, hi;       // interval of scores whose key starts with the prefix
    uint64_t prefix;  // the fixed digits
};

// Scores whose order key starts with `prefix` (digits 0..level) form an interval,
// since the key is strictly increasing in the score. Bisection inside [lo, hi],
// the interval of the enclosing prefix.
__device__ void prefix_interval(int level, uint64_t prefix, int& lo, int& hi) {
    const int sh = 24 - 12 * level;
    long long a = lo, b = (long long)hi + 1;   // first score with key prefix >= prefix
    while (a < b) {
        const long long m = (a + b) >> 1;
        if ((ext_key((int)m) >> sh) >= prefix) b = m; else a = m + 1;
    }
    const long long first = a;
    b = (long long)hi + 1;                     // first score with key prefix > prefix
    while (a < b) {
        const long long m = (a + b) >> 1;
        if ((ext_key((int)m) >> sh) > prefix) b = m; else a = m + 1;
    }
    lo = (int)first;
    hi = (int)(a - 1);
}

// The chunk's scores: element e sits at sc[e], in shared memory or, for chunks
// longer than kSmemScores, in this CTA's spill area (padding past n is ignored).
// Each warp walks one contiguous range of 32-element steps (lane = element in
// the step), so a warp meets its elements in position order and the warps'
// ranges follow each other.
template <bool kSpill>
__device__ __forceinline__ int ld_score(const int* sc, int e) {
    if constexpr (kSpill) return __ldcg(sc + e);
    else return sc[e];
}

__device__ __forceinline__ void warp_steps(int n, int& s0, int& s1) {
    const int nstep = (n + 31) >> 5;
    const int spw = (nstep + kSelWarps - 1) / kSelWarps;
    s0 = min(nstep, (threadIdx.x >> 5) * spw);
    s1 = min(nstep, s0 + spw);
}

__device__ __forceinline__ int4 warp_sum4(int4 v) {
    return make_int4(__reduce_add_sync(0xffffffffu, v.x), __reduce_add_sync(0xffffffffu, v.y),
                     __reduce_add_sync(0xffffffffu, v.z), __reduce_add_sync(0xffffffffu, v.w));
}

// Totals of two int4 over the select threads (two barriers).
__device__ __forceinline__ void sel_total8(int4& a, int4& b, int* red) {
    a = warp_sum4(a);
    b = warp_sum4(b);
    sel_sync();
    int4* r4 = reinterpret_cast<int4*>(red);
    if ((threadIdx.x & 31) == 0) { r4[2 * (threadIdx.x >> 5)] = a; r4[2 * (threadIdx.x >> 5) + 1] = b; }
    sel_sync();
    a = make_int4(0, 0, 0, 0);
    b = a;
#pragma unroll 1
    for (int w = 0; w < kSelWarps; ++w) {
        const int4 x = r4[2 * w], y = r4[2 * w + 1];
        a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
        b.x += y.x; b.y += y.y; b.z += y.z; b.w += y.w;
    }
}

// Candidates of both tracks (scores in [lo0, hi0] / [lo1, hi1]; lo > hi = off)
// into lbuf[0..) and lbuf[kCandCap..) as (score, element index + base). A warp
// reserves room once per step that holds candidates; the order is free.
// The same pass appends to the warp's ordered list (lists + warp * kListCap)
// every element that is above a track's interval or inside it, as
// e | flags << 28 (flag bits: above 0, inside 0, above 1, inside 1), and stores
// the list lengths in wn; a list longer than kListCap sets *ovf. kCands = false
// builds the lists only.
template <bool kSpill, bool kCands = true>
__device__ __forceinline__ void gather_cands(const int* sc, int n, int base, int lo0, int hi0, int lo1, int hi1,
                                             int2* lbuf, int* lcnt, int* lists, int* wn, int* ovf,
                                             int* above = nullptr) {
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const unsigned below = (1u << lane) - 1u;
    const bool on0 = lo0 <= hi0, on1 = lo1 <= hi1;
    int* list = lists + wp * kListCap;
    int ln = 0, na0 = 0, na1 = 0;
    int s0, s1;
    warp_steps(n, s0, s1);
#pragma unroll 4
    for (int st = s0; st < s1; ++st) {
        const int e = st * 32 + lane;
        const int x = e < n ? ld_score<kSpill>(sc, e) : 0;
        const bool m0 = e < n && x >= lo0 && x <= hi0, m1 = e < n && x >= lo1 && x <= hi1;
        const bool a0 = e < n && on0 && x > hi0, a1 = e < n && on1 && x > hi1;
        const unsigned f = (a0 ? 1u : 0u) | (m0 ? 2u : 0u) | (a1 ? 4u : 0u) | (m1 ? 8u : 0u);
        na0 += a0;
        na1 += a1;
        const unsigned bk = __ballot_sync(0xffffffffu, f != 0u);
        if (bk) {
            const int at = ln + __popc(bk & below);
            if (f != 0u && at < kListCap) list[at] = e | (int)(f << 28);
            ln += __popc(bk);
        }
        if (!kCands) continue;
        const unsigned b0 = __ballot_sync(0xffffffffu, m0), b1 = __ballot_sync(0xffffffffu, m1);
        if ((b0 | b1) == 0u) continue;
        int w0 = 0, w1 = 0;
        if (lane == 0) {
            w0 = b0 ? atomicAdd(lcnt, __popc(b0)) : 0;
            w1 = b1 ? atomicAdd(lcnt + 1, __popc(b1)) : 0;
        }
        w0 = __shfl_sync(0xffffffffu, w0, 0) + __popc(b0 & below);
        w1 = __shfl_sync(0xffffffffu, w1, 0) + __popc(b1 & below);
        const int2 cv = make_int2(x, base + e);
        if (m0 && w0 < kCandCap) lbuf[w0] = cv;
        if (m1 && w1 < kCandCap) lbuf[kCandCap + w1] = cv;
    }
    if (above != nullptr) {   // this CTA's elements above each interval (above[] zeroed by the caller)
        na0 = __reduce_add_sync(0xffffffffu, na0);
        na1 = __reduce_add_sync(0xffffffffu, na1);
        if (lane == 0) { atomicAdd(above, na0); atomicAdd(above + 1, na1); }
    }
    if (lane == 0) {
        wn[wp] = min(ln, kListCap);
        if (ln > kListCap) *ovf = 1;
    }
}

// The ordered lists and the counts above each interval, as in gather_cands with
// kCands = false, two elements per lane per step: lane l holds elements 2l and 2l + 1
// of a 64-element step, and ballots over both keep the entries in position order.
template <bool kSpill>
__device__ __forceinline__ void gather_lists2(const int* sc, int n, int lo0, int hi0, int lo1, int hi1, int* lists,
                                              int* wn, int* ovf, int* above) {
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const unsigned below = (1u << lane) - 1u;
    const bool on0 = lo0 <= hi0, on1 = lo1 <= hi1;
    int* list = lists + wp * kListCap;
    int ln = 0, na0 = 0, na1 = 0;
    const int nstep = (n + 63) >> 6;
    const int spw = (nstep + kSelWarps - 1) / kSelWarps;
    const int s0 = min(nstep, wp * spw), s1 = min(nstep, s0 + spw);
    // kIn steps' loads are issued before any of their list stores (which the compiler
    // cannot tell apart from the scores, so it would not move a later load above them);
    // spilled scores come from L2, so more of them are in flight
    constexpr int kIn = kSpill ? 16 : 4;
#pragma unroll 1
    for (int st0 = s0; st0 < s1; st0 += kIn) {
        int2 xv[kIn];
#pragma unroll
        for (int u4 = 0; u4 < kIn; ++u4) {
            const int e = (st0 + u4) * 64 + 2 * lane;
            xv[u4] = make_int2(0, 0);
            if (st0 + u4 < s1) {
                if constexpr (kSpill) xv[u4] = __ldcg(reinterpret_cast<const int2*>(sc + e));
                else xv[u4] = *reinterpret_cast<const int2*>(sc + e);
            }
        }
#pragma unroll
        for (int u4 = 0; u4 < kIn; ++u4) {
            if (st0 + u4 >= s1) break;   // warp-uniform
            const int e = (st0 + u4) * 64 + 2 * lane;
            unsigned f[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int x = q == 0 ? xv[u4].x : xv[u4].y;
                const bool ok = e + q < n;
                const bool a0 = ok && on0 && x > hi0, m0 = ok && x >= lo0 && x <= hi0;
                const bool a1 = ok && on1 && x > hi1, m1 = ok && x >= lo1 && x <= hi1;
                f[q] = (a0 ? 1u : 0u) | (m0 ? 2u : 0u) | (a1 ? 4u : 0u) | (m1 ? 8u : 0u);
                na0 += a0;
                na1 += a1;
            }
            const unsigned k0 = __ballot_sync(0xffffffffu, f[0] != 0u), k1 = __ballot_sync(0xffffffffu, f[1] != 0u);
            if ((k0 | k1) == 0u) continue;
            const int at = ln + __popc(k0 & below) + __popc(k1 & below);
            if (f[0] != 0u && at < kListCap) list[at] = e | (int)(f[0] << 28);
            const int at1 = at + (f[0] != 0u ? 1 : 0);
            if (f[1] != 0u && at1 < kListCap) list[at1] = (e + 1) | (int)(f[1] << 28);
            ln += __popc(k0) + __popc(k1);
        }
    }
    if (above != nullptr) {   // this CTA's elements above each interval (above[] zeroed by the caller)
        na0 = __reduce_add_sync(0xffffffffu, na0);
        na1 = __reduce_add_sync(0xffffffffu, na1);
        if (lane == 0) { atomicAdd(above, na0); atomicAdd(above + 1, na1); }
    }
    if (lane == 0) {
        wn[wp] = min(ln, kListCap);
        if (ln > kListCap) *ovf = 1;
    }
}

// Candidates of both tracks (list entries inside a track's interval) from the warps'
// ordered lists into lbuf[0..) and lbuf[kCandCap..) as (score, element index + base);
// counts to lcnt[0..1]. Valid when no list overflowed. wsum: 2 * kSelWarps ints.
template <bool kSpill>
__device__ __forceinline__ void cands_from_lists(const int* sc, int base, const int* lists, const int* wn,
                                                 int2* lbuf, int* lcnt, int* wsum) {
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const unsigned below = (1u << lane) - 1u;
    const int* list = lists + wp * kListCap;
    const int n = wn[wp];
    int c0 = 0, c1 = 0;
#pragma unroll 1
    for (int i = lane; i < n; i += 32) {
        const unsigned f = (unsigned)list[i] >> 28;
        c0 += (f & 2u) != 0u;
        c1 += (f & 8u) != 0u;
    }
    c0 = __reduce_add_sync(0xffffffffu, c0);
    c1 = __reduce_add_sync(0xffffffffu, c1);
    if (lane == 0) { wsum[2 * wp] = c0; wsum[2 * wp + 1] = c1; }
    sel_sync();
    int o0 = 0, o1 = 0, t0 = 0, t1 = 0;
#pragma unroll 1
    for (int w = 0; w < kSelWarps; ++w) {
        const int a = wsum[2 * w], b = wsum[2 * w + 1];
        o0 += w < wp ? a : 0;
        o1 += w < wp ? b : 0;
        t0 += a;
        t1 += b;
    }
    if (threadIdx.x == 0) { lcnt[0] = t0; lcnt[1] = t1; }
#pragma unroll 1
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        const int ent = i < n ? list[i] : 0;
        const unsigned f = i < n ? ((unsigned)ent >> 28) : 0u;
        const bool in0 = (f & 2u) != 0u, in1 = (f & 8u) != 0u;
        const unsigned b0 = __ballot_sync(0xffffffffu, in0), b1 = __ballot_sync(0xffffffffu, in1);
        if (in0 || in1) {
            const int e = ent & 0x0FFFFFFF;
            const int2 cv = make_int2(ld_score<kSpill>(sc, e), base + e);
            if (in0) { const int k = o0 + __popc(b0 & below); if (k < kCandCap) lbuf[k] = cv; }
            if (in1) { const int k = o1 + __popc(b1 & below); if (k < kCandCap) lbuf[kCandCap + k] = cv; }
        }
        o0 += __popc(b0);
        o1 += __popc(b1);
    }
}

// Scores of the list entries that carry flag bit `fb` (inside a track's interval),
// in list order, to out[0..); returns their number. Valid when no list overflowed.
// wsum: kSelWarps ints.
__device__ __forceinline__ int vals_from_lists(const int* sc, const int* lists, const int* wn, unsigned fb, int* out,
                                               int* wsum) {
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const unsigned below = (1u << lane) - 1u;
    const int* list = lists + wp * kListCap;
    const int n = wn[wp];
    int c = 0;
#pragma unroll 1
    for (int i = lane; i < n; i += 32) c += (((unsigned)list[i] >> 28) & fb) != 0u;
    c = __reduce_add_sync(0xffffffffu, c);
    if (lane == 0) wsum[wp] = c;
    sel_sync();
    int o = 0, tot = 0;
#pragma unroll 1
    for (int w = 0; w < kSelWarps; ++w) {
        const int a = wsum[w];
        o += w < wp ? a : 0;
        tot += a;
    }
#pragma unroll 1
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        const int ent = i < n ? list[i] : 0;
        const bool in = i < n && (((unsigned)ent >> 28) & fb) != 0u;
        const unsigned b = __ballot_sync(0xffffffffu, in);
        if (in) out[o + __popc(b & below)] = sc[ent & 0x0FFFFFFF];
        o += __popc(b);
    }
    sel_sync();   // wsum is free again
    return tot;
}

// Histogram of digit `lv` over the elements in [lo_t, hi_t] (they share digits 0..lv-1).
// Spilled scores are read four steps at a time, all loads in flight before the first
// use (the histogram's atomics would otherwise keep the next load from issuing).
template <bool kSpill>
__device__ __noinline__ void radix_hist(const int* sc, int n, int lo_t, int hi_t, int lv, int* hist) {
    int s0, s1;
    warp_steps(n, s0, s1);
    const int lane = threadIdx.x & 31;
    if constexpr (kSpill) {
#pragma unroll 1
        for (int st = s0; st < s1; st += 4) {
            int xs[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int e = (st + q) * 32 + lane;
                xs[q] = (st + q < s1 && e < n) ? __ldcg(sc + e) : 0;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int e = (st + q) * 32 + lane;
                if (st + q < s1 && e < n && xs[q] >= lo_t && xs[q] <= hi_t)
                    atomicAdd(&hist[digit_at(ext_key(xs[q]), lv)], 1);
            }
        }
    } else {
#pragma unroll 1
        for (int st = s0; st < s1; ++st) {
            const int e = st * 32 + lane;
            const int x = e < n ? ld_score<kSpill>(sc, e) : 0;
            if (e < n && x >= lo_t && x <= hi_t) atomicAdd(&hist[digit_at(ext_key(x), lv)], 1);
        }
    }
}

// Number of this thread's elements in [lo_t, hi_t].
template <bool kSpill>
__device__ __noinline__ int count_range(const int* sc, int n, int lo_t, int hi_t) {
    int s0, s1, cnt = 0;
    warp_steps(n, s0, s1);
#pragma unroll 4
    for (int st = s0; st < s1; ++st) {
        const int e = st * 32 + (threadIdx.x & 31);
        const int x = e < n ? ld_score<kSpill>(sc, e) : 0;
        cnt += (e < n && x >= lo_t && x <= hi_t);
    }
    return cnt;
}

// Where one track's cut leaves this CTA: elements above T are taken, and so are the
// first `quota` elements equal to T in position order (all = take every element).
// The taken elements go to out[base ..] in position order.
struct ListCut {
    int T, all, quota, base, r;
    int32_t* out;      // nullptr: track off
    int32_t* status;   // status word (reports of the range-checked build)
};

// The global cache rows of one sequence that its top-k list selects are pulled into
// L2 as the list is written, so that the attention launch after the indexer
// gathers them from L2 (fp4 nullptr: off).
struct RowPrefetch {
    const uint8_t* fp4;     // the sequence's codes [N][code_bytes]
    const uint8_t* scale;   // the sequence's scales [N][scale_bytes]
    int code_bytes, scale_bytes;
};

__device__ __forceinline__ RowPrefetch row_prefetch(const IdxParams& p, int u) {
    RowPrefetch f{nullptr, nullptr, 0, 0};
    if (p.pf_fp4 != nullptr) {
        const size_t b = (size_t)(u / p.Tq);
        f.fp4 = p.pf_fp4 + b * p.pf_N * p.pf_code_bytes;
        f.scale = p.pf_scale + b * p.pf_N * p.pf_scale_bytes;
        f.code_bytes = p.pf_code_bytes;
        f.scale_bytes = p.pf_scale_bytes;
    }
    return f;
}

__device__ __forceinline__ void prefetch_row(const RowPrefetch& f, int pos) {
    if (f.fp4 == nullptr || pos < 0) return;
    asm volatile("prefetch.global.L2 [%0];" ::"l"(f.fp4 + (size_t)pos * f.code_bytes));
    asm volatile("prefetch.global.L2 [%0];" ::"l"(f.scale + (size_t)pos * f.scale_bytes));
}

__device__ __forceinline__ void take_flags(int x, bool ok, const ListCut& c, bool& g, bool& e) {
    g = ok && c.out != nullptr && (c.all || x > c.T);
    e = ok && c.out != nullptr && !c.all && x == c.T;
}

// Ordered write of both tracks: pass 1 counts per warp, pass 2 walks the same
// ranges with running counts and ballots for the ranks inside a step.
template <bool kSpill>
__device__ __forceinline__ void write_lists(const int* sc, int n, int base, const int32_t* pool, ListCut c0,
                                         ListCut c1, int* wsum, RowPrefetch pf) {
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const unsigned below = (1u << lane) - 1u;
    int s0, s1;
    warp_steps(n, s0, s1);
    int4 cnt = make_int4(0, 0, 0, 0);   // gt0, eq0, gt1, eq1
#pragma unroll 4
    for (int st = s0; st < s1; ++st) {
        const int e = st * 32 + lane;
        const int x = e < n ? ld_score<kSpill>(sc, e) : 0;
        bool g, q;
        take_flags(x, e < n, c0, g, q);
        cnt.x += g; cnt.y += q;
        take_flags(x, e < n, c1, g, q);
        cnt.z += g; cnt.w += q;
    }
    cnt = warp_sum4(cnt);
    int4* w4 = reinterpret_cast<int4*>(wsum);
    if (lane == 0) w4[wp] = cnt;
    sel_sync();
    int rg0 = 0, re0 = 0, rg1 = 0, re1 = 0;
#pragma unroll 1
    for (int w = 0; w < wp; ++w) {
        const int4 a = w4[w];
        rg0 += a.x; re0 += a.y; rg1 += a.z; re1 += a.w;
    }
#pragma unroll 4
    for (int st = s0; st < s1; ++st) {
        const int e = st * 32 + lane;
        const int x = e < n ? ld_score<kSpill>(sc, e) : 0;
        bool g0, q0, g1, q1;
        take_flags(x, e < n, c0, g0, q0);
        take_flags(x, e < n, c1, g1, q1);
        const unsigned bg0 = __ballot_sync(0xffffffffu, g0), bq0 = __ballot_sync(0xffffffffu, q0);
        const unsigned bg1 = __ballot_sync(0xffffffffu, g1), bq1 = __ballot_sync(0xffffffffu, q1);
        if ((bg0 | bq0 | bg1 | bq1) == 0u) continue;
        const int og0 = rg0 + __popc(bg0 & below), oq0 = re0 + __popc(bq0 & below);
        const int og1 = rg1 + __popc(bg1 & below), oq1 = re1 + __popc(bq1 & below);
        const bool t0 = g0 || (q0 && oq0 < c0.quota), t1 = g1 || (q1 && oq1 < c1.quota);
        if (t0 || t1) {
            const int pos = pool ? pool[base + e] : base + e;
            if (t0) { const int k = c0.base + og0 + min(oq0, c0.quota); if (CSA2_GUARD((unsigned)k < (unsigned)c0.r, c0.status, 2201)) { c0.out[k] = pos; } }
            if (t1) { const int k = c1.base + og1 + min(oq1, c1.quota); if (CSA2_GUARD((unsigned)k < (unsigned)c1.r, c1.status, 2202)) { c1.out[k] = pos; prefetch_row(pf, pos); } }
        }
        rg0 += __popc(bg0); re0 += __popc(bq0); rg1 += __popc(bg1); re1 += __popc(bq1);
    }
}

// Ordered write of both tracks from the warps' ordered lists (built by
// gather_cands with the tracks' final intervals): an entry above a track's
// interval is taken, one inside it is taken if its score is above T, or equal to
// T within the quota. Same ranks as write_lists, over ~P/G entries instead of the
// whole chunk.
template <bool kSpill>
__device__ __forceinline__ void write_from_lists(const int* sc, int base, const int32_t* pool, const int* lists,
                                                 const int* wn, ListCut c0, ListCut c1, int* wsum, RowPrefetch pf) {
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const unsigned below = (1u << lane) - 1u;
    const int* list = lists + wp * kListCap;
    const int n = wn[wp];
    auto flags = [&](int ent, bool ok, bool& g0, bool& q0, bool& g1, bool& q1) {
        const unsigned f = ok ? ((unsigned)ent >> 28) : 0u;
        const int x = (f & 10u) ? ld_score<kSpill>(sc, ent & 0x0FFFFFFF) : 0;
        g0 = c0.out && ((f & 1u) || ((f & 2u) && x > c0.T));
        q0 = c0.out && (f & 2u) && x == c0.T;
        g1 = c1.out && ((f & 4u) || ((f & 8u) && x > c1.T));
        q1 = c1.out && (f & 8u) && x == c1.T;
    };
    int4 cnt = make_int4(0, 0, 0, 0);   // gt0, eq0, gt1, eq1
#pragma unroll 1
    for (int i = lane; i < n; i += 32) {
        bool g0, q0, g1, q1;
        flags(list[i], true, g0, q0, g1, q1);
        cnt.x += g0; cnt.y += q0; cnt.z += g1; cnt.w += q1;
    }
    cnt = warp_sum4(cnt);
    int4* w4 = reinterpret_cast<int4*>(wsum);
    if (lane == 0) w4[wp] = cnt;
    sel_sync();
    int rg0 = 0, re0 = 0, rg1 = 0, re1 = 0;
#pragma unroll 1
    for (int w = 0; w < wp; ++w) {
        const int4 a = w4[w];
        rg0 += a.x; re0 += a.y; rg1 += a.z; re1 += a.w;
    }
#pragma unroll 1
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        const int ent = i < n ? list[i] : 0;
        bool g0, q0, g1, q1;
        flags(ent, i < n, g0, q0, g1, q1);
        const unsigned bg0 = __ballot_sync(0xffffffffu, g0), bq0 = __ballot_sync(0xffffffffu, q0);
        const unsigned bg1 = __ballot_sync(0xffffffffu, g1), bq1 = __ballot_sync(0xffffffffu, q1);
        const int og0 = rg0 + __popc(bg0 & below), oq0 = re0 + __popc(bq0 & below);
        const int og1 = rg1 + __popc(bg1 & below), oq1 = re1 + __popc(bq1 & below);
        const bool t0 = g0 || (q0 && oq0 < c0.quota), t1 = g1 || (q1 && oq1 < c1.quota);
        if (t0 || t1) {
            const int e = base + (ent & 0x0FFFFFFF);
            const int pos = pool ? pool[e] : e;
            if (t0) { const int k = c0.base + og0 + min(oq0, c0.quota); if (CSA2_GUARD((unsigned)k < (unsigned)c0.r, c0.status, 2201)) { c0.out[k] = pos; } }
            if (t1) { const int k = c1.base + og1 + min(oq1, c1.quota); if (CSA2_GUARD((unsigned)k < (unsigned)c1.r, c1.status, 2202)) { c1.out[k] = pos; prefetch_row(pf, pos); } }
        }
        rg0 += __popc(bg0); re0 += __popc(bq0); rg1 += __popc(bg1); re1 += __popc(bq1);
    }
}

// Exact pool/top-k cut for one unit and the write of this CTA's selected
// positions. Runs on threads [0, kSel). `sc` holds the chunk's scores (element
// index order) and S.hist0 their level-0 histogram. The two tracks (pool P and
// top-k) share every pass and every group barrier. Returns false on a timeout.
template <bool kSpill>
__device__ __forceinline__ bool select_unit(const IdxParams& p, IdxSmem& S, const Slot& sl, const UnitCtx& c,
                                         int& bar_target, const int* sc) {
    const int tid = threadIdx.x;
    const bool full = p.mode == CSA2_FULL;
    const int lo = c.lo, my_n = c.my_n;

    // ---- step 0: histogram of level 0; zero the buffers the next steps use
    int* g0cur = sl.g0 + ((c.epoch + c.j) % 3) * kG0Stride;
    int* g0nxt = sl.g0 + ((c.epoch + c.j + 1) % 3) * kG0Stride;
    push_hist(S.hist0, g0cur);
    if (!full && tid == 0 && my_n > 0) atomicAdd(g0cur + kBins, my_n);   // the group's element count
    {
        const int per = (kBins + p.G - 1) / p.G;
        const int zlo = c.cta * per, zhi = min(kBins, zlo + per);
#pragma unroll 1
        for (int i = zlo + tid; i < zhi; i += kSel) {
            g0nxt[i] = 0;
            sl.gl[i] = 0; sl.gl[kBins + i] = 0; sl.gl[2 * kBins + i] = 0; sl.gl[3 * kBins + i] = 0;
        }
        if (c.cta == 0 && tid == 0) { sl.ctrl[CTRL_CAND0] = 0; sl.ctrl[CTRL_CAND1] = 0; g0nxt[kBins] = 0; }
    }
    bar_target += p.G;
    if (!group_barrier(sl.ctrl + CTRL_BAR, bar_target, p.status, p.wait_budget,
                       p.skip_arrival && c.cta == p.G - 1))
        return false;
    CSA2_TRACE(3);   // histograms exchanged

    const int n_total = full ? c.n_all : min(max(__ldcg(g0cur + kBins), 0), p.P_in);
    Track tk[2];
    int rq[2];
#pragma unroll
    for (int tr = 0; tr < 2; ++tr) {
        tk[tr] = Track{TS_OFF, 0, 0, 0, 0, 1, 0, 0};
        const int r = p.r[tr];
        rq[tr] = 0;
        if (r <= 0) continue;
        if (n_total <= r) { tk[tr].state = TS_ALL; continue; }
        rq[tr] = r;
    }
    if (rq[0] > 0 || rq[1] > 0) {
        find_rank_bins2(g0cur, rq, S.red, S.info);
#pragma unroll
        for (int tr = 0; tr < 2; ++tr) {
            if (rq[tr] <= 0) continue;
            Track& k = tk[tr];
            const int d = S.info[8 * tr + 0];
            k.rrem = rq[tr] - S.info[8 * tr + 1];
            k.C = S.info[8 * tr + 2];
            k.prefix = (uint64_t)d;
            bin0_interval((uint32_t)d, k.lo, k.hi);
            k.state = (k.C <= kCandCap) ? TS_CAND : TS_RADIX;
        }
        // this CTA's elements above the threshold bin: counted by the candidate gather,
        // or here from the local histogram for a track that goes to the radix rounds
        if (tk[0].state == TS_RADIX || tk[1].state == TS_RADIX) {
            int a0 = 0, a1 = 0;
            const int d0 = S.info[0], d1 = S.info[8];
#pragma unroll 1
            for (int i = tid; i < kBins; i += kSel) {
                const int v = S.hist0[i];
                a0 += (rq[0] > 0 && i > d0) ? v : 0;
                a1 += (rq[1] > 0 && i > d1) ? v : 0;
            }
            int4 ta = make_int4(a0, a1, 0, 0), tb = make_int4(0, 0, 0, 0);
            sel_total8(ta, tb, S.red);
            if (tk[0].state == TS_RADIX) tk[0].above = ta.x;
            if (tk[1].state == TS_RADIX) tk[1].above = ta.y;
        }
    }

    CSA2_TRACE(4);   // threshold bins found
    int list_tracks = 0;   // tracks whose final intervals the ordered lists hold (bit per track)
    // ---- rounds until every track knows its cut (usually one)
#pragma unroll 1
    while (true) {
        bool any = false;
        const bool g0on = tk[0].state == TS_CAND, g1on = tk[1].state == TS_CAND;
        if (g0on || g1on) {
            any = true;
            int2* lbuf = reinterpret_cast<int2*>(&S.stage[0][0]);
            int* lcnt = S.info + 40;
            const bool lvl0 = tk[0].level == 0 && tk[1].level == 0;   // "above" counts are complete at level 0
            if (tid == 0) { lcnt[0] = 0; lcnt[1] = 0; S.wlist_ovf = 0; S.info[48] = 0; S.info[49] = 0; }
            sel_sync();
            const int glo0 = g0on ? tk[0].lo : 1, ghi0 = g0on ? tk[0].hi : 0;
            const int glo1 = g1on ? tk[1].lo : 1, ghi1 = g1on ? tk[1].hi : 0;
            gather_lists2<kSpill>(sc, my_n, glo0, ghi0, glo1, ghi1, wlists(S), S.wlist_n, &S.wlist_ovf,
                                  lvl0 ? S.info + 48 : nullptr);
            list_tracks = (g0on ? 1 : 0) | (g1on ? 2 : 0);   // a gather rebuilds the lists
            sel_sync();
            CSA2_TRACE(5);   // ordered lists built
            if (S.wlist_ovf == 0) {
                cands_from_lists<kSpill>(sc, lo, wlists(S), S.wlist_n, lbuf, lcnt, S.wsum);
            } else {   // a list overflowed: gather the candidates by reservation
                gather_cands<kSpill, true>(sc, my_n, lo, glo0, ghi0, glo1, ghi1, lbuf, lcnt, wlists(S), S.wlist_n,
                                           &S.wlist_ovf);
            }
            sel_sync();
            if (lvl0) {
                if (g0on) tk[0].above = S.info[48];
                if (g1on) tk[1].above = S.info[49];
            }
            if (tid == 0 || tid == 32) {
                const int tr = tid >> 5;
                const bool on = tr == 0 ? g0on : g1on;
                const int n_mine = min(lcnt[tr], kCandCap);
                S.info[44 + tr] = (on && n_mine) ? atomicAdd(sl.ctrl + CTRL_CAND0 + tr, n_mine) : 0;
                S.info[46 + tr] = on ? n_mine : 0;
                if (on) sl.pub[(tr * 3 + 0) * kMaxG + c.cta] = tk[tr].above;
            }
            sel_sync();
#pragma unroll
            for (int tr = 0; tr < 2; ++tr) {
                const int n_mine = S.info[46 + tr], gbase = S.info[44 + tr];
#pragma unroll 1
                for (int i = tid; i < n_mine; i += kSel)
                    if ((unsigned)(gbase + i) < (unsigned)kCandCap) sl.cand[tr * kCandCap + gbase + i] = lbuf[tr * kCandCap + i];
            }
        }
#pragma unroll
        for (int tr = 0; tr < 2; ++tr) {
            Track& k = tk[tr];
            if (k.state == TS_RADIX) {
                // histogram of the next digit over own elements inside the prefix
                any = true;
                int* hl = histl(S, tr);
#pragma unroll 1
                for (int i = tid; i < kBins; i += kSel) hl[i] = 0;
                sel_sync();
                radix_hist<kSpill>(sc, my_n, k.lo, k.hi, k.level + 1, hl);
                sel_sync();
                push_hist(hl, sl.gl + (2 * tr + k.level) * kBins);
            } else if (k.state == TS_EQ) {
                // the prefix is the whole key: the score is exact; count own ties
                any = true;
                const int eq = sel_sum(count_range<kSpill>(sc, my_n, k.lo, k.hi), S.red);
                if (tid == 0) {
                    sl.pub[(tr * 3 + 0) * kMaxG + c.cta] = k.above;
                    sl.pub[(tr * 3 + 1) * kMaxG + c.cta] = eq;
                }
            }
        }
        if (!any) break;
        bar_target += p.G;
        if (!group_barrier(sl.ctrl + CTRL_BAR, bar_target, p.status, p.wait_budget)) return false;
        CSA2_TRACE(7);   // candidates exchanged
        bool pending = false;
#pragma unroll
        for (int tr = 0; tr < 2; ++tr) {
            Track& k = tk[tr];
            if (k.state == TS_RADIX) {
                const int lv = k.level + 1;
                find_rank_bin_global(sl.gl + (2 * tr + (lv - 1)) * kBins, k.rrem, S.red, S.info + 8 * tr);
                const int d = S.info[8 * tr + 0];
                k.rrem -= S.info[8 * tr + 1];
                k.C = S.info[8 * tr + 2];
                k.prefix = (k.prefix << 12) | (uint64_t)d;
                k.level = lv;
                k.above += sel_sum(sum_above(histl(S, tr), d), S.red);
                prefix_interval(lv, k.prefix, k.lo, k.hi);
                k.state = (k.C <= kCandCap) ? TS_CAND : (lv < 2 ? TS_RADIX : TS_EQ);
                pending = true;
            } else if (k.state == TS_CAND) {
                k.state = TS_FIN_CAND;
            } else if (k.state == TS_EQ) {
                k.state = TS_FIN_EQ;
            }
        }
        if (!pending) break;
    }

    CSA2_TRACE(8);
    // ---- finalize both tracks: threshold T, tie quota and this CTA's output offset
    ListCut cut[2];
    {
        // published counts of the earlier CTAs, one parallel load round
        const int grp = tid >> 6, ci = tid & 63;     // grp: 0 above0, 1 above1, 2 eq0, 3 eq1
        const int tr_g = grp & 1;
        const int st_g = tk[tr_g].state;
        const bool fin = st_g == TS_FIN_CAND || st_g == TS_FIN_EQ;
        // the published counts and the candidates of both tracks: one load round
        int v = 0;
        if (grp < 4 && fin && ci < c.cta && (grp < 2 || st_g == TS_FIN_EQ))
            v = __ldcg(sl.pub + (tr_g * 3 + (grp >> 1)) * kMaxG + ci);
        int* cx0 = reinterpret_cast<int*>(&S.stage[0][0]);
        const int n0 = tk[0].state == TS_FIN_CAND ? tk[0].C : 0, n1 = tk[1].state == TS_FIN_CAND ? tk[1].C : 0;
#pragma unroll 1
        for (int i = tid; i < n0 + n1; i += kSel) {
            const int tr = i < n0 ? 0 : 1, k = i < n0 ? i : i - n0;
            const int2 cv = __ldcg(sl.cand + tr * kCandCap + k);
            cx0[tr * 2 * kCandCap + k] = cv.x;
            cx0[tr * 2 * kCandCap + kCandCap + k] = cv.y;
        }
        v = __reduce_add_sync(0xffffffffu, v);
        if ((tid & 31) == 0 && tid < 256) S.red[tid >> 5] = v;
        sel_sync();
        const int prev[2] = {S.red[0] + S.red[1], S.red[2] + S.red[3]};
        const int eqb[2] = {S.red[4] + S.red[5], S.red[6] + S.red[7]};
        int T[2] = {INT_MAX, INT_MAX}, need[2] = {0, 0};
        if (n0 > 0 || n1 > 0) {
            CSA2_TRACE(12);   // candidates loaded
            CSA2_TRACE_VAL(16, n0);
            CSA2_TRACE_VAL(17, n1);
            const int4 ls = local_select2(cx0, n0, tk[0].rrem, tk[0].lo, tk[0].hi, cx0 + 2 * kCandCap, n1, tk[1].rrem,
                                          tk[1].lo, tk[1].hi, histl(S, 0), S.red, S.info);
            if (n0 > 0) { T[0] = ls.x; need[0] = ls.y; }
            if (n1 > 0) { T[1] = ls.z; need[1] = ls.w; }
        }
#pragma unroll
        for (int tr = 0; tr < 2; ++tr) {
            if (tk[tr].state == TS_FIN_EQ) {
                T[tr] = tk[tr].lo;
                need[tr] = tk[tr].rrem;
            }
        }
        // larger candidates and ties before this CTA, and this CTA's ties (both tracks)
        int4 ca = make_int4(0, 0, 0, 0), cb = make_int4(0, 0, 0, 0);
        const int e_end = lo + my_n;
#pragma unroll 1
        for (int i = tid; i < n0 + n1; i += kSel) {
            const int tr = i < n0 ? 0 : 1, k = i < n0 ? i : i - n0;
            const int x = cx0[tr * 2 * kCandCap + k], idx = cx0[tr * 2 * kCandCap + kCandCap + k];
            const int gtb = x > T[tr] && idx < lo, eqb2 = x == T[tr] && idx < lo;
            const int mine = x == T[tr] && idx >= lo && idx < e_end;
            if (tr == 0) { ca.x += gtb; ca.y += eqb2; cb.x += mine; }
            else         { ca.z += gtb; ca.w += eqb2; cb.y += mine; }
        }
        sel_total8(ca, cb, S.red);
        CSA2_TRACE(13);   // thresholds and counts
        const int gtb[2] = {ca.x, ca.z}, eqc[2] = {ca.y, ca.w}, mye[2] = {cb.x, cb.y};
#pragma unroll
        for (int tr = 0; tr < 2; ++tr) {
            const int st = tk[tr].state;
            ListCut& lc = cut[tr];
            lc.r = p.r[tr];
            lc.out = lc.r > 0 ? p.out[tr] + (size_t)c.u * lc.r : nullptr;
            lc.status = p.status;
            lc.all = st == TS_ALL;
            lc.T = T[tr];
            lc.quota = 0;
            lc.base = lo;
            if (st != TS_FIN_CAND && st != TS_FIN_EQ) continue;
            const bool cand = st == TS_FIN_CAND;
            const int gt_before = cand ? gtb[tr] : 0;
            const int eq_before = cand ? eqc[tr] : eqb[tr];
            const int my_eq = cand ? mye[tr] : __ldcg(sl.pub + (tr * 3 + 1) * kMaxG + c.cta);
            lc.quota = max(0, min(need[tr] - eq_before, my_eq));
            lc.base = prev[tr] + gt_before + min(need[tr], eq_before);
        }
    }

    CSA2_TRACE(9);
    // ---- ordered write of both tracks: from the ordered lists when every active
    // track was cut inside its last gathered interval, else over the whole chunk
    const bool from_lists = list_tracks != 0 && S.wlist_ovf == 0 &&
                            (tk[0].state == TS_OFF || (tk[0].state == TS_FIN_CAND && (list_tracks & 1))) &&
                            (tk[1].state == TS_OFF || (tk[1].state == TS_FIN_CAND && (list_tracks & 2)));
    if (from_lists)
        write_from_lists<kSpill>(sc, lo, full ? nullptr : c.pool, wlists(S), S.wlist_n, cut[0], cut[1], S.wsum,
                                 row_prefetch(p, c.u));
    else
        write_lists<kSpill>(sc, my_n, lo, full ? nullptr : c.pool, cut[0], cut[1], S.wsum, row_prefetch(p, c.u));
    CSA2_TRACE(10);   // lists written
    // padding: entries [min(r, n_total), r) = -1
    if (c.cta == p.G - 1) {
#pragma unroll
        for (int tr = 0; tr < 2; ++tr)
            if (cut[tr].out)
#pragma unroll 1
                for (int i = min(cut[tr].r, n_total) + tid; i < cut[tr].r; i += kSel) cut[tr].out[i] = -1;
    }
    sel_sync();
    return true;
}

// ------------------------------------------------------------ Reindex: one select per group
// A Reindex pool fits in one CTA's shared memory, so the group does not run the
// distributed select: every CTA publishes its scores (element order), its element
// count and its level-0 histogram, and meets the group at one barrier. Then every CTA
// loads all of the unit's scores and the group's histogram and finds the same exact cut (the order key's level-0 bin of the k-th best
// score, the bin's scores as candidates, the exact threshold T and the number of ties
// at T to take), and writes its own chunk's selected entries at its offset in the
// list (the entries taken before its chunk), in pool order, which is position order.
__device__ __forceinline__ bool reindex_local_unit(const IdxParams& p, IdxSmem& S, const Slot& sl, const UnitCtx& c,
                                                   int& bar_target) {
    const int tid = threadIdx.x, lane = tid & 31;
    int32_t* rs = p.rscore + (size_t)c.u * p.rstride;
    int* g0cur = sl.g0 + ((c.epoch + c.j) % 3) * kG0Stride;
    int* cnt = g0cur + kBins;
    int* cnt_next = sl.g0 + ((c.epoch + c.j + 1) % 3) * kG0Stride + kBins;
#pragma unroll 1
    for (int e = tid; e < c.my_n; e += kSel) rs[c.lo + e] = S.sc[e];
    push_hist(S.hist0, g0cur);   // (built over this CTA's valid scores)
    if (tid == 0 && c.my_n > 0) atomicAdd(cnt, c.my_n);
    {
        // the next level-0 buffer (bins and count) must be zero when the next unit,
        // in this kernel or the next one, starts: each CTA clears its share
        int* g0nxt = cnt_next - kBins;
        const int per = (kBins + p.G - 1) / p.G;
        const int zlo = c.cta * per, zhi = min(kBins, zlo + per);
#pragma unroll 1
        for (int i = zlo + tid; i < zhi; i += kSel) g0nxt[i] = 0;
        if (tid == 0 && c.cta == 0) *cnt_next = 0;
    }
    if (tid == 0) S.info[20] = 0;
    // every CTA waits: the first CTA's zeroing of the next unit's count (above) is then
    // ordered before any CTA's add for that unit
    bar_target += p.G;
    if (!group_barrier(sl.ctrl + CTRL_BAR, bar_target, p.status, p.wait_budget,
                       p.skip_arrival && c.cta == p.G - 1))
        return false;
    CSA2_TRACE(3);   // scores published

    // the group's histogram (kBpt bins a thread) and all scores of the unit (valid pool
    // entries form a prefix), as int4 vectors with every load of a thread in flight at
    // once. The score loads cover the whole row (rstride >= P_in, a multiple of 4) and
    // are issued with the count's, which decides which of them are used.
    const int n = min(max(__ldcg(cnt), 0), p.P_in);
    int hg[kBpt];
    {
        const int4* g4 = reinterpret_cast<const int4*>(g0cur + kBpt * tid);
#pragma unroll
        for (int i = 0; i < kBpt / 4; ++i) {
            const int4 v = __ldcg(g4 + i);
            hg[4 * i] = v.x; hg[4 * i + 1] = v.y; hg[4 * i + 2] = v.z; hg[4 * i + 3] = v.w;
        }
    }
    {
        const int nv = (n + 3) >> 2;
        const int nv_cap = (p.P_in + 3) >> 2;
        const int4* rs4 = reinterpret_cast<const int4*>(rs);
#pragma unroll 1
        for (int v0 = tid; v0 < nv_cap; v0 += 4 * kSel) {
            int4 x4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) x4[q] = (v0 + q * kSel < nv_cap) ? __ldcg(rs4 + v0 + q * kSel) : make_int4(0, 0, 0, 0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int v = v0 + q * kSel;
                if (v >= nv) continue;
                reinterpret_cast<int4*>(S.sc)[v] = x4[q];
            }
        }
    }
    sel_sync();
    CSA2_TRACE(4);   // all scores loaded
    const int r = p.r[1];
    ListCut none{INT_MAX, 0, 0, 0, 0, nullptr, p.status};
    ListCut cut{INT_MAX, 0, 0, 0, r, p.out[1] + (size_t)c.u * r, p.status};
    int T = INT_MAX, need = 0;
    if (n <= r) {
        cut.all = 1;
    } else {
        // level-0 bin holding rank r, from the group's histogram
        int sum = 0;
#pragma unroll
        for (int i = 0; i < kBpt; ++i) sum += hg[i];
        int total;
        const int excl = sel_scan_excl(sum, S.red, total);
        int above = total - excl - sum;
        if (above < r && r <= above + sum) {
#pragma unroll
            for (int i = kBpt - 1; i >= 0; --i) {
                if (above < r && r <= above + hg[i]) { S.info[0] = kBpt * tid + i; S.info[1] = above; }
                above += hg[i];
            }
        }
        sel_sync();
        int blo, bhi;
        bin0_interval((uint32_t)S.info[0], blo, bhi);
        const int rrem = r - S.info[1];
        // the bin's scores (any order) are the candidates; one reservation per warp and step
        int* cx = reinterpret_cast<int*>(&S.stage[0][0]);
        const unsigned below = (1u << lane) - 1u;
#pragma unroll 4
        for (int e0 = 0; e0 < n; e0 += kSel) {
            const int e = e0 + tid;
            const int x = e < n ? S.sc[e] : 0;
            const bool in = e < n && x >= blo && x <= bhi;
            const unsigned b = __ballot_sync(0xffffffffu, in);
            if (b == 0u) continue;
            int w = 0;
            if (lane == 0) w = atomicAdd(&S.info[20], __popc(b));
            w = __shfl_sync(0xffffffffu, w, 0);
            if (in) cx[w + __popc(b & below)] = x;
        }
        sel_sync();
        const int nx = S.info[20];
        CSA2_TRACE(5);   // candidates
        CSA2_TRACE_VAL(16, nx);
        const int4 ls = local_select2(S.sc, 0, 0, 1, 0, cx, nx, rrem, blo, bhi, histl(S, 0), S.red, S.info);
        T = ls.z;
        need = ls.w;   // the ties at T ranked within the first r
        CSA2_TRACE(6);   // threshold
    }
    // this CTA's offset: the entries taken before its chunk; its own share of the ties
    {
        int4 a = make_int4(0, 0, 0, 0), bb = make_int4(0, 0, 0, 0);
        const int e_end = min(c.lo + c.my_n, n);
#pragma unroll 4
        for (int e = tid; e < e_end; e += kSel) {
            const int x = S.sc[e];
            if (e < c.lo) { a.x += x > T; a.y += x == T; }
            else a.z += x == T;
        }
        sel_total8(a, bb, S.red);
        if (cut.all) {
            cut.base = c.lo;
        } else {
            cut.T = T;
            cut.base = a.x + min(need, a.y);
            cut.quota = max(0, min(need - a.y, a.z));
        }
    }
    CSA2_TRACE(7);   // offsets
    // the chunk's pool positions sit in the list region (stored as its rows were gathered;
    // the candidates and the radix histogram above lie below it)
    if (c.my_n > 0)
        write_lists<false>(S.sc + c.lo, c.my_n, 0, wlists(S), none, cut, S.wsum, row_prefetch(p, c.u));
    if (c.cta == p.G - 1) {
#pragma unroll 1
        for (int i = min(r, n) + tid; i < r; i += kSel) cut.out[i] = -1;
    }
    sel_sync();
    return true;
}

// Reindex with one CTA per query (more queries than SMs): the pool's scores and their
// level-0 histogram are already in this CTA's shared memory, so the cut runs on them
// directly (no publishing, no barrier): the bin of the k-th best score, that bin's scores
// as candidates, the exact threshold and ties, and one ordered write of the pool.
__device__ __forceinline__ bool reindex_single_unit(const IdxParams& p, IdxSmem& S, const Slot& sl, const UnitCtx& c) {
    const int tid = threadIdx.x, lane = tid & 31;
    const int n = c.my_n;   // valid pool entries (a prefix), all in this CTA
    const int r = p.r[1];
    ListCut none{INT_MAX, 0, 0, 0, 0, nullptr, p.status};
    ListCut cut{INT_MAX, 0, 0, 0, r, p.out[1] + (size_t)c.u * r, p.status};
    if (tid == 0) S.info[20] = 0;
    if (n <= r) {
        cut.all = 1;
        sel_sync();
    } else {
        int h[kBpt], sum = 0;
#pragma unroll
        for (int i = 0; i < kBpt; ++i) { h[i] = S.hist0[kBpt * tid + i]; sum += h[i]; }
        int total;
        const int excl = sel_scan_excl(sum, S.red, total);
        int above = total - excl - sum;
        if (above < r && r <= above + sum) {
#pragma unroll
            for (int i = kBpt - 1; i >= 0; --i) {
                if (above < r && r <= above + h[i]) { S.info[0] = kBpt * tid + i; S.info[1] = above; }
                above += h[i];
            }
        }
        sel_sync();
        int blo, bhi;
        bin0_interval((uint32_t)S.info[0], blo, bhi);
        const int rrem = r - S.info[1];
        int* cx = reinterpret_cast<int*>(&S.stage[0][0]);
        const unsigned below = (1u << lane) - 1u;
#pragma unroll 4
        for (int e0 = 0; e0 < n; e0 += kSel) {
            const int e = e0 + tid;
            const int x = e < n ? S.sc[e] : 0;
            const bool in = e < n && x >= blo && x <= bhi;
            const unsigned b = __ballot_sync(0xffffffffu, in);
            if (b == 0u) continue;
            int w = 0;
            if (lane == 0) w = atomicAdd(&S.info[20], __popc(b));
            w = __shfl_sync(0xffffffffu, w, 0);
            if (in) cx[w + __popc(b & below)] = x;
        }
        sel_sync();
        const int nx = S.info[20];
        const int4 ls = local_select2(S.sc, 0, 0, 1, 0, cx, nx, rrem, blo, bhi, histl(S, 0), S.red, S.info);
        cut.T = ls.z;
        cut.quota = ls.w;   // the ties at T ranked within the first r
    }
    CSA2_TRACE(4);   // threshold found
    if (n > 0) write_lists<false>(S.sc, n, 0, c.pool, none, cut, S.wsum, row_prefetch(p, c.u));
    CSA2_TRACE(10);   // list written
#pragma unroll 1
    for (int i = min(r, n) + tid; i < r; i += kSel) cut.out[i] = -1;
    {   // the next level-0 buffer (bins and count) must be zero when the next unit starts
        int* g0nxt = sl.g0 + ((c.epoch + c.j + 1) % 3) * kG0Stride;
#pragma unroll 1
        for (int i = tid; i <= kBins; i += kSel) g0nxt[i] = 0;
    }
    sel_sync();
    return true;
}

// ------------------------------------------------------------ scoring helpers
// Score of one key row (DI/16 int4 chunks) against the index query held in
// shared memory (HI heads of DI bytes, read as broadcasts). Heads at or past
// the call's Hi have weight 0.
template <int HI, int DI>
__device__ __forceinline__ int score_smem(const int4* rowc, const int8_t* qs, const int32_t* w) {
    int s = 0;
#pragma unroll
    for (int h = 0; h < HI; ++h) {
        int acc = 0;
        const int4* qh = reinterpret_cast<const int4*>(qs + h * DI);
#pragma unroll
        for (int c = 0; c < DI / 16; ++c) {
            const int4 k = rowc[c], qq = qh[c];
            acc = __dp4a(k.x, qq.x, acc);
            acc = __dp4a(k.y, qq.y, acc);
            acc = __dp4a(k.z, qq.z, acc);
            acc = __dp4a(k.w, qq.w, acc);
        }
        s += w[h] * max(acc, 0);
    }
    return s;
}

// Scores of two key rows at once: each read of the index query from shared memory
// serves both rows.
template <int HI, int DI>
__device__ __forceinline__ void score2_smem(const int4* ra, const int4* rb, const int8_t* qs, const int32_t* w,
                                            int& xa, int& xb) {
    int sa = 0, sb = 0;
#pragma unroll
    for (int h = 0; h < HI; ++h) {
        int aa = 0, ab = 0;
        const int4* qh = reinterpret_cast<const int4*>(qs + h * DI);
#pragma unroll
        for (int c = 0; c < DI / 16; ++c) {
            const int4 qq = qh[c], ka = ra[c], kb = rb[c];
            aa = __dp4a(ka.x, qq.x, aa); aa = __dp4a(ka.y, qq.y, aa); aa = __dp4a(ka.z, qq.z, aa); aa = __dp4a(ka.w, qq.w, aa);
            ab = __dp4a(kb.x, qq.x, ab); ab = __dp4a(kb.y, qq.y, ab); ab = __dp4a(kb.z, qq.z, ab); ab = __dp4a(kb.w, qq.w, ab);
        }
        sa += w[h] * max(aa, 0);
        sb += w[h] * max(ab, 0);
    }
    xa = sa;
    xb = sb;
}

// Generic shapes: Hi <= 16, Di <= 128, queries read from shared memory.
__device__ __forceinline__ int score_generic(const int4* rowc, int nchunk, const int8_t* qs, int Hi, int Di,
                                             const int32_t* w) {
    int s = 0;
    for (int h = 0; h < Hi; ++h) {
        int acc = 0;
        const int4* qh = reinterpret_cast<const int4*>(qs + h * Di);
        for (int c = 0; c < nchunk; ++c) {
            const int4 k = rowc[c], qq = qh[c];
            acc = __dp4a(k.x, qq.x, acc);
            acc = __dp4a(k.y, qq.y, acc);
            acc = __dp4a(k.z, qq.z, acc);
            acc = __dp4a(k.w, qq.w, acc);
        }
        s += w[h] * max(acc, 0);
    }
    return s;
}

// byte offset of chunk c of row r in a TMA tile whose rows are `di` bytes and
// whose swizzle span equals the row length (no swizzle for 16-byte rows)
__device__ __forceinline__ uint32_t tile_off(int r, int c, int di) {
    const uint32_t off = (uint32_t)(r * di + c * 16);
    const uint32_t b = (di == 32) ? 1u : (di == 64) ? 2u : (di == 128) ? 3u : 0u;
    return off ^ (((off >> 7) & ((1u << b) - 1u)) << 4);
}

// Key tiles are read once per launch: they are loaded with an L2 evict-first
// policy, so the stream does not push the kernel's own instructions and the
// select state out of L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void tma_load_keys(void* dst, const CUtensorMap* map, int x, int y, int z,
                                              uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, "
        "{%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ IdxSmem& idx_smem() {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    return *reinterpret_cast<IdxSmem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
}

// ------------------------------------------------------------ Full mode on the tensor cores
// Warps 0-15: epilogue and select; warp 16: TMA producer; warp 17: MMA issuer.
template <int DI>
__global__ void __launch_bounds__(kTcThreads, 1)
    index_full_tc_kernel(const __grid_constant__ IdxParams p, const __grid_constant__ CUtensorMap kmap) {
    static_assert(DI == 32 || DI == 64 || DI == 128, "tensor-core key widths");
    CSA2_TRACE_INIT();
    IdxSmem& S = idx_smem();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int group = blockIdx.x / p.G;
    const int cta = blockIdx.x % p.G;
    const Slot sl = slot_of(p, group);
    int* spill = (p.chunk > kSmemScores) ? p.spill + (size_t)blockIdx.x * p.chunk : nullptr;
    constexpr int kRows = (kStageBytes / DI) < 256 ? (kStageBytes / DI) : 256;   // rows per tile
    constexpr int kBlocks = kRows / 128;                                          // MMA row blocks per tile
    constexpr uint32_t kSwz = DI == 32 ? 6u : DI == 64 ? 4u : 2u;
    constexpr uint32_t kSbo = 8 * DI;                                             // bytes per 8-row group
    constexpr uint32_t kIdesc = idesc_i8(128, 16);

    if (warp == 0) tmem_alloc(&S.tmem_base, 32 * kTmemBufs);
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) { mbar_init(&S.full_bar[i], 1); mbar_init(&S.empty_bar[i], 1); }
        for (int i = 0; i < kTmemBufs; ++i) { mbar_init(&S.tfull_bar[i], 1); mbar_init(&S.tempty_bar[i], kSel / 64); }
        S.abort = 0;
        mbar_fence_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch_dependents();   // the next kernel may start its own set-up
    // The workspace and the index query may come from the previous kernel: wait for
    // it. When the keys and positions were complete before that kernel began, the
    // TMA producer starts the key stream at once and fills its stages meanwhile.
    const bool producer = warp == kSel / 32;
    if (!(producer && p.keys_ready)) pdl_wait();
    CSA2_TRACE(1);
    const int epoch = producer ? 0 : __ldcg(sl.ctrl + CTRL_EPOCH);
    int bar_target = producer ? 0 : __ldcg(sl.ctrl + CTRL_BAR_BASE);
    const uint32_t tmem = S.tmem_base;
    uint32_t seq = 0;   // tiles processed by this CTA so far (same count in every role)

    // every unit, or the ones a list names (the queries the shared-key cut left over)
    const int nlist = p.unit_list ? __ldcg(p.unit_list) : p.units;
    int j = 0;
    for (int i = group; i < nlist; i += p.groups, ++j) {
        const int u = p.unit_list ? __ldcg(p.unit_list + 1 + i) : i;
        const int b = u / p.Tq;
        int t = p.q_pos[u];
        int tg = last_entry(t, p.m);   // the last global entry the query reads
        if (t < 0 || tg >= p.N) {
            if (tid == 0 && cta == 0) report(p.status, CSA2_ERR_RANGE, u);
            t = -1;
            tg = -1;
        }
        const int n_all = tg + 1;
        const int lo = min(cta * p.chunk, n_all);
        const int my_n = min(lo + p.chunk, n_all) - lo;
        const int nst = (my_n + kRows - 1) / kRows;

        // index query -> B operand (16 rows: heads, zero past Hi); zero the histogram. The
        // TMA warp takes no part: it starts streaming keys at once, and the others meet on
        // named barrier 2 (the previous unit's select ended at a block barrier).
        if (warp != kSel / 32) {
            constexpr int kStg = kTcThreads - 32;
            const int li = tid < kSel ? tid : tid - 32;
            fence_proxy_async_smem();
            for (int i = li; i < p.Hi * DI / 16; i += kStg)
                reinterpret_cast<int4*>(S.q)[i] = reinterpret_cast<const int4*>(p.qi + (size_t)u * p.Hi * DI)[i];
            for (int i = li; i < kBins; i += kStg) S.hist0[i] = 0;
            asm volatile("bar.sync 2, %0;" ::"n"(kStg) : "memory");
            for (int i = li; i < DI; i += kStg) {
                const int h = i / (DI / 16), c2 = i % (DI / 16);
                int4 v = make_int4(0, 0, 0, 0);
                if (h < p.Hi) v = reinterpret_cast<const int4*>(S.q + h * DI)[c2];
                *reinterpret_cast<int4*>(S.qtc + tile_off(h, c2, DI)) = v;
            }
            fence_proxy_async_smem();
            asm volatile("bar.sync 2, %0;" ::"n"(kStg) : "memory");
        }

        if (warp == kSel / 32) {
            // ---- TMA producer
            if (lane == 0) {
                const uint64_t pol = l2_evict_first_policy();
                for (int s2 = 0; s2 < nst; ++s2) {
                    const uint32_t i = seq + s2, slot = i % kStages;
                    if (i >= (uint32_t)kStages &&
                        !mbar_wait(&S.empty_bar[slot], ((i / kStages) - 1) & 1u, p.status, 5)) { S.abort = 1; break; }
                    mbar_arrive_expect_tx(&S.full_bar[slot], (uint32_t)(kRows * DI));
                    tma_load_keys(S.stage[slot], &kmap, 0, lo + s2 * kRows, b, &S.full_bar[slot], pol);
                }
            }
        } else if (warp == kSel / 32 + 1) {
            // ---- MMA issuer
            if (lane == 0) {
                const uint32_t b0 = smem_u32(S.qtc);
                for (int s2 = 0; s2 < nst; ++s2) {
                    const uint32_t i = seq + s2, slot = i % kStages, buf = i % kTmemBufs;
                    if (!mbar_wait(&S.full_bar[slot], (i / kStages) & 1u, p.status, 3)) { S.abort = 1; break; }
                    if (i >= (uint32_t)kTmemBufs &&
                        !mbar_wait(&S.tempty_bar[buf], ((i / kTmemBufs) - 1) & 1u, p.status, 6)) { S.abort = 1; break; }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(S.stage[slot]);
                    const uint32_t d0 = tmem + buf * 32u;
#pragma unroll
                    for (int blk = 0; blk < kBlocks; ++blk) {
#pragma unroll
                        for (int kk = 0; kk < DI / 32; ++kk)
                            mma_i8(d0 + blk * 16, smem_desc(a0 + blk * 128 * DI + kk * 32, 16, kSbo, kSwz),
                                   smem_desc(b0 + kk * 32, 16, kSbo, kSwz), kIdesc, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&S.empty_bar[slot]);
                    mma_commit(&S.tfull_bar[buf]);
                }
            }
        } else {
            // ---- epilogue: ReLU and head weights on the int32 accumulators. Two
            // groups of 8 warps take alternate tiles; in a group, warp wl reads
            // TMEM lane quarter wl % 4 of row block wl / 4.
            const int egrp = warp >> 3, wl = warp & 7, tl = tid & 255;
            const bool in_block = (wl >> 2) < kBlocks;                // warp-uniform
            const uint32_t lane_base = tmem + (uint32_t)(wl >> 2) * 16u + ((uint32_t)(wl & 3) * 32u << 16);
            for (int s2 = egrp; s2 < nst; s2 += 2) {
                const uint32_t i = seq + s2, buf = i % kTmemBufs;
                const bool got = mbar_wait(&S.tfull_bar[buf], (i / kTmemBufs) & 1u, p.status, 4);
                if (!__all_sync(0xffffffffu, got)) { S.abort = 1; break; }   // warp-uniform exit
                tc_fence_after();
                int x = 0;
                if (in_block) {
                    int acc[8];
                    const uint32_t ta = lane_base + buf * 32u;
                    tmem_ld8(ta, acc);
                    tmem_ld_wait();
#pragma unroll
                    for (int h = 0; h < 8; ++h) x += p.w[h] * max(acc[h], 0);
                    if (p.Hi > 8) {
                        tmem_ld8(ta + 8, acc);
                        tmem_ld_wait();
#pragma unroll
                        for (int h = 0; h < 8; ++h) x += p.w[8 + h] * max(acc[h], 0);
                    }
                }
                // one arrival per warp (the buffer's barrier counts the group's 8 warps):
                // 256 arrivals on one mbarrier per tile were serialised by shared memory
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.tempty_bar[buf]);
                const int e = s2 * kRows + tl;
                if (in_block && e < my_n) {
                    if (spill) spill[e] = x; else S.sc[e] = x;
                    atomicAdd(&S.hist0[bin0(x)], 1);
                }
            }
        }
        seq += nst;
        __syncthreads();
        CSA2_TRACE(2);   // scan done
        if (S.abort) break;

        if (tid < kSel) {
            UnitCtx c{u, t, lo, my_n, n_all, cta, j, epoch, nullptr};
            const bool ok = spill ? select_unit<true>(p, S, sl, c, bar_target, spill)
                                  : select_unit<false>(p, S, sl, c, bar_target, S.sc);
            if (!ok && tid == 0) S.abort = 1;
        }
        __syncthreads();
        if (S.abort) break;
    }
    CSA2_TRACE(11);
    CSA2_TRACE_END(1);
    if (!S.abort && cta == 0 && tid == 0) {
        sl.ctrl[CTRL_EPOCH] = epoch + j;
        sl.ctrl[CTRL_BAR_BASE] = bar_target;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 32 * kTmemBufs);
}

// ------------------------------------------------------------ Full mode, queries that share keys
// Several queries of one sequence (Tq >= kMqMin) score the same keys. A CTA takes a
// block of up to kMqQ queries of a sequence and a range of 128-row key tiles. One
// kind::i8 MMA per 32-byte K step scores a tile against all of the block's queries:
// B row 8q + h holds query q's head h (zero past Hi or past the block), so N = 8 kMqQ,
// and each key tile is read once per block instead of once per query. No query's
// scores are kept in full. The call runs in four steps:
//   1. sample (this kernel, kMqSample): every tstep-th tile only; each query's scores
//      there, up to its own position, go to a compact per-unit sample;
//   2. estimate (index_mq_estimate_kernel): per query and track, a threshold estimate
//      from the sample, the sample's value at 1.2 times the rank the track's cut would
//      have in it, plus 16; tlo is the lower of the two;
//   3. mark (this kernel, kMqMark): every tile; per query, a bit per position for the
//      scores at or above tlo (the candidates), one 32-bit word per 32 positions;
//   4. cut (index_mq_select_kernel): per query, the candidates' positions in order,
//      their scores recomputed from the keys, a check that each track has at least r
//      candidates at or above its estimate (then its r best scores and every tie at
//      its threshold are candidates), the exact cut and the ordered write. A query
//      that fails the check, or has more candidates than shared memory holds, is
//      listed for the cooperative Full kernel, which scans and cuts it in full.
constexpr int kMqQ = 16;                                  // queries per block
constexpr int kMqN = kMqQ * 8;                            // MMA N
constexpr int kMqRows = 128;                              // key rows per tile (one M = 128 block)
constexpr int kMqStages = 8;
constexpr int kMqBufs = 4;                                // TMEM buffers of kMqN columns (512 in all)
constexpr int kMqGroups = 4;                              // epilogue groups of 4 warps, alternate tiles
constexpr int kMqThreads = (kMqGroups * 4 + 2) * 32;      // + the TMA and MMA warps
constexpr int kMqMin = 4;                                 // Tq from which a Full call takes this path
constexpr int kMqMinN = 8192;                             // ... on a key set of at least this many positions

enum { kMqSample = 0, kMqMark = 1 };

struct MqParams {
    int B, Tq, N, Hi, nblk, splits;
    int m;               // sequence compression rate of the global entries
    int32_t w[8];
    const int32_t* q_pos;
    const int8_t* qi;
    int32_t* out;        // sample: [B*Tq][ostride] scores; mark: [B*Tq][ostride] candidate words
    int64_t ostride;
    int tstep;           // sample: every tstep-th key tile (mark: 1)
    const int4* est;     // mark: per unit {tlo, te0, te1, tracks}
    int32_t* status;
};

template <int DI>
struct __align__(1024) MqSmem {
    uint8_t stage[kMqStages][kMqRows * DI];
    uint8_t qb[kMqN * DI];               // the block's index queries as the B operand
    uint64_t full_bar[kMqStages], empty_bar[kMqStages], tfull_bar[kMqBufs], tempty_bar[kMqBufs];
    int tq[kMqQ];
    int tlo[kMqQ];
    int tile_lo, tile_hi;
    uint32_t tmem_base;
};

__device__ __forceinline__ void tmem_ld16i(uint32_t taddr, int (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}

template <int DI, int MODE>
__global__ void __launch_bounds__(kMqThreads, 1)
    index_mq_score_kernel(const __grid_constant__ MqParams p, const __grid_constant__ CUtensorMap kmap) {
    CSA2_TRACE_INIT();
    static_assert(DI == 32 || DI == 64 || DI == 128, "tensor-core key widths");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    MqSmem<DI>& S = *reinterpret_cast<MqSmem<DI>*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    constexpr uint32_t kSwz = DI == 32 ? 6u : DI == 64 ? 4u : 2u;
    constexpr uint32_t kSbo = 8 * DI;
    constexpr uint32_t kIdesc = idesc_i8(128, kMqN);
    constexpr int kEpiWarps = kMqGroups * 4;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x % p.splits;
    const int bq = blockIdx.x / p.splits;
    const int b = bq / p.nblk, j0 = (bq % p.nblk) * kMqQ;
    const int nq = min(kMqQ, p.Tq - j0);

    if (warp == 0) tmem_alloc(&S.tmem_base, kMqBufs * kMqN);
    if (tid == 0) {
        for (int i = 0; i < kMqStages; ++i) { mbar_init(&S.full_bar[i], 1); mbar_init(&S.empty_bar[i], 1); }
        for (int i = 0; i < kMqBufs; ++i) { mbar_init(&S.tfull_bar[i], 1); mbar_init(&S.tempty_bar[i], 4); }
        mbar_fence_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch_dependents();
    pdl_wait();   // positions and index queries may come from the previous kernel

    if (tid < kMqQ) {
        int t = -1;
        if (tid < nq) {
            t = p.q_pos[(size_t)b * p.Tq + j0 + tid];
            const int tg = last_entry(t, p.m);
            t = (t < 0 || tg >= p.N) ? -1 : tg;   // no scores past the last entry; the cut reports a bad position
        }
        S.tq[tid] = t;
        if (MODE == kMqMark) S.tlo[tid] = tid < nq ? p.est[(size_t)b * p.Tq + j0 + tid].x : INT_MAX;
    }
    fence_proxy_async_smem();
    for (int i = tid; i < kMqN * (DI / 16); i += kMqThreads) {
        const int r = i / (DI / 16), c2 = i % (DI / 16);
        const int q = r >> 3, h = r & 7;
        int4 v = make_int4(0, 0, 0, 0);
        if (q < nq && h < p.Hi)
            v = reinterpret_cast<const int4*>(p.qi + (((size_t)b * p.Tq + j0 + q) * p.Hi + h) * DI)[c2];
        *reinterpret_cast<int4*>(S.qb + tile_off(r, c2, DI)) = v;
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {   // this split's share of the tiles that cover [0, the block's last position]
        int tmax = -1;
        for (int q = 0; q < kMqQ; ++q) tmax = max(tmax, S.tq[q]);
        const int ntile = ((tmax + kMqRows) / kMqRows + p.tstep - 1) / p.tstep;   // (sample: the sampled tiles)
        S.tile_lo = (int)((long long)ntile * split / p.splits);
        S.tile_hi = (int)((long long)ntile * (split + 1) / p.splits);
    }
    __syncthreads();
    const int tile_lo = S.tile_lo, nt = S.tile_hi - S.tile_lo;
    const uint32_t tmem = S.tmem_base;

    if (warp == kEpiWarps) {
        if (lane == 0) {   // TMA producer
            const uint64_t pol = l2_evict_first_policy();
            for (int i = 0; i < nt; ++i) {
                const int slot = i % kMqStages;
                if (i >= kMqStages && !mbar_wait(&S.empty_bar[slot], ((i / kMqStages) - 1) & 1u, p.status, 21)) break;
                mbar_arrive_expect_tx(&S.full_bar[slot], (uint32_t)(kMqRows * DI));
                tma_load_keys(S.stage[slot], &kmap, 0, (tile_lo + i) * p.tstep * kMqRows, b, &S.full_bar[slot], pol);
            }
        }
    } else if (warp == kEpiWarps + 1) {
        if (lane == 0) {   // MMA issuer
            const uint32_t b0 = smem_u32(S.qb);
            for (int i = 0; i < nt; ++i) {
                const int slot = i % kMqStages, buf = i % kMqBufs;
                if (!mbar_wait(&S.full_bar[slot], (i / kMqStages) & 1u, p.status, 22)) break;
                if (i >= kMqBufs && !mbar_wait(&S.tempty_bar[buf], ((i / kMqBufs) - 1) & 1u, p.status, 23)) break;
                tc_fence_after();
                const uint32_t a0 = smem_u32(S.stage[slot]);
#pragma unroll
                for (int kk = 0; kk < DI / 32; ++kk)
                    mma_i8(tmem + (uint32_t)(buf * kMqN), smem_desc(a0 + kk * 32, 16, kSbo, kSwz),
                           smem_desc(b0 + kk * 32, 16, kSbo, kSwz), kIdesc, kk > 0 ? 1u : 0u);
                mma_commit(&S.empty_bar[slot]);
                mma_commit(&S.tfull_bar[buf]);
            }
        }
    } else {
        // epilogue: group g takes tiles g, g + 4, ...; warp wl of a group reads TMEM lane
        // quarter wl, i.e. key rows 32 wl .. 32 wl + 31 of the tile
        const int g = warp >> 2, wl = warp & 3;
        int tq[kMqQ], w[8];
#pragma unroll
        for (int q = 0; q < kMqQ; ++q) tq[q] = S.tq[q];
#pragma unroll
        for (int h = 0; h < 8; ++h) w[h] = p.w[h];
        for (int i = g; i < nt; i += kMqGroups) {
            const int buf = i % kMqBufs;
            const bool got = mbar_wait(&S.tfull_bar[buf], (i / kMqBufs) & 1u, p.status, 24);
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            int x[kMqQ];
            const uint32_t ta = tmem + (uint32_t)(buf * kMqN) + ((uint32_t)(wl * 32) << 16);
#pragma unroll
            for (int q2 = 0; q2 < kMqQ / 2; ++q2) {
                int acc[16];
                tmem_ld16i(ta + (uint32_t)(q2 * 16), acc);
                tmem_ld_wait();
                int xa = 0, xb = 0;
#pragma unroll
                for (int h = 0; h < 8; ++h) {
                    xa += w[h] * max(acc[h], 0);
                    xb += w[h] * max(acc[8 + h], 0);
                }
                x[2 * q2] = xa;
                x[2 * q2 + 1] = xb;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.tempty_bar[buf]);
            const int kt = (tile_lo + i) * p.tstep;            // the key tile
            const int s = kt * kMqRows + wl * 32 + lane;       // this lane's position
            if (MODE == kMqSample) {
                // sample entry (tile ordinal) * 128 + row, for the positions up to the query's own
                const int e = (tile_lo + i) * kMqRows + wl * 32 + lane;
#pragma unroll
                for (int q = 0; q < kMqQ; ++q)
                    if (s <= tq[q]) p.out[((size_t)b * p.Tq + j0 + q) * p.ostride + e] = x[q];
            } else {
                // candidate word of each query for these 32 positions; lane q stores query q's
                unsigned mine = 0u;
#pragma unroll
                for (int q = 0; q < kMqQ; ++q) {
                    const unsigned m = __ballot_sync(0xffffffffu, s <= tq[q] && x[q] >= S.tlo[q]);
                    if (lane == q) mine = m;
                }
                if (lane < nq)
                    p.out[((size_t)b * p.Tq + j0 + lane) * p.ostride + kt * 4 + wl] = (int32_t)mine;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kMqBufs * kMqN);
    CSA2_TRACE_END(5);
}

// ------------------------------------------------------------ shared keys: estimates and the cut
constexpr int kMqSampleMax = 16384;  // sample entries per query (at most 128 sampled tiles)
constexpr int kMqCap = 16384;        // candidates per query that the cut holds
constexpr int kMqCapSmall = 8192;    // ... in its two-CTAs-per-SM form

size_t mq_estimate_smem_bytes(int sstride) { return (size_t)(sstride + 1088 + 8 * kSelWarps + 64) * 4; }

// Step 2: one CTA per query. The sampled tiles' entries up to the query's position form a
// prefix of its sample (a sampled tile is whole or the last one); the estimate of each
// track with 0 < r < n is the sample's value at rank min(m, r m / n * 1.2 + 16).
__global__ void __launch_bounds__(kSel, 2) index_mq_estimate_kernel(const __grid_constant__ IdxParams p) {
    extern __shared__ __align__(16) int sme[];
    struct {
        int* sc;     // [sstride] the sample
        int* hist;   // [1088]
        int* red;    // [8 * kSelWarps]
        int* info;   // [64]
    } S{sme, sme + p.mq_sstride, sme + p.mq_sstride + 1088, sme + p.mq_sstride + 1088 + 8 * kSelWarps};
    const int tid = threadIdx.x, lane = tid & 31;
    const int u = blockIdx.x;
    pdl_launch_dependents();
    pdl_wait();
    if (u == 0 && tid == 0) p.fb_list[0] = 0;   // the call's fallback list starts empty
    const int t = p.q_pos[u], tg = last_entry(t, p.m);
    const int n = (t < 0 || tg >= p.N) ? 0 : tg + 1;
    int act[2];
#pragma unroll
    for (int tr = 0; tr < 2; ++tr) act[tr] = p.r[tr] > 0 && p.r[tr] < n;
    int4 e = make_int4(INT_MAX, INT_MAX, INT_MAX, 0);
    if (act[0] || act[1]) {
        const int span = p.mq_tstep * kMqRows;
        int m = 0;
        for (int j = 0; j * span <= tg && j * kMqRows < p.mq_sstride; ++j) m += min(kMqRows, tg - j * span + 1);
        const int32_t* src = p.mq_sample + (size_t)u * p.mq_sstride;
        int smin = INT_MAX, smax = INT_MIN;
        for (int i = tid; i < m; i += kSel) {
            const int x = __ldcg(src + i);
            S.sc[i] = x;
            smin = min(smin, x);
            smax = max(smax, x);
        }
        smin = __reduce_min_sync(0xffffffffu, smin);
        smax = __reduce_max_sync(0xffffffffu, smax);
        if (tid == 0) { S.info[26] = INT_MAX; S.info[27] = INT_MIN; }
        sel_sync();
        if (lane == 0) { atomicMin(&S.info[26], smin); atomicMax(&S.info[27], smax); }
        sel_sync();
        smin = S.info[26];
        smax = S.info[27];
        int qr[2];
#pragma unroll
        for (int tr = 0; tr < 2; ++tr)
            qr[tr] = act[tr] ? min(m, (int)((long long)p.r[tr] * m / n * 6 / 5) + 16) : 0;
        const int4 est = local_select2(S.sc, act[0] ? m : 0, qr[0], smin, smax, S.sc, act[1] ? m : 0, qr[1], smin,
                                       smax, S.hist, S.red, S.info);
        const int te0 = act[0] ? est.x : INT_MAX, te1 = act[1] ? est.z : INT_MAX;
        e = make_int4(min(te0, te1), te0, te1, act[0] | (act[1] << 1));
    }
    if (tid == 0) p.mq_est[u] = e;
}

// Step 4 (and Reindex with more queries than SMs): one CTA per query. Shared memory
// (1024-aligned): kRB 128-row blocks of gathered key rows and the index query as
// tensor-core operands, [cap] positions and [cap] scores (cap = kMqCap, or kMqCapSmall in
// the two-CTAs-per-SM form), the histogram, reduction and count scratch, the barrier and
// the TMEM address.
// 128-row blocks per batch: 8, or 4 in the small form and for 128-byte keys
template <int DI, bool SMALL> constexpr int mq_rb() { return (SMALL || DI == 128) ? 4 : 8; }

template <int DI, bool SMALL>
__global__ void __launch_bounds__(kSel, SMALL ? 2 : 1) index_mq_select_kernel(const __grid_constant__ IdxParams p) {
    extern __shared__ __align__(1024) uint8_t smq_raw[];
    uint8_t* sbase = smq_raw + ((1024u - (smem_u32(smq_raw) & 1023u)) & 1023u);
    constexpr int kRB = mq_rb<DI, SMALL>();
    const int cap = SMALL ? kMqCapSmall : kMqCap;
    uint8_t* stage = sbase;                                   // [kRB][128 rows][DI], TMA-tile layout
    uint8_t* qtc = stage + kRB * 128 * DI;                    // [16 rows][DI]: heads, zero past Hi
    int* cpos = reinterpret_cast<int*>(qtc + (16 * DI > 1024 ? 16 * DI : 1024));
    int* csc = cpos + cap;
    int* hist = csc + cap;
    int* red = hist + 1088;
    int* info = red + 8 * kSelWarps;
    int* wsum = info + 64;
    uint64_t* bar = reinterpret_cast<uint64_t*>(wsum + 4 * kSelWarps);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int u = blockIdx.x, b = u / p.Tq;
    CSA2_TRACE_INIT();
    pdl_launch_dependents();
    pdl_wait();
    const int t = p.q_pos[u], tg = last_entry(t, p.m);
    const bool bad = t < 0 || tg >= p.N;
    if (bad && tid == 0) report(p.status, CSA2_ERR_RANGE, u);
    // Reindex with one CTA per query: the candidates are the unit's pool, whose valid
    // entries (0 <= s <= the query's last entry) form a prefix, -1 padding after
    const int32_t* pool = p.pool_in ? p.pool_in + (size_t)u * p.P_in : nullptr;
    int n = bad ? 0 : tg + 1;
    if (pool) {
        int fb = p.P_in;
        for (int i = tid; i < p.P_in; i += kSel) {
            const int s = __ldg(pool + i);
            if (!(s >= 0 && s <= tg)) fb = min(fb, i);
        }
        fb = sel_min(fb, red);
        for (int i = fb + tid; i < p.P_in; i += kSel)   // past the first invalid entry: padding only
            if (__ldg(pool + i) >= 0) report(p.status, CSA2_ERR_RANGE, u);
        n = fb;
    }
    // a track with r >= n takes every entry in order (none at a bad position), then -1
#pragma unroll
    for (int tr = 0; tr < 2; ++tr) {
        const int r = p.r[tr];
        if (r > 0 && r >= n) {
            int32_t* out = p.out[tr] + (size_t)u * r;
            for (int i = tid; i < r; i += kSel) out[i] = i < n ? (pool ? __ldg(pool + i) : i) : -1;
        }
    }
    // the tracks to cut and their estimates (a pool: every entry is a candidate)
    const bool pk = pool && p.r[1] > 0 && p.r[1] < n;
    const int4 e = pool ? make_int4(INT_MIN, INT_MIN, INT_MIN, pk ? 2 : 0) : p.mq_est[u];
    const bool act0 = (e.w & 1) != 0, act1 = (e.w & 2) != 0;
    if (!act0 && !act1) { CSA2_TRACE_END(7); return; }

    // ---- the candidates' positions in order: warp w takes the words [w W, (w + 1) W), its
    // lanes read 32 consecutive words at a time; counted, scanned over the warps, expanded
    const int nw = pool ? 0 : (n + 31) >> 5;
    const int wpw = (nw + kSelWarps * 32 - 1) / (kSelWarps * 32) * 32;   // words per warp
    const int ww0 = min(nw, (tid >> 5) * wpw), ww1 = min(nw, ww0 + wpw);
    const int32_t* words = pool ? nullptr : p.mq_words + (size_t)u * p.mq_wstride;
    auto word_at = [&](int w) -> unsigned {
        if (w >= ww1) return 0u;
        unsigned m = (unsigned)__ldcg(words + w);
        const int valid = n - 32 * w;   // positions of this word up to the query's own
        return valid >= 32 ? m : (m & ((1u << valid) - 1u));
    };
    int cnt = 0;
#pragma unroll 4
    for (int w = ww0 + lane; w < ww1; w += 32) cnt += __popc(word_at(w));
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    int total;
    int off = sel_scan_excl(lane == 0 ? cnt : 0, red, total);   // the warp's first slot
    off = __shfl_sync(0xffffffffu, off, 0);
    if (pool) total = n;
    CSA2_TRACE(22);   // candidates counted
    bool fail = total > cap;
    if (!fail) {
        if (pool)
            for (int i = tid; i < n; i += kSel) cpos[i] = __ldg(pool + i);
        for (int w0 = ww0; w0 < ww1; w0 += 32) {
            unsigned m = word_at(w0 + lane);
            const int c = __popc(m);
            int incl = c;   // inclusive scan of the counts over the lanes
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            int k = off + incl - c;
            while (m) {
                const int bit = __ffs(m) - 1;
                m &= m - 1u;
                cpos[k++] = 32 * (w0 + lane) + bit;
            }
            off += __shfl_sync(0xffffffffu, incl, 31);
        }
        // the index query as the B operand (16 rows: heads, zero past Hi), the barrier, TMEM
        for (int i = tid; i < 16 * DI / 16; i += kSel) {
            const int h = i / (DI / 16), c2 = i % (DI / 16);
            int4 v = make_int4(0, 0, 0, 0);
            if (h < p.Hi) v = reinterpret_cast<const int4*>(p.qi + ((size_t)u * p.Hi + h) * DI)[c2];
            *reinterpret_cast<int4*>(qtc + tile_off(h, c2, DI)) = v;
        }
        if (tid == 0) {
            mbar_init(bar, 1);
            mbar_fence_init();
        }
        if (warp == 0) tmem_alloc(tmem_slot, 16 * kRB);
        fence_proxy_async_smem();
        tc_fence_before();
        sel_sync();
        tc_fence_after();
        const uint32_t tmem = *tmem_slot;
        // ---- the candidates' scores on the tensor cores, kRB blocks of 128 rows a batch:
        // the rows are gathered into operand tiles (DI / 16 threads per row, 16 bytes each),
        // one kind::i8 MMA per block and 32-byte K step (N = 16), then warp w reads TMEM lane
        // quarter w % 4 of blocks w / 4 and w / 4 + 4
        constexpr uint32_t kSwz = DI == 32 ? 6u : DI == 64 ? 4u : 2u;
        constexpr uint32_t kSbo = 8 * DI;
        constexpr uint32_t kIdesc = idesc_i8(128, 16);
        constexpr int CPR = DI / 16, CPT = kRB * 128 * CPR / kSel;   // chunks per row, per thread
        const int8_t* kb = p.ki + (size_t)b * p.ki_seq_stride;
        int c0 = 0, c1 = 0, cmax = INT_MIN, cmin = INT_MAX;
        uint32_t phase = 0;
        bool ok = true;
        // this batch's chunks in registers; the next batch's loads are issued once this
        // batch's MMAs are, so they are in flight during its wait and epilogue
        int4 v[CPT];
        auto load_batch = [&](int b0) {
#pragma unroll
            for (int k = 0; k < CPT; ++k) {
                const int ci = tid + k * kSel, r = ci / CPR, g = b0 + r;
                v[k] = g < total ? __ldg(reinterpret_cast<const int4*>(kb + (size_t)cpos[g] * DI) + ci % CPR)
                                 : make_int4(0, 0, 0, 0);
            }
        };
        load_batch(0);
        for (int base = 0; base < total && ok; base += kRB * 128) {
            const int nblk = min(kRB, (total - base + 127) / 128);
#pragma unroll
            for (int k = 0; k < CPT; ++k) {
                const int ci = tid + k * kSel, r = ci / CPR;
                *reinterpret_cast<int4*>(stage + (r >> 7) * 128 * DI + tile_off(r & 127, ci % CPR, DI)) = v[k];
            }
            fence_proxy_async_smem();
            tc_fence_before();
            sel_sync();
            tc_fence_after();
            if (tid == 0) {
                const uint32_t a0 = smem_u32(stage), b0 = smem_u32(qtc);
                for (int blk = 0; blk < nblk; ++blk)
#pragma unroll
                    for (int kk = 0; kk < DI / 32; ++kk)
                        mma_i8(tmem + blk * 16, smem_desc(a0 + blk * 128 * DI + kk * 32, 16, kSbo, kSwz),
                               smem_desc(b0 + kk * 32, 16, kSbo, kSwz), kIdesc, kk > 0 ? 1u : 0u);
                mma_commit(bar);
            }
            if (base + kRB * 128 < total) load_batch(base + kRB * 128);
            ok = sel_and(mbar_wait(bar, phase, p.status, 31) ? 1 : 0) != 0;   // (the same in every thread)
            phase ^= 1u;
            tc_fence_after();
#pragma unroll
            for (int bb = 0; bb < kRB; bb += 4) {
                const int blk = warp / 4 + bb;
                if (blk < nblk && ok) {   // (warp-uniform)
                    int acc[8];
                    tmem_ld8(tmem + blk * 16 + ((uint32_t)(warp & 3) * 32u << 16), acc);
                    tmem_ld_wait();
                    int x = 0;
#pragma unroll
                    for (int h = 0; h < 8; ++h) x += p.w[h] * max(acc[h], 0);
                    const int g = base + blk * 128 + (warp & 3) * 32 + lane;
                    if (g < total) {
                        csc[g] = x;
                        c0 += x >= e.y;
                        c1 += x >= e.z;
                        cmax = max(cmax, x);
                        cmin = min(cmin, x);
                    }
                }
            }
            tc_fence_before();
            sel_sync();   // the tiles and TMEM are free for the next batch
        }
        tc_fence_after();
        if (warp == 0) tmem_dealloc(tmem, 16 * kRB);
        fail = !ok;
        cmax = __reduce_max_sync(0xffffffffu, cmax);
        cmin = __reduce_min_sync(0xffffffffu, cmin);
        if (tid == 0) { info[28] = INT_MIN; info[29] = INT_MAX; }
        int4 ca = make_int4(c0, c1, 0, 0), cb = make_int4(0, 0, 0, 0);
        sel_total8(ca, cb, red);   // (its first barrier also orders info[28..29] before the extremes below)
        if (lane == 0) { atomicMax(&info[28], cmax); atomicMin(&info[29], cmin); }
        sel_sync();
        cmax = info[28];
        // the radix passes' range: the candidates' own, from the lower estimate on
        const int clo = max(e.x, info[29]);
        CSA2_TRACE(23);   // candidates scored
        // every track needs r candidates at or above its estimate: then its r best scores
        // and all ties at its threshold are candidates
        fail = fail || (act0 && ca.x < p.r[0]) || (act1 && ca.y < p.r[1]);
        if (!fail) {
            const int4 ls = local_select2(csc, act0 ? total : 0, p.r[0], clo, cmax, csc, act1 ? total : 0, p.r[1],
                                          clo, cmax, hist, red, info);
            CSA2_TRACE(24);   // threshold
            ListCut cut[2];
#pragma unroll
            for (int tr = 0; tr < 2; ++tr) {
                const bool on = tr == 0 ? act0 : act1;
                cut[tr].T = tr == 0 ? ls.x : ls.z;
                cut[tr].quota = tr == 0 ? ls.y : ls.w;   // the ties at T ranked within the first r
                cut[tr].all = 0;
                cut[tr].base = 0;
                cut[tr].r = p.r[tr];
                cut[tr].out = on ? p.out[tr] + (size_t)u * p.r[tr] : nullptr;
                cut[tr].status = p.status;
            }
            write_lists<false>(csc, total, 0, cpos, cut[0], cut[1], wsum, row_prefetch(p, u));
            CSA2_TRACE(25);   // lists written
        }
    }
    if (fail && tid == 0 && p.fb_list) {   // the Full kernel scans and cuts this query in full
        const int i = atomicAdd(p.fb_list, 1);
        p.fb_list[1 + i] = u;
    }
    CSA2_TRACE_END(7);
}

size_t mq_select_smem_bytes(bool small, int di) {
    const int cap = small ? kMqCapSmall : kMqCap;
    const int rb = (small || di == 128) ? 4 : 8;
    return 1024 + (size_t)rb * 128 * di + (size_t)std::max(1024, 16 * di) +
           (size_t)(2 * cap + 1088 + 8 * kSelWarps + 64 + 4 * kSelWarps) * 4 + 16;
}

// ------------------------------------------------------------ Reindex, and Full for other key widths
template <int HI, int DI>
__global__ void __launch_bounds__(kSel, 1)
    index_dp4a_kernel(const __grid_constant__ IdxParams p, const __grid_constant__ CUtensorMap kmap) {
    IdxSmem& S = idx_smem();
    CSA2_TRACE_INIT();
    const int tid = threadIdx.x;
    const int group = blockIdx.x / p.G;
    const int cta = blockIdx.x % p.G;
    const Slot sl = slot_of(p, group);
    const bool full = p.mode == CSA2_FULL;
    constexpr bool generic = (HI == 0);
    int* spill = (p.chunk > kSmemScores) ? p.spill + (size_t)blockIdx.x * p.chunk : nullptr;

    const int rows_per_stage = (full ? min(256, kStageBytes / p.Di) : 0);
    const int nchunk = p.Di / 16;

    if (tid < kStages) mbar_init(&S.full_bar[tid], 1);
    mbar_fence_init();
    __syncthreads();
    pdl_launch_dependents();   // the next kernel may start its own set-up
    pdl_wait();                // the workspace, pool and index query may come from the previous kernel
    CSA2_TRACE(1);
    const int epoch = __ldcg(sl.ctrl + CTRL_EPOCH);
    int bar_target = __ldcg(sl.ctrl + CTRL_BAR_BASE);
    uint32_t stage_seq = 0;   // key tiles issued by this CTA so far
    bool alive = true;

    int j = 0;
    for (int u = group; u < p.units && alive; u += p.groups, ++j) {
        const int b = u / p.Tq;
        const int32_t* pool = full ? nullptr : p.pool_in + (size_t)u * p.P_in;
        constexpr int RB = 2;   // Reindex: rows per thread in flight (one pair)
        // Reindex: this CTA's slice of the pool does not depend on the query position
        // (the position only validates the entries), so its first entries and the index
        // query are loaded before the position arrives
        // 64-byte keys with at most 8 heads: four lanes per key row (the row's 16-byte
        // chunks), 128 rows per round, kQuadRounds rounds in flight
        constexpr bool kQuad = (HI == 8 && DI == 64);
        constexpr int kQuadRounds = 8;
        int sidx0[kQuad ? kQuadRounds : RB];
        if (!full) {
            const int lo_r = min(cta * p.chunk, p.P_in), hi_r = min(lo_r + p.chunk, p.P_in);
#pragma unroll
            for (int q2 = 0; q2 < (kQuad ? kQuadRounds : RB); ++q2) {
                const int e = kQuad ? q2 * (kSel / 4) + (tid >> 2) : q2 * kSel + tid;
                sidx0[q2] = (e < hi_r - lo_r) ? __ldg(pool + lo_r + e) : -1;
            }
        }
        const int nq = p.Hi * p.Di / 16;   // int4 chunks of the index query (<= 128)
        const int4 qv = tid < nq ? reinterpret_cast<const int4*>(p.qi + (size_t)u * p.Hi * p.Di)[tid] : make_int4(0, 0, 0, 0);
        int t = p.q_pos[u];
        int tg = last_entry(t, p.m);   // the last global entry the query reads
        const bool bad_t = (t < 0 || tg >= p.N);
        if (bad_t) {
            if (tid == 0 && cta == 0) report(p.status, CSA2_ERR_RANGE, u);
            t = -1;
            tg = -1;
        }
        const int n_all = full ? (tg + 1) : (bad_t ? 0 : p.P_in);
        const int lo = min(cta * p.chunk, n_all);
        const int hi = min(lo + p.chunk, n_all);

        fence_proxy_async_smem();
        if (tid < nq) reinterpret_cast<int4*>(S.q)[tid] = qv;
        for (int i = tid; i < kBins; i += kSel) S.hist0[i] = 0;
        __syncthreads();

        int my_n = hi - lo;
        if (full) {
            const int nst = (my_n + rows_per_stage - 1) / rows_per_stage;
            const uint64_t pol = l2_evict_first_policy();
            if (tid == 0) {
                for (int s2 = 0; s2 < min(kStages, nst); ++s2) {
                    const uint32_t k = stage_seq + s2;
                    mbar_arrive_expect_tx(&S.full_bar[k % kStages], (uint32_t)(rows_per_stage * p.Di));
                    tma_load_keys(S.stage[k % kStages], &kmap, 0, lo + s2 * rows_per_stage, b,
                                  &S.full_bar[k % kStages], pol);
                }
            }
            for (int s2 = 0; s2 < nst; ++s2) {
                const uint32_t k = stage_seq + s2;
                if (!mbar_wait(&S.full_bar[k % kStages], (k / kStages) & 1u, p.status, 2)) alive = false;
                if (__syncthreads_or(!alive)) { alive = false; break; }
                const int e = s2 * rows_per_stage + tid;
                if (tid < rows_per_stage && e < my_n) {
                    const uint8_t* tile = S.stage[k % kStages];
                    int4 rowc[8];
#pragma unroll
                    for (int c2 = 0; c2 < 8; ++c2)
                        if (c2 < nchunk) rowc[c2] = *reinterpret_cast<const int4*>(tile + tile_off(tid, c2, p.Di));
                    const int x = generic ? score_generic(rowc, nchunk, S.q, p.Hi, p.Di, p.w)
                                          : score_smem<(HI > 0 ? HI : 1), (DI > 0 ? DI : 16)>(rowc, S.q, p.w);
                    if (spill) spill[e] = x; else S.sc[e] = x;
                    atomicAdd(&S.hist0[bin0(x)], 1);
                }
                __syncthreads();
                if (tid == 0 && s2 + kStages < nst) {
                    const uint32_t k2 = k + kStages;
                    mbar_arrive_expect_tx(&S.full_bar[k2 % kStages], (uint32_t)(rows_per_stage * p.Di));
                    tma_load_keys(S.stage[k2 % kStages], &kmap, 0, lo + (s2 + kStages) * rows_per_stage, b,
                                  &S.full_bar[k2 % kStages], pol);
                }
            }
            stage_seq += nst;
            if (!alive) break;
        } else {
            // Reindex: valid pool entries (0 <= s <= t) form a prefix, -1 padding after.
            // Entries, their check and the key rows come in one dependent chain; the
            // histogram is built once the valid prefix is known.
            const int8_t* kb = p.ki + (size_t)b * p.ki_seq_stride;
            constexpr int kCh = DI > 0 ? DI / 16 : 8;   // 16-byte chunks per key row
            int first_bad = my_n;
            int* lpos = p.local_sel ? wlists(S) : nullptr;   // the chunk's positions, for the ordered write
            if constexpr (kQuad) {
                // lane l of a quad holds chunk l % 4 of its row: one load instruction of a
                // warp covers 8 rows (8 lines instead of 32). Each lane's partial dot products
                // of the 8 heads are summed over the quad by two halving exchanges (each lane
                // ends with two heads), then ReLU, weights and a quad sum give the score.
                const int sub = tid & 3, rw = tid >> 2;
                const int hb = ((sub >> 1) & 1) * 4 + (sub & 1) * 2;   // this lane's two heads
                const int wa = hb == 0 ? p.w[0] : hb == 2 ? p.w[2] : hb == 4 ? p.w[4] : p.w[6];
                const int wb = hb == 0 ? p.w[1] : hb == 2 ? p.w[3] : hb == 4 ? p.w[5] : p.w[7];
                int4 qc[8];
#pragma unroll
                for (int h = 0; h < 8; ++h) qc[h] = reinterpret_cast<const int4*>(S.q + h * 64)[sub];
#pragma unroll 1
                for (int e0 = 0; e0 < my_n; e0 += kQuadRounds * (kSel / 4)) {
                    int sidx[kQuadRounds];
                    bool okr[kQuadRounds];
                    int4 kv[kQuadRounds];
#pragma unroll
                    for (int rd = 0; rd < kQuadRounds; ++rd) {
                        const int e = e0 + rd * (kSel / 4) + rw;
                        sidx[rd] = (e0 == 0) ? sidx0[rd] : ((e < my_n) ? __ldg(pool + lo + e) : -1);
                    }
#pragma unroll
                    for (int rd = 0; rd < kQuadRounds; ++rd) {
                        const int e = e0 + rd * (kSel / 4) + rw;
                        okr[rd] = e < my_n && sidx[rd] >= 0 && sidx[rd] <= tg;
                        if (e < my_n && !okr[rd]) first_bad = min(first_bad, e);
                        kv[rd] = okr[rd] ? __ldg(reinterpret_cast<const int4*>(kb + (size_t)sidx[rd] * 64) + sub)
                                         : make_int4(0, 0, 0, 0);
                        if (lpos != nullptr && sub == 0 && okr[rd]) lpos[e] = sidx[rd];
                    }
#pragma unroll
                    for (int rd = 0; rd < kQuadRounds; ++rd) {
                        if (e0 + rd * (kSel / 4) >= my_n) break;   // warp-uniform
                        int acc[8];
#pragma unroll
                        for (int h = 0; h < 8; ++h) {
                            int a2 = __dp4a(kv[rd].x, qc[h].x, 0);
                            a2 = __dp4a(kv[rd].y, qc[h].y, a2);
                            a2 = __dp4a(kv[rd].z, qc[h].z, a2);
                            acc[h] = __dp4a(kv[rd].w, qc[h].w, a2);
                        }
                        const bool up2 = (sub & 2) != 0, up1 = (sub & 1) != 0;
                        int v4[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            const int send = up2 ? acc[h] : acc[h + 4], keep = up2 ? acc[h + 4] : acc[h];
                            v4[h] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                        }
                        int v2[2];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int send = up1 ? v4[h] : v4[h + 2], keep = up1 ? v4[h + 2] : v4[h];
                            v2[h] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
                        }
                        int x = wa * max(v2[0], 0) + wb * max(v2[1], 0);
                        x += __shfl_xor_sync(0xffffffffu, x, 1);
                        x += __shfl_xor_sync(0xffffffffu, x, 2);
                        const int e = e0 + rd * (kSel / 4) + rw;
                        if (sub == 0 && okr[rd]) { if (spill) spill[e] = x; else S.sc[e] = x; }
                    }
                }
            } else {
#pragma unroll 1
            for (int e0 = 0; e0 < my_n; e0 += RB * kSel) {
                int sidx[RB];
                bool okr[RB];
                int4 rows[RB][kCh];
#pragma unroll
                for (int q2 = 0; q2 < RB; ++q2) {
                    const int e = e0 + q2 * kSel + tid;
                    sidx[q2] = (e0 == 0) ? sidx0[q2] : ((e < my_n) ? __ldg(pool + lo + e) : -1);
                    okr[q2] = e < my_n && sidx[q2] >= 0 && sidx[q2] <= tg;
                    if (lpos != nullptr && okr[q2]) lpos[e] = sidx[q2];
                    if (e < my_n && !okr[q2]) first_bad = min(first_bad, e);
                    if (okr[q2]) {
                        const int4* row = reinterpret_cast<const int4*>(kb + (size_t)sidx[q2] * p.Di);
#pragma unroll
                        for (int c2 = 0; c2 < kCh; ++c2)
                            if (c2 < nchunk) rows[q2][c2] = __ldg(row + c2);
                    }
                }
#pragma unroll
                for (int q2 = 0; q2 < RB; q2 += 2) {
                    if (!okr[q2] && !okr[q2 + 1]) continue;
                    int xa, xb;
                    if (generic) {
                        xa = okr[q2] ? score_generic(rows[q2], nchunk, S.q, p.Hi, p.Di, p.w) : 0;
                        xb = okr[q2 + 1] ? score_generic(rows[q2 + 1], nchunk, S.q, p.Hi, p.Di, p.w) : 0;
                    } else {
                        score2_smem<(HI > 0 ? HI : 1), (DI > 0 ? DI : 16)>(rows[q2], rows[q2 + 1], S.q, p.w, xa, xb);
                    }
                    const int ea = e0 + q2 * kSel + tid, eb = ea + kSel;
                    if (okr[q2]) { if (spill) spill[ea] = xa; else S.sc[ea] = xa; }
                    if (okr[q2 + 1]) { if (spill) spill[eb] = xb; else S.sc[eb] = xb; }
                }
            }
            }
            const int fb = sel_min(first_bad, S.red);
            if (fb < my_n) {
                // an entry past the first invalid one must be padding, never a position
                for (int e = fb + tid; e < my_n; e += kSel)
                    if (__ldg(pool + lo + e) >= 0) report(p.status, CSA2_ERR_RANGE, u);
                my_n = fb;
            }
            if (my_n > 0 && lo > 0 && tid == 0 && __ldg(pool + lo - 1) < 0) report(p.status, CSA2_ERR_RANGE, u);
#pragma unroll 1
            for (int e = tid; e < my_n; e += kSel) atomicAdd(&S.hist0[bin0(spill ? spill[e] : S.sc[e])], 1);
        }
        __syncthreads();
        CSA2_TRACE(2);   // scores done
        UnitCtx c{u, t, lo, my_n, n_all, cta, j, epoch, pool};
        if (!full && p.local_sel)
            alive = reindex_local_unit(p, S, sl, c, bar_target);
        else if (!full && p.G == 1 && !spill)
            alive = reindex_single_unit(p, S, sl, c);
        else
            alive = spill ? select_unit<true>(p, S, sl, c, bar_target, spill)
                          : select_unit<false>(p, S, sl, c, bar_target, S.sc);
        __syncthreads();
    }
    CSA2_TRACE(11);
    CSA2_TRACE_END(2);
    if (alive && cta == 0 && tid == 0) {
        sl.ctrl[CTRL_EPOCH] = epoch + j;
        sl.ctrl[CTRL_BAR_BASE] = bar_target;
    }
}

// ------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// Failure-detection controls (csa2_set_wait_controls): process-wide, read at launch.
static std::atomic<long long> g_wait_budget{kSpinBudgetCycles};
static std::atomic<int> g_skip_arrival{0};

long long group_wait_budget() { return g_wait_budget.load(); }
int group_skip_arrival() { return g_skip_arrival.load(); }

void set_wait_controls(long long budget, int skip) {
    g_wait_budget.store(budget > 0 ? budget : kSpinBudgetCycles);
    g_skip_arrival.store(skip ? 1 : 0);
}

struct IdxPlan {
    int units, G, groups, chunk;
    int local_sel, rstride;
    int mq;              // Full with queries sharing keys: sample, estimate, mark, cut (+ Full for the rest)
    int mq_tstep, mq_cap;
    int64_t mq_sstride, mq_wstride;
    int fb_groups, fb_G, fb_chunk;   // the Full kernel for the queries the cut leaves
    size_t off_sample, off_words, off_est, off_fb;   // scratch offsets (the fallback's spill at 0)
    size_t spill_bytes;
};

int num_sms() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Fixed layout of the persistent indexer region: one slot per SM, so a slot's
// state (barrier counter, epoch, histogram buffers) sits at the same address in
// every call that shares the workspace.
struct IdxRegion {
    size_t off_ctrl, off_g0, off_gl, off_cand, off_pub, bytes;
};

IdxRegion idx_region(int slots) {
    IdxRegion r{};
    size_t off = 0;
    r.off_ctrl = off; off += align_up((size_t)slots * kCtrlInts * 4, 256);
    r.off_g0 = off;   off += align_up((size_t)slots * 3 * kG0Stride * 4, 256);
    r.off_gl = off;   off += align_up((size_t)slots * 4 * kBins * 4, 256);
    r.off_cand = off; off += align_up((size_t)slots * 2 * kCandCap * 8, 256);
    r.off_pub = off;  off += align_up((size_t)slots * 6 * kMaxG * 4, 256);
    r.bytes = off;
    return r;
}

size_t index_region_bytes() { return idx_region(num_sms()).bytes; }

IdxPlan plan_index(const csa2_index_args& a, int sms) {
    IdxPlan pl{};
    pl.units = a.B * a.Tq;
    const int n_max = (a.mode == CSA2_FULL) ? a.N : a.P_in;
    // A Reindex pool that one CTA's shared memory holds is cut without the distributed select,
    // whose 64-element steps want 256-aligned chunks: its groups take chunks down to 512 entries.
    const bool rx_small = a.mode == CSA2_REINDEX && a.P_in <= kSmemScores;
    const int min_chunk = rx_small ? 512 : 1024;
    if (pl.units >= sms) {
        pl.G = 1;
        pl.groups = sms;
    } else {
        pl.groups = pl.units;
        pl.G = std::max(1, std::min(kMaxG, sms / pl.units));
        pl.G = std::max(1, std::min(pl.G, (n_max + min_chunk - 1) / min_chunk));
    }
    int chunk = (n_max + pl.G - 1) / pl.G;
    chunk = (int)align_up((size_t)std::max(chunk, 1), rx_small ? 64 : 256);
    pl.chunk = chunk;
    pl.spill_bytes = 0;
    // (+ 512 bytes: the select's 64-element steps may read up to 63 elements past a chunk's end)
    if (chunk > kSmemScores) pl.spill_bytes = align_up((size_t)pl.groups * pl.G * chunk * 4 + 512, 256);
    // Reindex with a pool that fits one CTA: published scores, one select per group
    pl.local_sel = (a.mode == CSA2_REINDEX && pl.G > 1 && a.P_in <= kSmemScores) ? 1 : 0;
    pl.rstride = (int)align_up((size_t)std::max(a.P_in, 1), 4);
    if (pl.local_sel) pl.spill_bytes = std::max(pl.spill_bytes, align_up((size_t)pl.units * pl.rstride * 4, 256));
    // (below kMqMinN keys the second launch costs more than the shared tiles save)
    pl.mq = (a.mode == CSA2_FULL && a.Tq >= kMqMin && a.N >= kMqMinN && a.Hi <= 8 &&
             (a.Di == 32 || a.Di == 64 || a.Di == 128)) ? 1 : 0;
    if (pl.mq) {
        // (replaces the plan above) 32 to 128 sampled tiles, at least one in 64 (the estimate
        // then ranks about r / 64 samples or more); a candidate word per 32 positions
        const int ntile = (a.N + kMqRows - 1) / kMqRows;
        const int want = std::min(128, std::max(32, (ntile + 63) / 64));
        pl.mq_tstep = std::max(1, (ntile + want - 1) / want);
        pl.mq_sstride = (int64_t)((ntile + pl.mq_tstep - 1) / pl.mq_tstep) * kMqRows;
        pl.mq_wstride = (int64_t)ntile * 4;
        // candidates expected: about 1.2 r + 16 n / m a track (r the larger track); the two-CTAs-per-SM
        // cut when half its room covers that
        const int m_s = (int)std::min<int64_t>(pl.mq_sstride, (int64_t)a.N);
        const int r_max = std::max(a.P, a.k);
        const long long expect = (long long)r_max * 6 / 5 + 16LL * a.N / std::max(m_s, 1);
        pl.mq_cap = (2 * expect <= kMqCapSmall && a.Di <= 64) ? kMqCapSmall : kMqCap;
        // the fallback (a few queries a call at most, as a rule): up to 16 queries at a time, groups of
        // fb_G CTAs each over the SMs, their scores spilled where a chunk exceeds shared memory (at most 64 MB)
        const size_t all = align_up((size_t)a.N, 256) * 4;
        pl.fb_groups = (int)std::max<size_t>(1, std::min<size_t>({(size_t)16, (size_t)pl.units, ((size_t)64 << 20) / all}));
        pl.fb_G = std::max(1, std::min({kMaxG, sms / pl.fb_groups, (a.N + 1023) / 1024}));
        pl.fb_chunk = (int)align_up((size_t)((a.N + pl.fb_G - 1) / pl.fb_G), 256);
        const size_t per = (size_t)pl.fb_chunk * 4;
        size_t off = pl.fb_chunk > kSmemScores ? align_up((size_t)pl.fb_groups * pl.fb_G * per + 512, 256) : 0;
        pl.off_sample = off;  off += align_up((size_t)pl.units * pl.mq_sstride * 4, 256);
        pl.off_words = off;   off += align_up((size_t)pl.units * pl.mq_wstride * 4, 256);
        pl.off_est = off;     off += align_up((size_t)pl.units * 16, 256);
        pl.off_fb = off;      off += align_up((size_t)(pl.units + 1) * 4, 256);
        pl.spill_bytes = off;
    }
    return pl;
}

size_t index_smem_bytes() { return sizeof(IdxSmem) + 1024; }

template <typename Kern>
static cudaError_t launch_coop(Kern kern, int threads, const IdxParams& p, const CUtensorMap& map, int grid,
                               cudaStream_t stream) {
    const size_t smem = index_smem_bytes();
    cudaError_t e = set_smem_once(reinterpret_cast<const void*>(kern), (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    // Programmatic dependent launch on top of the cooperative one: the kernel may be
    // scheduled while the previous kernel drains (every kernel of this library calls
    // griddepcontrol.launch_dependents only once all of its own CTAs are resident, so
    // neither grid can keep the other's CTAs off the device). A runtime that refuses
    // the pair gets the plain cooperative launch from then on.
    static std::atomic<int> coop_pdl{1};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = coop_pdl.load() ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, kern, p, map);
    if (e != cudaSuccess && cfg.numAttrs == 2) {
        (void)cudaGetLastError();
        coop_pdl.store(0);
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kern, p, map);
    }
    return e;
}

// Cluster launch of the Full kernel: clusters of q.G CTAs, q.groups clusters, programmatic
// stream serialisation (the kernel reads nothing the previous kernel writes before
// griddepcontrol.wait, except that a producer with keys_ready starts the key stream).
template <int DI, int MODE>
static cudaError_t launch_mq(const MqParams& mp, const CUtensorMap& map, int grid, cudaStream_t stream) {
    auto kern = index_mq_score_kernel<DI, MODE>;
    // at least 116 KB, so that one CTA (and its 512 TMEM columns) holds an SM
    const size_t smem = std::max(sizeof(MqSmem<DI>) + 1024, (size_t)116 * 1024);
    cudaError_t e = set_smem_once(reinterpret_cast<const void*>(kern), (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kMqThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mp, map);
}

// One CTA per query, programmatic dependent launch (nothing is read before griddepcontrol.wait).
// smem_max: the kernel's largest dynamic shared memory over all calls (its attribute is set once).
template <typename Kern>
static cudaError_t launch_per_query(Kern kern, const IdxParams& p, size_t smem, size_t smem_max, cudaStream_t stream) {
    if (smem_max > 48 * 1024) {
        cudaError_t e = set_smem_once(reinterpret_cast<const void*>(kern), (int)smem_max);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(p.units);
    cfg.blockDim = dim3(kSel);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

// The cut, in its two-CTAs-per-SM form (8192 candidates) or its one-CTA form (16384).
template <int DI>
static cudaError_t launch_cut(const IdxParams& p, bool small, cudaStream_t stream) {
    const size_t ssm = mq_select_smem_bytes(small, DI);
    return small ? launch_per_query(index_mq_select_kernel<DI, true>, p, ssm, ssm, stream)
                 : launch_per_query(index_mq_select_kernel<DI, false>, p, ssm, ssm, stream);
}

// The shared-key steps (sample, estimate, mark, cut) and the Full kernel for the
// queries the cut leaves over.
template <int DI>
static cudaError_t launch_mq_steps(const csa2_index_args& a, const IdxPlan& pl, const IdxParams& p0,
                                   const CUtensorMap& map, const CUtensorMap& mmap, uint8_t* scratch, int sms,
                                   cudaStream_t stream) {
    IdxParams p = p0;
    p.mq_sample = reinterpret_cast<int32_t*>(scratch + pl.off_sample);
    p.mq_sstride = pl.mq_sstride;
    p.mq_tstep = pl.mq_tstep;
    p.mq_est = reinterpret_cast<int4*>(scratch + pl.off_est);
    p.mq_words = reinterpret_cast<int32_t*>(scratch + pl.off_words);
    p.mq_wstride = pl.mq_wstride;
    p.fb_list = reinterpret_cast<int32_t*>(scratch + pl.off_fb);
    MqParams mp{};
    mp.B = a.B; mp.Tq = a.Tq; mp.N = a.N; mp.Hi = a.Hi;
    mp.nblk = (a.Tq + kMqQ - 1) / kMqQ;
    const int items = a.B * mp.nblk;
    for (int h = 0; h < 8; ++h) mp.w[h] = h < a.Hi ? a.w[h] : 0;
    mp.q_pos = a.q_pos; mp.qi = a.qi;
    mp.m = a.m;
    mp.status = p.status;
    // 1. the sampled tiles
    mp.splits = std::max(1, std::min(sms / std::max(items, 1), (int)(pl.mq_sstride / kMqRows) / 8));
    mp.tstep = pl.mq_tstep;
    mp.out = const_cast<int32_t*>(p.mq_sample);
    mp.ostride = pl.mq_sstride;
    cudaError_t e = launch_mq<DI, kMqSample>(mp, mmap, items * mp.splits, stream);
    if (e != cudaSuccess) return e;
    // 2. the estimates
    e = launch_per_query(index_mq_estimate_kernel, p, mq_estimate_smem_bytes((int)pl.mq_sstride),
                         mq_estimate_smem_bytes(kMqSampleMax), stream);
    if (e != cudaSuccess) return e;
    // 3. the candidate words: each block's tiles split so that the grid covers the SMs, at least 8 tiles a split
    mp.splits = std::max(1, std::min(sms / std::max(items, 1), (a.N / kMqRows + 7) / 8));
    mp.tstep = 1;
    mp.out = const_cast<int32_t*>(p.mq_words);
    mp.ostride = pl.mq_wstride;
    mp.est = p.mq_est;
    e = launch_mq<DI, kMqMark>(mp, mmap, items * mp.splits, stream);
    if (e != cudaSuccess) return e;
    // 4. the cut
    e = launch_cut<DI>(p, pl.mq_cap == kMqCapSmall, stream);
    if (e != cudaSuccess) return e;
    // 5. the queries it left: the Full kernel over the list
    IdxParams f = p0;
    f.G = pl.fb_G;
    f.groups = pl.fb_groups;
    f.chunk = pl.fb_chunk;
    f.spill = reinterpret_cast<int32_t*>(scratch);
    f.unit_list = p.fb_list;
    f.keys_ready = 0;
    f.local_sel = 0;
    return launch_coop(index_full_tc_kernel<DI>, kTcThreads, f, map, pl.fb_groups * pl.fb_G, stream);
}

// Launch one indexer call. `ws` holds plan_index(a).ws_bytes bytes (zero at first use).
csa2_status launch_index(const csa2_index_args& a, const int32_t* pool_in, int P_in, void* region, void* scratch,
                         int32_t* d_status, cudaStream_t stream, const csa2_attn_args* pf, int keys_ready) {
    const int sms = num_sms();
    csa2_index_args aa = a;
    aa.P_in = P_in;
    IdxPlan pl = plan_index(aa, sms);
    IdxParams p{};
    p.mode = a.mode;
    p.B = a.B; p.Tq = a.Tq; p.N = a.N; p.Hi = a.Hi; p.Di = a.Di;
    p.r[0] = (a.mode == CSA2_FULL) ? a.P : 0;
    p.r[1] = a.k;
    p.out[0] = a.pool_out;
    p.out[1] = a.topk_out;
    p.q_pos = a.q_pos; p.qi = a.qi;
    for (int h = 0; h < 16; ++h) p.w[h] = h < a.Hi ? a.w[h] : 0;
    p.ki = a.ki; p.ki_seq_stride = a.ki_seq_stride;
    p.pool_in = pool_in; p.P_in = P_in;
    p.units = pl.units; p.G = pl.G; p.groups = pl.groups; p.chunk = pl.chunk;
    const IdxRegion rg = idx_region(sms);
    uint8_t* base = static_cast<uint8_t*>(region);
    p.ctrl = reinterpret_cast<int*>(base + rg.off_ctrl);
    p.g0 = reinterpret_cast<int*>(base + rg.off_g0);
    p.gl = reinterpret_cast<int*>(base + rg.off_gl);
    p.cand = reinterpret_cast<int2*>(base + rg.off_cand);
    p.pub = reinterpret_cast<int*>(base + rg.off_pub);
    p.spill = (pl.chunk > kSmemScores && !pl.mq) ? static_cast<int32_t*>(scratch) : nullptr;
    p.local_sel = pl.local_sel;
    p.rstride = pl.rstride;
    p.rscore = pl.local_sel ? static_cast<int32_t*>(scratch) : nullptr;
    if (pf != nullptr && pf->kv_fp4 != nullptr && pf->kv_scale != nullptr && pf->B == a.B) {
        p.pf_fp4 = pf->kv_fp4;
        p.pf_scale = pf->kv_scale;
        p.pf_N = pf->N;
        p.pf_code_bytes = pf->D / 2;
        p.pf_scale_bytes = pf->D / 16;
    }
    p.keys_ready = keys_ready;
    p.m = a.m;
    p.status = d_status;
    p.wait_budget = group_wait_budget();
    p.skip_arrival = group_skip_arrival();

    CUtensorMap map;
    memset(&map, 0, sizeof(map));
    if (a.mode == CSA2_FULL) {
        EncodeTiledFn enc = get_encode_fn();
        if (!enc) return CSA2_ERR_CUDA;
        const int rows = std::min(256, kStageBytes / a.Di);
        cuuint64_t dims[3] = {(cuuint64_t)a.Di, (cuuint64_t)a.N, (cuuint64_t)a.B};
        cuuint64_t strides[2] = {(cuuint64_t)a.Di, (cuuint64_t)a.ki_seq_stride};
        cuuint32_t box[3] = {(cuuint32_t)a.Di, (cuuint32_t)rows, 1};
        cuuint32_t estr[3] = {1, 1, 1};
        CUtensorMapSwizzle swz = a.Di == 32    ? CU_TENSOR_MAP_SWIZZLE_32B
                                 : a.Di == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
                                 : a.Di == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                               : CU_TENSOR_MAP_SWIZZLE_NONE;
        CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t*>(a.ki), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return CSA2_ERR_CUDA;
    }
    const int grid = pl.groups * pl.G;
    cudaError_t e;
    if (pl.mq) {
        // key tiles shared by blocks of kMqQ queries
        EncodeTiledFn enc = get_encode_fn();
        if (!enc) return CSA2_ERR_CUDA;
        CUtensorMap mmap;
        memset(&mmap, 0, sizeof(mmap));
        cuuint64_t dims[3] = {(cuuint64_t)a.Di, (cuuint64_t)a.N, (cuuint64_t)a.B};
        cuuint64_t strides[2] = {(cuuint64_t)a.Di, (cuuint64_t)a.ki_seq_stride};
        cuuint32_t box[3] = {(cuuint32_t)a.Di, (cuuint32_t)kMqRows, 1};
        cuuint32_t estr[3] = {1, 1, 1};
        CUtensorMapSwizzle swz = a.Di == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                 : a.Di == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                              : CU_TENSOR_MAP_SWIZZLE_128B;
        CUresult r = enc(&mmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t*>(a.ki), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return CSA2_ERR_CUDA;
        uint8_t* sc = static_cast<uint8_t*>(scratch);
        e = a.Di == 64   ? launch_mq_steps<64>(a, pl, p, map, mmap, sc, sms, stream)
            : a.Di == 32 ? launch_mq_steps<32>(a, pl, p, map, mmap, sc, sms, stream)
                         : launch_mq_steps<128>(a, pl, p, map, mmap, sc, sms, stream);
        return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
    }
    if (a.mode == CSA2_REINDEX && pl.units >= sms && P_in > 0 && P_in <= kMqCap && a.Hi <= 8 &&
        (a.Di == 32 || a.Di == 64 || a.Di == 128)) {
        // one CTA per query: the pool is the cut's candidate list, rescored on the tensor cores
        const bool small = P_in <= kMqCapSmall && a.Di <= 64;
        e = a.Di == 64 ? launch_cut<64>(p, small, stream) : a.Di == 32 ? launch_cut<32>(p, small, stream)
                                                                       : launch_cut<128>(p, small, stream);
        return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
    }
    if (a.mode == CSA2_FULL && a.Di == 64) e = launch_coop(index_full_tc_kernel<64>, kTcThreads, p, map, grid, stream);
    else if (a.mode == CSA2_FULL && a.Di == 32) e = launch_coop(index_full_tc_kernel<32>, kTcThreads, p, map, grid, stream);
    else if (a.mode == CSA2_FULL && a.Di == 128) e = launch_coop(index_full_tc_kernel<128>, kTcThreads, p, map, grid, stream);
    else if (a.Hi <= 8 && a.Di == 64) e = launch_coop(index_dp4a_kernel<8, 64>, kSel, p, map, grid, stream);
    else if (a.Hi <= 4 && a.Di == 32) e = launch_coop(index_dp4a_kernel<4, 32>, kSel, p, map, grid, stream);
    else e = launch_coop(index_dp4a_kernel<0, 0>, kSel, p, map, grid, stream);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

size_t index_scratch_bytes(const csa2_index_args& a, int P_in) {
    csa2_index_args aa = a;
    aa.P_in = P_in;
    return plan_index(aa, num_sms()).spill_bytes;
}

}  // namespace csa2

CSA2_TRACE_SETTER(csa2_trace_set_idx)
