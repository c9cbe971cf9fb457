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
// candidates into shared memory (Full: key tiles arrive by TMA into a 4-stage
// ring; Reindex: pool rows are gathered with 16-byte loads), then the group
// finds the exact k-th best with a distributed radix select on a 36-bit
// order-preserving key of the score: a 12-bit log-scale digit first, then two
// 12-bit digits of the remaining bits. Each round costs one group barrier
// (an atomic counter with a bounded spin). Once the threshold digit holds at
// most kCandCap elements, they are gathered and every CTA sorts them (score,
// position) in shared memory and knows the exact cut; exact ties at the last
// digit are cut by position through per-CTA counts. Every CTA then writes its
// selected positions at its offset, in ascending order, with no further sync.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "csa2_common.cuh"

namespace csa2 {

constexpr int kIdxThreads = 256;
constexpr int kBins = 4096;
constexpr int kCandCap = 4096;
constexpr int kStageBytes = 16384;
constexpr int kStages = 4;
constexpr int kSmemScores = 16384;                  // scores kept in shared memory
constexpr int kSkewLen = kSmemScores / 64 * 65;     // padded: one spare word per 64
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
    int32_t* spill;      // [groups*G][skewed chunk] when chunk > kSmemScores
    int* ctrl;           // [groups][kCtrlInts]
    int* g0;             // [groups][3][kBins]
    int* gl;             // [groups][2 tracks][2 levels][kBins]
    int2* cand;          // [groups][2 tracks][kCandCap]
    int* pub;            // [groups][2 tracks][2][kMaxG]
    int32_t* status;
};

struct __align__(16) IdxSmem {
    uint8_t stage[kStages][kStageBytes];   // key tiles; later the candidate sort buffer
    int sc[kSkewLen];                      // scores of this CTA's chunk (skewed index)
    int hist0[kBins];
    int histl[2][kBins];
    int8_t q[16 * 128];
    uint64_t full_bar[kStages];
    int red[64];
    int info[64];
};
static_assert(sizeof(uint64_t) * kCandCap <= sizeof(((IdxSmem*)0)->stage), "candidate buffer");

__device__ __forceinline__ int skew(int e) { return (e >> 6) * 65 + (e & 63); }

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

// composite key: larger = ranked earlier (higher score, then lower index)
__device__ __forceinline__ uint64_t comp_key(int32_t x, int idx) {
    return (ext_key(x) << 27) | (uint64_t)(0x7FFFFFF - idx);
}

// ------------------------------------------------------------ block helpers
// Exclusive scan over the block (256 threads); returns the block total in `total`.
__device__ __forceinline__ int block_scan_excl(int v, int* red, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    __syncthreads();
    if (lane == 31) red[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int s = lane < (kIdxThreads / 32) ? red[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < kIdxThreads / 32) red[32 + lane] = s;
    }
    __syncthreads();
    const int warp_excl = warp ? red[32 + warp - 1] : 0;
    total = red[32 + kIdxThreads / 32 - 1];
    return warp_excl + x - v;
}

__device__ __forceinline__ int block_sum(int v, int* red) {
    int total;
    block_scan_excl(v, red, total);
    return total;
}

// Group barrier over the G CTAs of a slot: counter increments once per CTA.
__device__ bool group_barrier(int* counter, int target, int32_t* st) {
    __syncthreads();
    int ok = 1;
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(counter, 1);
        if (ld_acquire_gpu(counter) < target) {
            const long long t0 = clock64();
            while (ld_acquire_gpu(counter) < target) {
                if (clock64() - t0 > kSpinBudgetCycles) {
                    report(st, CSA2_ERR_TIMEOUT, 1);
                    ok = 0;
                    break;
                }
                __nanosleep(32);
            }
        }
        __threadfence();
    }
    return __syncthreads_and(ok) != 0;
}

// In a global 4096-bin histogram, find the bin holding the r-th largest element
// (1-based). Writes {bin, count above the bin, count in the bin} to out[0..2].
__device__ void find_rank_bin(const int* hist, int r, int* red, int* out) {
    const int t = threadIdx.x;
    int h[16];
    const int4* src = reinterpret_cast<const int4*>(hist + 16 * t);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int4 v = __ldcg(src + i);
        h[4 * i] = v.x; h[4 * i + 1] = v.y; h[4 * i + 2] = v.z; h[4 * i + 3] = v.w;
    }
    int s = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) s += h[i];
    int total;
    const int excl = block_scan_excl(s, red, total);
    int above = total - excl - s;    // elements in bins above this thread's range
    if (above < r && r <= above + s) {
#pragma unroll
        for (int i = 15; i >= 0; --i) {
            if (above < r && r <= above + h[i]) {
                out[0] = 16 * t + i;
                out[1] = above;
                out[2] = h[i];
            }
            above += h[i];
        }
    }
    __syncthreads();
}

// Push the non-zero bins of a shared histogram into a global one.
__device__ __forceinline__ void push_hist(const int* sh, int* gh) {
    for (int i = threadIdx.x; i < kBins; i += kIdxThreads) {
        const int v = sh[i];
        if (v) atomicAdd(gh + i, v);
    }
}

__device__ __forceinline__ int sum_above(const int* sh, int bin) {
    int s = 0;
    for (int i = threadIdx.x; i < kBins; i += kIdxThreads) s += (i > bin) ? sh[i] : 0;
    return s;
}

// Bitonic sort of n (power of two) 64-bit keys in shared memory, descending.
__device__ void bitonic_desc(uint64_t* a, int n) {
    for (int k = 2; k <= n; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < n; i += kIdxThreads) {
                const int l = i ^ j;
                if (l > i) {
                    const uint64_t x = a[i], y = a[l];
                    const bool desc = (i & k) == 0;
                    if (desc ? (x < y) : (x > y)) { a[i] = y; a[l] = x; }
                }
            }
            __syncthreads();
        }
    }
}

// ------------------------------------------------------------ scoring
template <int HI, int DI>
struct RegQ {
    int q[HI][DI / 4];
    __device__ void load(const int8_t* qs) {
#pragma unroll
        for (int h = 0; h < HI; ++h)
#pragma unroll
            for (int d = 0; d < DI / 4; ++d) q[h][d] = reinterpret_cast<const int*>(qs + h * DI)[d];
    }
    // score of one key row given as DI/16 int4 chunks (chunk c = bytes 16c..16c+15)
    __device__ __forceinline__ int score(const int4* rowc, const int32_t* w) const {
        int acc[HI];
#pragma unroll
        for (int h = 0; h < HI; ++h) acc[h] = 0;
#pragma unroll
        for (int c = 0; c < DI / 16; ++c) {
            const int4 k = rowc[c];
#pragma unroll
            for (int h = 0; h < HI; ++h) {
                acc[h] = __dp4a(k.x, q[h][4 * c + 0], acc[h]);
                acc[h] = __dp4a(k.y, q[h][4 * c + 1], acc[h]);
                acc[h] = __dp4a(k.z, q[h][4 * c + 2], acc[h]);
                acc[h] = __dp4a(k.w, q[h][4 * c + 3], acc[h]);
            }
        }
        int s = 0;
#pragma unroll
        for (int h = 0; h < HI; ++h) s += w[h] * max(acc[h], 0);
        return s;
    }
};

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

__device__ __forceinline__ void tma_load_keys(void* dst, const CUtensorMap* map, int x, int y, int z,
                                              uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
        "%4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------------------ the kernel
template <int HI, int DI>
__global__ void __launch_bounds__(kIdxThreads, 1)
    index_select_kernel(const __grid_constant__ IdxParams p, const __grid_constant__ CUtensorMap kmap) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    IdxSmem& S = *reinterpret_cast<IdxSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    const int group = blockIdx.x / p.G;
    const int cta = blockIdx.x % p.G;
    const bool full = p.mode == CSA2_FULL;
    const bool generic = (HI == 0);

    int* ctrl = p.ctrl + (size_t)group * kCtrlInts;
    int* g0 = p.g0 + (size_t)group * 3 * kBins;
    int* gl = p.gl + (size_t)group * 4 * kBins;
    int2* cand = p.cand + (size_t)group * 2 * kCandCap;
    int* pub = p.pub + (size_t)group * 4 * kMaxG;
    int* sc = (p.chunk > kSmemScores) ? p.spill + (size_t)blockIdx.x * ((p.chunk + 63) / 64 * 65) : S.sc;

    const int epoch = __ldcg(ctrl + CTRL_EPOCH);
    int bar_target = __ldcg(ctrl + CTRL_BAR_BASE);
    const int rows_per_stage = (full ? min(256, kStageBytes / p.Di) : 0);
    const int nchunk = p.Di / 16;

    if (tid < kStages) mbar_init(&S.full_bar[tid], 1);
    mbar_fence_init();
    __syncthreads();
    uint32_t stage_seq = 0;   // stages issued by this CTA so far
    bool alive = true;

    int j = 0;
    for (int u = group; u < p.units && alive; u += p.groups, ++j) {
        const int b = u / p.Tq;
        int t = p.q_pos[u];
        bool bad_t = (t < 0 || t >= p.N);
        if (bad_t) {
            if (tid == 0 && cta == 0) report(p.status, CSA2_ERR_RANGE, u);
            t = -1;
        }
        // candidates of this unit: Full -> positions 0..t; Reindex -> pool entries
        const int n_all = full ? (t + 1) : (bad_t ? 0 : p.P_in);
        const int lo = min(cta * p.chunk, n_all);
        const int hi = min(lo + p.chunk, n_all);
        const int32_t* pool = full ? nullptr : p.pool_in + (size_t)u * p.P_in;

        // ---- indexer query and local histogram
        for (int i = tid; i < p.Hi * p.Di / 16; i += kIdxThreads)
            reinterpret_cast<int4*>(S.q)[i] = reinterpret_cast<const int4*>(p.qi + (size_t)u * p.Hi * p.Di)[i];
        for (int i = tid; i < kBins; i += kIdxThreads) S.hist0[i] = 0;
        __syncthreads();
        RegQ<(HI > 0 ? HI : 1), (DI > 0 ? DI : 16)> rq;
        if (!generic) rq.load(S.q);

        // ---- score own chunk
        int my_n = hi - lo;
        if (full) {
            const int nst = (my_n + rows_per_stage - 1) / rows_per_stage;
            if (tid == 0) {
                for (int s = 0; s < min(kStages, nst); ++s) {
                    const uint32_t k = stage_seq + s;
                    mbar_arrive_expect_tx(&S.full_bar[k % kStages], (uint32_t)(rows_per_stage * p.Di));
                    tma_load_keys(S.stage[k % kStages], &kmap, 0, lo + s * rows_per_stage, b,
                                  &S.full_bar[k % kStages]);
                }
            }
            for (int s = 0; s < nst; ++s) {
                const uint32_t k = stage_seq + s;
                if (!mbar_wait(&S.full_bar[k % kStages], (k / kStages) & 1u, p.status, 2)) { alive = false; }
                if (__syncthreads_or(!alive)) { alive = false; break; }
                const int e = s * rows_per_stage + tid;
                if (tid < rows_per_stage && e < my_n) {
                    const uint8_t* tile = S.stage[k % kStages];
                    int4 rowc[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        if (c < nchunk) rowc[c] = *reinterpret_cast<const int4*>(tile + tile_off(tid, c, p.Di));
                    const int x = generic ? score_generic(rowc, nchunk, S.q, p.Hi, p.Di, p.w)
                                          : rq.score(rowc, p.w);
                    sc[skew(e)] = x;
                    atomicAdd(&S.hist0[digit_at(ext_key(x), 0)], 1);
                }
                __syncthreads();
                if (tid == 0 && s + kStages < nst) {
                    const uint32_t k2 = k + kStages;
                    mbar_arrive_expect_tx(&S.full_bar[k2 % kStages], (uint32_t)(rows_per_stage * p.Di));
                    tma_load_keys(S.stage[k2 % kStages], &kmap, 0, lo + (s + kStages) * rows_per_stage, b,
                                  &S.full_bar[k2 % kStages]);
                }
            }
            stage_seq += nst;
            if (!alive) break;
        } else {
            // Reindex: valid pool entries form a prefix (ascending, -1 padded at the end)
            int first_bad = my_n;
            for (int e = tid; e < my_n; e += kIdxThreads) {
                const int s = pool[lo + e];
                if (s < 0 || s > t) first_bad = min(first_bad, e);
            }
            int fb = first_bad;
            {
                // block min
                for (int o = 16; o > 0; o >>= 1) fb = min(fb, __shfl_xor_sync(0xffffffffu, fb, o));
                if ((tid & 31) == 0) S.red[tid >> 5] = fb;
                __syncthreads();
                fb = S.red[0];
                for (int w2 = 1; w2 < kIdxThreads / 32; ++w2) fb = min(fb, S.red[w2]);
                __syncthreads();
            }
            if (fb < my_n) {
                // an entry past the first invalid one must be padding, never a position
                for (int e = fb + tid; e < my_n; e += kIdxThreads)
                    if (pool[lo + e] >= 0) report(p.status, CSA2_ERR_RANGE, u);
                my_n = fb;
            }
            if (my_n > 0 && lo > 0 && tid == 0 && pool[lo - 1] < 0) report(p.status, CSA2_ERR_RANGE, u);
            const int8_t* kb = p.ki + (size_t)b * p.ki_seq_stride;
            for (int e = tid; e < my_n; e += kIdxThreads) {
                const int s = pool[lo + e];
                const int4* row = reinterpret_cast<const int4*>(kb + (size_t)s * p.Di);
                int4 rowc[8];
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    if (c < nchunk) rowc[c] = __ldg(row + c);
                const int x = generic ? score_generic(rowc, nchunk, S.q, p.Hi, p.Di, p.w) : rq.score(rowc, p.w);
                sc[skew(e)] = x;
                atomicAdd(&S.hist0[digit_at(ext_key(x), 0)], 1);
            }
        }
        __syncthreads();

        // ---- round 0: histogram of level 0, zero the buffers the next steps use
        int* g0cur = g0 + ((epoch + j) % 3) * kBins;
        int* g0nxt = g0 + ((epoch + j + 1) % 3) * kBins;
        push_hist(S.hist0, g0cur);
        {
            const int per = (kBins + p.G - 1) / p.G;
            const int zlo = cta * per, zhi = min(kBins, zlo + per);
            for (int i = zlo + tid; i < zhi; i += kIdxThreads) {
                g0nxt[i] = 0;
                gl[i] = 0; gl[kBins + i] = 0; gl[2 * kBins + i] = 0; gl[3 * kBins + i] = 0;
            }
            if (cta == 0 && tid == 0) { ctrl[CTRL_CAND0] = 0; ctrl[CTRL_CAND1] = 0; }
        }
        bar_target += p.G;
        if (!group_barrier(ctrl + CTRL_BAR, bar_target, p.status)) { alive = false; break; }

        // ---- per-track state (identical in every CTA of the group)
        // info layout per track: [0]=state [1]=r_rem [2]=C [3]=level [4..5]=prefix lo/hi [6]=above_local
        // state: 0 off, 1 all, 2 radix in progress, 3 cand gather, 4 eq counts, 9 finished
        int n_total;
        if (full) n_total = n_all;
        else {
            int s = 0;
            for (int i = tid; i < kBins; i += kIdxThreads) s += __ldcg(g0cur + i);
            n_total = block_sum(s, S.red);
        }
        int state[2], rrem[2], C[2], level[2], above_loc[2];
        uint64_t prefix[2];
        for (int tr = 0; tr < 2; ++tr) {
            state[tr] = 0; rrem[tr] = 0; C[tr] = 0; level[tr] = 0; above_loc[tr] = 0; prefix[tr] = 0;
            const int r = p.r[tr];
            if (r <= 0) continue;
            if (n_total <= r) { state[tr] = 1; continue; }
            find_rank_bin(g0cur, r, S.red, S.info + 8 * tr);
            const int d = S.info[8 * tr + 0];
            rrem[tr] = r - S.info[8 * tr + 1];
            C[tr] = S.info[8 * tr + 2];
            prefix[tr] = (uint64_t)d;
            level[tr] = 0;
            above_loc[tr] = block_sum(sum_above(S.hist0, d), S.red);
            state[tr] = (C[tr] <= kCandCap) ? 3 : 2;
        }

        // ---- rounds until every track knows its cut
        while (alive) {
            bool any = false;
            for (int tr = 0; tr < 2; ++tr) {
                if (state[tr] == 2) {
                    // histogram of the next digit over elements matching the prefix
                    any = true;
                    int* hl = S.histl[tr];
                    for (int i = tid; i < kBins; i += kIdxThreads) hl[i] = 0;
                    __syncthreads();
                    const int lv = level[tr] + 1;
                    for (int e = tid; e < my_n; e += kIdxThreads) {
                        const uint64_t ek = ext_key(sc[skew(e)]);
                        if ((ek >> (36 - 12 * lv)) == prefix[tr]) atomicAdd(&hl[digit_at(ek, lv)], 1);
                    }
                    __syncthreads();
                    push_hist(hl, gl + (2 * tr + (lv - 1)) * kBins);
                } else if (state[tr] == 3) {
                    // gather the elements of the threshold bin
                    any = true;
                    const int lv = level[tr] + 1;
                    for (int e0 = 0; e0 < my_n; e0 += kIdxThreads) {
                        const int e = e0 + tid;
                        int x = 0;
                        bool m = false;
                        if (e < my_n) {
                            x = sc[skew(e)];
                            m = (ext_key(x) >> (36 - 12 * lv)) == prefix[tr];
                        }
                        const unsigned bal = __ballot_sync(0xffffffffu, m);
                        if (bal) {
                            int basei = 0;
                            if ((tid & 31) == 0) basei = atomicAdd(ctrl + CTRL_CAND0 + tr, __popc(bal));
                            basei = __shfl_sync(0xffffffffu, basei, 0);
                            if (m) {
                                const int slot = basei + __popc(bal & ((1u << (tid & 31)) - 1u));
                                if (slot < kCandCap) cand[tr * kCandCap + slot] = make_int2(x, lo + e);
                            }
                        }
                    }
                    if (tid == 0) pub[(tr * 2 + 0) * kMaxG + cta] = above_loc[tr];
                } else if (state[tr] == 4) {
                    any = true;
                    int eq = 0;
                    for (int e = tid; e < my_n; e += kIdxThreads) eq += (ext_key(sc[skew(e)]) == prefix[tr]);
                    eq = block_sum(eq, S.red);
                    if (tid == 0) {
                        pub[(tr * 2 + 0) * kMaxG + cta] = above_loc[tr];
                        pub[(tr * 2 + 1) * kMaxG + cta] = eq;
                    }
                }
            }
            if (!any) break;
            bar_target += p.G;
            if (!group_barrier(ctrl + CTRL_BAR, bar_target, p.status)) { alive = false; break; }
            for (int tr = 0; tr < 2; ++tr) {
                if (state[tr] == 2) {
                    const int lv = level[tr] + 1;
                    const int* gh = gl + (2 * tr + (lv - 1)) * kBins;
                    find_rank_bin(gh, rrem[tr], S.red, S.info + 8 * tr);
                    const int d = S.info[8 * tr + 0];
                    rrem[tr] -= S.info[8 * tr + 1];
                    C[tr] = S.info[8 * tr + 2];
                    prefix[tr] = (prefix[tr] << 12) | (uint64_t)d;
                    level[tr] = lv;
                    above_loc[tr] += block_sum(sum_above(S.histl[tr], d), S.red);
                    state[tr] = (C[tr] <= kCandCap) ? 3 : (lv < 2 ? 2 : 4);
                } else if (state[tr] == 3) {
                    state[tr] = 5;   // finalize from candidates
                } else if (state[tr] == 4) {
                    state[tr] = 6;   // finalize from equal counts
                }
            }
            bool pending = false;
            for (int tr = 0; tr < 2; ++tr) pending |= (state[tr] == 2 || state[tr] == 3 || state[tr] == 4);
            if (!pending) break;
        }
        if (!alive) break;

        // ---- write each track's list
        for (int tr = 0; tr < 2; ++tr) {
            const int r = p.r[tr];
            if (r <= 0) continue;
            int32_t* outp = p.out[tr] + (size_t)u * r;
            int base_off = 0;
            uint64_t kcut = 0;         // cand: select comp_key >= kcut
            uint64_t ecut = 0;         // eq: select ext > ecut, or == with quota
            int quota = 0;
            const int st = state[tr];
            if (st == 1) {
                base_off = lo;   // every candidate is taken; valid entries are a prefix
            } else if (st == 5) {
                // exact cut among the candidates
                uint64_t* keys = reinterpret_cast<uint64_t*>(&S.stage[0][0]);
                const int Cn = C[tr];
                int np2 = 1;
                while (np2 < Cn) np2 <<= 1;
                for (int i = tid; i < np2; i += kIdxThreads) {
                    if (i < Cn) {
                        const int2 cv = __ldcg(cand + tr * kCandCap + i);
                        keys[i] = comp_key(cv.x, cv.y);
                    } else {
                        keys[i] = 0;
                    }
                }
                __syncthreads();
                bitonic_desc(keys, np2);
                kcut = keys[rrem[tr] - 1];
                int before = 0;
                for (int i = tid; i < Cn; i += kIdxThreads) {
                    const int idx = 0x7FFFFFF - (int)(keys[i] & 0x7FFFFFFull);
                    before += (keys[i] >= kcut && idx < lo);
                }
                before = block_sum(before, S.red);
                int prev = 0;
                for (int c2 = 0; c2 < cta; ++c2) prev += __ldcg(pub + (tr * 2 + 0) * kMaxG + c2);
                base_off = prev + before;
            } else if (st == 6) {
                ecut = prefix[tr];
                int prev = 0, eqb = 0;
                for (int c2 = 0; c2 < cta; ++c2) {
                    prev += __ldcg(pub + (tr * 2 + 0) * kMaxG + c2);
                    eqb += __ldcg(pub + (tr * 2 + 1) * kMaxG + c2);
                }
                const int my_eq = __ldcg(pub + (tr * 2 + 1) * kMaxG + cta);
                quota = max(0, min(rrem[tr] - eqb, my_eq));
                base_off = prev + min(rrem[tr], eqb);
            }
            // ordered compaction: thread tid owns elements [tid*R, tid*R+R)
            const int R = (my_n + kIdxThreads - 1) / kIdxThreads;
            const int e0 = min(tid * R, my_n), e1 = min(e0 + R, my_n);
            int cnt = 0, ceq = 0;
            for (int e = e0; e < e1; ++e) {
                const int x = sc[skew(e)];
                if (st == 1) cnt++;
                else if (st == 5) cnt += comp_key(x, lo + e) >= kcut;
                else {
                    const uint64_t ek = ext_key(x);
                    cnt += ek > ecut;
                    ceq += ek == ecut;
                }
            }
            int tot;
            int eq_excl = 0;
            if (st == 6) eq_excl = block_scan_excl(ceq, S.red, tot);
            const int eq_take = (st == 6) ? max(0, min(quota - eq_excl, ceq)) : 0;
            const int off = base_off + block_scan_excl(cnt + eq_take, S.red, tot);
            int k2 = off, eq_seen = 0;
            for (int e = e0; e < e1; ++e) {
                const int x = sc[skew(e)];
                bool sel;
                if (st == 1) sel = true;
                else if (st == 5) sel = comp_key(x, lo + e) >= kcut;
                else {
                    const uint64_t ek = ext_key(x);
                    sel = ek > ecut;
                    if (ek == ecut) { sel = eq_seen < eq_take; eq_seen++; }
                }
                if (sel) {
                    const int pos = full ? (lo + e) : pool[lo + e];
                    if (k2 < r) outp[k2] = pos;
                    k2++;
                }
            }
            // padding: entries [min(r, n_total), r) = -1
            if (cta == p.G - 1) {
                for (int i = min(r, n_total) + tid; i < r; i += kIdxThreads) outp[i] = -1;
            }
            __syncthreads();
        }
    }
    // persist the slot state for the next launch
    if (alive && cta == 0 && tid == 0) {
        ctrl[CTRL_EPOCH] = epoch + j;
        ctrl[CTRL_BAR_BASE] = bar_target;
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

struct IdxPlan {
    int units, G, groups, chunk;
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
    r.off_g0 = off;   off += align_up((size_t)slots * 3 * kBins * 4, 256);
    r.off_gl = off;   off += align_up((size_t)slots * 4 * kBins * 4, 256);
    r.off_cand = off; off += align_up((size_t)slots * 2 * kCandCap * 8, 256);
    r.off_pub = off;  off += align_up((size_t)slots * 4 * kMaxG * 4, 256);
    r.bytes = off;
    return r;
}

size_t index_region_bytes() { return idx_region(num_sms()).bytes; }

IdxPlan plan_index(const csa2_index_args& a, int sms) {
    IdxPlan pl{};
    pl.units = a.B * a.Tq;
    const int n_max = (a.mode == CSA2_FULL) ? a.N : a.P_in;
    if (pl.units >= sms) {
        pl.G = 1;
        pl.groups = sms;
    } else {
        pl.groups = pl.units;
        pl.G = std::max(1, std::min(kMaxG, sms / pl.units));
        pl.G = std::max(1, std::min(pl.G, (n_max + 1023) / 1024));
    }
    int chunk = (n_max + pl.G - 1) / pl.G;
    chunk = (int)align_up((size_t)std::max(chunk, 1), 256);
    pl.chunk = chunk;
    pl.spill_bytes = 0;
    if (chunk > kSmemScores) pl.spill_bytes = align_up((size_t)pl.groups * pl.G * ((chunk + 63) / 64 * 65) * 4, 256);
    return pl;
}

size_t index_smem_bytes() { return sizeof(IdxSmem) + 1024; }

template <int HI, int DI>
static cudaError_t launch_variant(const IdxParams& p, const CUtensorMap& map, int grid, cudaStream_t stream) {
    auto kern = index_select_kernel<HI, DI>;
    const size_t smem = index_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kIdxThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p, map);
}

// Launch one indexer call. `ws` holds plan_index(a).ws_bytes bytes (zero at first use).
csa2_status launch_index(const csa2_index_args& a, const int32_t* pool_in, int P_in, void* region, void* scratch,
                         int32_t* d_status, cudaStream_t stream) {
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
    p.spill = (pl.chunk > kSmemScores) ? static_cast<int32_t*>(scratch) : nullptr;
    p.status = d_status;

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
    if (a.Hi <= 8 && a.Di == 64) e = launch_variant<8, 64>(p, map, grid, stream);
    else if (a.Hi <= 4 && a.Di == 32) e = launch_variant<4, 32>(p, map, grid, stream);
    else e = launch_variant<0, 0>(p, map, grid, stream);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

size_t index_scratch_bytes(const csa2_index_args& a, int P_in) {
    csa2_index_args aa = a;
    aa.P_in = P_in;
    return plan_index(aa, num_sms()).spill_bytes;
}

}  // namespace csa2
