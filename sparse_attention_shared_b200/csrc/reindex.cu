// Reindex mode: rescore a query's candidate pool with the layer's own indexer and
// keep the exact top-k.
//
// "CED: Continuing Context with a Causal Encoder and Decoder", "What Full,
// Reindex, and Reuse Share" (Fig. 5): a Reindex layer chooses again, with its own
// indexer query, among the candidates of the pool the Full layer built; it may
// pick positions the previous top-k lacked, never one outside the pool. Score
// (a reading of the pages): sum_h w[h] * max(0, qi[h] . ki[s]), exact in int32;
// ranking by score descending, then position ascending; the list is written in
// ascending position order, padded with -1.
//
// Design (B200): one thread-block cluster of C <= 8 CTAs per query. CTA r gathers
// the key rows of its slice of the pool with 16-byte loads, all of a thread's
// rows in flight at once, scores them with dp4a, and pushes (score, position)
// into the shared memory of the cluster's first CTA (distributed shared memory).
// After one cluster barrier that CTA alone finds the exact cut:
//   1. a 4096-bin histogram of a 12-bit log-scale digit of the score finds the
//      bin that holds the k-th best score;
//   2. the bin's entries (a few dozen on random data) go to a candidate list, and
//      two 12-bit digits of the score's offset in the bin find the exact k-th
//      best score T;
//   3. one ordered pass over the pool (8 warps, each a contiguous range, ballots
//      inside 32-entry steps) writes every entry above T and the first ties at T
//      in position order, which is pool order.
// In a layer stack the pool was written two or more kernels earlier, so the pool
// entries and key rows are loaded before the dependency wait; only the index
// query waits for the previous kernel. The list writes prefetch the FP4 rows the
// layer's attention gathers next into L2.
#include <algorithm>
#include <climits>

#include "csa2_common.cuh"

namespace csa2 {

constexpr int kRxThreads = 256;
constexpr int kRxWarps = kRxThreads / 32;
constexpr int kRxMaxCluster = 8;
constexpr int kRxBins = 4096;

// entries per CTA: every row of a thread in registers (at most 32 16-byte chunks)
template <int DI>
struct RxGeom {
    static constexpr int RPT = (512 / DI) < 8 ? (512 / DI) : 8;   // rows per thread
    static constexpr int kSlice = RPT * kRxThreads;               // entries per CTA
    static constexpr int kMaxPool = kSlice * kRxMaxCluster;
};

struct RxParams {
    int B, Tq, N, Hi, Di, k, P_in, slice;
    const int32_t* q_pos;
    const int8_t* qi;
    int32_t w[16];
    const int8_t* ki;
    int64_t ki_seq_stride;
    const int32_t* pool;
    int32_t* topk_out;
    int pool_ready;      // the pool and the keys were complete before the previous kernel began
    int m;               // sequence compression rate of the global entries
    const uint8_t* pf_fp4;
    const uint8_t* pf_scale;
    int pf_N, pf_code_bytes, pf_scale_bytes;
    int32_t* status;
};

// Shared memory (dynamic, 16-byte aligned regions), for a pool capacity Pc:
//   sc   [Pc] int32     leader: every entry's score
//   ps   [Pc] int32     leader: every entry's position (-1: none)
//   c1   [Pc] uint16    leader: candidate indices, level 1
//   c2   [Pc] uint16    leader: candidate indices, level 2
//   hist [kRxBins] int32
//   q    [16 * 128] int8  the index query
//   misc
struct RxMisc {
    int red[64];
    int info[8];
    int cnt[2];
    int wabove[kRxWarps], wtie[kRxWarps];
};

__device__ __forceinline__ uint32_t rx_mag_bin(uint32_t y) {
    if (y < 64u) return y;
    const int e = 31 - __clz(y);
    return 64u + (uint32_t)(e - 6) * 64u + ((y >> (e - 6)) & 63u);
}

// 12-bit log-scale digit of a score; increasing in the score
__device__ __forceinline__ uint32_t rx_d0(int32_t x) {
    return x >= 0 ? 2048u + rx_mag_bin((uint32_t)x) : 2047u - rx_mag_bin((uint32_t)(-1 - x));
}

// lowest score whose level-0 digit is d
__device__ __forceinline__ int32_t rx_d0_lo(uint32_t d) {
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
    return pos ? (int32_t)ylo : (int32_t)(-1 - yhi);
}

// In a histogram of kRxBins bins, the bin holding the r-th largest element
// (1-based): info[0] = bin, info[1] = elements in higher bins.
__device__ void rx_rank_bin(const int* hist, int r, RxMisc& M) {
    constexpr int PER = kRxBins / kRxThreads;   // 16 bins per thread, thread 0 the highest
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int hi = kRxBins - PER * t;           // this thread's bins: [hi - PER, hi)
    int h[PER];
    int s = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        h[i] = hist[hi - 1 - i];                // descending bin order
        s += h[i];
    }
    int x = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) M.red[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int v = lane < kRxWarps ? M.red[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += y;
        }
        if (lane < kRxWarps) M.red[32 + lane] = v;
    }
    __syncthreads();
    int above = (warp ? M.red[32 + warp - 1] : 0) + x - s;   // elements in bins above this thread's
    if (above < r && r <= above + s) {
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            if (above < r && r <= above + h[i]) {
                M.info[0] = hi - 1 - i;
                M.info[1] = above;
            }
            above += h[i];
        }
    }
    __syncthreads();
}

template <int HI, int DI>
__device__ __forceinline__ int rx_score(const int4 (&row)[DI / 16], const int8_t* qs, const int32_t* w) {
    int s = 0;
#pragma unroll
    for (int h = 0; h < HI; ++h) {
        int acc = 0;
        const int4* qh = reinterpret_cast<const int4*>(qs + h * DI);
#pragma unroll
        for (int c = 0; c < DI / 16; ++c) {
            const int4 k = row[c], q = qh[c];
            acc = __dp4a(k.x, q.x, acc);
            acc = __dp4a(k.y, q.y, acc);
            acc = __dp4a(k.z, q.z, acc);
            acc = __dp4a(k.w, q.w, acc);
        }
        s += w[h] * max(acc, 0);
    }
    return s;
}

__device__ __forceinline__ void st_dsmem_i32(uint32_t addr, int v) {
    asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

template <int HI, int DI>
__global__ void __launch_bounds__(kRxThreads, 1) index_reindex_cl_kernel(const __grid_constant__ RxParams p, int Pc) {
    using G = RxGeom<DI>;
    constexpr int RPT = G::RPT;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    int* sc = reinterpret_cast<int*>(smem_raw);
    int* ps = sc + Pc;
    uint16_t* c1 = reinterpret_cast<uint16_t*>(ps + Pc);
    uint16_t* c2 = c1 + Pc;
    int* hist = reinterpret_cast<int*>(c2 + Pc);
    int8_t* qs = reinterpret_cast<int8_t*>(hist + kRxBins);
    RxMisc& M = *reinterpret_cast<RxMisc*>(qs + 16 * 128);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rank = (int)cluster_ctarank();
    const int u = blockIdx.y;
    const int b = u / p.Tq;
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");   // waited on before the first push

    int t = last_entry(p.q_pos[u], p.m);   // the last global entry the query reads
    const bool t_ok = p.q_pos[u] >= 0 && t < p.N;
    if (!t_ok) {
        if (tid == 0 && rank == 0) report(p.status, CSA2_ERR_RANGE, u);
        t = -1;
    }
    const int lo = rank * p.slice;
    const int32_t* pool = p.pool + (size_t)u * p.P_in;
    const int8_t* kb = p.ki + (size_t)b * p.ki_seq_stride;
    int spos[RPT];
    int4 rows[RPT][DI / 16];
    auto gather = [&]() {
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int e = lo + i * kRxThreads + tid;
            int s = -1;
            if (e < min(lo + p.slice, p.P_in)) {
                s = __ldg(pool + e);
                const int prev = e > 0 ? __ldg(pool + e - 1) : -1;
                // valid entries are ascending positions <= t, -1 padding only at the end
                if (s >= 0 && (s > t || s >= p.N || (e > 0 && (prev < 0 || prev >= s)))) {
                    report(p.status, CSA2_ERR_RANGE, u);
                    s = -1;
                }
            }
            spos[i] = s;
        }
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            if (spos[i] < 0) continue;
            const int4* src = reinterpret_cast<const int4*>(kb + (size_t)spos[i] * DI);
#pragma unroll
            for (int c = 0; c < DI / 16; ++c) rows[i][c] = __ldg(src + c);
        }
    };
    if (p.pool_ready) gather();
    pdl_wait();
    pdl_launch_dependents();
    if (!p.pool_ready) gather();
    // the index query depends on the previous layer
    for (int i = tid; i < HI * DI / 16; i += kRxThreads) {
        const int h = i / (DI / 16);
        int4 v = make_int4(0, 0, 0, 0);
        if (h < p.Hi) v = __ldg(reinterpret_cast<const int4*>(p.qi + (size_t)u * p.Hi * p.Di) + i);
        reinterpret_cast<int4*>(qs)[i] = v;
    }
    __syncthreads();

    // ---- scores, pushed with their positions into the first CTA of the cluster
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    const uint32_t sc0 = dsmem_addr(sc, 0), ps0 = dsmem_addr(ps, 0);
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int e = lo + i * kRxThreads + tid;
        if (e >= min(lo + p.slice, p.P_in)) continue;
        const int x = spos[i] >= 0 ? rx_score<HI, DI>(rows[i], qs, p.w) : 0;
        if (!CSA2_CHECK(e < Pc, p.status, 2201)) continue;
        st_dsmem_i32(sc0 + 4u * (uint32_t)e, x);
        st_dsmem_i32(ps0 + 4u * (uint32_t)e, spos[i]);
    }
    cluster_sync_all();
    if (rank != 0) return;   // no CTA reads another's shared memory after the barrier

    // ---- the first CTA: exact cut over the whole pool
    const int n = p.P_in;
    int32_t* out = p.topk_out + (size_t)u * p.k;
    const bool pf = p.pf_fp4 != nullptr;
    auto emit = [&](int idx, int s) {
        if (!CSA2_CHECK(idx >= 0 && idx < p.k, p.status, 2203)) return;
        out[idx] = s;
        if (pf) {
            const size_t row = (size_t)b * p.pf_N + s;
            prefetch_l2(p.pf_fp4 + row * p.pf_code_bytes);
            prefetch_l2(p.pf_scale + row * p.pf_scale_bytes);
        }
    };
    int nv = 0;
    for (int i = tid; i < n; i += kRxThreads) nv += ps[i] >= 0;
    for (int i = tid; i < kRxBins; i += kRxThreads) hist[i] = 0;
    if (tid < 2) M.cnt[tid] = 0;
    for (int o = 16; o > 0; o >>= 1) nv += __shfl_xor_sync(0xffffffffu, nv, o);
    if (lane == 0) M.red[warp] = nv;
    __syncthreads();
    nv = 0;
#pragma unroll
    for (int w = 0; w < kRxWarps; ++w) nv += M.red[w];
    int T = INT_MIN, need = 0;   // entries above T are taken, and the first `need` ties at T
    if (nv > p.k) {
        for (int i = tid; i < n; i += kRxThreads)
            if (ps[i] >= 0) atomicAdd(&hist[rx_d0(sc[i])], 1);
        __syncthreads();
        rx_rank_bin(hist, p.k, M);
        const uint32_t B0 = (uint32_t)M.info[0];
        const int above0 = M.info[1];
        const int32_t blo = rx_d0_lo(B0);
        for (int i = tid; i < n; i += kRxThreads)
            if (ps[i] >= 0 && rx_d0(sc[i]) == B0) {
                const int slot = atomicAdd(&M.cnt[0], 1);
                if (CSA2_CHECK(slot < Pc, p.status, 2202)) c1[slot] = (uint16_t)i;
            }
        for (int i = tid; i < kRxBins; i += kRxThreads) hist[i] = 0;
        __syncthreads();
        const int n1 = M.cnt[0];
        // level 1: bits 12..23 of the offset in the bin
        for (int j = tid; j < n1; j += kRxThreads) atomicAdd(&hist[((uint32_t)(sc[c1[j]] - blo) >> 12) & 4095u], 1);
        __syncthreads();
        rx_rank_bin(hist, p.k - above0, M);
        const uint32_t B1 = (uint32_t)M.info[0];
        const int above1 = M.info[1];
        for (int j = tid; j < n1; j += kRxThreads) {
            const int i = c1[j];
            if ((((uint32_t)(sc[i] - blo) >> 12) & 4095u) == B1) {
                const int slot = atomicAdd(&M.cnt[1], 1);
                if (CSA2_CHECK(slot < Pc, p.status, 2202)) c2[slot] = (uint16_t)i;
            }
        }
        for (int i = tid; i < kRxBins; i += kRxThreads) hist[i] = 0;
        __syncthreads();
        const int n2 = M.cnt[1];
        // level 2: bits 0..11 of the offset
        for (int j = tid; j < n2; j += kRxThreads) atomicAdd(&hist[(uint32_t)(sc[c2[j]] - blo) & 4095u], 1);
        __syncthreads();
        rx_rank_bin(hist, p.k - above0 - above1, M);
        const uint32_t B2 = (uint32_t)M.info[0];
        T = blo + (int32_t)((B1 << 12) | B2);
        need = p.k - above0 - above1 - M.info[1];
    }

    // ---- ordered write: warp w scans entries [w * span, (w + 1) * span) in 32-entry steps
    const int span = ((n + kRxWarps - 1) / kRxWarps + 31) / 32 * 32;
    const int w0 = warp * span, w1 = min(w0 + span, n);
    int n_above = 0, n_tie = 0;
    for (int s0 = w0; s0 < w1; s0 += 32) {
        const int i = s0 + lane;
        const bool v = i < w1 && ps[i] >= 0;
        const int x = v ? sc[i] : 0;
        n_above += __popc(__ballot_sync(0xffffffffu, v && x > T));
        n_tie += __popc(__ballot_sync(0xffffffffu, v && x == T));
    }
    if (lane == 0) {
        M.wabove[warp] = n_above;
        M.wtie[warp] = n_tie;
    }
    __syncthreads();
    int tie_before = 0, out_before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kRxWarps; ++w) {
        const int take_t = (nv > p.k) ? max(0, min(M.wtie[w], need - tie_before)) : M.wtie[w];
        const int sel = M.wabove[w] + take_t;
        if (w < warp) {
            out_before += sel;
            tie_before += M.wtie[w];
        }
        total += sel;
    }
    int ties_seen = tie_before, written = out_before;
    for (int s0 = w0; s0 < w1; s0 += 32) {
        const int i = s0 + lane;
        const bool v = i < w1 && ps[i] >= 0;
        const int x = v ? sc[i] : 0;
        const bool is_tie = v && x == T;
        const unsigned tb = __ballot_sync(0xffffffffu, is_tie);
        const int tie_rank = ties_seen + __popc(tb & ((1u << lane) - 1u));
        const bool take = v && (x > T || (is_tie && (nv <= p.k || tie_rank < need)));
        const unsigned sb = __ballot_sync(0xffffffffu, take);
        if (take) emit(written + __popc(sb & ((1u << lane) - 1u)), ps[i]);
        written += __popc(sb);
        ties_seen += __popc(tb);
    }
    for (int i = total + tid; i < p.k; i += kRxThreads) out[i] = -1;
}

// ------------------------------------------------------------ host side
static size_t rx_smem_bytes(int Pc) {
    return (size_t)Pc * (4 + 4 + 2 + 2) + kRxBins * 4 + 16 * 128 + sizeof(RxMisc);
}

// Clustered Reindex for these sizes: CTAs per query (0: not this kernel).
int reindex_cluster_size(const csa2_index_args& a, int P_in) {
    if (a.mode != CSA2_REINDEX || a.Hi > 16 || P_in < 1 || (int64_t)a.B * a.Tq > 65535) return 0;
    int slice = 0, maxp = 0;
    if (a.Di == 32) { slice = RxGeom<32>::kSlice; maxp = RxGeom<32>::kMaxPool; }
    else if (a.Di == 64) { slice = RxGeom<64>::kSlice; maxp = RxGeom<64>::kMaxPool; }
    else if (a.Di == 128) { slice = RxGeom<128>::kSlice; maxp = RxGeom<128>::kMaxPool; }
    else return 0;
    if (P_in > maxp || P_in > 65535) return 0;
    return std::max(1, (P_in + slice - 1) / slice);
}

template <int HI, int DI>
static cudaError_t launch_rx_variant(const RxParams& p, int cs, int units, int Pc, cudaStream_t stream) {
    auto kern = index_reindex_cl_kernel<HI, DI>;
    const size_t smem = rx_smem_bytes(Pc);
    cudaError_t e = set_smem_once(reinterpret_cast<const void*>(kern), (int)rx_smem_bytes(RxGeom<DI>::kMaxPool));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(cs, units);
    cfg.blockDim = dim3(kRxThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // reads no output of the previous kernel before griddepcontrol.wait, except
    // (pool_ready) the pool and keys, which were complete before that kernel began
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, p, Pc);
}

csa2_status launch_reindex_cl(const csa2_index_args& a, const int32_t* pool_in, int P_in, int pool_ready,
                              const csa2_attn_args* pf, int32_t* d_status, cudaStream_t stream) {
    const int cs = reindex_cluster_size(a, P_in);
    if (cs == 0) return CSA2_ERR_UNSUPPORTED;
    RxParams p{};
    p.B = a.B; p.Tq = a.Tq; p.N = a.N; p.Hi = a.Hi; p.Di = a.Di; p.k = a.k; p.P_in = P_in;
    p.slice = (P_in + cs - 1) / cs;
    p.q_pos = a.q_pos; p.qi = a.qi;
    for (int h = 0; h < 16; ++h) p.w[h] = h < a.Hi ? a.w[h] : 0;
    p.ki = a.ki; p.ki_seq_stride = a.ki_seq_stride;
    p.pool = pool_in;
    p.topk_out = a.topk_out;
    p.pool_ready = pool_ready;
    p.m = a.m;
    if (pf != nullptr && pf->kv_fp4 != nullptr && pf->kv_scale != nullptr && pf->B == a.B) {
        p.pf_fp4 = pf->kv_fp4;
        p.pf_scale = pf->kv_scale;
        p.pf_N = pf->N;
        p.pf_code_bytes = pf->D / 2;
        p.pf_scale_bytes = pf->D / 16;
    }
    p.status = d_status;
    const int Pc = (P_in + 31) / 32 * 32;
    const int units = a.B * a.Tq;
    cudaError_t e;
    const bool h8 = a.Hi <= 8;
    if (a.Di == 64) e = h8 ? launch_rx_variant<8, 64>(p, cs, units, Pc, stream) : launch_rx_variant<16, 64>(p, cs, units, Pc, stream);
    else if (a.Di == 32) e = h8 ? launch_rx_variant<8, 32>(p, cs, units, Pc, stream) : launch_rx_variant<16, 32>(p, cs, units, Pc, stream);
    else e = h8 ? launch_rx_variant<8, 128>(p, cs, units, Pc, stream) : launch_rx_variant<16, 128>(p, cs, units, Pc, stream);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

}  // namespace csa2
