// Sparse attention over {selected global FP4 rows} U {sliding-window local rows}.
//
// "CED: Continuing Context with a Causal Encoder and Decoder", "Selecting
// Positions and Reading Values with Attention" (Fig. 4): the selected global
// entries are concatenated with the layer's local KV and Main Q attends over
// the union with one softmax; a position present in both sets counts twice.
// Global entries are FP4 (E2M1 codes, one E4M3 scale per 16 values:
// "DeepSeek-V4.1 Flash Pushes KV Cache Compression for Agent Workloads",
// "Ana Gelisme") and serve as both key and value.
//
// Design (B200): one CTA (128 threads) per 128-key tile of one query: either a
// tile of the query's global list or a tile of its window. The CTA stages the
// tile in shared memory as bf16 in the 128-byte-swizzled layout that tcgen05
// reads (FP4 rows are dequantised exactly on the way: e2m1 * e4m3 has at most
// six significant bits), computes S = K Q^T with keys as M = 128 and heads as
// N into tensor memory, takes the tile's softmax partial (max, sum, P in bf16),
// and computes O^T = V^T P with the head dim as M, reading the same key tile
// as an M-major operand. Partials go to the workspace; the last CTA of the
// query (atomic ticket, no waiting) merges them by log-sum-exp and writes the
// bf16 output and the fp32 log-sum-exp.
#include <cuda_bf16.h>

#include "csa2_common.cuh"

namespace csa2 {

constexpr int kAttnThreads = 128;
constexpr int kTileKeys = 128;
constexpr int kPanelBytes = kTileKeys * 128;   // 128 rows x 128 bytes

struct AttnParams {
    int B, Tq, N, Hq, D, k, W, Lloc;
    int ngt, nlt, ntiles;
    float scale_log2;   // log2(e) / sqrt(D)
    const int32_t* q_pos;
    const uint16_t* q;
    const uint8_t* kv_fp4;
    const uint8_t* kv_scale;
    const int32_t* topk;
    const uint16_t* kl;
    const uint16_t* vl;
    const int32_t* local_base;
    uint16_t* out;
    float* lse;
    float* part;    // [units][ntiles][HQP * (D + 2)]
    int* tickets;   // [units]
    int32_t* status;
};

template <int HQP>
struct __align__(1024) AttnSmem {
    uint8_t kbuf[2 * kPanelBytes];      // key tile (also the value tile of a global tile)
    uint8_t vbuf[2 * kPanelBytes];      // value tile of a local tile
    uint8_t qbuf[2 * HQP * 128];        // queries, [HQP rows x D] in 64-element panels
    uint8_t pbuf[2 * HQP * 128];        // probabilities, [HQP rows x 128 keys] in 64-key panels
    uint32_t lut[256];                  // code byte -> two bf16 E2M1 values
    float red[4][HQP];
    uint64_t bar_s, bar_o;
    uint32_t tmem_base;
    int is_last;
};

__device__ __forceinline__ uint32_t e2m1_bf16_bits(uint32_t c) {
    const uint32_t mag = c & 7u;
    uint32_t bits = (mag == 0u) ? 0u : (mag == 1u) ? 0x3F00u : ((((mag >> 1) + 126u) << 7) | ((mag & 1u) << 6));
    return bits | ((c & 8u) << 12);
}

__device__ __forceinline__ uint32_t e4m3_bf16_bits(uint32_t b) {
    const uint32_t e = (b >> 3) & 15u, m = b & 7u;
    const float v = (e == 0) ? (float)m * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
    return (__float_as_uint(v) >> 16) | ((b & 0x80u) << 8);
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
    __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a);
    __nv_bfloat162 y = *reinterpret_cast<__nv_bfloat162*>(&b);
    __nv_bfloat162 z = __hmul2(x, y);
    return *reinterpret_cast<uint32_t*>(&z);
}

template <int HQP, int D>
__global__ void __launch_bounds__(kAttnThreads) sparse_attn_kernel(const __grid_constant__ AttnParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    AttnSmem<HQP>& S =
        *reinterpret_cast<AttnSmem<HQP>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr uint32_t kCols = (2 * HQP < 32) ? 32 : 2 * HQP;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int tau = blockIdx.x;
    const int u = blockIdx.y;
    const int b = u / p.Tq;
    const bool global_tile = tau < p.ngt;

    if (warp == 0) tmem_alloc(&S.tmem_base, kCols);
    if (tid == 0) {
        mbar_init(&S.bar_s, 1);
        mbar_init(&S.bar_o, 1);
        mbar_fence_init();
    }
    for (int i = tid; i < 256; i += kAttnThreads)
        S.lut[i] = e2m1_bf16_bits(i & 15u) | (e2m1_bf16_bits(i >> 4) << 16);

    int t = p.q_pos[u];
    if (t < 0 || t >= p.N) {
        if (tid == 0 && tau == 0) report(p.status, CSA2_ERR_RANGE, u);
        t = -1;
    }
    const int base = p.local_base[b];

    // ---- queries -> qbuf (rows >= Hq are zero)
    for (int i = tid; i < HQP * (D / 8); i += kAttnThreads) {
        const int h = i / (D / 8), c = i % (D / 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (h < p.Hq) v = __ldg(reinterpret_cast<const uint4*>(p.q + ((size_t)u * p.Hq + h) * D) + c);
        *reinterpret_cast<uint4*>(S.qbuf + (c >> 3) * (HQP * 128) + sw128(h, c & 7)) = v;
    }
    if (D == 64) {   // second M-half of the value operand stays zero
        for (int i = tid; i < kPanelBytes / 16; i += kAttnThreads) {
            reinterpret_cast<uint4*>(S.kbuf + kPanelBytes)[i] = make_uint4(0, 0, 0, 0);
            reinterpret_cast<uint4*>(S.vbuf + kPanelBytes)[i] = make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();

    // ---- the tile's 128 key rows
    const int r = tid;       // this thread's key row
    bool valid = false;
    if (global_tile) {
        const int j = tau * kTileKeys + r;
        int s = (j < p.k) ? p.topk[(size_t)u * p.k + j] : -1;
        if (s >= 0 && (s > t || s >= p.N)) {
            report(p.status, CSA2_ERR_RANGE, u);
            s = -1;
        }
        valid = s >= 0;
        if (valid) {
            const size_t row = (size_t)b * p.N + s;
            const uint4* cp = reinterpret_cast<const uint4*>(p.kv_fp4 + row * (D / 2));
            uint4 codes[D / 32];
#pragma unroll
            for (int i = 0; i < D / 32; ++i) codes[i] = __ldg(cp + i);
            uint32_t sw[D / 64];
            if (D == 128) {
                const uint2 s2 = __ldg(reinterpret_cast<const uint2*>(p.kv_scale + row * 8));
                sw[0] = s2.x; sw[1 % (D / 64)] = s2.y;
            } else {
                sw[0] = __ldg(reinterpret_cast<const uint32_t*>(p.kv_scale + row * 4));
            }
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {           // 8 elements (4 code bytes) per chunk
                const uint4 cw = codes[c >> 2];
                const uint32_t w = (c & 3) == 0 ? cw.x : (c & 3) == 1 ? cw.y : (c & 3) == 2 ? cw.z : cw.w;
                const uint32_t g = c >> 1;              // 16-element scale group
                const uint32_t sb = (sw[g >> 2] >> (8 * (g & 3))) & 0xFFu;
                const uint32_t s16 = e4m3_bf16_bits(sb);
                const uint32_t s2x = s16 | (s16 << 16);
                uint4 o;
                o.x = bf16x2_mul(S.lut[w & 0xFFu], s2x);
                o.y = bf16x2_mul(S.lut[(w >> 8) & 0xFFu], s2x);
                o.z = bf16x2_mul(S.lut[(w >> 16) & 0xFFu], s2x);
                o.w = bf16x2_mul(S.lut[w >> 24], s2x);
                *reinterpret_cast<uint4*>(S.kbuf + (c >> 3) * kPanelBytes + sw128(r, c & 7)) = o;
            }
        } else {
#pragma unroll
            for (int c = 0; c < D / 8; ++c)
                *reinterpret_cast<uint4*>(S.kbuf + (c >> 3) * kPanelBytes + sw128(r, c & 7)) = make_uint4(0, 0, 0, 0);
        }
    } else {
        // local tile: window positions [lo, t], rows lo-base .. ; coalesced 16-byte loads
        const int lt = tau - p.ngt;
        const int lo = max(max(base, t - p.W + 1), 0);
        const int p0 = lo + lt * kTileKeys;
        {
            const int pr = p0 + r;
            valid = (t >= 0) && (p.W > 0) && (pr <= t);
            if (valid && (pr - base < 0 || pr - base >= p.Lloc)) {
                report(p.status, CSA2_ERR_RANGE, u);
                valid = false;
            }
        }
        const uint4* kls = reinterpret_cast<const uint4*>(p.kl);
        const uint4* vls = reinterpret_cast<const uint4*>(p.vl);
        constexpr int CPR = D / 8;                              // 16-byte chunks per row
        constexpr int ITERS = kTileKeys * CPR / kAttnThreads;   // chunks per thread per tensor
        constexpr int BATCH = ITERS < 8 ? ITERS : 8;            // loads in flight per tensor
#pragma unroll
        for (int i0 = 0; i0 < ITERS; i0 += BATCH) {
            uint4 kv[BATCH], vv[BATCH];
#pragma unroll
            for (int j = 0; j < BATCH; ++j) {
                const int i = tid + (i0 + j) * kAttnThreads;
                const int rr = i / CPR, c = i % CPR;
                const int pr = p0 + rr;
                const int lrow = pr - base;
                const bool ok = (t >= 0) && (p.W > 0) && (pr <= t) && lrow >= 0 && lrow < p.Lloc;
                kv[j] = make_uint4(0, 0, 0, 0);
                vv[j] = make_uint4(0, 0, 0, 0);
                if (ok) {
                    const size_t off = ((size_t)b * p.Lloc + lrow) * CPR + c;
                    kv[j] = __ldg(kls + off);
                    vv[j] = __ldg(vls + off);
                }
            }
#pragma unroll
            for (int j = 0; j < BATCH; ++j) {
                const int i = tid + (i0 + j) * kAttnThreads;
                const int rr = i / CPR, c = i % CPR;
                const uint32_t dst = (c >> 3) * kPanelBytes + sw128(rr, c & 7);
                *reinterpret_cast<uint4*>(S.kbuf + dst) = kv[j];
                *reinterpret_cast<uint4*>(S.vbuf + dst) = vv[j];
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const uint32_t tmem_s = tmem, tmem_o = tmem + HQP;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    // ---- S = K Q^T  (M = 128 keys, N = HQP heads, K = D)
    if (tid == 0) {
        const uint32_t ka = smem_u32(S.kbuf), qa = smem_u32(S.qbuf);
        constexpr uint32_t idesc = idesc_bf16(128, HQP, 0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = smem_desc(ka + (kk >> 2) * kPanelBytes + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc(qa + (kk >> 2) * (HQP * 128) + (kk & 3) * 32, 16, 1024);
            mma_bf16(tmem_s, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&S.bar_s);
    }
    bool ok = mbar_wait(&S.bar_s, 0, p.status, 10);
    tc_fence_after();

    // ---- tile softmax partial
    float sv[HQP];
#pragma unroll
    for (int h = 0; h < HQP; ++h) sv[h] = 0.f;
    if (!ok) valid = false;
    if (ok) {
        float tmp[16];
#pragma unroll
        for (int c0 = 0; c0 < HQP; c0 += 16) {
            tmem_ld16(tmem_s + lane_off + c0, tmp);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) sv[c0 + i] = tmp[i];
        }
    }
#pragma unroll
    for (int h = 0; h < HQP; ++h) sv[h] = valid ? sv[h] * p.scale_log2 : -INFINITY;
    float mh[HQP];
#pragma unroll
    for (int h = 0; h < HQP; ++h) {
        float m = sv[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        mh[h] = m;
    }
    if ((tid & 31) == 0) {
#pragma unroll
        for (int h = 0; h < HQP; ++h) S.red[warp][h] = mh[h];
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < HQP; ++h) mh[h] = fmaxf(fmaxf(S.red[0][h], S.red[1][h]), fmaxf(S.red[2][h], S.red[3][h]));
    __syncthreads();
    float lh[HQP];
#pragma unroll
    for (int h = 0; h < HQP; ++h) {
        const float pv = valid ? exp2f(sv[h] - mh[h]) : 0.f;
        const __nv_bfloat16 pb = __float2bfloat16_rn(pv);
        *reinterpret_cast<__nv_bfloat16*>(S.pbuf + (r >> 6) * (HQP * 128) + sw128(h, (r & 63) >> 3) + (r & 7) * 2) = pb;
        float l = pv;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        lh[h] = l;
    }
    if ((tid & 31) == 0) {
#pragma unroll
        for (int h = 0; h < HQP; ++h) S.red[warp][h] = lh[h];
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
#pragma unroll
    for (int h = 0; h < HQP; ++h) lh[h] = S.red[0][h] + S.red[1][h] + S.red[2][h] + S.red[3][h];

    // ---- O^T = V^T P  (M = 128 = head dim (padded), N = HQP, K = 128 keys)
    if (tid == 0 && ok) {
        const uint32_t va = smem_u32(global_tile ? S.kbuf : S.vbuf), pa = smem_u32(S.pbuf);
        constexpr uint32_t idesc = idesc_bf16(128, HQP, 1);
#pragma unroll
        for (int kk = 0; kk < kTileKeys / 16; ++kk) {
            const uint64_t ad = smem_desc(va + kk * 2048, kPanelBytes, 1024);
            const uint64_t bd = smem_desc(pa + (kk >> 2) * (HQP * 128) + (kk & 3) * 32, 16, 1024);
            mma_bf16(tmem_o, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&S.bar_o);
    }
    ok = ok && mbar_wait(&S.bar_o, 0, p.status, 11);
    tc_fence_after();

    // ---- partial -> workspace: o[h][d] (unnormalised), m[h] (log2 units), l[h]
    float* part = p.part + ((size_t)u * p.ntiles + tau) * (HQP * (D + 2));
    if (ok) {
        float tmp[16];
#pragma unroll
        for (int c0 = 0; c0 < HQP; c0 += 16) {
            tmem_ld16(tmem_o + lane_off + c0, tmp);
            tmem_ld_wait();
            if (tid < D) {
#pragma unroll
                for (int i = 0; i < 16; ++i) part[(c0 + i) * D + tid] = tmp[i];
            }
        }
    }
    if (tid < HQP) {
        float mv = 0.f, lv = 0.f;
#pragma unroll
        for (int h = 0; h < HQP; ++h)
            if (h == tid) { mv = mh[h]; lv = lh[h]; }
        part[HQP * D + tid] = mv;
        part[HQP * D + HQP + tid] = lv;
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        S.is_last = (atomicAdd(p.tickets + u, 1) == p.ntiles - 1);
    }
    __syncthreads();

    if (S.is_last) {
        // Merge the query's tile partials: weights exp2(m_s - M) / L per (tile, head)
        // into shared memory, then every thread accumulates float4 slices of o.
        __threadfence();
        const float* pu = p.part + (size_t)u * p.ntiles * (HQP * (D + 2));
        const size_t stride = HQP * (D + 2);
        const int nt = p.ntiles;
        float* wgt = reinterpret_cast<float*>(S.kbuf);             // [nt][HQP]
        float* Mh = reinterpret_cast<float*>(S.vbuf);              // [HQP]
        float* Lh = Mh + HQP;                                      // [HQP]
        float* lsum = reinterpret_cast<float*>(S.kbuf + kPanelBytes);   // [nt][HQP] tile sums
        for (int i = tid; i < nt * HQP; i += kAttnThreads) {
            const int s2 = i / HQP, h = i % HQP;
            wgt[i] = __ldcg(pu + s2 * stride + HQP * D + h);
            lsum[i] = __ldcg(pu + s2 * stride + HQP * D + HQP + h);
        }
        __syncthreads();
        if (tid < HQP) {
            float M = -INFINITY;
            for (int s2 = 0; s2 < nt; ++s2) M = fmaxf(M, wgt[s2 * HQP + tid]);
            float L = 0.f;
            if (M != -INFINITY)
                for (int s2 = 0; s2 < nt; ++s2) {
                    const float ms = wgt[s2 * HQP + tid];
                    if (ms != -INFINITY) L += exp2f(ms - M) * lsum[s2 * HQP + tid];
                }
            Mh[tid] = M;
            Lh[tid] = L;
        }
        __syncthreads();
        for (int i = tid; i < nt * HQP; i += kAttnThreads) {
            const int h = i % HQP;
            const float ms = wgt[i];
            wgt[i] = (ms == -INFINITY || !(Lh[h] > 0.f)) ? 0.f : exp2f(ms - Mh[h]) / Lh[h];
        }
        __syncthreads();
        constexpr int D4 = D / 4;
        for (int it = tid; it < p.Hq * D4; it += kAttnThreads) {
            const int h = it / D4, d4 = it % D4;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            const float4* src = reinterpret_cast<const float4*>(pu + h * D) + d4;
#pragma unroll 8
            for (int s2 = 0; s2 < nt; ++s2) {
                const float4 v = __ldcg(src + s2 * (stride / 4));
                const float w = wgt[s2 * HQP + h];
                acc.x += w * v.x; acc.y += w * v.y; acc.z += w * v.z; acc.w += w * v.w;
            }
            __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
            uint2 pk;
            pk.x = *reinterpret_cast<uint32_t*>(&lo);
            pk.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(p.out + ((size_t)u * p.Hq + h) * D + 4 * d4) = pk;
        }
        if (tid < p.Hq && p.lse != nullptr) {
            const float L = Lh[tid];
            p.lse[(size_t)u * p.Hq + tid] = (L > 0.f) ? (Mh[tid] + log2f(L)) * 0.69314718055994530942f : -INFINITY;
        }
        if (tid == 0) p.tickets[u] = 0;
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kCols);
}

// ------------------------------------------------------------ host side
struct AttnPlan {
    int units, ngt, nlt, ntiles, HQP;
    size_t part_bytes;
};

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

AttnPlan plan_attn(const csa2_attn_args& a) {
    AttnPlan pl{};
    pl.units = a.B * a.Tq;
    pl.ngt = (a.k + kTileKeys - 1) / kTileKeys;
    pl.nlt = (a.W + kTileKeys - 1) / kTileKeys;
    pl.ntiles = pl.ngt + pl.nlt;
    pl.HQP = a.Hq <= 16 ? 16 : 32;
    pl.part_bytes = align256((size_t)pl.units * pl.ntiles * pl.HQP * (a.D + 2) * 4);
    return pl;
}

template <int HQP, int D>
static cudaError_t launch_attn_variant(const AttnParams& p, int units, cudaStream_t stream) {
    auto kern = sparse_attn_kernel<HQP, D>;
    const size_t smem = sizeof(AttnSmem<HQP>) + 1024;
    cudaError_t e = set_smem_once(reinterpret_cast<const void*>(kern), (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.ntiles, units);
    kern<<<grid, kAttnThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

// tickets: [units] ints, zero at rest (every call leaves them zero); scratch: partials
csa2_status launch_attn(const csa2_attn_args& a, const int32_t* topk, int* tickets, void* scratch,
                        int32_t* d_status, cudaStream_t stream) {
    AttnPlan pl = plan_attn(a);
    if (pl.units == 0) return CSA2_OK;
    AttnParams p{};
    p.B = a.B; p.Tq = a.Tq; p.N = a.N; p.Hq = a.Hq; p.D = a.D; p.k = a.k; p.W = a.W; p.Lloc = a.Lloc;
    p.ngt = pl.ngt; p.nlt = pl.nlt; p.ntiles = pl.ntiles;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)a.D));
    p.q_pos = a.q_pos; p.q = a.q; p.kv_fp4 = a.kv_fp4; p.kv_scale = a.kv_scale; p.topk = topk;
    p.kl = a.kl; p.vl = a.vl; p.local_base = a.local_base; p.out = a.out; p.lse = a.lse;
    p.tickets = tickets;
    p.part = static_cast<float*>(scratch);
    p.status = d_status;
    cudaError_t e;
    if (pl.HQP == 16 && a.D == 128) e = launch_attn_variant<16, 128>(p, pl.units, stream);
    else if (pl.HQP == 16 && a.D == 64) e = launch_attn_variant<16, 64>(p, pl.units, stream);
    else if (pl.HQP == 32 && a.D == 128) e = launch_attn_variant<32, 128>(p, pl.units, stream);
    else e = launch_attn_variant<32, 64>(p, pl.units, stream);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

size_t attn_scratch_bytes(const csa2_attn_args& a) { return plan_attn(a).part_bytes; }

}  // namespace csa2
