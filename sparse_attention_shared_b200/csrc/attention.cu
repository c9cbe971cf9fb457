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
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstddef>
#include <cstring>

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
    int list_ready; // the list and the cache were complete before the previous kernel began
    int m;          // sequence compression rate of the global entries
};

template <int HQP>
struct __align__(1024) AttnSmem {
    uint8_t kbuf[2 * kPanelBytes];      // key tile (also the value tile of a global tile)
    // value tile of a local tile, and the merge's tile sums; at 16 heads the key buffer takes
    // the values once S has read the keys, and 9 KB hold the sums of up to 144 tiles (a
    // multiple of 1024 bytes keeps the operands below aligned)
    uint8_t vbuf[HQP == 16 ? 9216 : 2 * kPanelBytes];
    uint8_t qbuf[2 * HQP * 128];        // queries, [HQP rows x D] in 64-element panels
    uint8_t pbuf[2 * HQP * 128];        // probabilities, [HQP rows x 128 keys] in 64-key panels
    float red[4][HQP];
    uint64_t bar_s, bar_o;
    uint32_t tmem_base;
    int is_last;
};
static_assert(offsetof(AttnSmem<16>, qbuf) % 1024 == 0 && offsetof(AttnSmem<32>, qbuf) % 1024 == 0,
              "operand alignment");

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Eight E2M1 codes (a 32-bit word, lowest nibble first) as four bf16x2 words, lower
// element in the lower half, by byte permutes: the three magnitude bits of each of four
// codes pick its value's high and low byte from two 8-entry byte tables (|v| = 0, 0.5,
// 1, 1.5, 2, 3, 4, 6 as bf16), two permutes interleave the bytes into values, and one
// more per pair of values moves the codes' sign bits to bit 15 of each. Registers only:
// no table in shared memory and no bank conflicts.
__device__ __forceinline__ uint4 e2m1x8_bf16(uint32_t w) {
    constexpr uint32_t kHi03 = 0x3F3F3F00u, kHi47 = 0x40404040u;   // high bytes, magnitudes 0-3 and 4-7
    constexpr uint32_t kLo03 = 0xC0800000u, kLo47 = 0xC0804000u;   // low bytes
    const uint32_t m = w & 0x77777777u, mh = m >> 16, w4 = w << 4;
    const uint32_t ha = prmt(kHi03, kHi47, m), la = prmt(kLo03, kLo47, m);
    const uint32_t hb = prmt(kHi03, kHi47, mh), lb = prmt(kLo03, kLo47, mh);
    uint4 r;
    // sign of code 2i: bit 7 of byte i of w << 4; of code 2i + 1: bit 7 of byte i of w
    r.x = prmt(la, ha, 0x5140u) | (prmt(w4, w, 0x4000u) & 0x80008000u);
    r.y = prmt(la, ha, 0x7362u) | (prmt(w4, w, 0x5010u) & 0x80008000u);
    r.z = prmt(lb, hb, 0x5140u) | (prmt(w4, w, 0x6020u) & 0x80008000u);
    r.w = prmt(lb, hb, 0x7362u) | (prmt(w4, w, 0x7030u) & 0x80008000u);
    return r;
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

// Eight E2M1 codes (a 32-bit word, lowest nibble first) as four f16x2 words, lower
// element in the lower half. The hardware conversion is exact: every E2M1 value is
// an f16 value.
__device__ __forceinline__ void e2m1x8_f16(uint32_t w, uint32_t (&d)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(w));
}

// Two E4M3 scales (lower byte first) as f16x2; exact (E4M3 values are f16 values).
__device__ __forceinline__ uint32_t e4m3x2_f16(uint32_t two) {
    uint32_t d;
    const uint16_t h = (uint16_t)two;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(h));
    return d;
}

__device__ __forceinline__ uint32_t f16x2_mul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// bf16x2 -> f16x2 after scaling by a power of two f (exact unless the scaled value
// falls below f16's normal range)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v, float f) {
    const float lo = __uint_as_float(v << 16) * f, hi = __uint_as_float(v & 0xFFFF0000u) * f;
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// largest bf16 exponent field among the eight values of a 16-byte chunk
__device__ __forceinline__ uint32_t bf16x8_max_exp(const uint4& v) {
    const uint32_t a = max((v.x >> 7) & 0xFFu, (v.x >> 23) & 0xFFu), b = max((v.y >> 7) & 0xFFu, (v.y >> 23) & 0xFFu);
    const uint32_t c = max((v.z >> 7) & 0xFFu, (v.z >> 23) & 0xFFu), d = max((v.w >> 7) & 0xFFu, (v.w >> 23) & 0xFFu);
    return max(max(a, b), max(c, d));
}

template <int HQP, int D>
__global__ void __launch_bounds__(kAttnThreads) sparse_attn_kernel(const __grid_constant__ AttnParams p) {
    CSA2_TRACE_INIT();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    AttnSmem<HQP>& S =
        *reinterpret_cast<AttnSmem<HQP>*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
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

    int t = p.q_pos[u];
    int tg = last_entry(t, p.m);   // the last global entry the query reads
    if (t < 0 || tg >= p.N) {
        if (tid == 0 && tau == 0) report(p.status, CSA2_ERR_RANGE, u);
        t = -1;
        tg = -1;
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
            if constexpr (HQP != 16) reinterpret_cast<uint4*>(S.vbuf + kPanelBytes)[i] = make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();

    // ---- the tile's 128 key rows
    const int r = tid;       // this thread's key row
    bool valid = false;
    if (global_tile) {
        const int j = tau * kTileKeys + r;
        int s = (j < p.k) ? p.topk[(size_t)u * p.k + j] : -1;
        if (s >= 0 && (s > tg || s >= p.N)) {
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
                const uint4 e = e2m1x8_bf16(w);
                uint4 o;
                o.x = bf16x2_mul(e.x, s2x);
                o.y = bf16x2_mul(e.y, s2x);
                o.z = bf16x2_mul(e.z, s2x);
                o.w = bf16x2_mul(e.w, s2x);
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
                    if constexpr (HQP != 16) vv[j] = __ldg(vls + off);
                }
            }
#pragma unroll
            for (int j = 0; j < BATCH; ++j) {
                const int i = tid + (i0 + j) * kAttnThreads;
                const int rr = i / CPR, c = i % CPR;
                const uint32_t dst = (c >> 3) * kPanelBytes + sw128(rr, c & 7);
                *reinterpret_cast<uint4*>(S.kbuf + dst) = kv[j];
                if constexpr (HQP != 16) *reinterpret_cast<uint4*>(S.vbuf + dst) = vv[j];
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
    if constexpr (HQP == 16) {
        if (!global_tile) {   // the local tile's values go into the key buffer, which S has read
            const int lo = max(max(base, t - p.W + 1), 0);
            const int p0 = lo + (tau - p.ngt) * kTileKeys;
            const uint4* vls = reinterpret_cast<const uint4*>(p.vl);
            constexpr int CPR = D / 8, ITERS = kTileKeys * CPR / kAttnThreads, BATCH = ITERS < 8 ? ITERS : 8;
#pragma unroll
            for (int i0 = 0; i0 < ITERS; i0 += BATCH) {
                uint4 vv[BATCH];
#pragma unroll
                for (int j = 0; j < BATCH; ++j) {
                    const int i = tid + (i0 + j) * kAttnThreads;
                    const int rr = i / CPR, c = i % CPR;
                    const int pr = p0 + rr, lrow = pr - base;
                    const bool okr = (t >= 0) && (p.W > 0) && (pr <= t) && lrow >= 0 && lrow < p.Lloc;
                    vv[j] = okr ? __ldg(vls + ((size_t)b * p.Lloc + lrow) * CPR + c) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int j = 0; j < BATCH; ++j) {
                    const int i = tid + (i0 + j) * kAttnThreads;
                    const int rr = i / CPR, c = i % CPR;
                    *reinterpret_cast<uint4*>(S.kbuf + (c >> 3) * kPanelBytes + sw128(rr, c & 7)) = vv[j];
                }
            }
        }
    }

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
        const uint32_t va = smem_u32((global_tile || HQP == 16) ? S.kbuf : S.vbuf), pa = smem_u32(S.pbuf);
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
        // (k + W <= 16384 gives at most 129 tiles: each buffer holds at least 144)
        const int nt = CSA2_CHECK(p.ntiles * HQP * 4 <= (int)sizeof(S.vbuf), p.status, 2104) ? p.ntiles : 0;
        float* wgt = reinterpret_cast<float*>(S.kbuf);             // [nt][HQP]
        float* lsum = reinterpret_cast<float*>(S.vbuf);            // [nt][HQP] tile sums
        float* Mh = S.red[0];                                      // [HQP]
        float* Lh = S.red[1];                                      // [HQP]
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

    CSA2_TRACE_END(4);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kCols);
}

// ------------------------------------------------------------ clustered variant
// One thread-block cluster per query: CTA r < ngt2 takes 256 entries of the
// global list (two 128-row MMA blocks), the others one 128-row tile of the
// window each. Every CTA issues all of its loads at once (the list entries,
// then its FP4 rows; local tiles by TMA), computes its softmax partial on the
// tensor cores, parks it in shared memory, and the cluster merges the
// partials through distributed shared memory: CTA r writes the heads
// h = r, r + CS, ... . No partial goes through global memory.
constexpr int kCLBuf = 4 * kPanelBytes;   // 64 KB: a 256-row global tile or a local K+V tile
constexpr int kClThreads = 256;           // one key row of a global tile per thread

template <int HQP>
struct AttnClSmem {   // placed at a 1024-byte-aligned address (operand tiles need it)
    uint8_t tbuf[kCLBuf];
    // Q as [HQP rows x D] (two 64-element panels), then, once S = K Q^T has been
    // computed, P as [HQP rows x 256 keys] in four 64-key panels
    uint8_t qpbuf[4 * HQP * 128];
    float qmul[HQP];                      // per head: the softmax scale (log2 units) over the Q scaling
    float red[kClThreads / 32][HQP];      // per-warp head maxima, then sums
    float mfin[HQP], lfin[HQP];
    // partials pushed by the cluster's CTAs for the heads this CTA merges: head h
    // (merged by CTA h % CS) from CTA c sits in row (h / CS) * CS + c
    float recv_o[HQP + 16][128];
    float recv_m[HQP + 16], recv_l[HQP + 16];
    uint64_t bar_tma, bar_s, bar_o;
    uint32_t tmem_base;
};

static_assert(offsetof(AttnClSmem<16>, qpbuf) % 1024 == 0 && offsetof(AttnClSmem<32>, qpbuf) % 1024 == 0,
              "operand alignment");
static_assert(sizeof(AttnClSmem<32>) + 1024 <= 113 * 1024, "two clustered-attention CTAs per SM");

// Reduce V values per lane (V = 8, 16 or 32, one per head) across the 32 lanes of a
// warp with halving exchanges: after the call, lane l holds in v[0] the result for
// value (l / (32 / V)) % V: head l & 31 (V = 32), (l >> 1) & 15 (V = 16) or (l >> 2) & 7
// (V = 8). V - 1 + log2(32 / V) shuffles instead of 5*V.
template <int V, bool kMax>
__device__ __forceinline__ float warp_transpose_reduce(float (&v)[V]) {
    static_assert(V == 8 || V == 16 || V == 32, "values per lane");
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int half = V / 2, bit = 16; half >= 1; half >>= 1, bit >>= 1) {
        const bool up = (lane & bit) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = up ? v[i] : v[i + half];
            const float keep = up ? v[i + half] : v[i];
            const float recv = __shfl_xor_sync(0xffffffffu, send, bit);
            v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
        }
    }
#pragma unroll
    for (int bit = 16 / V; bit >= 1; bit >>= 1) {   // lanes that still hold partials of the same value
        const float recv = __shfl_xor_sync(0xffffffffu, v[0], bit);
        v[0] = kMax ? fmaxf(v[0], recv) : v[0] + recv;
    }
    return v[0];
}

template <int HQP, int D>
__global__ void __launch_bounds__(kClThreads, 2)
    sparse_attn_cl_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap kl_map,
                          const __grid_constant__ CUtensorMap vl_map) {
    static_assert(HQP == 16 || HQP == 32, "head padding");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    AttnClSmem<HQP>& S =
        *reinterpret_cast<AttnClSmem<HQP>*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    constexpr uint32_t kCols = (3 * HQP <= 32) ? 32 : (3 * HQP <= 64 ? 64 : 128);
    constexpr int kPanels = D / 64;
    constexpr int kWarps = kClThreads / 32;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int CS = gridDim.x;
    const int rank = (int)cluster_ctarank();
    const int u = blockIdx.y;
    CSA2_TRACE_INIT();
    const int b = u / p.Tq;
    const int ngt2 = (p.k + 2 * kTileKeys - 1) / (2 * kTileKeys);
    const bool glob = rank < ngt2;

    // ---- 0. set-up that reads no input; it may overlap the previous kernel
    if (warp == 0) tmem_alloc(&S.tmem_base, kCols);
    if (tid == 0) {
        mbar_init(&S.bar_tma, 1);
        mbar_init(&S.bar_s, 1);
        mbar_init(&S.bar_o, 1);
        mbar_fence_init();
    }
    // A global CTA of a layer whose list and cache were complete before the previous
    // kernel began (a Reuse layer of a stack) issues its list and row loads before
    // waiting for that kernel; everything else (Q, the window) is read after the wait.
    const bool pre = glob && p.list_ready;
    constexpr int kQv = (HQP * D / 8 + kClThreads - 1) / kClThreads;   // 16-byte chunks of Q per thread
    uint4 qv[kQv];
    auto load_q = [&]() {   // the query depends on the previous layer: only after the wait
#pragma unroll
        for (int q = 0; q < kQv; ++q) {
            const int i = tid + q * kClThreads;
            const int h = i / (D / 8), c = i % (D / 8);
            qv[q] = make_uint4(0, 0, 0, 0);
            if (i < HQP * (D / 8) && h < p.Hq) qv[q] = __ldg(reinterpret_cast<const uint4*>(p.q + ((size_t)u * p.Hq + h) * D) + c);
        }
    };
    if (!pre) {
        pdl_wait();
        pdl_launch_dependents();
        load_q();   // in flight while the list and the rows are fetched
    }
    CSA2_TRACE(1);

    // ---- 1. positions and list entries; row tid of the tile is this thread's
    int t = p.q_pos[u];
    const int base = p.local_base[b];
    int s0 = -1;
    if (glob) {
        const int j0 = rank * 2 * kTileKeys + tid;
        s0 = (j0 < p.k) ? __ldcg(p.topk + (size_t)u * p.k + j0) : -1;
    }
    int tg = last_entry(t, p.m);   // the last global entry the query reads
    if (t < 0 || tg >= p.N) {
        if (tid == 0 && rank == 0) report(p.status, CSA2_ERR_RANGE, u);
        t = -1;
        tg = -1;
    }
    const int lo_w = max(max(base, t - p.W + 1), 0);
    CSA2_TRACE(2);   // positions

    // ---- 2. the tile's rows
    bool v0 = false;
    uint4 c0[D / 32];
    uint32_t sc0[D / 64];
    if (glob) {
        if (s0 >= 0 && (s0 > tg || s0 >= p.N)) { report(p.status, CSA2_ERR_RANGE, u); s0 = -1; }
        v0 = s0 >= 0;
        if (v0) {
            const size_t row = (size_t)b * p.N + s0;
            const uint4* cp = reinterpret_cast<const uint4*>(p.kv_fp4 + row * (D / 2));
#pragma unroll
            for (int q = 0; q < D / 32; ++q) c0[q] = __ldg(cp + q);
            if (D == 128) {
                const uint2 s2 = __ldg(reinterpret_cast<const uint2*>(p.kv_scale + row * 8));
                sc0[0] = s2.x;
                sc0[(D / 64) - 1] = s2.y;
            } else {
                sc0[0] = __ldg(reinterpret_cast<const uint32_t*>(p.kv_scale + row * 4));
            }
        }
    } else {
        const int lt = rank - ngt2;
        const int pos = lo_w + lt * kTileKeys + tid;
        v0 = tid < kTileKeys && (t >= 0) && (p.W > 0) && (pos <= t) && (pos - base) < p.Lloc;
        if (tid == 0) {
            mbar_arrive_expect_tx(&S.bar_tma, 2u * kPanels * kPanelBytes);
            const int y = lo_w - base + lt * kTileKeys;
#pragma unroll
            for (int pn = 0; pn < kPanels; ++pn) {
                tma_load_3d(S.tbuf + pn * kPanelBytes, &kl_map, pn * 64, y, b, &S.bar_tma);
                tma_load_3d(S.tbuf + 2 * kPanelBytes + pn * kPanelBytes, &vl_map, pn * 64, y, b, &S.bar_tma);
            }
        }
    }
    if (glob && D == 64) {   // the value operand's second M-half stays zero
        for (int i = tid; i < 2 * kPanelBytes / 16; i += kClThreads)
            reinterpret_cast<uint4*>(S.tbuf + 2 * kPanelBytes)[i] = make_uint4(0, 0, 0, 0);
    }
    if (!glob && D == 64) {
        for (int i = tid; i < kPanelBytes / 16; i += kClThreads) {
            reinterpret_cast<uint4*>(S.tbuf + kPanelBytes)[i] = make_uint4(0, 0, 0, 0);
            reinterpret_cast<uint4*>(S.tbuf + 3 * kPanelBytes)[i] = make_uint4(0, 0, 0, 0);
        }
    }
    if (pre) {
        // the rows are in flight: wait for the previous kernel here, so that a CTA that
        // starts after it has ended has its query load in flight during the dequantisation
        pdl_wait();
        pdl_launch_dependents();
        load_q();
    }
    __syncthreads();   // the barriers (initialised by thread 0) and TMEM address are set
    CSA2_TRACE(3);
    bool ok = true;
    if (glob) {
        // A global tile is dequantised to f16 (code times scale is exact in f16) and
        // multiplied in f16: Q is brought into f16's range by a power of two per head
        // below. Panels hold 256 rows: panel p at p * 2 * kPanelBytes; row tid.
        uint32_t sp[D / 32];   // f16x2 scale pairs (groups 2i, 2i + 1)
#pragma unroll
        for (int i = 0; i < D / 32; ++i) sp[i] = e4m3x2_f16(sc0[i >> 1] >> (16 * (i & 1)));
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
            uint4 o = make_uint4(0, 0, 0, 0);
            if (v0) {
                const uint4 w4 = c0[c >> 2];
                const uint32_t w = (c & 3) == 0 ? w4.x : (c & 3) == 1 ? w4.y : (c & 3) == 2 ? w4.z : w4.w;
                const uint32_t g = c >> 1;   // scale group of 16
                const uint32_t pr = sp[g >> 1];
                const uint32_t s2x = (g & 1) ? ((pr >> 16) | (pr & 0xFFFF0000u)) : ((pr & 0xFFFFu) | (pr << 16));
                uint32_t d[4];
                e2m1x8_f16(w, d);
                o.x = f16x2_mul(d[0], s2x);
                o.y = f16x2_mul(d[1], s2x);
                o.z = f16x2_mul(d[2], s2x);
                o.w = f16x2_mul(d[3], s2x);
            }
            *reinterpret_cast<uint4*>(S.tbuf + (c >> 3) * (2 * kPanelBytes) + sw128(tid, c & 7)) = o;
        }
    }
#pragma unroll
    for (int q = 0; q < kQv; ++q) {
        const int i = tid + q * kClThreads;
        const int h = i / (D / 8), c = i % (D / 8);
        uint4 v = qv[q];
        float mul = p.scale_log2;
        if (glob) {
            // head h's D / 8 chunks sit in D / 8 consecutive lanes: the largest exponent
            // over the head sets 2^k, which puts the head's largest value in [2^14, 2^15)
            uint32_t e = bf16x8_max_exp(v);
#pragma unroll
            for (int o = 1; o < D / 8; o <<= 1) e = max(e, __shfl_xor_sync(0xffffffffu, e, o));
            const int k = (e == 0u) ? 0 : min(141 - (int)e, 126);
            const float f = __uint_as_float((uint32_t)(127 + k) << 23);
            v.x = bf16x2_to_f16x2(v.x, f);
            v.y = bf16x2_to_f16x2(v.y, f);
            v.z = bf16x2_to_f16x2(v.z, f);
            v.w = bf16x2_to_f16x2(v.w, f);
            mul = p.scale_log2 * __uint_as_float((uint32_t)(127 - k) << 23);
        }
        if (i < HQP * (D / 8)) {
            *reinterpret_cast<uint4*>(S.qpbuf + (c >> 3) * (HQP * 128) + sw128(h, c & 7)) = v;
            if (c == 0) S.qmul[h] = mul;
        }
    }
    if (!glob) ok = mbar_wait(&S.bar_tma, 0, p.status, 12);
    CSA2_TRACE(4);   // tile staged
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const int nblk = glob ? 2 : 1;
    const uint32_t panel_stride = glob ? 2 * kPanelBytes : kPanelBytes;

    // ---- 3. S = K Q^T per 128-row block
    if (tid == 0) {
        const uint32_t ka = smem_u32(S.tbuf), qa = smem_u32(S.qpbuf);
        const uint32_t idesc = glob ? idesc_f16(128, HQP, 0) : idesc_bf16(128, HQP, 0);
        for (int blk = 0; blk < nblk; ++blk) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t ad = smem_desc(ka + (kk >> 2) * panel_stride + blk * kPanelBytes + (kk & 3) * 32, 16, 1024);
                const uint64_t bd = smem_desc(qa + (kk >> 2) * (HQP * 128) + (kk & 3) * 32, 16, 1024);
                mma_bf16(tmem + blk * HQP, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
        }
        mma_commit(&S.bar_s);
    }
    ok = mbar_wait(&S.bar_s, 0, p.status, 10) && ok;
    CSA2_TRACE(5);   // S done
    tc_fence_after();

    // ---- 4. softmax partial over the tile's rows: thread tid holds key tid, which
    // sits in row block tid / 128, TMEM lane tid % 128 (warp w reads lane quarter w % 4)
    float a[HQP];
    {
        const uint32_t ta = tmem + (uint32_t)(tid >> 7) * HQP + ((uint32_t)(warp & 3) * 32u << 16);
        float tmp[16];
#pragma unroll
        for (int c0i = 0; c0i < HQP; c0i += 16) {
            tmem_ld16(ta + c0i, tmp);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 16; ++q) a[c0i + q] = tmp[q];
        }
    }
    const bool r0 = v0 && ok;
#pragma unroll
    for (int h = 0; h < HQP; ++h) a[h] = r0 ? a[h] * S.qmul[h] : -INFINITY;
    const int hl = (HQP == 16) ? ((lane >> 1) & 15) : lane;   // the head this lane ends up holding
    {
        float v[HQP];
#pragma unroll
        for (int h = 0; h < HQP; ++h) v[h] = a[h];
        const float m = warp_transpose_reduce<HQP, true>(v);
        if (HQP == 32 || (lane & 1) == 0) S.red[warp][hl] = m;
    }
    __syncthreads();
    if (tid < HQP) {
        float m = S.red[0][tid];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) m = fmaxf(m, S.red[w][tid]);
        S.mfin[tid] = m;
    }
    __syncthreads();
    float pv[HQP];
#pragma unroll
    for (int h = 0; h < HQP; ++h) {
        const float mh = S.mfin[h];
        pv[h] = (r0 && mh != -INFINITY) ? exp2f(a[h] - mh) : 0.f;
        // key tid -> panel tid / 64, column tid % 64
        const float pr = pv[h];
        *reinterpret_cast<uint16_t*>(S.qpbuf + (tid >> 6) * (HQP * 128) + sw128(h, (tid & 63) >> 3) + (tid & 7) * 2) =
            glob ? __half_as_ushort(__float2half_rn(pr)) : __bfloat16_as_ushort(__float2bfloat16_rn(pr));
    }
    {
        const float l = warp_transpose_reduce<HQP, false>(pv);
        if (HQP == 32 || (lane & 1) == 0) S.red[warp][hl] = l;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid < HQP) {
        float l = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) l += S.red[w][tid];
        S.lfin[tid] = l;
    }

    CSA2_TRACE(6);   // softmax done
    // ---- 5. O^T = V^T P (keys as the reduction; the head dim as M)
    if (tid == 0) {
        const uint32_t va = smem_u32(glob ? S.tbuf : S.tbuf + 2 * kPanelBytes), pa = smem_u32(S.qpbuf);
        const uint32_t idesc = glob ? idesc_f16(128, HQP, 1) : idesc_bf16(128, HQP, 1);
        const int nk = nblk * (kTileKeys / 16);
        for (int kk = 0; kk < nk; ++kk) {
            const uint64_t ad = smem_desc(va + kk * 2048, panel_stride, 1024);
            const uint64_t bd = smem_desc(pa + (kk >> 2) * (HQP * 128) + (kk & 3) * 32, 16, 1024);
            mma_bf16(tmem + 2 * HQP, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&S.bar_o);
    }
    ok = mbar_wait(&S.bar_o, 0, p.status, 11) && ok;
    CSA2_TRACE(7);   // O done
    tc_fence_after();
    float ov[HQP];
    if (warp < 4) {   // O^T rows (the head dim) sit in TMEM lanes 0..127
        float tmp[16];
#pragma unroll
        for (int c0i = 0; c0i < HQP; c0i += 16) {
            tmem_ld16(tmem + 2 * HQP + ((uint32_t)(warp * 32) << 16) + c0i, tmp);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 16; ++q) ov[c0i + q] = tmp[q];
        }
    }
    tc_fence_before();

    // ---- 6. merge: every CTA pushes its partial of head h into the shared memory of
    // the CTA that merges h (CTA h % CS); one cluster barrier publishes the pushes,
    // then each CTA merges its heads from its own shared memory
    if (tid < D) {
#pragma unroll
        for (int h = 0; h < HQP; ++h) {
            if (h >= p.Hq) break;
            if (!CSA2_CHECK((h / CS) * CS + rank < HQP + 16 && h % CS < CS, p.status, 2101)) break;
            st_dsmem(dsmem_addr(&S.recv_o[(h / CS) * CS + rank][tid], h % CS), ok ? ov[h] : 0.f);
        }
    }
    if (tid < p.Hq) {
        const int row = (tid / CS) * CS + rank, owner = tid % CS;
        if (CSA2_CHECK(row < HQP + 16, p.status, 2102)) {
            st_dsmem(dsmem_addr(&S.recv_m[row], owner), ok ? S.mfin[tid] : -INFINITY);
            st_dsmem(dsmem_addr(&S.recv_l[row], owner), ok ? S.lfin[tid] : 0.f);
        }
    }
    cluster_sync_all();   // after it no CTA touches another's shared memory
    CSA2_TRACE(8);   // partials exchanged
    constexpr int kSlots = kClThreads / D;
    const int slot = tid / D, dim = tid % D;
    for (int h = rank + slot * CS; h < p.Hq; h += kSlots * CS) {
        const int r0 = (h / CS) * CS;
        if (!CSA2_CHECK(r0 + CS <= HQP + 16, p.status, 2103)) break;
        float M = -INFINITY;
#pragma unroll
        for (int c = 0; c < 16; ++c)
            if (c < CS) M = fmaxf(M, S.recv_m[r0 + c]);
        float L = 0.f, acc = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                if (c >= CS) break;
                const float mc = S.recv_m[r0 + c];
                const float wgt = (mc == -INFINITY) ? 0.f : exp2f(mc - M);
                L += wgt * S.recv_l[r0 + c];
                acc += wgt * S.recv_o[r0 + c][dim];
            }
        }
        p.out[((size_t)u * p.Hq + h) * D + dim] = __bfloat16_as_ushort(__float2bfloat16_rn(L > 0.f ? acc / L : 0.f));
        if (dim == 0 && p.lse != nullptr)
            p.lse[(size_t)u * p.Hq + h] = (L > 0.f) ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
    }
    CSA2_TRACE(9);
    CSA2_TRACE_END(3);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kCols);
}

// ------------------------------------------------------------ one CTA per query
// For calls with many queries (a prefill chunk, a bounded replay), where throughput
// counts rather than one query's latency: one CTA (NT = 128 or 256 threads) takes every
// tile of its query in turn, the global tiles of its list and then its window tiles, 128
// rows each, with an online softmax. Per tile: S = K Q^T into TMEM, the tile's maximum per
// head updates the running maximum m, P = exp2(s - m) goes to shared memory, O_tile^T =
// V^T P into a fresh TMEM accumulator, and each thread (one row of O^T, one head
// dimension, its part of the heads) rescales its running o[h] by exp2(m_old - m_new) and
// adds the tile's. The query's output is o / l at the end: no partials leave the CTA and
// nothing is merged. NT / 128 threads stage each row of a tile (a part of the row each);
// in the softmax and the O update, warp w reads TMEM lanes 32 (w % 4) .. + 31 and the
// columns of head part w / 4. 16 padded heads run 128 threads at four CTAs per SM (a
// window tile's values then follow its keys through one buffer), 32 heads 256 threads at
// two (shared memory holds two of those).
// Global rows are dequantised to bf16 (code times scale has at most seven significant
// bits, so bf16 holds it exactly) and Q is bf16 for both kinds of tile.
template <int HQP>
struct __align__(1024) AttnSeqSmem {
    uint8_t kbuf[2 * kPanelBytes];      // key tile (also the value tile of a global tile)
    // value tile of a window tile; at 16 heads the key buffer takes it once S has read the
    // keys (1 KB here keeps the operands below 1024-byte aligned)
    uint8_t vbuf[HQP == 16 ? 1024 : 2 * kPanelBytes];
    uint8_t qbuf[2 * HQP * 128];        // queries, [HQP rows x D] in 64-element panels
    uint8_t pbuf[2 * HQP * 128];        // probabilities, [HQP rows x 128 keys] in 64-key panels
    float red_m[4][HQP], red_l[4][HQP];
    float m_run[HQP], l_run[HQP];       // running maximum (log2 units) and sum per head
    float cf[HQP];                      // the tile's rescale exp2(m_old - m_new) per head
    int rowok[kTileKeys];               // the tile's rows that hold an entry
    uint64_t bar_s, bar_o;
    uint32_t tmem_base;
};

// HH consecutive TMEM columns of this warp's 32 lanes (HH = 8 or 16).
template <int HH>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&v)[HH]) {
    if constexpr (HH == 16) {
        tmem_ld16(taddr, v);
    } else {
        int t[8];
        tmem_ld8(taddr, t);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __int_as_float(t[i]);
    }
}

static_assert(offsetof(AttnSeqSmem<16>, qbuf) % 1024 == 0 && offsetof(AttnSeqSmem<32>, qbuf) % 1024 == 0,
              "operand alignment");

template <int HQP> constexpr int seq_threads() { return HQP == 16 ? 128 : 256; }

template <int HQP, int D, int NT = seq_threads<HQP>()>
__global__ void __launch_bounds__(NT, NT == 128 && HQP == 16 ? 4 : 2)
    sparse_attn_seq_kernel(const __grid_constant__ AttnParams p) {
    CSA2_TRACE_INIT();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    AttnSeqSmem<HQP>& S =
        *reinterpret_cast<AttnSeqSmem<HQP>*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    constexpr uint32_t kCols = (2 * HQP < 32) ? 32 : 2 * HQP;
    constexpr int TPR = NT / 128;          // threads per row of a tile
    constexpr int HH = HQP / TPR;          // heads per warp in the softmax and the O update
    constexpr int kLpv = 32 / HH;          // lanes that hold one head after a transpose-reduce
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, hh0 = (warp >> 2) * HH;   // TMEM lane quarter, first head of this warp
    const int u = blockIdx.x;
    const int b = u / p.Tq;

    if (warp == 0) tmem_alloc(&S.tmem_base, kCols);
    if (tid == 0) {
        mbar_init(&S.bar_s, 1);
        mbar_init(&S.bar_o, 1);
        mbar_fence_init();
    }
    pdl_wait();   // the list, the query and the window's newest rows may come from the previous kernel
    pdl_launch_dependents();

    int t = p.q_pos[u];
    int tg = last_entry(t, p.m);   // the last global entry the query reads
    if (t < 0 || tg >= p.N) {
        if (tid == 0) report(p.status, CSA2_ERR_RANGE, u);
        t = -1;
        tg = -1;
    }
    const int base = p.local_base[b];
    const int lo_w = max(max(base, t - p.W + 1), 0);

    // ---- queries -> qbuf (rows >= Hq are zero); a D = 64 value operand's second half is zero
    for (int i = tid; i < HQP * (D / 8); i += NT) {
        const int h = i / (D / 8), c = i % (D / 8);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (h < p.Hq) v = __ldg(reinterpret_cast<const uint4*>(p.q + ((size_t)u * p.Hq + h) * D) + c);
        *reinterpret_cast<uint4*>(S.qbuf + (c >> 3) * (HQP * 128) + sw128(h, c & 7)) = v;
    }
    if (D == 64) {
        for (int i = tid; i < kPanelBytes / 16; i += NT) {
            reinterpret_cast<uint4*>(S.kbuf + kPanelBytes)[i] = make_uint4(0, 0, 0, 0);
            if constexpr (HQP != 16) reinterpret_cast<uint4*>(S.vbuf + kPanelBytes)[i] = make_uint4(0, 0, 0, 0);
        }
    }
    float o[HH];   // this thread's row of O^T (head dimension 32 * quarter + lane), heads hh0 ..
#pragma unroll
    for (int h = 0; h < HH; ++h) o[h] = 0.f;
    if (tid < HQP) { S.m_run[tid] = -INFINITY; S.l_run[tid] = 0.f; }
    const int hl = hh0 + ((lane / kLpv) % HH);   // the head a lane holds after a transpose-reduce
    const bool hl_writer = (lane % kLpv) == 0;
    const int rs = tid / TPR, part = tid % TPR;  // staging: this thread's row of a tile and its part
    const int rm = quarter * 32 + lane;          // softmax: this thread's key row (TMEM lane)
    bool ok = true;
    const int ntiles = p.ngt + p.nlt;
    int s_next = -1;     // the next global tile's list entry for row rs, loaded during this tile
#pragma unroll 1
    for (int tau = 0; tau < ntiles; ++tau) {
        const bool global_tile = tau < p.ngt;
        // ---- the tile's 128 rows, two threads a row
        if (global_tile) {
            const int jj = tau * kTileKeys + rs;
            int s = tau == 0 ? ((jj < p.k) ? __ldcg(p.topk + (size_t)u * p.k + jj) : -1) : s_next;
            if (s >= 0 && (s > tg || s >= p.N)) {
                if (part == 0) report(p.status, CSA2_ERR_RANGE, u);
                s = -1;
            }
            if (part == 0) S.rowok[rs] = s >= 0;
            constexpr int CH = D / 8 / TPR;   // 8-element chunks in this thread's part of a row
            constexpr int SB = D / 16 / TPR;  // its scale bytes, one per 16-element group
            if (s >= 0) {
                const size_t row = (size_t)b * p.N + s;
                const uint4* cp = reinterpret_cast<const uint4*>(p.kv_fp4 + row * (D / 2) + part * (D / 2 / TPR));
                uint4 codes[CH / 4];
#pragma unroll
                for (int i = 0; i < CH / 4; ++i) codes[i] = __ldg(cp + i);
                const uint8_t* sp = p.kv_scale + row * (D / 16) + part * SB;
                uint64_t sw;
                if constexpr (SB == 8) {
                    const uint2 s2 = __ldg(reinterpret_cast<const uint2*>(sp));
                    sw = (uint64_t)s2.x | ((uint64_t)s2.y << 32);
                } else if constexpr (SB == 4) {
                    sw = __ldg(reinterpret_cast<const uint32_t*>(sp));
                } else {
                    sw = __ldg(reinterpret_cast<const uint16_t*>(sp));
                }
#pragma unroll
                for (int c = 0; c < CH; ++c) {           // 8 elements (4 code bytes) per chunk
                    const uint4 cw = codes[c >> 2];
                    const uint32_t w = (c & 3) == 0 ? cw.x : (c & 3) == 1 ? cw.y : (c & 3) == 2 ? cw.z : cw.w;
                    const uint32_t s16 = e4m3_bf16_bits((uint32_t)(sw >> (8 * (c >> 1))) & 0xFFu);
                    const uint32_t s2x = s16 | (s16 << 16);
                    const uint4 e = e2m1x8_bf16(w);
                    uint4 ov;
                    ov.x = bf16x2_mul(e.x, s2x);
                    ov.y = bf16x2_mul(e.y, s2x);
                    ov.z = bf16x2_mul(e.z, s2x);
                    ov.w = bf16x2_mul(e.w, s2x);
                    const int cg = part * CH + c;        // the chunk within the row
                    *reinterpret_cast<uint4*>(S.kbuf + (cg >> 3) * kPanelBytes + sw128(rs, cg & 7)) = ov;
                }
            } else {
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    const int cg = part * CH + c;
                    *reinterpret_cast<uint4*>(S.kbuf + (cg >> 3) * kPanelBytes + sw128(rs, cg & 7)) =
                        make_uint4(0, 0, 0, 0);
                }
            }
        } else {
            // window rows [lo_w, t], tile lt: coalesced 16-byte loads of K and V
            const int p0 = lo_w + (tau - p.ngt) * kTileKeys;
            if (tid < kTileKeys) {
                const int pr = p0 + tid;
                bool valid = (t >= 0) && (p.W > 0) && (pr <= t);
                if (valid && (pr - base < 0 || pr - base >= p.Lloc)) {
                    report(p.status, CSA2_ERR_RANGE, u);
                    valid = false;
                }
                S.rowok[tid] = valid;
            }
            const uint4* kls = reinterpret_cast<const uint4*>(p.kl);
            const uint4* vls = reinterpret_cast<const uint4*>(p.vl);
            constexpr int CPR = D / 8;                              // 16-byte chunks per row
            constexpr int ITERS = kTileKeys * CPR / NT;    // chunks per thread per tensor
            constexpr int BATCH = ITERS < 8 ? ITERS : 8;            // loads in flight per tensor
#pragma unroll
            for (int i0 = 0; i0 < ITERS; i0 += BATCH) {
                uint4 kv[BATCH], vv[BATCH];
#pragma unroll
                for (int jb = 0; jb < BATCH; ++jb) {
                    const int i = tid + (i0 + jb) * NT;
                    const int rr = i / CPR, c = i % CPR;
                    const int pr = p0 + rr;
                    const int lrow = pr - base;
                    const bool okr = (t >= 0) && (p.W > 0) && (pr <= t) && lrow >= 0 && lrow < p.Lloc;
                    kv[jb] = make_uint4(0, 0, 0, 0);
                    vv[jb] = make_uint4(0, 0, 0, 0);
                    if (okr) {
                        const size_t off = ((size_t)b * p.Lloc + lrow) * CPR + c;
                        kv[jb] = __ldg(kls + off);
                        if constexpr (HQP != 16) vv[jb] = __ldg(vls + off);
                    }
                }
#pragma unroll
                for (int jb = 0; jb < BATCH; ++jb) {
                    const int i = tid + (i0 + jb) * NT;
                    const int rr = i / CPR, c = i % CPR;
                    const uint32_t dst = (c >> 3) * kPanelBytes + sw128(rr, c & 7);
                    *reinterpret_cast<uint4*>(S.kbuf + dst) = kv[jb];
                    if constexpr (HQP != 16) *reinterpret_cast<uint4*>(S.vbuf + dst) = vv[jb];
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();   // the tile (and, at the first tile, Q, the barriers and TMEM) is in place
        tc_fence_after();
        const int tslot = tau == 0 ? 1 : tau == ntiles - 1 ? 6 : 0;   // phase-trace slots (first, last tile)
        if (tslot) { CSA2_TRACE(tslot); }   // tile staged
        if (tau + 1 < p.ngt) {   // the next tile's list entry, in flight during this tile
            const int jn = (tau + 1) * kTileKeys + rs;
            s_next = jn < p.k ? __ldcg(p.topk + (size_t)u * p.k + jn) : -1;
        }
        const uint32_t tmem_s = S.tmem_base, tmem_o = S.tmem_base + HQP;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;

        // ---- S = K Q^T  (M = 128 keys, N = HQP heads, K = D)
        if (tid == 0 && ok) {
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
        ok = ok && mbar_wait(&S.bar_s, (uint32_t)(tau & 1), p.status, 13);
        tc_fence_after();
        if constexpr (HQP == 16) {
            if (!global_tile) {   // the window tile's values go into the key buffer, which S has read
                const int p0 = lo_w + (tau - p.ngt) * kTileKeys;
                const uint4* vls = reinterpret_cast<const uint4*>(p.vl);
                constexpr int CPR = D / 8, ITERS = kTileKeys * CPR / NT, BATCH = ITERS < 8 ? ITERS : 8;
#pragma unroll
                for (int i0 = 0; i0 < ITERS; i0 += BATCH) {
                    uint4 vv[BATCH];
#pragma unroll
                    for (int jb = 0; jb < BATCH; ++jb) {
                        const int i = tid + (i0 + jb) * NT;
                        const int rr = i / CPR, c = i % CPR;
                        const int pr = p0 + rr, lrow = pr - base;
                        const bool okr = (t >= 0) && (p.W > 0) && (pr <= t) && lrow >= 0 && lrow < p.Lloc;
                        vv[jb] = okr ? __ldg(vls + ((size_t)b * p.Lloc + lrow) * CPR + c) : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int jb = 0; jb < BATCH; ++jb) {
                        const int i = tid + (i0 + jb) * NT;
                        const int rr = i / CPR, c = i % CPR;
                        *reinterpret_cast<uint4*>(S.kbuf + (c >> 3) * kPanelBytes + sw128(rr, c & 7)) = vv[jb];
                    }
                }
            }
        }
        if (tslot) { CSA2_TRACE(tslot + 1); }   // S done

        // ---- online softmax: the tile's maximum per head, then P and the tile's sums
        float sv[HH];
#pragma unroll
        for (int h = 0; h < HH; ++h) sv[h] = 0.f;
        if (ok) {
            tmem_ld_cols<HH>(tmem_s + lane_off + hh0, sv);
            tmem_ld_wait();
        }
        const bool rv = ok && S.rowok[rm] != 0;
        {
            float v[HH];
#pragma unroll
            for (int h = 0; h < HH; ++h) {
                sv[h] = rv ? sv[h] * p.scale_log2 : -INFINITY;
                v[h] = sv[h];
            }
            const float mx = warp_transpose_reduce<HH, true>(v);
            if (hl_writer) S.red_m[quarter][hl] = mx;
        }
        __syncthreads();
        if (tid < HQP) {   // one thread per head: the new running maximum and the rescale
            const float mt = fmaxf(fmaxf(S.red_m[0][tid], S.red_m[1][tid]), fmaxf(S.red_m[2][tid], S.red_m[3][tid]));
            const float mo = S.m_run[tid], mn = fmaxf(mo, mt);
            S.cf[tid] = (mn == -INFINITY) ? 1.f : exp2f(mo - mn);
            S.m_run[tid] = mn;
        }
        __syncthreads();
        {
            float pv[HH];
#pragma unroll
            for (int h = 0; h < HH; ++h) {
                const float mn = S.m_run[hh0 + h];
                pv[h] = (rv && mn != -INFINITY) ? exp2f(sv[h] - mn) : 0.f;
                *reinterpret_cast<__nv_bfloat16*>(S.pbuf + (rm >> 6) * (HQP * 128) + sw128(hh0 + h, (rm & 63) >> 3) +
                                                  (rm & 7) * 2) = __float2bfloat16_rn(pv[h]);
            }
            const float l = warp_transpose_reduce<HH, false>(pv);
            if (hl_writer) S.red_l[quarter][hl] = l;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();   // P and the tile sums are in place
        tc_fence_after();
        if (tslot) { CSA2_TRACE(tslot + 2); }   // softmax done

        // ---- O_tile^T = V^T P  (M = 128 = head dim (padded), N = HQP, K = 128 keys)
        if (tid == 0 && ok) {
            const uint32_t va = smem_u32((global_tile || HQP == 16) ? S.kbuf : S.vbuf), pa = smem_u32(S.pbuf);
            constexpr uint32_t idesc = idesc_bf16(128, HQP, 1);
#pragma unroll
            for (int kk = 0; kk < kTileKeys / 16; ++kk) {
                const uint64_t ad = smem_desc(va + kk * 2048, kPanelBytes, 1024);
                const uint64_t bd = smem_desc(pa + (kk >> 2) * (HQP * 128) + (kk & 3) * 32, 16, 1024);
                mma_bf16(tmem_o, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
            mma_commit(&S.bar_o);
        }
        if (tid < HQP)   // (the thread that owns head tid's running values)
            S.l_run[tid] = S.l_run[tid] * S.cf[tid] + (S.red_l[0][tid] + S.red_l[1][tid]) + (S.red_l[2][tid] + S.red_l[3][tid]);
        if (tau + 1 < p.ngt && part == 0 && s_next >= 0 && s_next < p.N) {   // the next tile's row towards L1
            const size_t row = (size_t)b * p.N + s_next;
            asm volatile("prefetch.global.L1 [%0];" ::"l"(p.kv_fp4 + row * (D / 2)));
            asm volatile("prefetch.global.L1 [%0];" ::"l"(p.kv_scale + row * (D / 16)));
        }
        ok = ok && mbar_wait(&S.bar_o, (uint32_t)(tau & 1), p.status, 14);
        tc_fence_after();
        if (tslot) { CSA2_TRACE(tslot + 3); }   // O done
        if (ok) {
            float tmp[HH];
            tmem_ld_cols<HH>(tmem_o + lane_off + hh0, tmp);
            tmem_ld_wait();
#pragma unroll
            for (int h = 0; h < HH; ++h) o[h] = o[h] * S.cf[hh0 + h] + tmp[h];
        }
        tc_fence_before();
        __syncthreads();   // every read of this tile's buffers, TMEM and sums is done
        if (tslot) { CSA2_TRACE(tslot + 4); }   // tile done
    }

    // ---- out = o / l (thread = head dimension, its part of the heads), lse in natural-log units
    {
        const int dim = quarter * 32 + lane;
        if (dim < D) {
#pragma unroll
            for (int h = 0; h < HH; ++h) {
                const int hg = hh0 + h;
                if (hg >= p.Hq) break;
                const float L = S.l_run[hg];
                p.out[((size_t)u * p.Hq + hg) * D + dim] =
                    __bfloat16_as_ushort(__float2bfloat16_rn((ok && L > 0.f) ? o[h] / L : 0.f));
            }
        }
    }
    if (tid < p.Hq && p.lse != nullptr) {
        const float mv = S.m_run[tid], lv = S.l_run[tid];
        p.lse[(size_t)u * p.Hq + tid] = (ok && lv > 0.f) ? (mv + log2f(lv)) * 0.69314718055994530942f : -INFINITY;
    }
    CSA2_TRACE(11);
    CSA2_TRACE_END(6);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(S.tmem_base, kCols);
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
    p.m = a.m;
    cudaError_t e;
    if (pl.HQP == 16 && a.D == 128) e = launch_attn_variant<16, 128>(p, pl.units, stream);
    else if (pl.HQP == 16 && a.D == 64) e = launch_attn_variant<16, 64>(p, pl.units, stream);
    else if (pl.HQP == 32 && a.D == 128) e = launch_attn_variant<32, 128>(p, pl.units, stream);
    else e = launch_attn_variant<32, 64>(p, pl.units, stream);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

size_t attn_scratch_bytes(const csa2_attn_args& a) { return plan_attn(a).part_bytes; }

template <int HQP, int D>
static cudaError_t launch_seq_variant(const AttnParams& p, int units, cudaStream_t stream) {
    constexpr int NT = seq_threads<HQP>();
    auto kern = sparse_attn_seq_kernel<HQP, D, NT>;
    const size_t smem = sizeof(AttnSeqSmem<HQP>) + 1024;
    cudaError_t e = set_smem_once(reinterpret_cast<const void*>(kern), (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(units);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    // the kernel reads no input before pdl_wait(): it may start while the previous kernel runs
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

// One CTA per query over all of its tiles (calls with many queries).
csa2_status launch_attn_seq(const csa2_attn_args& a, const int32_t* topk, int32_t* d_status, cudaStream_t stream) {
    AttnPlan pl = plan_attn(a);
    if (pl.units == 0) return CSA2_OK;
    AttnParams p{};
    p.B = a.B; p.Tq = a.Tq; p.N = a.N; p.Hq = a.Hq; p.D = a.D; p.k = a.k; p.W = a.W; p.Lloc = a.Lloc;
    p.ngt = pl.ngt; p.nlt = pl.nlt; p.ntiles = pl.ntiles;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)a.D));
    p.q_pos = a.q_pos; p.q = a.q; p.kv_fp4 = a.kv_fp4; p.kv_scale = a.kv_scale; p.topk = topk;
    p.kl = a.kl; p.vl = a.vl; p.local_base = a.local_base; p.out = a.out; p.lse = a.lse;
    p.status = d_status;
    p.m = a.m;
    cudaError_t e;
    if (pl.HQP == 16 && a.D == 128) e = launch_seq_variant<16, 128>(p, pl.units, stream);
    else if (pl.HQP == 16 && a.D == 64) e = launch_seq_variant<16, 64>(p, pl.units, stream);
    else if (pl.HQP == 32 && a.D == 128) e = launch_seq_variant<32, 128>(p, pl.units, stream);
    else e = launch_seq_variant<32, 64>(p, pl.units, stream);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

}  // namespace csa2

namespace csa2 {

typedef CUresult (*EncodeTiledFnA)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFnA encode_fn() {
    static EncodeTiledFnA fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFnA>(ptr);
    }
    return fn;
}

// [B, Lloc, D] bf16 local K or V as a 3-D map with 128-row x 64-element boxes,
// 128-byte swizzle (the tcgen05 operand layout).
static bool encode_local_map(CUtensorMap* m, const uint16_t* ptr, int B, int Lloc, int D) {
    EncodeTiledFnA enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Lloc, (cuuint64_t)B};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Lloc * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kTileKeys, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Dynamic shared memory of a clustered-attention CTA: at least 80 KB, so that at
// most two CTAs share an SM. Packing three per SM puts a call's clusters on fewer
// SMs, and the kernel is latency-bound: measured 22.5 us per launch against
// 15.3 us with two per SM.
template <int HQP>
constexpr size_t attn_cl_smem_bytes() {
    return sizeof(AttnClSmem<HQP>) + 1024 > 80 * 1024 ? sizeof(AttnClSmem<HQP>) + 1024 : 80 * 1024;
}

template <int HQP, int D>
static cudaError_t launch_cl_variant(const AttnParams& p, const CUtensorMap& km, const CUtensorMap& vm, int cs,
                                     int units, cudaStream_t stream) {
    auto kern = sparse_attn_cl_kernel<HQP, D>;
    const size_t smem = attn_cl_smem_bytes<HQP>();
    cudaError_t e = set_smem_once(reinterpret_cast<const void*>(kern), (int)smem);
    if (e != cudaSuccess) return e;
    if (cs > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(cs, units);
    cfg.blockDim = dim3(kClThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // the kernel reads no input before pdl_wait(), so it may start while the
    // previous kernel of the stream is still running
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, p, km, vm);
}

// Clustered attention: one cluster of ceil(k/256) + ceil(W/128) <= 16 CTAs per
// query; false when the call needs more CTAs than a cluster holds.
bool attn_cluster_fits(const csa2_attn_args& a) {
    const int cs = (a.k + 2 * kTileKeys - 1) / (2 * kTileKeys) + (a.W + kTileKeys - 1) / kTileKeys;
    return cs >= 1 && cs <= 16 && (int64_t)a.B * a.Tq <= 65535;
}

csa2_status launch_attn_cluster(const csa2_attn_args& a, const int32_t* topk, int list_ready, int32_t* d_status,
                                cudaStream_t stream) {
    const int units = a.B * a.Tq;
    if (units == 0) return CSA2_OK;
    AttnParams p{};
    p.B = a.B; p.Tq = a.Tq; p.N = a.N; p.Hq = a.Hq; p.D = a.D; p.k = a.k; p.W = a.W; p.Lloc = a.Lloc;
    const int ngt2 = (a.k + 2 * kTileKeys - 1) / (2 * kTileKeys);
    p.nlt = (a.W + kTileKeys - 1) / kTileKeys;
    p.ngt = ngt2;
    p.ntiles = ngt2 + p.nlt;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)a.D));
    p.q_pos = a.q_pos; p.q = a.q; p.kv_fp4 = a.kv_fp4; p.kv_scale = a.kv_scale; p.topk = topk;
    p.kl = a.kl; p.vl = a.vl; p.local_base = a.local_base; p.out = a.out; p.lse = a.lse;
    p.part = nullptr;
    p.tickets = nullptr;
    p.status = d_status;
    p.list_ready = list_ready;
    p.m = a.m;
    CUtensorMap km, vm;
    memset(&km, 0, sizeof(km));
    memset(&vm, 0, sizeof(vm));
    if (a.W > 0) {
        if (!encode_local_map(&km, a.kl, a.B, a.Lloc, a.D) || !encode_local_map(&vm, a.vl, a.B, a.Lloc, a.D))
            return CSA2_ERR_CUDA;
    }
    const int HQP = a.Hq <= 16 ? 16 : 32;
    const int cs = p.ntiles;
    cudaError_t e;
    if (HQP == 16 && a.D == 128) e = launch_cl_variant<16, 128>(p, km, vm, cs, units, stream);
    else if (HQP == 16 && a.D == 64) e = launch_cl_variant<16, 64>(p, km, vm, cs, units, stream);
    else if (HQP == 32 && a.D == 128) e = launch_cl_variant<32, 128>(p, km, vm, cs, units, stream);
    else e = launch_cl_variant<32, 64>(p, km, vm, cs, units, stream);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}


}  // namespace csa2

CSA2_TRACE_SETTER(csa2_trace_set_attn)
