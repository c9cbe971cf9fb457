// Plain CPU oracle for CSA2 sparse attention over a shared FP4 global KV cache,
// in C++17: exact int64 index scores, a full sort for the selection, fp64
// attention with one softmax over the union of the selected global rows and the
// local window. Threads (std::thread) run independent (sequence, query) units.
//
// TEST INFRASTRUCTURE. Only the tests, __graft_entry__.smoke() and bench.py's
// CPU-baseline and reference legs may load or run this library. It shares no
// code with the CUDA path: its own format tables, its own selection, its own
// softmax. It is written to be read against the pages, not to be fast.
//
// Sources (page titles; sections and figures named on each page):
//   [CED] "CED: Continuing Context with a Causal Encoder and Decoder":
//         "One Token Sequence and Causal Access" (Fig. 2): a query at position t
//           reads positions 0..t;
//         "Selecting Positions and Reading Values with Attention" (Fig. 4): the
//           indexer returns positions; their global entries are fetched and
//           concatenated with the layer's local KV; Main Q attends over the
//           concatenation; a position in both sets is read twice;
//         "What Full, Reindex, and Reuse Share" (Fig. 5): Full scores every
//           position and keeps a pool wider than top-k, Reindex rescores the
//           pool, Reuse takes the previous list.
//   [KVC] "DeepSeek-V4.1 Flash Pushes KV Cache Compression for Agent
//         Workloads", section "Ana Gelisme": FP4 E2M1 values, one E4M3 scale per
//         16 channels.
//   [OCP] OCP Microscaling Formats (MX) v1.0: the E2M1 and E4M3 definitions.
// Readings where the pages are silent (score formula, tie rule, rounding):
//   score(s) = sum_h w[h] * max(0, sum_d qi[h][d] * k[s][d]);  ranking by score
//   descending, then position ascending; lists ascending, padded with -1;
//   FP4 scale = E4M3 nearest amax/6 (ties to even, saturating at 448), code =
//   E2M1 nearest x/scale (ties to even, saturating at +-6), -0 never emitted.
// Parity status: every function is pinned in tests/test_oracle_cpp.py; the score
// formula itself is a reading, unpinned against a trained model.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <utility>
#include <vector>

namespace {

// ------------------------------------------------------------ formats [OCP]
// E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 is
// subnormal (0.5 * mantissa). No infinity or NaN.
double e2m1_value(int code) {
    const double sign = (code & 8) ? -1.0 : 1.0;
    const int e = (code >> 1) & 3, m = code & 1;
    const double mag = (e == 0) ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
    return sign * mag;
}

// E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is
// subnormal (2^-6 * m / 8); exponent 15 with mantissa 7 is NaN; no infinity.
double e4m3_value(int byte) {
    const double sign = (byte & 0x80) ? -1.0 : 1.0;
    const int e = (byte >> 3) & 15, m = byte & 7;
    if (e == 15 && m == 7) return std::numeric_limits<double>::quiet_NaN();
    const double mag = (e == 0) ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
    return sign * mag;
}

// Code of the non-negative value nearest to x >= 0 among codes 0..ncodes-1
// (whose values ascend with the code); a tie goes to the even code; values at or
// above the largest saturate to it.
int round_nearest_even(double x, double (*value)(int), int ncodes) {
    const double top = value(ncodes - 1);
    if (x >= top) return ncodes - 1;
    int hi = 0;
    while (value(hi) < x) ++hi;           // first code whose value is >= x
    if (hi == 0) return 0;
    const int lo = hi - 1;
    const double d_lo = x - value(lo), d_hi = value(hi) - x;
    if (d_hi < d_lo) return hi;
    if (d_lo < d_hi) return lo;
    return (hi % 2 == 0) ? hi : lo;
}

int e4m3_round(double x) { return round_nearest_even(x, e4m3_value, 127); }   // 0x00..0x7E: 0..448

int e2m1_round(double x) {
    const int mag = round_nearest_even(std::fabs(x), e2m1_value, 8);          // 0..6
    return (x < 0 && mag != 0) ? (mag | 8) : mag;
}

double bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return (double)f;
}

// ------------------------------------------------------------ indexer [CED] Fig. 4, Fig. 5
int64_t index_score(const int8_t* qi, const int32_t* w, int Hi, int Di, const int8_t* key) {
    int64_t score = 0;
    for (int h = 0; h < Hi; ++h) {
        int64_t dot = 0;
        for (int d = 0; d < Di; ++d) dot += (int64_t)qi[h * Di + d] * (int64_t)key[d];
        score += (int64_t)w[h] * std::max<int64_t>(dot, 0);
    }
    return score;
}

// The `count` candidates ranked first by (score descending, position ascending),
// written in ascending position order to out[0..len), padded with -1.
void select_best(std::vector<std::pair<int64_t, int32_t>> cand, int count, int32_t* out, int len) {
    std::sort(cand.begin(), cand.end(), [](const std::pair<int64_t, int32_t>& a, const std::pair<int64_t, int32_t>& b) {
        if (a.first != b.first) return a.first > b.first;
        return a.second < b.second;
    });
    const int n = std::min<int>(count, (int)cand.size());
    std::vector<int32_t> pos(n);
    for (int i = 0; i < n; ++i) pos[i] = cand[i].second;
    std::sort(pos.begin(), pos.end());
    for (int i = 0; i < len; ++i) out[i] = i < n ? pos[i] : -1;
}

// Runs fn(i) for i in [0, n) on up to `threads` std::threads.
template <class Fn>
void parallel_for(int64_t n, int threads, Fn fn) {
    if (threads <= 1 || n <= 1) {
        for (int64_t i = 0; i < n; ++i) fn(i);
        return;
    }
    std::atomic<int64_t> next{0};
    std::vector<std::thread> pool;
    const int nt = (int)std::min<int64_t>(threads, n);
    for (int k = 0; k < nt; ++k)
        pool.emplace_back([&]() {
            for (int64_t i = next++; i < n; i = next++) fn(i);
        });
    for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

double orc_e2m1_value(int code) { return e2m1_value(code); }
double orc_e4m3_value(int byte) { return e4m3_value(byte); }
int orc_e2m1_round(double x) { return e2m1_round(x); }
int orc_e4m3_round(double x) { return e4m3_round(x); }

// FP4 quantisation [KVC]: x [rows][D] fp32 -> codes [rows][D/2] (element 2j in the
// low nibble), scales [rows][D/16] (E4M3 bits). The quotient x/scale is formed in
// fp64; an fp32 numerator over a scale of at most 4 significant bits lands on a
// rounding boundary of E2M1 only when the exact quotient does.
void orc_fp4_quantize(const float* x, int64_t rows, int D, uint8_t* codes, uint8_t* scales, int threads) {
    parallel_for(rows, threads, [&](int64_t r) {
        for (int g = 0; g < D / 16; ++g) {
            const float* v = x + r * D + g * 16;
            double amax = 0.0;
            for (int i = 0; i < 16; ++i) amax = std::max(amax, std::fabs((double)v[i]));
            const int sc = e4m3_round(amax / 6.0);
            const double s = e4m3_value(sc);
            scales[r * (D / 16) + g] = (uint8_t)sc;
            for (int i = 0; i < 16; i += 2) {
                const int c0 = s > 0 ? e2m1_round((double)v[i] / s) : 0;
                const int c1 = s > 0 ? e2m1_round((double)v[i + 1] / s) : 0;
                codes[r * (D / 2) + (g * 16 + i) / 2] = (uint8_t)(c0 | (c1 << 4));
            }
        }
    });
}

// Global entries of sequence compression rate m ([CED] "What Does the Sequence
// Compression Rate Reduce?": at m = 2 two positions become one entry). The pages
// give no combining rule; this reading takes the mean: entry g of x [groups*m][D]
// is (x[g*m] + ... + x[g*m + m - 1]) summed left to right in fp32, times 1/m.
void orc_compress_entries(const float* x, int64_t groups, int m, int D, float* out) {
    for (int64_t g = 0; g < groups; ++g)
        for (int d = 0; d < D; ++d) {
            float acc = x[(g * m) * D + d];
            for (int r = 1; r < m; ++r) acc = acc + x[(g * m + r) * D + d];
            out[g * D + d] = acc * (1.0f / (float)m);
        }
}

// The last global entry a query at position t may read: entries are positions at
// m <= 1; at m >= 2 entry j covers positions m*j .. m*j + m - 1 and is read once
// the whole group is causal.
int orc_last_entry(int t, int m) { return m <= 1 ? t : (t + 1) / m - 1; }

// Value of element d of an FP4 row: e2m1(code) * e4m3(scale of its 16-group).
double orc_fp4_value(const uint8_t* codes_row, const uint8_t* scales_row, int d) {
    const int byte = codes_row[d / 2];
    const int code = (d % 2 == 0) ? (byte & 15) : (byte >> 4);
    return e2m1_value(code) * e4m3_value(scales_row[d / 16]);
}

// Full mode for one query at position t: score every s in [0, min(t, N-1)]; write
// the top-P pool (P > 0) and the top-k list.
void orc_index_full(const int8_t* qi, const int32_t* w, int Hi, int Di, const int8_t* keys, int N, int t, int k, int P,
                    int32_t* pool_out, int32_t* topk_out) {
    std::vector<std::pair<int64_t, int32_t>> cand;
    const int last = std::min(t, N - 1);
    for (int s = 0; s <= last; ++s) cand.emplace_back(index_score(qi, w, Hi, Di, keys + (int64_t)s * Di), s);
    if (P > 0 && pool_out) select_best(cand, P, pool_out, P);
    select_best(cand, k, topk_out, k);
}

// Reindex mode: rescore only the pool's valid entries with this layer's indexer.
void orc_index_reindex(const int8_t* qi, const int32_t* w, int Hi, int Di, const int8_t* keys, const int32_t* pool,
                       int P_in, int k, int32_t* topk_out) {
    std::vector<std::pair<int64_t, int32_t>> cand;
    for (int i = 0; i < P_in; ++i)
        if (pool[i] >= 0) cand.emplace_back(index_score(qi, w, Hi, Di, keys + (int64_t)pool[i] * Di), pool[i]);
    select_best(cand, k, topk_out, k);
}

// Attention of one query (all heads), [CED] Fig. 4: the union of the listed global
// rows (dequantised FP4; each row is both key and value) and the local rows at
// positions [max(local_base, t-W+1, 0), t] (their own K and V); one softmax per
// head over the union with logits q.key / sqrt(D), in fp64. With no entries the
// output is 0 and the log-sum-exp -inf.
void orc_attention_unit(const uint16_t* q, int Hq, int D, const uint8_t* codes_seq, const uint8_t* scales_seq,
                        const int32_t* topk, int k, const uint16_t* kl_seq, const uint16_t* vl_seq, int local_base,
                        int t, int W, double* out, double* lse) {
    std::vector<std::vector<double>> keys, vals;
    for (int i = 0; i < k; ++i) {
        const int s = topk[i];
        if (s < 0) continue;
        std::vector<double> g(D);
        for (int d = 0; d < D; ++d)
            g[d] = orc_fp4_value(codes_seq + (int64_t)s * (D / 2), scales_seq + (int64_t)s * (D / 16), d);
        keys.push_back(g);
        vals.push_back(g);
    }
    if (W > 0) {
        const int lo = std::max(std::max(local_base, t - W + 1), 0);
        for (int p = lo; p <= t; ++p) {
            const int64_t r = p - local_base;
            std::vector<double> kk(D), vv(D);
            for (int d = 0; d < D; ++d) {
                kk[d] = bf16_value(kl_seq[r * D + d]);
                vv[d] = bf16_value(vl_seq[r * D + d]);
            }
            keys.push_back(kk);
            vals.push_back(vv);
        }
    }
    const double scale = 1.0 / std::sqrt((double)D);
    const size_t n = keys.size();
    for (int h = 0; h < Hq; ++h) {
        double* o = out + (int64_t)h * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (n == 0) {
            lse[h] = -std::numeric_limits<double>::infinity();
            continue;
        }
        std::vector<double> logit(n);
        double m = -std::numeric_limits<double>::infinity();
        for (size_t j = 0; j < n; ++j) {
            double dot = 0.0;
            for (int d = 0; d < D; ++d) dot += bf16_value(q[h * D + d]) * keys[j][d];
            logit[j] = dot * scale;
            m = std::max(m, logit[j]);
        }
        double l = 0.0;
        for (size_t j = 0; j < n; ++j) {
            const double p = std::exp(logit[j] - m);
            l += p;
            for (int d = 0; d < D; ++d) o[d] += p * vals[j][d];
        }
        for (int d = 0; d < D; ++d) o[d] /= l;
        lse[h] = m + std::log(l);
    }
}

// ------------------------------------------------------------ batched, threaded over units
// Unit u = b * Tq + j is query j of sequence b at position q_pos[u].

void orc_index_full_batch(int B, int Tq, int N, int Hi, int Di, const int32_t* q_pos, const int8_t* qi,
                          const int32_t* w, const int8_t* ki, int64_t ki_seq_stride, int k, int P, int32_t* pool_out,
                          int32_t* topk_out, int threads) {
    parallel_for((int64_t)B * Tq, threads, [&](int64_t u) {
        const int64_t b = u / Tq;
        orc_index_full(qi + u * Hi * Di, w, Hi, Di, ki + b * ki_seq_stride, N, q_pos[u], k, P,
                       P > 0 && pool_out ? pool_out + u * P : nullptr, topk_out + u * k);
    });
}

void orc_index_reindex_batch(int B, int Tq, int Hi, int Di, const int8_t* qi, const int32_t* w, const int8_t* ki,
                             int64_t ki_seq_stride, const int32_t* pool, int P_in, int k, int32_t* topk_out,
                             int threads) {
    parallel_for((int64_t)B * Tq, threads, [&](int64_t u) {
        const int64_t b = u / Tq;
        orc_index_reindex(qi + u * Hi * Di, w, Hi, Di, ki + b * ki_seq_stride, pool + u * P_in, P_in, k,
                          topk_out + u * k);
    });
}

// q [B*Tq][Hq][D] bf16; codes [B][N][D/2], scales [B][N][D/16]; topk [B*Tq][k];
// kl, vl [B][Lloc][D] bf16; local_base [B]; out [B*Tq][Hq][D], lse [B*Tq][Hq] fp64.
void orc_attention_batch(int B, int Tq, int N, int Hq, int D, const int32_t* q_pos, const uint16_t* q,
                         const uint8_t* codes, const uint8_t* scales, const int32_t* topk, int k, const uint16_t* kl,
                         const uint16_t* vl, int Lloc, const int32_t* local_base, int W, double* out, double* lse,
                         int threads) {
    parallel_for((int64_t)B * Tq, threads, [&](int64_t u) {
        const int64_t b = u / Tq;
        orc_attention_unit(q + u * Hq * D, Hq, D, codes + b * (int64_t)N * (D / 2), scales + b * (int64_t)N * (D / 16),
                           topk + u * k, k, kl ? kl + b * (int64_t)Lloc * D : nullptr,
                           vl ? vl + b * (int64_t)Lloc * D : nullptr, local_base ? local_base[b] : 0, q_pos[u], W,
                           out + u * Hq * D, lse + u * Hq);
    });
}

}  // extern "C"
