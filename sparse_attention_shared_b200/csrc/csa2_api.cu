// Host side of the C ABI declared in include/csa2.h: argument validation, the
// workspace layout and the per-layer launch sequence of the decoder stack
// ("CED: Continuing Context with a Causal Encoder and Decoder", "What Full,
// Reindex, and Reuse Share", Fig. 5: modes are fixed per layer; Reuse takes the
// list of the most recent Full or Reindex layer; Reindex rescores the pool of
// the Full layer before it).
//
// Workspace layout (bytes, every region 256-byte aligned):
//   [0, R)            indexer slots: per-SM barrier counters, epochs, histogram
//                     and candidate buffers. Persistent between calls.
//   [R, R + T)        attention merge tickets, one int per query (T fixed: room for
//                     65535 queries, the most a call accepts). Zero at rest.
//   [R + T, end)      scratch: attention partials or spilled indexer scores,
//                     rewritten by every call.
// The whole workspace must be zero-filled before its first use. Every call
// that completes without a device-reported error leaves it consistent for the
// next call; after a reported error, zero it again.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "csa2_common.cuh"

namespace csa2 {
// indexer.cu
int num_sms();
size_t index_region_bytes();
size_t index_scratch_bytes(const csa2_index_args& a, int P_in);
size_t index_smem_bytes();
csa2_status launch_index(const csa2_index_args& a, const int32_t* pool_in, int P_in, void* region, void* scratch,
                         int32_t* d_status, cudaStream_t stream, const csa2_attn_args* pf, int keys_ready);
// attention.cu
size_t attn_scratch_bytes(const csa2_attn_args& a);
csa2_status launch_attn(const csa2_attn_args& a, const int32_t* topk, int* tickets, void* scratch,
                        int32_t* d_status, cudaStream_t stream);
bool attn_cluster_fits(const csa2_attn_args& a);
csa2_status launch_attn_seq(const csa2_attn_args& a, const int32_t* topk, int32_t* d_status, cudaStream_t stream);
csa2_status launch_attn_cluster(const csa2_attn_args& a, const int32_t* topk, int list_ready, int32_t* d_status,
                                cudaStream_t stream);

// The attention kernel for a call: with many queries, one CTA per query over all of its
// tiles; else the cluster kernel (one CTA per 256 list entries or 128 window rows, the
// partials merged through distributed shared memory) while the call is latency-bound,
// else one CTA per 128-row tile with a ticket merge. Measured on one
// B200 at 16 heads: the cluster kernel wins while the call's clusters hold at most about
// four CTAs per SM (decode: 16-32 queries x 12 CTAs), the ticket kernel beyond (64 queries
// x 16 CTAs: 57 against 61 us; 2048 queries x 12 CTAs: 0.83 against 0.98 ms). At 32 heads
// (a prefill chunk of 4096 queries) the two are within 2%; the cluster kernel stays.
static csa2_status run_attn(const csa2_attn_args& a, const int32_t* topk, int list_ready, int* tickets,
                            void* scratch, int32_t* d_status, cudaStream_t stream) {
    // at least two queries per SM: one CTA per query over all of its tiles (a prefill chunk
    // of 4096 queries: 1.63 ms against 2.86 ms for the cluster kernel)
    if ((int64_t)a.B * a.Tq >= 2LL * num_sms()) return launch_attn_seq(a, topk, d_status, stream);
    const int cs = (a.k + 255) / 256 + (a.W + 127) / 128;
    const bool many = a.Hq <= 16 && (int64_t)a.B * a.Tq * cs > 4LL * num_sms();
    if (attn_cluster_fits(a) && !many) return launch_attn_cluster(a, topk, list_ready, d_status, stream);
    return launch_attn(a, topk, tickets, scratch, d_status, stream);
}
void set_wait_controls(long long budget, int skip);
// cache_append.cu
csa2_status launch_cache_append(const csa2_append_args& a, int32_t* d_status, cudaStream_t stream);
int append_max_sets();
int append_max_layers();
// fp4_quant.cu
cudaError_t launch_fp4_quantize(const float* x, int64_t rows, int D, uint8_t* codes, uint8_t* scales,
                                cudaStream_t stream);
cudaError_t launch_fp4_compress(const float* x, int64_t groups, int m, int D, uint8_t* codes, uint8_t* scales,
                                cudaStream_t stream);

static size_t a256(size_t x) { return (x + 255) / 256 * 256; }
static bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static csa2_status check_index(const csa2_index_args* a, bool in_stack) {
    if (!a) return CSA2_ERR_NULL;
    if (a->mode != CSA2_FULL && a->mode != CSA2_REINDEX) return CSA2_ERR_MODE;
    if (a->B < 1 || a->Tq < 1 || a->N < 1 || a->N >= (1 << 27)) return CSA2_ERR_SHAPE;
    if ((int64_t)a->B * a->Tq > (1 << 26)) return CSA2_ERR_SHAPE;
    if (a->Hi < 1 || a->Hi > 16 || a->Di < 16 || a->Di > 128 || a->Di % 16) return CSA2_ERR_SHAPE;
    if (a->m < 0 || a->m > 8) return CSA2_ERR_SHAPE;
    if (a->k < 1 || a->P < 0) return CSA2_ERR_SHAPE;
    if (a->mode == CSA2_FULL && a->P > 0 && a->k > a->P) return CSA2_ERR_SHAPE;
    if (!a->q_pos || !a->qi || !a->w || !a->ki || !a->topk_out) return CSA2_ERR_NULL;
    if (a->mode == CSA2_FULL && a->P > 0 && !a->pool_out) return CSA2_ERR_NULL;
    if (a->mode == CSA2_REINDEX && !in_stack) {
        if (!a->pool_in) return CSA2_ERR_NULL;
        if (a->P_in < 1) return CSA2_ERR_SHAPE;
    }
    if (a->ki_seq_stride < (int64_t)a->N * a->Di || a->ki_seq_stride % 16) return CSA2_ERR_ALIGN;
    if (!al16(a->q_pos) || !al16(a->qi) || !al16(a->ki) || !al16(a->topk_out)) return CSA2_ERR_ALIGN;
    if (a->pool_out && !al16(a->pool_out)) return CSA2_ERR_ALIGN;
    if (a->mode == CSA2_REINDEX && !in_stack && !al16(a->pool_in)) return CSA2_ERR_ALIGN;
    int64_t wmax = 0;
    for (int h = 0; h < a->Hi; ++h) wmax = std::max<int64_t>(wmax, std::llabs((long long)a->w[h]));
    if ((int64_t)a->Hi * wmax * a->Di * 16384 >= ((int64_t)1 << 31)) return CSA2_ERR_RANGE;
    return CSA2_OK;
}

static csa2_status check_attn(const csa2_attn_args* a, bool in_stack) {
    if (!a) return CSA2_ERR_NULL;
    if (a->B < 1 || a->Tq < 1 || a->N < 1 || a->N >= (1 << 27)) return CSA2_ERR_SHAPE;
    if ((int64_t)a->B * a->Tq > 65535) return CSA2_ERR_UNSUPPORTED;
    if (a->Hq < 1 || a->Hq > 32) return CSA2_ERR_UNSUPPORTED;
    if (a->D != 64 && a->D != 128) return CSA2_ERR_UNSUPPORTED;
    if (a->m < 0 || a->m > 8) return CSA2_ERR_SHAPE;
    if ((!in_stack && a->k < 1) || a->W < 0 || a->Lloc < 0) return CSA2_ERR_SHAPE;
    if ((int64_t)a->k + a->W > 16384) return CSA2_ERR_UNSUPPORTED;   // the merge keeps <= 128 tile weights
    if (!a->q_pos || !a->q || !a->kv_fp4 || !a->kv_scale || !a->out) return CSA2_ERR_NULL;
    if (!in_stack && !a->topk) return CSA2_ERR_NULL;
    if (a->W > 0 && (!a->kl || !a->vl || !a->local_base || a->Lloc < 1)) return CSA2_ERR_NULL;
    if (!al16(a->q_pos) || !al16(a->q) || !al16(a->kv_fp4) || !al16(a->kv_scale) || !al16(a->out))
        return CSA2_ERR_ALIGN;
    if (!in_stack && !al16(a->topk)) return CSA2_ERR_ALIGN;
    if (a->W > 0 && (!al16(a->kl) || !al16(a->vl) || !al16(a->local_base))) return CSA2_ERR_ALIGN;
    if (a->lse && !al16(a->lse)) return CSA2_ERR_ALIGN;
    return CSA2_OK;
}

// The ticket region has one size for every call (room for the most queries a call may
// have), so that no call's scratch ever lies where another call keeps its tickets: a
// workspace shared by calls of different sizes stays zero there between calls.
static size_t tickets_bytes(int /*units*/) { return a256((size_t)65535 * 4); }

static void* ws_at(void* ws, size_t off) { return static_cast<uint8_t*>(ws) + off; }

static csa2_status check_stack(const csa2_stack_args* s) {
    if (!s || !s->idx || !s->attn) return CSA2_ERR_NULL;
    if (s->L < 1) return CSA2_ERR_SHAPE;
    bool have_list = false, have_pool = false;
    const csa2_attn_args& a0 = s->attn[0];
    for (int l = 0; l < s->L; ++l) {
        const csa2_index_args& ix = s->idx[l];
        const csa2_attn_args& at = s->attn[l];
        if (ix.mode == CSA2_REUSE) {
            if (!have_list) return CSA2_ERR_MODE;
        } else {
            if (ix.mode == CSA2_REINDEX && !have_pool) return CSA2_ERR_MODE;
            csa2_status st = check_index(&ix, true);
            if (st != CSA2_OK) return st;
            if (ix.B != a0.B || ix.Tq != a0.Tq || ix.N != a0.N || ix.m != a0.m) return CSA2_ERR_SHAPE;
            have_list = true;
            if (ix.mode == CSA2_FULL && ix.P > 0) have_pool = true;
        }
        csa2_status st = check_attn(&at, true);
        if (st != CSA2_OK) return st;
        if (at.B != a0.B || at.Tq != a0.Tq || at.N != a0.N) return CSA2_ERR_SHAPE;
    }
    return CSA2_OK;
}

}  // namespace csa2

using namespace csa2;

extern "C" {

const char* csa2_status_string(csa2_status s) {
    switch (s) {
        case CSA2_OK: return "ok";
        case CSA2_ERR_NULL: return "a required pointer is NULL";
        case CSA2_ERR_SHAPE: return "a size is out of its allowed range";
        case CSA2_ERR_ALIGN: return "a pointer or stride is not 16-byte aligned";
        case CSA2_ERR_MODE: return "bad layer mode or mode order";
        case CSA2_ERR_RANGE: return "an index or position is outside its range";
        case CSA2_ERR_UNSUPPORTED: return "no kernel for these sizes";
        case CSA2_ERR_CUDA: return "a CUDA runtime call failed";
        case CSA2_ERR_TIMEOUT: return "a bounded device wait ran out";
        case CSA2_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

size_t csa2_workspace_bytes(int which, const void* args) {
    if (!args) return 0;
    const size_t R = index_region_bytes();
    if (which == 0) {
        const csa2_index_args* a = static_cast<const csa2_index_args*>(args);
        if (check_index(a, false) != CSA2_OK) return 0;
        return R + tickets_bytes(a->B * a->Tq) + index_scratch_bytes(*a, a->mode == CSA2_REINDEX ? a->P_in : 0);
    }
    if (which == 1) {
        const csa2_attn_args* a = static_cast<const csa2_attn_args*>(args);
        if (check_attn(a, false) != CSA2_OK) return 0;
        return R + tickets_bytes(a->B * a->Tq) + attn_scratch_bytes(*a);
    }
    if (which == 2) {
        const csa2_stack_args* s = static_cast<const csa2_stack_args*>(args);
        if (check_stack(s) != CSA2_OK) return 0;
        size_t scratch = 0;
        int cur_k = 0, pool_P = 0;
        for (int l = 0; l < s->L; ++l) {
            const csa2_index_args& ix = s->idx[l];
            if (ix.mode == CSA2_FULL) {
                scratch = std::max(scratch, index_scratch_bytes(ix, 0));
                cur_k = ix.k;
                if (ix.P > 0) pool_P = ix.P;
            } else if (ix.mode == CSA2_REINDEX) {
                scratch = std::max(scratch, index_scratch_bytes(ix, pool_P));
                cur_k = ix.k;
            }
            csa2_attn_args at = s->attn[l];
            at.k = cur_k;
            scratch = std::max(scratch, attn_scratch_bytes(at));
        }
        return R + tickets_bytes(s->attn[0].B * s->attn[0].Tq) + scratch;
    }
    return 0;
}

csa2_status csa2_index_topk(const csa2_index_args* args, void* workspace, size_t ws_bytes, int32_t* d_status,
                            void* stream) {
    csa2_status st = check_index(args, false);
    if (st != CSA2_OK) return st;
    const size_t need = csa2_workspace_bytes(0, args);
    if (!workspace || ws_bytes < need || !al16(workspace)) return CSA2_ERR_WORKSPACE;
    const size_t R = index_region_bytes();
    void* scratch = ws_at(workspace, R + tickets_bytes(args->B * args->Tq));
    const int P_in = args->mode == CSA2_REINDEX ? args->P_in : 0;
    return launch_index(*args, args->pool_in, P_in, workspace, scratch, d_status, static_cast<cudaStream_t>(stream),
                        nullptr, 0);
}

csa2_status csa2_sparse_attn(const csa2_attn_args* args, void* workspace, size_t ws_bytes, int32_t* d_status,
                             void* stream) {
    csa2_status st = check_attn(args, false);
    if (st != CSA2_OK) return st;
    const size_t need = csa2_workspace_bytes(1, args);
    if (!workspace || ws_bytes < need || !al16(workspace)) return CSA2_ERR_WORKSPACE;
    const size_t R = index_region_bytes();
    int* tickets = static_cast<int*>(ws_at(workspace, R));
    void* scratch = ws_at(workspace, R + tickets_bytes(args->B * args->Tq));
    csa2_attn_args a = *args;
    if (a.W == 0) {
        // no local branch: the kernel still reads local_base; point it at the
        // (always >= 1 entry) query-position array, whose values are unused then
        a.local_base = a.q_pos;
        a.Lloc = 0;
    }
    return run_attn(a, a.topk, 0, tickets, scratch, d_status, static_cast<cudaStream_t>(stream));
}

csa2_status csa2_layer_stack(const csa2_stack_args* s, void* workspace, size_t ws_bytes, int32_t* d_status,
                             void* stream) {
    csa2_status st = check_stack(s);
    if (st != CSA2_OK) return st;
    const size_t need = csa2_workspace_bytes(2, s);
    if (!workspace || ws_bytes < need || !al16(workspace)) return CSA2_ERR_WORKSPACE;
    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    const size_t R = index_region_bytes();
    const int units = s->attn[0].B * s->attn[0].Tq;
    int* tickets = static_cast<int*>(ws_at(workspace, R));
    void* scratch = ws_at(workspace, R + tickets_bytes(units));

    const int32_t* cur = nullptr;   // the current layer's list
    int cur_k = 0;
    const int32_t* pool = nullptr;  // the most recent Full layer's pool
    int pool_P = 0;
    for (int l = 0; l < s->L; ++l) {
        const csa2_index_args& ix = s->idx[l];
        bool copied = false;   // a list copy was issued for this layer
        // Past the first layer the kernel before an indexer is the previous layer's
        // attention, which writes no key, position or pool: those were complete when it began.
        const int keys_ready = l > 0 ? 1 : 0;
        if (ix.mode == CSA2_FULL) {
            st = launch_index(ix, nullptr, 0, workspace, scratch, d_status, strm, &s->attn[l], keys_ready);
            if (st != CSA2_OK) return st;
            cur = ix.topk_out;
            cur_k = ix.k;
            if (ix.P > 0) {
                pool = ix.pool_out;
                pool_P = ix.P;
            }
        } else if (ix.mode == CSA2_REINDEX) {
            st = launch_index(ix, pool, pool_P, workspace, scratch, d_status, strm, &s->attn[l], keys_ready);
            if (st != CSA2_OK) return st;
            cur = ix.topk_out;
            cur_k = ix.k;
        } else if (ix.topk_out && ix.topk_out != cur) {
            const size_t bytes = (size_t)units * cur_k * sizeof(int32_t);
            if (cudaMemcpyAsync(ix.topk_out, cur, bytes, cudaMemcpyDeviceToDevice, strm) != cudaSuccess)
                return CSA2_ERR_CUDA;
            copied = true;
        }
        csa2_attn_args a = s->attn[l];
        a.k = cur_k;
        a.topk = cur;
        if (a.W == 0) {
            a.local_base = a.q_pos;
            a.Lloc = 0;
        }
        // A Reuse layer's list was written two or more kernels earlier (the previous
        // kernel is the previous layer's attention), so its clusters may gather their
        // global rows before waiting for that kernel; not when a copy came between.
        const int list_ready = (ix.mode == CSA2_REUSE && !copied) ? 1 : 0;
        st = run_attn(a, cur, list_ready, tickets, scratch, d_status, strm);
        if (st != CSA2_OK) return st;
    }
    return CSA2_OK;
}

csa2_status csa2_fp4_compress(const float* x, int64_t groups, int32_t m, int32_t D, uint8_t* fp4, uint8_t* scale,
                              void* stream) {
    if (!x || !fp4 || !scale) return CSA2_ERR_NULL;
    if (groups < 0 || D < 16 || D % 16 || (m != 1 && m != 2 && m != 4 && m != 8)) return CSA2_ERR_SHAPE;
    if (!al16(x) || !al16(fp4) || !al16(scale)) return CSA2_ERR_ALIGN;
    return launch_fp4_compress(x, groups, m, D, fp4, scale, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? CSA2_OK
               : CSA2_ERR_CUDA;
}

csa2_status csa2_cache_append(const csa2_append_args* a, int32_t* d_status, void* stream) {
    if (!a) return CSA2_ERR_NULL;
    if (a->B < 1 || a->N < 1 || a->N >= (1 << 27) || a->D < 16 || a->D % 16) return CSA2_ERR_SHAPE;
    if (a->S < 0 || a->S > append_max_sets() || a->L < 0 || a->L > append_max_layers()) return CSA2_ERR_SHAPE;
    if (a->S > 0 && (a->Di < 16 || a->Di > 128 || a->Di % 16)) return CSA2_ERR_SHAPE;
    if (a->L > 0 && (a->W < 1 || a->Lcap < std::max(1, 2 * a->W - 1))) return CSA2_ERR_SHAPE;
    if (!a->pos || !a->kv_new || !a->kv_fp4 || !a->kv_scale) return CSA2_ERR_NULL;
    if (!al16(a->pos) || !al16(a->kv_new) || !al16(a->kv_fp4) || !al16(a->kv_scale)) return CSA2_ERR_ALIGN;
    if (a->S > 0) {
        if (!a->ki_new || !a->ki) return CSA2_ERR_NULL;
        if (!al16(a->ki_new)) return CSA2_ERR_ALIGN;
        for (int s = 0; s < a->S; ++s) {
            if (!a->ki[s]) return CSA2_ERR_NULL;
            if (!al16(a->ki[s])) return CSA2_ERR_ALIGN;
        }
    }
    if (a->L > 0) {
        if (!a->kl_new || !a->vl_new || !a->kl || !a->vl || !a->local_base) return CSA2_ERR_NULL;
        if (!al16(a->kl_new) || !al16(a->vl_new) || !al16(a->local_base)) return CSA2_ERR_ALIGN;
        for (int l = 0; l < a->L; ++l) {
            if (!a->kl[l] || !a->vl[l]) return CSA2_ERR_NULL;
            if (!al16(a->kl[l]) || !al16(a->vl[l])) return CSA2_ERR_ALIGN;
        }
    }
    return launch_cache_append(*a, d_status, static_cast<cudaStream_t>(stream));
}

csa2_status csa2_set_wait_controls(int64_t budget_cycles, int32_t skip_arrival) {
    if (budget_cycles < 0) return CSA2_ERR_SHAPE;
    set_wait_controls((long long)budget_cycles, skip_arrival);
    return CSA2_OK;
}

csa2_status csa2_fp4_quantize(const float* x, int64_t rows, int32_t D, uint8_t* fp4, uint8_t* scale, void* stream) {
    if (!x || !fp4 || !scale) return CSA2_ERR_NULL;
    if (rows < 0 || D < 16 || D % 16) return CSA2_ERR_SHAPE;
    if (!al16(x) || !al16(fp4) || !al16(scale)) return CSA2_ERR_ALIGN;
    return launch_fp4_quantize(x, rows, D, fp4, scale, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? CSA2_OK
               : CSA2_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// csa2_sparse_attn_noalloc: the attention call for callers that cannot allocate
// device memory. Its scratch (merge tickets, then per-tile partials) lives in the
// file-scope array below, which every GPU that loads this library holds until
// the process exits. Host code must not use the array's name as an address: on
// the host it is only a stand-in. The device address is looked up once per
// device with cudaGetSymbolAddress, on the first call made with that device
// current (so make that first call before any stream capture), and cached.
// All calls share the array and it keeps the last call's contents: the tickets
// are cleared on the stream before every launch, and two calls that overlap on
// the GPU (other streams, other host threads) race on it.
// ---------------------------------------------------------------------------
#include <mutex>

namespace csa2 {
constexpr size_t kStaticScratchBytes = (size_t)8 << 20;   // 8 MiB in total
constexpr size_t kStaticTicketBytes = (size_t)64 << 10;   // tickets for up to 16384 queries
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

static std::mutex g_static_mu;
static void* g_static_addr[kMaxDevices] = {nullptr};

static csa2_status static_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CSA2_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (g_static_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return CSA2_ERR_CUDA;
        g_static_addr[dev] = p;
    }
    *out = g_static_addr[dev];
    return CSA2_OK;
}
}  // namespace csa2

extern "C" csa2_status csa2_sparse_attn_noalloc(const csa2_attn_args* args, int32_t* d_status, void* stream) {
    csa2_status st = check_attn(args, false);
    if (st != CSA2_OK) return st;
    const int units = args->B * args->Tq;
    const size_t ticket_bytes = (size_t)units * sizeof(int);
    if (ticket_bytes > kStaticTicketBytes || attn_scratch_bytes(*args) > kStaticScratchBytes - kStaticTicketBytes)
        return CSA2_ERR_WORKSPACE;
    void* base = nullptr;
    st = static_scratch(&base);
    if (st != CSA2_OK) return st;
    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    int* tickets = static_cast<int*>(base);
    void* partials = static_cast<uint8_t*>(base) + kStaticTicketBytes;
    if (cudaMemsetAsync(tickets, 0, ticket_bytes, strm) != cudaSuccess) return CSA2_ERR_CUDA;
    csa2_attn_args a = *args;
    if (a.W == 0) {
        a.local_base = a.q_pos;
        a.Lloc = 0;
    }
    return launch_attn(a, a.topk, tickets, partials, d_status, strm);
}
