/*
 * csa2.h -- C ABI of the CSA2 sparse-attention hot path for NVIDIA B200 (sm_100a).
 *
 * What the library computes (sources by page title):
 *   [CED] "CED: Continuing Context with a Causal Encoder and Decoder":
 *         "One Token Sequence and Causal Access" (Fig. 2): a query at position t
 *           may read positions 0..t only.
 *         "Selecting Positions and Reading Values with Attention" (Fig. 4): an
 *           indexer (Indexer Q from the layer's h, Indexer K from the global
 *           cache) picks top-k positions; their global KV rows are concatenated
 *           with the layer's sliding-window local KV and Main Q attends over
 *           the union with one softmax.
 *         "What Full, Reindex, and Reuse Share" (Fig. 5): per-layer modes.
 *           Full scores every cached position and builds a candidate pool
 *           wider than top-k; Reindex rescores only that pool with the layer's
 *           own indexer; Reuse takes the most recent Full/Reindex list.
 *   [KVC] "DeepSeek-V4.1 Flash Pushes KV Cache Compression for Agent
 *         Workloads", section "Ana Gelisme": the global cache is FP4 with E2M1
 *         values and one E4M3 scale per 16 channels.
 * The index score, tie rule and rounding details that the pages leave open are
 * fixed as follows:
 *   score(s) = sum_h w[h] * max(0, sum_d qi[h][d] * ki[s][d])   (exact int32)
 *   ranking  = score descending, then position ascending
 *   lists    = ascending position order, padded with -1
 *
 * Conventions for every call
 *   - All tensor pointers are DEVICE pointers unless marked HOST. Layouts are
 *     dense row-major in the order of the brackets; bf16 values are passed as
 *     their 16-bit patterns (uint16_t).
 *   - The caller owns every buffer, including the workspace. The library never
 *     allocates device memory and keeps no per-call state outside the
 *     workspace (csa2_sparse_attn_noalloc, at the end, uses a static array). Calls are asynchronous on `stream` (a cudaStream_t; NULL =
 *     the legacy default stream).
 *   - Arguments are validated on the host before anything is launched; on an
 *     error the call returns a status and launches nothing.
 *   - Problems only the device can see (a position >= N in a caller-supplied
 *     list, a local row outside [0, Lloc), a wait that ran out of time) are
 *     written to d_status (device int32[2]: {code, detail}, first error wins;
 *     may be NULL). d_status is never cleared by the library: zero it before
 *     the call and read it after synchronising.
 *   - Alignment: every device pointer must be 16-byte aligned.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CSA2_OK = 0,
    CSA2_ERR_NULL = 1,        /* a required pointer is NULL */
    CSA2_ERR_SHAPE = 2,       /* a size is out of its allowed range */
    CSA2_ERR_ALIGN = 3,       /* a pointer or stride is not 16-byte aligned */
    CSA2_ERR_MODE = 4,        /* bad mode or mode order in a layer stack */
    CSA2_ERR_RANGE = 5,       /* device: an index or position outside its range */
    CSA2_ERR_UNSUPPORTED = 6, /* a size this build has no kernel for */
    CSA2_ERR_CUDA = 7,        /* a CUDA runtime call failed */
    CSA2_ERR_TIMEOUT = 8,     /* device: a bounded wait ran out */
    CSA2_ERR_WORKSPACE = 9    /* workspace missing or smaller than csa2_workspace_bytes() */
} csa2_status;

typedef enum { CSA2_FULL = 0, CSA2_REINDEX = 1, CSA2_REUSE = 2 } csa2_mode;

/*
 * One indexer call (Full or Reindex) for B sequences x Tq queries.
 *   q_pos    [B,Tq]        int32 position t of each query, 0 <= t < N
 *   qi       [B,Tq,Hi,Di]  int8 indexer queries
 *   w        HOST [Hi]     int32 head weights (|w| small enough that
 *                          Hi * max|w| * Di * 16384 < 2^31)
 *   ki       [B, N, Di]    int8 index keys; sequence b starts at
 *                          ki + b * ki_seq_stride (bytes, multiple of 16)
 *   Full:    scores every s <= t; writes topk_out [B,Tq,k] and, when P > 0,
 *            pool_out [B,Tq,P] (the top-P of the same scores; topk is a subset).
 *   Reindex: scores only the entries of pool_in [B,Tq,P_in] (ascending
 *            positions, -1 padding at the end, every entry <= t), normally
 *            the pool of the most recent Full call, and writes topk_out.
 * Limits: 1 <= Hi <= 16, 16 <= Di <= 128 with Di % 16 == 0, 1 <= k,
 *         N < 2^27, k <= P when P > 0.
 */
typedef struct {
    int32_t B, Tq, N, Hi, Di, k, P;
    csa2_mode mode;
    const int32_t* q_pos;
    const int8_t* qi;
    const int32_t* w;           /* HOST */
    const int8_t* ki;
    int64_t ki_seq_stride;      /* bytes between sequences of ki */
    const int32_t* pool_in;     /* Reindex only */
    int32_t P_in;               /* Reindex only */
    int32_t* pool_out;          /* Full with P > 0 */
    int32_t* topk_out;
    int32_t m;                  /* sequence compression rate of ki (see below); 0 or 1: one entry per position */
} csa2_index_args;

/*
 * Sequence compression rate m ([CED] "What Does the Sequence Compression Rate
 * Reduce?"): with m >= 2 (the encoder's CSA2 uses m = 2) row j of the global
 * cache and of the index keys is one entry that combines positions m*j ..
 * m*j + m - 1, N counts entries, and a query at position t reads entry j only
 * once the whole group is causal: j <= (t + 1) / m - 1. Lists then hold entry
 * indices; the local window stays on positions. csa2_fp4_compress builds such a
 * cache. 0 <= m <= 8.
 *
 * One attention call for B sequences x Tq queries.
 *   q        [B,Tq,Hq,D]   bf16 main queries
 *   kv_fp4   [B,N,D/2]     FP4 E2M1 codes, element 2j in the low nibble
 *   kv_scale [B,N,D/16]    E4M3 scale bytes, one per 16 elements
 *   topk     [B,Tq,k]      selected global positions (ascending, -1 padded)
 *   kl, vl   [B,Lloc,D]    bf16 local K and V; row r of sequence b holds
 *                          position local_base[b] + r
 *   local_base [B]         int32
 *   out      [B,Tq,Hq,D]   bf16 output; lse [B,Tq,Hq] fp32 natural-log
 *                          sum-exp of the logits (lse may be NULL)
 * Each query attends, with one softmax and logits q.key/sqrt(D), over the
 * dequantised global rows of its list (each row is both key and value) and
 * the local rows at positions [max(local_base, t-W+1, 0), t]. A position in
 * both sets counts twice. W = 0 disables the local branch.
 * Limits: Hq <= 32, D in {64, 128}, 1 <= k, 0 <= W, t - local_base < Lloc.
 */
typedef struct {
    int32_t B, Tq, N, Hq, D, k, W, Lloc;
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
    int32_t m;                  /* sequence compression rate of the global cache; 0 or 1: one row per position */
} csa2_attn_args;

/*
 * L decoder layers over one shared global cache, run in layer order on one
 * stream ([CED] Fig. 5). Layer l uses idx[l] and attn[l]:
 *   idx[l].mode FULL:    an indexer call as above (pool_out required if a
 *                        later REINDEX layer needs the pool).
 *   idx[l].mode REINDEX: pool_in/P_in are taken from the most recent FULL
 *                        layer (the caller's pool_in is ignored).
 *   idx[l].mode REUSE:   no indexer work; the layer's list is the list of the
 *                        most recent FULL/REINDEX layer. If idx[l].topk_out is
 *                        non-NULL that list is also copied there.
 *   attn[l]:             an attention call; its topk field is ignored and the
 *                        layer's list is used.
 * Errors: REUSE before any FULL/REINDEX, REINDEX before any FULL with P > 0.
 */
typedef struct {
    int32_t L;
    const csa2_index_args* idx;   /* HOST [L] */
    const csa2_attn_args* attn;   /* HOST [L] */
} csa2_stack_args;

/*
 * One decode step's cache update for B sequences ([CED] "Why Prefill Recomputes
 * a Recent Segment", closing paragraph: after each output, the new token's
 * global KV from the encoder output E is appended to the shared cache and each
 * decoder layer updates its local state; [KVC]: the appended row is FP4).
 *   pos        [B]        int32 position of the new token (its row), 0 <= pos < N
 *   kv_new     [B, D]     fp32 global KV row of the new token, quantised into
 *                         kv_fp4 [B,N,D/2] and kv_scale [B,N,D/16] at row pos[b]
 *                         with exactly the bytes csa2_fp4_quantize writes
 *   ki_new     [S, B, Di] int8 index key of the new token for each of S key sets,
 *                         copied to ki[s] + (b * N + pos[b]) * Di
 *   ki         HOST [S]   device pointers, each [B, N, Di]
 *   kl_new, vl_new [L, B, D] bf16 local K and V of the new token for each layer
 *   kl, vl     HOST [L]   device pointers, each [B, Lcap, D]: layer l's local
 *                         buffers; row r holds position local_base[b] + r
 *   local_base [B]        int32, read and updated
 * The new local row goes to row pos - local_base. When that is Lcap (the buffer
 * is full), the W - 1 rows before it first move to rows 0..W-2 in every layer and
 * local_base becomes pos - (W - 1); attention over the buffers then sees the
 * same window (positions [pos - W + 1, pos]). A position further past the end, or
 * before local_base, is reported as CSA2_ERR_RANGE on the device.
 * Limits: D % 16 == 0, 16 <= Di <= 128 with Di % 16 == 0, 0 <= S <= 32,
 *         0 <= L <= 64, and when L > 0: W >= 1 and Lcap >= 2W - 1.
 * No workspace; every write goes to the caller's buffers.
 */
typedef struct {
    int32_t B, N, D, Di, S, L, W, Lcap;
    const int32_t* pos;
    const float* kv_new;
    uint8_t* kv_fp4;
    uint8_t* kv_scale;
    const int8_t* ki_new;
    int8_t* const* ki;          /* HOST [S] */
    const uint16_t* kl_new;
    const uint16_t* vl_new;
    uint16_t* const* kl;        /* HOST [L] */
    uint16_t* const* vl;        /* HOST [L] */
    int32_t* local_base;
} csa2_append_args;

/* Workspace bytes a call with these arguments needs. which: 0 = csa2_index_topk
 * (args = csa2_index_args*), 1 = csa2_sparse_attn (csa2_attn_args*),
 * 2 = csa2_layer_stack (csa2_stack_args*). Returns 0 for invalid arguments.
 * A Full call whose sequences carry Tq >= 4 queries over N >= 8192 positions
 * (Hi <= 8, Di in {32, 64, 128}) scores its queries in blocks that share key
 * tiles and keeps no query's scores in full: its workspace then also holds a
 * sample of each query's scores (at most 16384 int32), one 32-bit candidate word
 * per 32 positions and query, per-query estimates, a list of the queries left
 * to the cooperative kernel, and that kernel's score spill (at most 64 MB).
 * One workspace may serve calls of any sizes in turn (on one stream): zero it once
 * before its first use; a call that ends without a device-reported error leaves it
 * ready for the next. */
size_t csa2_workspace_bytes(int which, const void* args);

/* Full- or Reindex-mode top-k (and pool) selection ([CED] Fig. 4, Fig. 5). */
csa2_status csa2_index_topk(const csa2_index_args* args, void* workspace, size_t ws_bytes,
                            int32_t* d_status, void* stream);

/* Attention over selected global FP4 rows plus the sliding window ([CED] Fig. 4). */
csa2_status csa2_sparse_attn(const csa2_attn_args* args, void* workspace, size_t ws_bytes,
                             int32_t* d_status, void* stream);

/* The whole layer stack ([CED] Fig. 5). */
csa2_status csa2_layer_stack(const csa2_stack_args* args, void* workspace, size_t ws_bytes,
                             int32_t* d_status, void* stream);

/* FP4 quantisation of fp32 rows ([KVC]): for each group of 16 values the scale
 * is the E4M3 value nearest amax/6 (ties to even, saturating at 448) and each
 * code is the E2M1 value nearest x/scale (ties to even, saturating at +-6); a
 * zero scale gives zero codes; -0 is never emitted.
 *   x [rows, D] fp32, D % 16 == 0 -> fp4 [rows, D/2], scale [rows, D/16]. */
csa2_status csa2_fp4_quantize(const float* x, int64_t rows, int32_t D, uint8_t* fp4,
                              uint8_t* scale, void* stream);

/* Global entries of compression rate m from per-position rows, FP4-quantised:
 * entry g of x [groups * m, D] fp32 combines rows g*m .. g*m + m - 1. The pages do
 * not give the combining rule; this library takes their mean, summed left to right
 * in fp32 and scaled by 1/m (exact for m in {1, 2, 4, 8}), and quantises it like
 * csa2_fp4_quantize -> fp4 [groups, D/2], scale [groups, D/16]. m = 1 is
 * csa2_fp4_quantize. */
csa2_status csa2_fp4_compress(const float* x, int64_t groups, int32_t m, int32_t D, uint8_t* fp4, uint8_t* scale,
                              void* stream);

/* Attention without a caller workspace, for callers that cannot allocate device
 * memory: code running inside a host framework that owns every device allocation
 * and forbids others, or a latency-critical decode loop that must not risk the
 * device-wide synchronisation a cudaMalloc or cudaFree can cause. The pages have
 * no counterpart: this is a deployment variant of csa2_sparse_attn, with the same
 * arguments, results and errors, and no workspace.
 * Scratch: a static 8 MiB device array per GPU (64 KiB of merge tickets, the rest
 * for per-tile partials of 4 * (Hq<=16 ? 16 : 32) * (D + 2) bytes per 128-key
 * tile and query). Calls needing more return CSA2_ERR_WORKSPACE and launch
 * nothing. The first call on a device looks up that array's address (make it
 * before any stream capture). Every call clears the tickets on `stream`; calls
 * that overlap on the GPU share the array and race. The looked-up address is
 * kept for the life of the process: a device reset (cudaDeviceReset) after the
 * first call on that device is not supported. */
csa2_status csa2_sparse_attn_noalloc(const csa2_attn_args* args, int32_t* d_status, void* stream);

/* Failure-detection controls, process-wide, read by every later indexer launch.
 * The indexer's CTAs of one query meet at group barriers (spins on a counter in
 * the workspace). A CTA that waits there longer than budget_cycles SM clock
 * cycles writes CSA2_ERR_TIMEOUT to d_status and leaves; the others of its group
 * leave as soon as they see that status (when d_status is not NULL), so the call
 * ends after about one budget. budget_cycles = 0 restores the default (4e9
 * cycles, about 2 s at the boost clock); a negative value returns CSA2_ERR_SHAPE.
 * skip_arrival != 0 is host-side fault injection for tests and health checks:
 * the last CTA of every group then leaves before its first group barrier, so the
 * others' waits run out. Never set it in production. After a call that reported
 * a timeout, zero the workspace before the next call.
 * Waits on a CTA's own copies and tensor-core operations keep the fixed budget. */
csa2_status csa2_set_wait_controls(int64_t budget_cycles, int32_t skip_arrival);

/* Append one token per sequence to the global cache, the index keys and every
 * layer's local buffers (csa2_append_args above). */
csa2_status csa2_cache_append(const csa2_append_args* args, int32_t* d_status, void* stream);

/* Static text for a status code. */
const char* csa2_status_string(csa2_status s);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_H */
