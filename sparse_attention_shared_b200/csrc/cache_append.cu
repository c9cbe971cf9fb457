// Decode-step cache append: the state update that runs before the hot path on
// every generated token.
//
// "CED: Continuing Context with a Causal Encoder and Decoder", "Why Prefill
// Recomputes a Recent Segment" (closing paragraph): after each output the new
// token's global KV, projected from the encoder's final output E, is appended to
// the one cache all decoder layers share, and each decoder layer updates its own
// local state. "DeepSeek-V4.1 Flash Pushes KV Cache Compression for Agent
// Workloads", "Ana Gelisme": the appended global row is stored as FP4 E2M1 with
// one E4M3 scale per 16 channels (the same bytes csa2_fp4_quantize writes).
//
// Local buffers are linear: row r of sequence b holds position local_base[b] + r,
// which is the layout the attention kernels read. A buffer of Lcap >= 2W - 1 rows
// is refilled in place: when the new token's row would fall past its end, the
// W - 1 rows before it move to rows 0..W-2 (a source and a destination that do not
// overlap) and local_base becomes pos - (W - 1). That moves W - 1 rows once every
// Lcap - W + 1 tokens instead of shifting the window on every token.
#include <algorithm>

#include "csa2_common.cuh"
#include "fp4_codec.cuh"

namespace csa2 {

constexpr int kAppendMaxSets = 32;
constexpr int kAppendMaxLayers = 64;
constexpr int kAppendThreads = 256;

struct AppendParams {
    int B, N, D, Di, S, L, W, Lcap;
    const int32_t* pos;
    const float* kv_new;
    uint8_t* kv_fp4;
    uint8_t* kv_scale;
    const int8_t* ki_new;
    int8_t* ki[kAppendMaxSets];
    const uint16_t* kl_new;
    const uint16_t* vl_new;
    uint16_t* kl[kAppendMaxLayers];
    uint16_t* vl[kAppendMaxLayers];
    const int32_t* local_base;
    int32_t* status;
};

// blockIdx.x = sequence; blockIdx.y = 0: the global row; 1..S: the index keys;
// S+1..S+L: layer l's local K and V. Every block reads the old local_base; the
// second kernel below writes the new one once these have finished.
__global__ void __launch_bounds__(kAppendThreads) cache_append_kernel(const __grid_constant__ AppendParams p) {
    const int b = blockIdx.x, y = blockIdx.y, tid = threadIdx.x;
    const int pos = p.pos[b];
    if (pos < 0 || pos >= p.N) {
        if (tid == 0 && y == 0) report(p.status, CSA2_ERR_RANGE, b);
        return;
    }
    if (y == 0) {
        const float* src = p.kv_new + (size_t)b * p.D;
        const size_t row = (size_t)b * p.N + pos;
        for (int g = tid; g < p.D / 16; g += kAppendThreads) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 f = reinterpret_cast<const float4*>(src + 16 * g)[i];
                v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
            }
            uint32_t packed[2];
            const uint32_t sc = fp4_quantize_group16(v, packed);
            reinterpret_cast<uint2*>(p.kv_fp4 + row * (p.D / 2))[g] = make_uint2(packed[0], packed[1]);
            p.kv_scale[row * (p.D / 16) + g] = (uint8_t)sc;
        }
        return;
    }
    if (y <= p.S) {
        const int s = y - 1;
        const int8_t* src = p.ki_new + ((size_t)s * p.B + b) * p.Di;
        int8_t* dst = p.ki[s] + ((size_t)b * p.N + pos) * p.Di;
        for (int i = tid; i < p.Di / 16; i += kAppendThreads)
            reinterpret_cast<int4*>(dst)[i] = reinterpret_cast<const int4*>(src)[i];
        return;
    }
    const int l = y - 1 - p.S;
    const int base = p.local_base[b];
    const int rel = pos - base;
    if (rel < 0 || rel > p.Lcap) {
        if (tid == 0) report(p.status, CSA2_ERR_RANGE, b);
        return;
    }
    constexpr int kChunk = 8;   // bf16 values per 16-byte load
    const int cpr = p.D / kChunk;
    uint4* kl = reinterpret_cast<uint4*>(p.kl[l] + (size_t)b * p.Lcap * p.D);
    uint4* vl = reinterpret_cast<uint4*>(p.vl[l] + (size_t)b * p.Lcap * p.D);
    int row = rel;
    if (rel == p.Lcap) {
        // refill: the W - 1 rows before the new token move to the front
        const int keep = p.W - 1, from = p.Lcap - keep;
        for (int i = tid; i < keep * cpr; i += kAppendThreads) {
            const int r = i / cpr, c = i % cpr;
            kl[(size_t)r * cpr + c] = kl[(size_t)(from + r) * cpr + c];
            vl[(size_t)r * cpr + c] = vl[(size_t)(from + r) * cpr + c];
        }
        row = keep;
    }
    const uint4* kn = reinterpret_cast<const uint4*>(p.kl_new + ((size_t)l * p.B + b) * p.D);
    const uint4* vn = reinterpret_cast<const uint4*>(p.vl_new + ((size_t)l * p.B + b) * p.D);
    if (!CSA2_CHECK(row >= 0 && row < p.Lcap, p.status, 2401)) return;
    for (int c = tid; c < cpr; c += kAppendThreads) {
        kl[(size_t)row * cpr + c] = kn[c];
        vl[(size_t)row * cpr + c] = vn[c];
    }
}

__global__ void cache_append_base_kernel(const int32_t* pos, int32_t* local_base, int B, int N, int W, int Lcap) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    const int p = pos[b], base = local_base[b];
    if (p >= 0 && p < N && p - base == Lcap) local_base[b] = p - (W - 1);
}

csa2_status launch_cache_append(const csa2_append_args& a, int32_t* d_status, cudaStream_t stream) {
    AppendParams p{};
    p.B = a.B; p.N = a.N; p.D = a.D; p.Di = a.Di; p.S = a.S; p.L = a.L; p.W = a.W; p.Lcap = a.Lcap;
    p.pos = a.pos;
    p.kv_new = a.kv_new; p.kv_fp4 = a.kv_fp4; p.kv_scale = a.kv_scale;
    p.ki_new = a.ki_new;
    for (int s = 0; s < a.S; ++s) p.ki[s] = a.ki[s];
    p.kl_new = a.kl_new; p.vl_new = a.vl_new;
    for (int l = 0; l < a.L; ++l) {
        p.kl[l] = a.kl[l];
        p.vl[l] = a.vl[l];
    }
    p.local_base = a.local_base;
    p.status = d_status;
    dim3 grid(a.B, 1 + a.S + a.L);
    cache_append_kernel<<<grid, kAppendThreads, 0, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return CSA2_ERR_CUDA;
    if (a.L > 0) {
        cache_append_base_kernel<<<(a.B + 127) / 128, 128, 0, stream>>>(a.pos, a.local_base, a.B, a.N, a.W, a.Lcap);
        if (cudaGetLastError() != cudaSuccess) return CSA2_ERR_CUDA;
    }
    return CSA2_OK;
}

int append_max_sets() { return kAppendMaxSets; }
int append_max_layers() { return kAppendMaxLayers; }

}  // namespace csa2
