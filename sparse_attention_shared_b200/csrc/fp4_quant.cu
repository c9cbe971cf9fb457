// FP4 (E2M1) quantisation with one E4M3 scale per 16 values ("DeepSeek-V4.1
// Flash Pushes KV Cache Compression for Agent Workloads", section "Ana Gelisme");
// the rounding rules are in fp4_codec.cuh. One thread per 16-value group.
#include "csa2_common.cuh"
#include "fp4_codec.cuh"

namespace csa2 {

__global__ void __launch_bounds__(256) fp4_quantize_kernel(const float* __restrict__ x, int64_t groups,
                                                           uint8_t* __restrict__ codes,
                                                           uint8_t* __restrict__ scales) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= groups) return;
    const float4* src = reinterpret_cast<const float4*>(x + g * 16);
    float v[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float4 f = src[i];
        v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
    }
    uint32_t packed[2];
    const uint32_t sc = fp4_quantize_group16(v, packed);
    reinterpret_cast<uint2*>(codes)[g] = make_uint2(packed[0], packed[1]);
    scales[g] = (uint8_t)sc;
}

// Entries of compression rate m: each 16-value group of an entry is the mean of the
// same group of m consecutive rows (fp32 sum left to right, times 1/m), quantised.
__global__ void __launch_bounds__(256) fp4_compress_kernel(const float* __restrict__ x, int64_t gpr, int64_t groups,
                                                           int m, float inv_m, uint8_t* __restrict__ codes,
                                                           uint8_t* __restrict__ scales) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // entry group: entry g / gpr
    if (g >= groups) return;
    const int64_t e = g / gpr, c = g % gpr;
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = 0.f;
    for (int r = 0; r < m; ++r) {
        const float4* src = reinterpret_cast<const float4*>(x + ((e * m + r) * gpr + c) * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 f = src[i];
            v[4 * i] += f.x; v[4 * i + 1] += f.y; v[4 * i + 2] += f.z; v[4 * i + 3] += f.w;
        }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] *= inv_m;
    uint32_t packed[2];
    const uint32_t sc = fp4_quantize_group16(v, packed);
    reinterpret_cast<uint2*>(codes)[g] = make_uint2(packed[0], packed[1]);
    scales[g] = (uint8_t)sc;
}

cudaError_t launch_fp4_compress(const float* x, int64_t groups, int m, int D, uint8_t* codes, uint8_t* scales,
                                cudaStream_t stream) {
    const int64_t gpr = D / 16, total = groups * gpr;
    if (total == 0) return cudaSuccess;
    fp4_compress_kernel<<<(unsigned)((total + 255) / 256), 256, 0, stream>>>(x, gpr, total, m, 1.0f / (float)m, codes,
                                                                             scales);
    return cudaGetLastError();
}

cudaError_t launch_fp4_quantize(const float* x, int64_t rows, int D, uint8_t* codes, uint8_t* scales,
                                cudaStream_t stream) {
    const int64_t groups = rows * (D / 16);
    if (groups == 0) return cudaSuccess;
    const int64_t blocks = (groups + 255) / 256;
    fp4_quantize_kernel<<<(unsigned)blocks, 256, 0, stream>>>(x, groups, codes, scales);
    return cudaGetLastError();
}

}  // namespace csa2
