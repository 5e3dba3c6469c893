// Seeded synthetic inputs, device side.
//
// Input generation only (no step of the CSA2 method).  Implements the same
// definition as synth_host.c -- SplitMix64 counters, Irwin-Hall(12) normals,
// fp32 channel scaling and RNE to bf16 -- with integer arithmetic and single
// IEEE fp32 operations (__fmul_rn), so values match the host bit for bit.
// Used by the benchmark and the full-size GPU tests to fill large device
// inputs without a host round trip.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kG = 0x9E3779B97F4A7C15ULL;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

__device__ __forceinline__ float normal_f32(uint64_t key, uint64_t i) {
    long long s = 0;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        uint64_t u = mix64(key + (3 * i + k + 1) * kG);
        s += (long long)(u & 0xFFFF) + (long long)((u >> 16) & 0xFFFF) +
             (long long)((u >> 32) & 0xFFFF) + (long long)(u >> 48);
    }
    return __fmul_rn((float)(int)(2 * s - 786420), 1.0f / 131072.0f);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
    uint32_t u = __float_as_uint(f);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

__global__ void k_normal_bf16(uint64_t key, uint64_t start, int64_t n, const float* scale,
                              int64_t nchan, uint16_t* out) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
         j += (int64_t)gridDim.x * blockDim.x) {
        uint64_t i = start + (uint64_t)j;
        float v = normal_f32(key, i);
        if (scale) v = __fmul_rn(v, scale[i % (uint64_t)nchan]);
        out[j] = f32_to_bf16_rne(v);
    }
}

__global__ void k_normal_scaled_f32(uint64_t key, uint64_t start, int64_t n, float scale,
                                    float* out) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
         j += (int64_t)gridDim.x * blockDim.x)
        out[j] = __fmul_rn(normal_f32(key, start + (uint64_t)j), scale);
}

__global__ void k_uniform_f32(uint64_t key, uint64_t start, int64_t n, float* out) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
         j += (int64_t)gridDim.x * blockDim.x)
        out[j] = __fmul_rn((float)(mix64(key + (start + j + 1) * kG) >> 40), 1.0f / 16777216.0f);
}

__global__ void k_normal_bf16_rows(uint64_t key, uint64_t start, uint64_t row_stride, int64_t rows,
                                  int64_t row_len, const float* scale, int64_t nchan, uint16_t* out) {
    const int64_t n = rows * row_len;
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
         j += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = j / row_len, c = j - r * row_len;
        const uint64_t i = start + (uint64_t)r * row_stride + (uint64_t)c;
        float v = normal_f32(key, i);
        if (scale) v = __fmul_rn(v, scale[i % (uint64_t)nchan]);
        out[j] = f32_to_bf16_rne(v);
    }
}

__global__ void k_normal_f32_rows(uint64_t key, uint64_t start, uint64_t row_stride, int64_t rows,
                                  int64_t row_len, float* out) {
    const int64_t n = rows * row_len;
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
         j += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = j / row_len, c = j - r * row_len;
        out[j] = normal_f32(key, start + (uint64_t)r * row_stride + (uint64_t)c);
    }
}

int grid_for(int64_t n) {
    int64_t g = (n + 255) / 256;
    if (g > 148 * 32) g = 148 * 32;
    return g < 1 ? 1 : (int)g;
}

}  // namespace

extern "C" int synth_dev_normal_bf16(uint64_t key, uint64_t start, int64_t n, const float* scale,
                                     int64_t nchan, uint16_t* out, cudaStream_t stream) {
    if (n <= 0) return 0;
    k_normal_bf16<<<grid_for(n), 256, 0, stream>>>(key, start, n, scale, nchan, out);
    return (int)cudaGetLastError();
}

extern "C" int synth_dev_normal_scaled_f32(uint64_t key, uint64_t start, int64_t n, float scale,
                                           float* out, cudaStream_t stream) {
    if (n <= 0) return 0;
    k_normal_scaled_f32<<<grid_for(n), 256, 0, stream>>>(key, start, n, scale, out);
    return (int)cudaGetLastError();
}

extern "C" int synth_dev_normal_bf16_rows(uint64_t key, uint64_t start, uint64_t row_stride,
                                          int64_t rows, int64_t row_len, const float* scale,
                                          int64_t nchan, uint16_t* out, cudaStream_t stream) {
    if (rows * row_len <= 0) return 0;
    k_normal_bf16_rows<<<grid_for(rows * row_len), 256, 0, stream>>>(key, start, row_stride, rows,
                                                                     row_len, scale, nchan, out);
    return (int)cudaGetLastError();
}

extern "C" int synth_dev_normal_f32_rows(uint64_t key, uint64_t start, uint64_t row_stride,
                                         int64_t rows, int64_t row_len, float* out,
                                         cudaStream_t stream) {
    if (rows * row_len <= 0) return 0;
    k_normal_f32_rows<<<grid_for(rows * row_len), 256, 0, stream>>>(key, start, row_stride, rows,
                                                                    row_len, out);
    return (int)cudaGetLastError();
}

extern "C" int synth_dev_uniform_f32(uint64_t key, uint64_t start, int64_t n, float* out,
                                     cudaStream_t stream) {
    if (n <= 0) return 0;
    k_uniform_f32<<<grid_for(n), 256, 0, stream>>>(key, start, n, out);
    return (int)cudaGetLastError();
}
