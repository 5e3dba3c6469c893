// Sparse + window attention (CSA2 chapter of "DeepSeek-V4.1-Flash, expliqué pas
// à pas": the main query reads the selected entries, decompressed, and the
// layer's local SWA KV), the SWA ring write, and the split combine.
//
// Items of (problem, sequence): positions [0, K) are the selected entries
// (index -1 or beyond n_entries is masked), positions [K, K + 128) the window
// slots (slot >= min(count, 128) is masked).  The latent item is both key and
// value.  Work unit = (problem, sequence, split of kSplit item positions):
// the CTA dequantises its items into shared memory (fp32, exact), then each
// warp takes one head at a time: scores (lane = item), softmax statistics by
// warp shuffles, output accumulation (lane = 16 channels).  Partials
// (max, sum, unnormalised output) are merged by k_attn_combine.
#include <cstdlib>

#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

namespace {

constexpr int kSplit = 64;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kStride = D + 1;  // padded item row (conflict-free column reads)

__host__ __device__ inline int n_splits(int K) { return (K + WIN + kSplit - 1) / kSplit; }

__global__ void __launch_bounds__(kThreads) k_attn_split(AttnBatch ab) {
    extern __shared__ float sm[];
    float* items = sm;                          // [kSplit][kStride]
    float* qsh = items + kSplit * kStride;      // [kWarps][512]
    __shared__ int valid[kSplit];
    const AttnProblem& P = ab.p[blockIdx.z];
    const int b = blockIdx.y;
    const int split = blockIdx.x;
    const int K = P.K;
    const int ns = n_splits(K);
    if (split >= ns) return;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int pos0 = split * kSplit;
    const int wcount = P.win_count[b];
    const int wlen = wcount < WIN ? (wcount < 0 ? 0 : wcount) : WIN;
    const int n = (K > 0) ? entries_of(P.cache, b) : 0;

    // ---- load + dequantise items (warp per item, lane = 16 channels = one scale)
    for (int it = wid; it < kSplit; it += kWarps) {
        const int pos = pos0 + it;
        float* row = items + it * kStride;
        int ok = 0;
        if (pos < K) {
            const int e = P.idx[(int64_t)b * K + pos];
            if (e >= 0 && e < n) {
                const int p = page_of(P.cache, b, e);
                if (p >= 0) {
                    ok = 1;
                    const int64_t ent = (int64_t)p * PAGE + (e % PAGE);
                    const uint2 cw = *reinterpret_cast<const uint2*>(P.cache.main_codes + ent * MCB + 8 * lane);
                    const float s = e4m3_decode_pos(P.cache.main_scales[ent * MSB + lane]);
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t by = ((k < 4 ? cw.x : cw.y) >> (8 * (k & 3))) & 0xFFu;
                        row[16 * lane + 2 * k] = __fmul_rn(e2m1_decode(by & 15u), s);
                        row[16 * lane + 2 * k + 1] = __fmul_rn(e2m1_decode(by >> 4), s);
                    }
                }
            }
        } else if (pos - K < wlen && P.win_fp8) {
            ok = 1;
            const uint8_t* src = static_cast<const uint8_t*>(P.win) + ((int64_t)b * WIN + (pos - K)) * D + 16 * lane;
            const uint4 u = *reinterpret_cast<const uint4*>(src);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
#pragma unroll
                for (int hlf = 0; hlf < 2; ++hlf) {
                    const uint32_t hb = e4m3x2_to_h2((w[k] >> (16 * hlf)) & 0xFFFFu);
                    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hb));
                    row[16 * lane + 4 * k + 2 * hlf] = f.x;
                    row[16 * lane + 4 * k + 2 * hlf + 1] = f.y;
                }
            }
        } else if (pos - K < wlen) {
            ok = 1;
            const uint16_t* src = static_cast<const uint16_t*>(P.win) + ((int64_t)b * WIN + (pos - K)) * D + 16 * lane;
            const uint4 u0 = *reinterpret_cast<const uint4*>(src);
            const uint4 u1 = *reinterpret_cast<const uint4*>(src + 8);
            const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                row[16 * lane + 2 * k] = __uint_as_float(w[k] << 16);
                row[16 * lane + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
            }
        }
        if (lane == 0) valid[it] = ok;
    }
    __syncthreads();

    // (problem, seq, split); the split stride is that of the largest K of the batch
    const int64_t part = ((int64_t)blockIdx.z * ab.batch + b) * n_splits(ab.Kmax) + split;
    float* q = qsh + wid * D;
    for (int h = wid; h < ab.H; h += kWarps) {
        const uint16_t* qs = P.q + ((int64_t)b * ab.H + h) * D;
        for (int c = lane; c < D; c += 32) q[c] = bf16_bits_to_f32(qs[c]);
        __syncwarp();
        float s0 = 0.0f, s1 = 0.0f;
        const float* r0 = items + lane * kStride;
        const float* r1 = items + (lane + 32) * kStride;
#pragma unroll 8
        for (int c = 0; c < D; ++c) {
            const float qc = q[c];
            s0 = fmaf(qc, r0[c], s0);
            s1 = fmaf(qc, r1[c], s1);
        }
        s0 = valid[lane] ? s0 * ab.scale : -INFINITY;
        s1 = valid[lane + 32] ? s1 * ab.scale : -INFINITY;
        float m = fmaxf(s0, s1);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float p0 = 0.0f, p1 = 0.0f;
        if (m != -INFINITY) {
            p0 = valid[lane] ? expf(s0 - m) : 0.0f;
            p1 = valid[lane + 32] ? expf(s1 - m) : 0.0f;
        }
        float l = p0 + p1;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        float acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
        for (int j = 0; j < 32; ++j) {
            const float pj0 = __shfl_sync(0xffffffffu, p0, j);
            const float pj1 = __shfl_sync(0xffffffffu, p1, j);
            const float* a0 = items + j * kStride + lane;
            const float* a1 = items + (j + 32) * kStride + lane;
            if (pj0 != 0.0f) {
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[i] = fmaf(pj0, a0[32 * i], acc[i]);
            }
            if (pj1 != 0.0f) {
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[i] = fmaf(pj1, a1[32 * i], acc[i]);
            }
        }
        float* po = ab.part_o + (part * ab.H + h) * D;
#pragma unroll
        for (int i = 0; i < 16; ++i) po[lane + 32 * i] = acc[i];
        if (lane == 0) {
            ab.part_ml[(part * ab.H + h) * 2 + 0] = m;
            ab.part_ml[(part * ab.H + h) * 2 + 1] = l;
        }
        __syncwarp();
    }
}

// out[b][h] = sum_s O_s e^(m_s - M) / sum_s l_s e^(m_s - M)
__global__ void k_attn_combine(AttnBatch ab) {
    const AttnProblem& P = ab.p[blockIdx.z];
    const int b = blockIdx.y, h = blockIdx.x;
    const int ns = n_splits(P.K);
    const int64_t base = ((int64_t)blockIdx.z * ab.batch + b) * n_splits(ab.Kmax);
    float M = -INFINITY;
    for (int s = 0; s < ns; ++s) M = fmaxf(M, ab.part_ml[((base + s) * ab.H + h) * 2]);
    float L = 0.0f;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
        for (int s = 0; s < ns; ++s) {
            const float m = ab.part_ml[((base + s) * ab.H + h) * 2];
            if (m == -INFINITY) continue;
            const float f = expf(m - M);
            L += ab.part_ml[((base + s) * ab.H + h) * 2 + 1] * f;
            const float* po = ab.part_o + ((base + s) * ab.H + h) * D;
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = fmaf(f, po[threadIdx.x + 128 * i], acc[i]);
        }
    }
    float* o = P.out + ((int64_t)b * ab.H + h) * D;
    const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) o[threadIdx.x + 128 * i] = acc[i] * inv;
}

// Eight bf16 channels (one 16-byte chunk) -> eight E4M3 codes: nearest finite
// value, ties to even, saturating at +-448 (cvt ... satfinite).
__device__ __forceinline__ uint2 bf16x8_to_e4m3x8(uint4 u) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        uint16_t lo, hi;
        // cvt packs its first source operand into the upper byte
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
            : "=h"(lo)
            : "f"(__uint_as_float(w[2 * k] & 0xFFFF0000u)), "f"(__uint_as_float(w[2 * k] << 16)));
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
            : "=h"(hi)
            : "f"(__uint_as_float(w[2 * k + 1] & 0xFFFF0000u)), "f"(__uint_as_float(w[2 * k + 1] << 16)));
        o[k] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    return make_uint2(o[0], o[1]);
}

__global__ void k_window_append(WinAppend wa) {
    const int l = blockIdx.y, b = blockIdx.x;
    const int cnt = wa.count[l][b];
    __syncthreads();
    const int slot = ((cnt % WIN) + WIN) % WIN;
    const uint4* src = reinterpret_cast<const uint4*>(wa.tok[l] + (int64_t)b * D);
    if (wa.fp8[l]) {
        uint2* dst = reinterpret_cast<uint2*>(static_cast<uint8_t*>(wa.tokens[l]) + ((int64_t)b * WIN + slot) * D);
        for (int i = threadIdx.x; i < D / 8; i += blockDim.x) dst[i] = bf16x8_to_e4m3x8(src[i]);
    } else {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(wa.tokens[l]) + ((int64_t)b * WIN + slot) * D);
        for (int i = threadIdx.x; i < D / 8; i += blockDim.x) dst[i] = src[i];
    }
    if (threadIdx.x == 0) wa.count[l][b] = cnt + 1;
}

}  // namespace

bool attn_mma_supported(const AttnBatch& ab);
size_t attn_mma_workspace_bytes(int n_problems, int batch, int H, int Kmax);
cudaError_t launch_attn_mma(const AttnBatch& ab, cudaStream_t st, cudaEvent_t* ev);

// CSA2_ATTN_CUDA_CORE=1 in the environment selects the CUDA-core attention for
// every head count (to compare the two kernels; the tensor-core one is the
// default for 1 .. 64 heads).  Read at every call, by the workspace query and
// the launch alike.
static bool attn_cuda_core_forced() {
    const char* e = std::getenv("CSA2_ATTN_CUDA_CORE");
    return e && e[0] == '1' && e[1] == 0;
}

size_t attn_workspace_bytes(int n_problems, int batch, int H, int Kmax) {
    if (H >= 1 && H <= 64 && !attn_cuda_core_forced()) return attn_mma_workspace_bytes(n_problems, batch, H, Kmax);
    const size_t units = (size_t)n_problems * batch * n_splits(Kmax) * H;
    return units * D * sizeof(float) + units * 2 * sizeof(float);
}

namespace {

// CUDA-core path (heads beyond the tensor-core kernel's 64).
cudaError_t launch_attn_cuda(const AttnBatch& ab, cudaStream_t st, cudaEvent_t* ev) {
    const size_t smem = sizeof(float) * (kSplit * kStride + kWarps * D);
    static std::atomic<uint64_t> attr_done{0};
    const cudaError_t ea = smem_opt_in(reinterpret_cast<const void*>(k_attn_split), (int)smem, attr_done);
    if (ea != cudaSuccess) return ea;
    dim3 grid(n_splits(ab.Kmax), ab.batch, ab.n);
    k_attn_split<<<grid, kThreads, smem, st>>>(ab);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (ev) cudaEventRecord(ev[0], st);
    dim3 g2(ab.H, ab.batch, ab.n);
    k_attn_combine<<<g2, 128, 0, st>>>(ab);
    e = cudaGetLastError();
    if (e == cudaSuccess && ev) cudaEventRecord(ev[1], st);
    return e;
}

}  // namespace

cudaError_t launch_sparse_attn(const AttnBatch& ab, cudaStream_t st, cudaEvent_t* ev) {
    if (attn_mma_supported(ab) && !attn_cuda_core_forced()) return launch_attn_mma(ab, st, ev);
    return launch_attn_cuda(ab, st, ev);
}

int attn_mma_launches(const AttnBatch& ab);

int sparse_attn_launches(const AttnBatch& ab) {
    if (attn_mma_supported(ab) && !attn_cuda_core_forced()) return attn_mma_launches(ab);
    return 2;
}

cudaError_t launch_window_append(const WinAppend& wa, cudaStream_t st) {
    dim3 grid(wa.batch, wa.n);
    k_window_append<<<grid, 64, 0, st>>>(wa);
    return cudaGetLastError();
}

}  // namespace csa2
