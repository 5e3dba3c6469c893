// Indexer scan (the pages' light indexer scores every main-KV entry from an
// indexer query and an indexer key: "DeepSeek-V4.1-Flash, expliqué pas à pas",
// CSA2 chapter) over MXFP4 keys and queries, and the per-sequence Top-K of the
// 512 best entries.
//
//   score[b][e] = sum_h w[b][h] * max(0, qhat[b][h] . khat[b][e])
//
// Query quantisation: one thread per (sequence, head, 32-channel block), same
// MXFP4 rule as the keys.
//
// CUDA-core scan: one thread per entry.  E2M1 values times 2 are the integers
// {0,1,2,3,4,6,8,12} (with sign), so each 32-channel block product is an exact
// int32 dot of int8 vectors (dp4a); the block's two E8M0 scales are applied to
// that exact integer and the four blocks summed in fp32.  A problem with a
// pool (hierarchical indexer) runs one thread per pool position instead.  Keys stream with
// 16-byte loads and an evict-first L2 policy (each key is read once per scan).
#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

namespace {

// 2 * E2M1 value as a signed byte, for all 16 codes.
__device__ __forceinline__ uint32_t e2m1x2_i8(uint32_t code) {
    // magnitudes*2 of codes 0..7: 0 1 2 3 4 6 8 12
    const uint32_t mag = (0xC8643210u >> (4 * (code & 7u))) & 0xFu;
    return (code & 8u) ? ((0x100u - mag) & 0xFFu) : mag;
}

// Four nibbles (two code bytes) -> four int8 lanes of one word.
__device__ __forceinline__ int32_t nib4_to_i8x4(uint32_t two_bytes) {
    return (int32_t)(e2m1x2_i8(two_bytes & 15u) | (e2m1x2_i8((two_bytes >> 4) & 15u) << 8) |
                     (e2m1x2_i8((two_bytes >> 8) & 15u) << 16) |
                     (e2m1x2_i8((two_bytes >> 12) & 15u) << 24));
}

// L2 policy for streamed keys: evict first (each key is read once per scan).
__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ uint4 ld_stream16(const void* p, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}

__device__ __forceinline__ uint32_t ld_stream4(const void* p, uint64_t pol) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.u32 %0, [%1], %2;"
                 : "=r"(v)
                 : "l"(p), "l"(pol));
    return v;
}

// ---- MXFP4 quantisation of the indexer queries
__global__ void k_quant_queries(ScanBatch sb, int batch) {
    const int prob = blockIdx.y;
    const ScanProblem& P = sb.p[prob];
    const int H = sb.H_idx;
    const int g = blockIdx.x * blockDim.x + threadIdx.x;  // (b, h, blk)
    if (g >= batch * H * 4) return;
    const int blk = g & 3, bh = g >> 2;
    // the block's 32 bf16 values: four 16-byte loads (rows are 256-byte aligned)
    const uint4* src = reinterpret_cast<const uint4*>(P.q_idx + (int64_t)bh * DI + 32 * blk);
    const int64_t qrow = (int64_t)prob * batch * H + bh;  // row of (problem, sequence, head)
    float v[32];
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint4 w = __ldg(src + c);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            v[8 * c + 2 * k] = __uint_as_float(ws[k] << 16);
            v[8 * c + 2 * k + 1] = __uint_as_float(ws[k] & 0xFFFF0000u);
        }
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    uint4* dst = reinterpret_cast<uint4*>(sb.qc + qrow * ICB + 16 * blk);
    if (amax == 0.0f) {
        *dst = make_uint4(0, 0, 0, 0);
        sb.qs[qrow * ISB + blk] = 0;
        return;
    }
    const int X = mx_shared_exp(amax);
    const float inv = pow2i(-X);
    uint32_t cw[4] = {0, 0, 0, 0};  // 32 codes, channel 2i in the low nibble of byte i
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t byte = e2m1_encode(__fmul_rn(v[2 * i], inv)) | (e2m1_encode(__fmul_rn(v[2 * i + 1], inv)) << 4);
        cw[i >> 2] |= byte << (8 * (i & 3));
    }
    *dst = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    sb.qs[qrow * ISB + blk] = (uint8_t)(X + 127);
}

// ---- CUDA-core scan: thread per entry
constexpr int kScanThreads = 256;

__global__ void __launch_bounds__(kScanThreads) k_scan_cuda(ScanBatch sb) {
    extern __shared__ int32_t sq[];  // [H][32] int8x4 query words, then [H][4] exps, then [H] w
    const int prob = blockIdx.z;
    const ScanProblem& P = sb.p[prob];
    const int b = blockIdx.y;
    const int H = sb.H_idx;
    int32_t* qexp = sq + H * 32;
    float* wv = reinterpret_cast<float*>(qexp + H * 4);
    const int64_t qrow0 = ((int64_t)prob * P.cache.batch + b) * H;
    for (int i = threadIdx.x; i < H * 32; i += blockDim.x) {
        const int h = i >> 5, wd = i & 31;
        const uint8_t* qc = sb.qc + (qrow0 + h) * ICB + 2 * wd;
        sq[i] = nib4_to_i8x4((uint32_t)qc[0] | ((uint32_t)qc[1] << 8));
    }
    for (int i = threadIdx.x; i < H * 4; i += blockDim.x)
        qexp[i] = (int)sb.qs[qrow0 * ISB + i] - 127;
    for (int i = threadIdx.x; i < H; i += blockDim.x) wv[i] = P.w[(int64_t)b * H + i];
    __syncthreads();

    // position i of the score row; entry e = i unless the problem scans a pool
    const int i = blockIdx.x * kScanThreads + threadIdx.x;
    if (i >= row_len(P, b)) return;
    const int e = row_entry(P, b, i);
    const int p = page_of(P.cache, b, e);
    if (p < 0) return;
    const int64_t ent = (int64_t)p * PAGE + (e % PAGE);
    const uint64_t pol = evict_first_policy();
    int32_t kv[32];
    const uint8_t* kc = P.cache.idx_codes + ent * ICB;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 u = ld_stream16(kc + 16 * i, pol);
        kv[8 * i + 0] = nib4_to_i8x4(u.x & 0xFFFFu);
        kv[8 * i + 1] = nib4_to_i8x4(u.x >> 16);
        kv[8 * i + 2] = nib4_to_i8x4(u.y & 0xFFFFu);
        kv[8 * i + 3] = nib4_to_i8x4(u.y >> 16);
        kv[8 * i + 4] = nib4_to_i8x4(u.z & 0xFFFFu);
        kv[8 * i + 5] = nib4_to_i8x4(u.z >> 16);
        kv[8 * i + 6] = nib4_to_i8x4(u.w & 0xFFFFu);
        kv[8 * i + 7] = nib4_to_i8x4(u.w >> 16);
    }
    const uint32_t ksw = ld_stream4(P.cache.idx_scales + ent * ISB, pol);
    int kexp[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) kexp[j] = (int)((ksw >> (8 * j)) & 0xFFu) - 127;

    float score = 0.0f;
#pragma unroll 2
    for (int h = 0; h < H; ++h) {
        float dot = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int acc = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) acc = __dp4a(kv[8 * j + k], sq[h * 32 + 8 * j + k], acc);
            // exact block dot = acc / 4 * 2^(xk + xq)
            dot += ldexpf((float)acc, kexp[j] + qexp[h * 4 + j] - 2);
        }
        score = fmaf(wv[h], fmaxf(dot, 0.0f), score);
    }
    P.scores[(int64_t)b * sb.score_stride + i] = score;
}

}  // namespace

bool scan_mma_supported(const ScanBatch& sb);
cudaError_t launch_scan_mma(const ScanBatch& sb, cudaStream_t st);

namespace {
constexpr size_t kWsAlign = 256;
inline size_t ws_align(size_t v) { return (v + kWsAlign - 1) / kWsAlign * kWsAlign; }
}  // namespace

size_t scan_workspace_bytes(int n, int batch, int max_entries, int H_idx) {
    return ws_align((size_t)n * batch * H_idx * ICB) + ws_align((size_t)n * batch * H_idx * ISB) +
           ws_align((size_t)n * batch * max_entries * sizeof(float));
}

void carve_scan_workspace(ScanBatch& sb, uint8_t* ws, int batch, int max_entries) {
    sb.qc = ws;
    ws += ws_align((size_t)sb.n * batch * sb.H_idx * ICB);
    sb.qs = ws;
    ws += ws_align((size_t)sb.n * batch * sb.H_idx * ISB);
    sb.score_stride = max_entries;
    for (int i = 0; i < sb.n; ++i)
        sb.p[i].scores = reinterpret_cast<float*>(ws) + (size_t)i * batch * max_entries;
}

namespace {
bool has_pool(const ScanBatch& sb) {
    for (int i = 0; i < sb.n; ++i)
        if (sb.p[i].pool) return true;
    return false;
}
}  // namespace

int index_topk_launches(const ScanBatch& sb) { return 3 + (has_pool(sb) ? 1 : 0); }

cudaError_t launch_index_topk(const ScanBatch& sb, cudaStream_t st, cudaEvent_t* ev) {
    cudaError_t e = launch_quant_scan(sb, st, ev);
    if (e != cudaSuccess) return e;
    e = launch_topk(sb, st);
    if (e == cudaSuccess && ev) cudaEventRecord(ev[2], st);
    return e;
}

cudaError_t launch_quant_scan(const ScanBatch& sb, cudaStream_t st, cudaEvent_t* ev) {
    const int batch = sb.p[0].cache.batch;
    if (has_pool(sb)) {
        cudaError_t e = launch_pool_count(sb, st);
        if (e != cudaSuccess) return e;
    }
    {
        const int total = batch * sb.H_idx * 4;
        dim3 grid((total + 127) / 128, sb.n);
        k_quant_queries<<<grid, 128, 0, st>>>(sb, batch);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        if (ev) cudaEventRecord(ev[0], st);
    }
    if (scan_mma_supported(sb)) {
        cudaError_t e = launch_scan_mma(sb, st);
        if (e != cudaSuccess) return e;
        if (ev) cudaEventRecord(ev[1], st);
    } else {
        int cap = 0;  // positions per score row at most
        for (int i = 0; i < sb.n; ++i)
            cap = max(cap, sb.p[i].pool ? kPoolBlock * sb.p[i].pool_blocks : sb.p[i].cache.max_pages * PAGE);
        dim3 grid((cap + kScanThreads - 1) / kScanThreads, batch, sb.n);
        const size_t smem = (size_t)sb.H_idx * (32 + 4 + 1) * 4;
        k_scan_cuda<<<grid, kScanThreads, smem, st>>>(sb);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        if (ev) cudaEventRecord(ev[1], st);
    }
    return cudaSuccess;
}

}  // namespace csa2
