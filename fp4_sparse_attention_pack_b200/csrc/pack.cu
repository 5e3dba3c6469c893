// Cache write: ratio-m compression, E2M1/E4M3 main pack, indexer-key
// projection and MXFP4 pack ("Le cache KV en FP4"; CSA2 chapter: disjoint
// groups, indexer K projected from the main KV).
//
// One CTA of 128 threads builds up to kEnt = 32 consecutive new entries of one
// sequence.  Phase 1 walks the entries: each thread owns 4 channels (a block
// of 16 channels is 4 adjacent lanes), compresses the token pair, packs the
// main entry and leaves the exact dequantised entry in shared memory.  Phase 2
// is the 512 -> 128 projection: thread o keeps the 32 accumulators k[.][o] in
// registers and streams W[c][o] once per CTA (not once per entry), in the
// fixed order c = 0..511 the bit-exact contract requires.  Phase 3 packs each
// key to MXFP4: warp w owns channel block w (32 channels = one E8M0 scale).
#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

namespace {

constexpr int kEnt = 32;
constexpr int kThreads = 128;

template <bool kF32>
__device__ __forceinline__ void load4(const void* x, int64_t off, float v[4]) {
    if (kF32) {
        float4 f = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + off);
        v[0] = f.x, v[1] = f.y, v[2] = f.z, v[3] = f.w;
    } else {
        uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(x) + off);
        v[0] = __uint_as_float(u.x << 16);
        v[1] = __uint_as_float(u.x & 0xFFFF0000u);
        v[2] = __uint_as_float(u.y << 16);
        v[3] = __uint_as_float(u.y & 0xFFFF0000u);
    }
}

// New entries this call makes for sequence b, or -1 when they do not fit.
__device__ __forceinline__ int new_entries(const CacheView& c, int b, int T, int n0, int* pend) {
    *pend = (c.ratio == 2) ? (c.pend_valid[b] ? 1 : 0) : 0;
    int nn = (c.ratio == 2) ? (*pend + T) / 2 : T;
    if (n0 + nn > c.max_pages * PAGE) return -1;
    return nn;
}

constexpr int kWc = 32;  // projection rows staged per step (32 x 128 fp32 = 16 KB)

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Rows [k*kWc, (k+1)*kWc) of W -> wb (128 threads, 8 x 16 B each).
__device__ __forceinline__ void stage_w(float* wb, const float* W, int k) {
    const float4* src = reinterpret_cast<const float4*>(W + (size_t)k * kWc * DI);
    float4* dst = reinterpret_cast<float4*>(wb);
#pragma unroll
    for (int i = 0; i < kWc * DI / 4 / kThreads; ++i)
        cp_async16(dst + threadIdx.x + i * kThreads, src + threadIdx.x + i * kThreads);
    cp_async_commit();
}

// k[jj][o] for jj < ne <= NE: fma over c = 0..511 in order (thread o = threadIdx.x).
template <int NE>
__device__ __forceinline__ void project(float (&acc)[kEnt], const float* deq, float* wbuf, const float* W, int ne) {
#pragma unroll
    for (int jj = 0; jj < kEnt; ++jj) acc[jj] = 0.0f;
    const int o = threadIdx.x;
    constexpr int kSteps = D / kWc;
    stage_w(wbuf, W, 0);
#pragma unroll 1
    for (int k = 0; k < kSteps; ++k) {
        if (k + 1 < kSteps) {
            stage_w(wbuf + ((k + 1) & 1) * kWc * DI, W, k + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const float* wb = wbuf + (k & 1) * kWc * DI;
#pragma unroll 4
        for (int cc = 0; cc < kWc; ++cc) {
            const float w = wb[cc * DI + o];
            const int ch = k * kWc + cc;
#pragma unroll
            for (int jj = 0; jj < NE; ++jj)
                if (jj < ne) acc[jj] = __fmaf_rn(w, deq[jj * D + ch], acc[jj]);
        }
        __syncthreads();
    }
}

template <bool kF32>
__global__ void __launch_bounds__(kThreads) k_pack_entries(const __grid_constant__ PackBatch pb, int T) {
    extern __shared__ float deq[];  // [kEnt][512], then W staging [2][kWc][128]
    float* wbuf = deq + kEnt * D;
    __shared__ int s_page[kEnt];
    const CacheView& c = pb.cache[blockIdx.z];
    const void* x = pb.x[blockIdx.z];
    const float* gates = pb.gates[blockIdx.z];
    const float* W = pb.W[blockIdx.z];
    const int b = blockIdx.y;
    const int t = threadIdx.x;
    const int n0 = entries_of(c, b);
    int pend;
    const int nn = new_entries(c, b, T, n0, &pend);
    if (nn < 0) {
        if (blockIdx.x == 0 && t == 0) atomicOr(c.status, CSA2_DEVERR_CAPACITY);
        return;
    }
    const int j0 = blockIdx.x * kEnt;
    if (j0 >= nn) return;
    const int ne = min(kEnt, nn - j0);
    if (t < ne) s_page[t] = page_of(c, b, n0 + j0 + t);
    __syncthreads();

    const int64_t xrow = (int64_t)b * T;  // token row base of sequence b
    // ---- phase 1: compress + main pack + dequantise
    for (int jj = 0; jj < ne; ++jj) {
        const int j = j0 + jj;
        float e[4];
        if (c.ratio == 1) {
            load4<kF32>(x, (xrow + j) * D + 4 * t, e);
        } else {
            const int t0 = 2 * j - pend;
            float x0[4], x1[4], g0;
            if (t0 < 0) {
                const float4 p = *reinterpret_cast<const float4*>(c.pend_x + (int64_t)b * D + 4 * t);
                x0[0] = p.x, x0[1] = p.y, x0[2] = p.z, x0[3] = p.w;
                g0 = c.pend_g[b];
            } else {
                load4<kF32>(x, (xrow + t0) * D + 4 * t, x0);
                g0 = gates[xrow + t0];
            }
            load4<kF32>(x, (xrow + t0 + 1) * D + 4 * t, x1);
            const float g1 = gates[xrow + t0 + 1];
            // (w0, w1) = softmax(g0, g1)
            const float E = spec_exp(__fsub_rn(g1, g0));
            const float w0 = __fdiv_rn(1.0f, __fadd_rn(1.0f, E));
            const float w1 = __fsub_rn(1.0f, w0);
#pragma unroll
            for (int k = 0; k < 4; ++k) e[k] = __fmaf_rn(w1, x1[k], __fmul_rn(w0, x0[k]));
        }
        // block of 16 channels = 4 adjacent lanes
        float amax = fmaxf(fmaxf(fabsf(e[0]), fabsf(e[1])), fmaxf(fabsf(e[2]), fabsf(e[3])));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const uint32_t sc = e4m3_encode(__fdiv_rn(amax, 6.0f));
        const float s = e4m3_decode_pos(sc);
        uint32_t q[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            q[k] = (s == 0.0f) ? 0u : e2m1_encode(__fdiv_rn(e[k], s));
            deq[jj * D + 4 * t + k] = __fmul_rn(e2m1_decode(q[k]), s);
        }
        const int p = s_page[jj];
        if (p >= 0) {
            const int64_t ent = (int64_t)p * PAGE + ((n0 + j) % PAGE);
            const uint16_t two = (uint16_t)(q[0] | (q[1] << 4) | (q[2] << 8) | (q[3] << 12));
            *reinterpret_cast<uint16_t*>(c.main_codes + ent * MCB + 2 * t) = two;
            if ((t & 3) == 0) c.main_scales[ent * MSB + (t >> 2)] = (uint8_t)sc;
        }
    }
    __syncthreads();

    // ---- phase 2: k[jj][o] = sum_c W[c][o] * deq[jj][c], fma order c = 0..511,
    // W rows staged through shared memory (double-buffered cp.async).  A CTA with
    // at most 4 entries (decode: one token per step) keeps 4 accumulators instead
    // of kEnt, so it does not issue kEnt predicated FMAs per channel.
    float acc[kEnt];
    if (ne <= 4)
        project<4>(acc, deq, wbuf, W, ne);
    else
        project<kEnt>(acc, deq, wbuf, W, ne);

    // ---- phase 3: MXFP4 per 32 channels (warp w = block w)
    const int o = t;
    const int lane = t & 31, blk = t >> 5;
#pragma unroll
    for (int jj = 0; jj < kEnt; ++jj) {
        if (jj >= ne) break;
        const float v = acc[jj];
        float amax = fabsf(v);
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
        uint32_t code, sc;
        if (amax == 0.0f) {
            code = 0u;
            sc = 0u;
        } else {
            const int X = mx_shared_exp(amax);
            sc = (uint32_t)(X + 127);
            code = e2m1_encode(__fmul_rn(v, pow2i(-X)));
        }
        const uint32_t hi = __shfl_down_sync(0xffffffffu, code, 1);
        const int p = s_page[jj];
        if (p >= 0) {
            const int64_t ent = (int64_t)p * PAGE + ((n0 + j0 + jj) % PAGE);
            if ((lane & 1) == 0) c.idx_codes[ent * ICB + (o >> 1)] = (uint8_t)(code | (hi << 4));
            if (lane == 0) c.idx_scales[ent * ISB + blk] = (uint8_t)sc;
        }
    }
}

// Entry count and pending-slot update, after every entry was written.
template <bool kF32>
__global__ void k_pack_finalize(const __grid_constant__ PackBatch pb, int T) {
    const CacheView& c = pb.cache[blockIdx.y];
    const void* x = pb.x[blockIdx.y];
    const float* gates = pb.gates[blockIdx.y];
    const int b = blockIdx.x;
    const int n0 = entries_of(c, b);
    int pend;
    const int nn = new_entries(c, b, T, n0, &pend);
    __syncthreads();  // every thread has read the old state
    if (nn < 0) return;
    if (c.ratio == 2) {
        const int rest = (pend + T) & 1;
        if (rest && T > 0) {
            const int64_t row = ((int64_t)b * T + (T - 1)) * D;
            for (int ch = threadIdx.x; ch < D; ch += blockDim.x) {
                float v = kF32 ? reinterpret_cast<const float*>(x)[row + ch]
                               : bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(x)[row + ch]);
                c.pend_x[(int64_t)b * D + ch] = v;
            }
            if (threadIdx.x == 0) c.pend_g[b] = gates[(int64_t)b * T + T - 1];
        }
        if (threadIdx.x == 0) c.pend_valid[b] = rest;
    }
    if (threadIdx.x == 0) c.n_entries[b] = n0 + nn;
}

}  // namespace

cudaError_t launch_pack(const PackBatch& pb, bool x_f32, int T, cudaStream_t st) {
    if (pb.n < 1 || T < 1) return cudaSuccess;
    int max_new = (T + 1) / 2;
    for (int i = 0; i < pb.n; ++i)
        if (pb.cache[i].ratio == 1) max_new = T;
    const int chunks = (max_new + kEnt - 1) / kEnt;
    const int batch = pb.cache[0].batch;
    const size_t smem = sizeof(float) * (kEnt * D + 2 * kWc * DI);
    static std::atomic<uint64_t> attr_done_f32{0}, attr_done_bf16{0};
    const cudaError_t ea =
        x_f32 ? smem_opt_in(reinterpret_cast<const void*>(k_pack_entries<true>), (int)smem, attr_done_f32)
              : smem_opt_in(reinterpret_cast<const void*>(k_pack_entries<false>), (int)smem, attr_done_bf16);
    if (ea != cudaSuccess) return ea;
    dim3 grid(chunks, batch, pb.n);
    if (x_f32)
        k_pack_entries<true><<<grid, kThreads, smem, st>>>(pb, T);
    else
        k_pack_entries<false><<<grid, kThreads, smem, st>>>(pb, T);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 g2(batch, pb.n);
    if (x_f32)
        k_pack_finalize<true><<<g2, 128, 0, st>>>(pb, T);
    else
        k_pack_finalize<false><<<g2, 128, 0, st>>>(pb, T);
    return cudaGetLastError();
}

}  // namespace csa2
