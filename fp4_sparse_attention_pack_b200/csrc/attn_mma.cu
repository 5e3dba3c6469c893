// Sparse + window attention on the 5th-generation tensor cores (tcgen05.mma
// kind::f16, fp16 operands, fp32 accumulation in TMEM).
//
// Per (problem, sequence) the items are the K selected entries (dequantised
// from E2M1 x E4M3: exact in fp16) and the valid window tokens (bf16 -> fp16,
// exact for |x| in fp16's normal range); the latent item is key and value.
// Items go through 128-item tiles with an online softmax:
//
//   S^T[128 items x 64 heads] = Items . Q^T            (M = 128, N = 64, K = 512)
//   P^T = exp(scale * S^T - m_head)                    (fp16, per item lane)
//   O^T[4 x 128 latent x 64 heads] += Items^T . P^T    (M = 128, N = 64, K = 128)
//
// One shared-memory image of the tile serves both MMAs: 128-byte-swizzled
// slabs of 64 latent channels, read as the K-major A operand of S^T and as the
// MN-major A operand of O^T.  The running per-head maximum is only moved when
// a tile's maximum exceeds it by more than 8 (so p <= e^8 fits fp16), which
// makes the O rescale (TMEM load, scale, store) rare.  Heads are padded to 64.
//
// CTA = 256 threads, one unit (problem, sequence, split of tiles) per CTA.  All
// warps gather + dequantise a tile (8 threads per item, one 64-channel slab
// each); thread 0 issues the MMAs; warps 0-3 (one TMEM lane quadrant each) run
// the softmax; all 8 warps rescale / write O.
#include <algorithm>
#include <cstring>

#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace csa2 {

namespace {

using namespace sm100;

constexpr int kT = 128;            // items per tile (MMA M of S^T)
constexpr int kHp = 64;            // heads, padded (MMA N)
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // S^T: 64 columns
constexpr uint32_t kColO = 64;     // O^T: 4 x 64 columns
constexpr float kRescaleGap = 8.0f;

struct __align__(1024) Smem {
    uint8_t items[8][kT * 128];    // 8 slabs x 128 rows x 128 B (SW128)
    uint8_t q[8][kHp * 128];       // 8 slabs x 64 rows x 128 B (SW128)
    uint8_t p[kT * 128];           // P^T: 128 item rows x 64 heads fp16 (SW128)
    __half2 lut[256];              // code byte -> two E2M1 values
    float red[4][kHp];             // per-warp partial max / sum
    float m_used[kHp];
    float l[kHp];
    float alpha[kHp];
    int valid[kT];
    uint64_t bar;
    uint32_t tmem_base;
};

__device__ __forceinline__ float e2m1_mag(uint32_t m) {
    return m < 2 ? 0.5f * (float)m : __uint_as_float(((126u + (m >> 1)) << 23) | ((m & 1u) << 22));
}

// Byte offset of 16-byte chunk c of row r inside a 128B-swizzled slab.
__device__ __forceinline__ uint32_t sw128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

// Reduce-scatter over the warp: v[64] per lane -> lane l holds the reduction of
// heads 2l and 2l+1 over the 32 lanes in v[0], v[1].
template <bool kMax>
__device__ __forceinline__ void warp_reduce_scatter64(float (&v)[64]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int o = 16 >> step;
        const int half = 32 >> step;
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float keep = upper ? v[half + i] : v[i];
            const float send = upper ? v[i] : v[half + i];
            const float got = __shfl_xor_sync(0xffffffffu, send, o);
            v[i] = kMax ? fmaxf(keep, got) : keep + got;
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1) k_attn_mma(const __grid_constant__ AttnBatch ab, int splits,
                                                           int tiles_per_split) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int unit = blockIdx.x;
    const int split = unit % splits;
    const int pb = unit / splits;
    const int b = pb % ab.batch;
    const int prob = pb / ab.batch;
    const AttnProblem& P = ab.p[prob];
    const int K = P.K;
    const int H = ab.H;
    const int n_tiles = (K + WIN + kT - 1) / kT;
    const int t_begin = split * tiles_per_split;
    const int t_end = min(n_tiles, t_begin + tiles_per_split);

    if (tid == 0) {
        mbar_init(&sm.bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(&sm.tmem_base, kTmemCols);
    for (int i = tid; i < 256; i += kThreads) {
        const uint32_t lo = i & 15u, hi = i >> 4;
        const float a = (lo & 8u) ? -e2m1_mag(lo & 7u) : e2m1_mag(lo & 7u);
        const float c = (hi & 8u) ? -e2m1_mag(hi & 7u) : e2m1_mag(hi & 7u);
        sm.lut[i] = __floats2half2_rn(a, c);
    }
    if (tid < kHp) {
        sm.m_used[tid] = -INFINITY;
        sm.l[tid] = 0.0f;
    }
    // Q -> fp16 slabs (rows >= H are zero)
    for (int u = tid; u < kHp * 8; u += kThreads) {
        const int h = u >> 3, j = u & 7;
        uint8_t* slab = sm.q[j];
        if (h < H) {
            const uint4* src = reinterpret_cast<const uint4*>(P.q + ((int64_t)b * H + h) * D + 64 * j);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 w = src[c];
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
                uint4 o;
                uint32_t* os = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const __half2 hv = __floats2half2_rn(__uint_as_float(ws[k] << 16),
                                                         __uint_as_float(ws[k] & 0xFFFF0000u));
                    os[k] = *reinterpret_cast<const uint32_t*>(&hv);
                }
                *reinterpret_cast<uint4*>(slab + sw128(h, c)) = o;
            }
        } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(slab + sw128(h, c)) = make_uint4(0, 0, 0, 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sm.tmem_base;
    const int wcount = P.win_count[b];
    const int wlen = wcount < WIN ? (wcount < 0 ? 0 : wcount) : WIN;
    const int n = (K > 0) ? entries_of(P.cache, b) : 0;
    uint32_t phase = 0;
    bool o_init = false;
    bool timed_out = false;

    const uint32_t idesc_s = idesc_f16(128, kHp, 0, 0, 0);
    const uint32_t idesc_o = idesc_f16(128, kHp, 0, 1, 1);

    for (int t = t_begin; t < t_end && !timed_out; ++t) {
        // ---- gather + dequantise 128 items: thread = slab j of items r0 + 32 i (i < 4).
        // The dependent loads (index -> page -> bytes) of the four items are issued
        // stage by stage so their latencies overlap.
        {
            const int j = tid & 7, r0 = tid >> 3;
            int ent_i[4];
            int64_t ent_row[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int pos = t * kT + r0 + 32 * i;
                ent_i[i] = (pos < K) ? __ldg(P.idx + (int64_t)b * K + pos) : -1;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                ent_row[i] = -1;
                const int e = ent_i[i];
                if (e >= 0 && e < n) {
                    const int pg = page_of(P.cache, b, e);
                    if (pg >= 0) ent_row[i] = (int64_t)pg * PAGE + (e % PAGE);
                }
            }
            uint4 c0[4], c1[4];
            uint32_t swd[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (ent_row[i] >= 0) {
                    const uint4* cs = reinterpret_cast<const uint4*>(P.cache.main_codes + ent_row[i] * MCB + 32 * j);
                    c0[i] = __ldg(cs);
                    c1[i] = __ldg(cs + 1);
                    swd[i] = __ldg(reinterpret_cast<const uint32_t*>(P.cache.main_scales + ent_row[i] * MSB + 4 * j));
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = r0 + 32 * i;
                const int pos = t * kT + r;
                uint8_t* slab = sm.items[j];
                bool ok = false;
                if (ent_row[i] >= 0) {
                    ok = true;
                    const uint32_t cw[8] = {c0[i].x, c0[i].y, c0[i].z, c0[i].w, c1[i].x, c1[i].y, c1[i].z, c1[i].w};
#pragma unroll
                    for (int c = 0; c < 8; ++c) {  // chunk c: channels 8c..8c+7, scale byte c/2
                        const __half2 s2 = __float2half2_rn(e4m3_decode_pos((swd[i] >> (8 * (c >> 1))) & 0xFFu));
                        uint4 o;
                        uint32_t* os = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const __half2 v = __hmul2(sm.lut[(cw[c] >> (8 * k)) & 0xFFu], s2);
                            os[k] = *reinterpret_cast<const uint32_t*>(&v);
                        }
                        *reinterpret_cast<uint4*>(slab + sw128(r, c)) = o;
                    }
                } else if (pos >= K && pos - K < wlen) {
                    ok = true;
                    const uint4* src = reinterpret_cast<const uint4*>(P.win + ((int64_t)b * WIN + (pos - K)) * D + 64 * j);
                    uint4 wv[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) wv[c] = __ldg(src + c);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t ws[4] = {wv[c].x, wv[c].y, wv[c].z, wv[c].w};
                        uint4 o;
                        uint32_t* os = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const __half2 hv = __floats2half2_rn(__uint_as_float(ws[k] << 16),
                                                                 __uint_as_float(ws[k] & 0xFFFF0000u));
                            os[k] = *reinterpret_cast<const uint32_t*>(&hv);
                        }
                        *reinterpret_cast<uint4*>(slab + sw128(r, c)) = o;
                    }
                }
                if (!ok) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(slab + sw128(r, c)) = make_uint4(0, 0, 0, 0);
                }
                if (j == 0) sm.valid[r] = ok;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- S^T = Items . Q^T
        if (tid == 0) {
            tc_fence_after();
#pragma unroll 1
            for (int ks = 0; ks < 32; ++ks) {  // 16 latent channels per MMA
                const int j = ks >> 2, off = (ks & 3) * 32;
                const uint64_t a = smem_desc(sm.items[j] + off, 16, 1024, kLayoutSw128);
                const uint64_t bq = smem_desc(sm.q[j] + off, 16, 1024, kLayoutSw128);
                tc_mma_f16(tbase + kColS, a, bq, idesc_s, ks > 0 ? 1u : 0u);
            }
            tc_commit(&sm.bar);
        }
        if (!mbar_wait(&sm.bar, phase)) timed_out = true;
        phase ^= 1;
        if (__syncthreads_or(timed_out)) {
            timed_out = true;
            break;
        }
        tc_fence_after();

        // ---- softmax statistics (warps 0-3: thread = item row)
        const uint32_t s_addr = tbase + ((uint32_t)((warp & 3) * 32) << 16) + kColS;
        if (warp < 4) {
            float v[64];
            tmem_ld_32x32b_x64(s_addr, v);
            const bool ok = sm.valid[warp * 32 + lane] != 0;
#pragma unroll
            for (int h = 0; h < 64; ++h) v[h] = ok ? v[h] * ab.scale : -INFINITY;
            warp_reduce_scatter64<true>(v);
            sm.red[warp][2 * lane] = v[0];
            sm.red[warp][2 * lane + 1] = v[1];
        }
        __syncthreads();
        bool rescale = false;
        if (tid < kHp) {
            const float mt = fmaxf(fmaxf(sm.red[0][tid], sm.red[1][tid]), fmaxf(sm.red[2][tid], sm.red[3][tid]));
            const float mo = sm.m_used[tid];
            float a = 1.0f;
            if (mt > mo + kRescaleGap || (mo == -INFINITY && mt != -INFINITY)) {
                a = (mo == -INFINITY) ? 0.0f : expf(mo - mt);
                sm.m_used[tid] = mt;
                rescale = o_init && mo != -INFINITY;
            }
            sm.alpha[tid] = a;
        }
        rescale = __syncthreads_or(rescale);

        // ---- P^T = exp(s - m) in fp16 (S reloaded from TMEM), row sums of the rounded p
        if (warp < 4) {
            const int r = warp * 32 + lane;
            float v[64];
            tmem_ld_32x32b_x64(s_addr, v);
            const bool ok = sm.valid[r] != 0;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint4 o;
                uint32_t* os = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int h = 8 * c + 2 * k;
                    const float p0 = ok ? __expf(v[h] * ab.scale - sm.m_used[h]) : 0.0f;
                    const float p1 = ok ? __expf(v[h + 1] * ab.scale - sm.m_used[h + 1]) : 0.0f;
                    const __half2 hv = __floats2half2_rn(p0, p1);
                    const float2 back = __half22float2(hv);
                    v[h] = back.x;
                    v[h + 1] = back.y;
                    os[k] = *reinterpret_cast<const uint32_t*>(&hv);
                }
                *reinterpret_cast<uint4*>(sm.p + sw128(r, c)) = o;
            }
            warp_reduce_scatter64<false>(v);
            sm.red[warp][2 * lane] = v[0];
            sm.red[warp][2 * lane + 1] = v[1];
        }
        // ---- rescale O^T where a head's reference maximum moved
        if (rescale) {
            const int quad = warp & 3;
            for (int c = (warp >> 2) * 2; c < (warp >> 2) * 2 + 2; ++c) {
                const uint32_t ta = tbase + ((uint32_t)(quad * 32) << 16) + kColO + 64 * c;
                float o[64];
                tmem_ld_32x32b_x64(ta, o);
#pragma unroll
                for (int h = 0; h < 64; ++h) o[h] *= sm.alpha[h];
                tmem_st_32x32b_x64(ta, o);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid < kHp)
            sm.l[tid] = sm.l[tid] * sm.alpha[tid] + (sm.red[0][tid] + sm.red[1][tid]) + (sm.red[2][tid] + sm.red[3][tid]);

        // ---- O^T += Items^T . P^T
        if (tid == 0) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
#pragma unroll 1
                for (int i = 0; i < 8; ++i) {  // 16 items per MMA
                    const uint64_t a = smem_desc(sm.items[2 * c] + 2048 * i, 16384, 1024, kLayoutSw128);
                    const uint64_t bp = smem_desc(sm.p + 2048 * i, 16384, 1024, kLayoutSw128);
                    tc_mma_f16(tbase + kColO + 64 * c, a, bp, idesc_o, (o_init || i > 0) ? 1u : 0u);
                }
            }
            tc_commit(&sm.bar);
        }
        o_init = true;
        if (!mbar_wait(&sm.bar, phase)) timed_out = true;
        phase ^= 1;
        if (__syncthreads_or(timed_out)) {
            timed_out = true;
            break;
        }
        tc_fence_after();
    }

    if (timed_out) {
        if (tid == 0 && K > 0) atomicOr(P.cache.status, CSA2_DEVERR_TIMEOUT);
    } else {
        // ---- write O (normalised) or the split's partial (O, m, l)
        const int quad = warp & 3;
        const bool partial = splits > 1;
        float* dst = partial ? ab.part_o + (int64_t)unit * H * D : P.out + (int64_t)b * H * D;
        for (int c = (warp >> 2) * 2; c < (warp >> 2) * 2 + 2; ++c) {
            float o[64];
            if (o_init) {
                tmem_ld_32x32b_x64(tbase + ((uint32_t)(quad * 32) << 16) + kColO + 64 * c, o);
            } else {
#pragma unroll
                for (int h = 0; h < 64; ++h) o[h] = 0.0f;
            }
            const int lat = 128 * c + quad * 32 + lane;
#pragma unroll
            for (int h = 0; h < 64; ++h) {
                if (h < H) {
                    const float l = sm.l[h];
                    dst[(int64_t)h * D + lat] = partial ? o[h] : (l > 0.0f ? o[h] / l : 0.0f);
                }
            }
        }
        if (partial && tid < H) {
            ab.part_ml[((int64_t)unit * H + tid) * 2 + 0] = sm.m_used[tid];
            ab.part_ml[((int64_t)unit * H + tid) * 2 + 1] = sm.l[tid];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

// out = sum_s O_s e^(m_s - M) / sum_s l_s e^(m_s - M) over the splits of (problem, sequence)
__global__ void k_attn_mma_combine(const __grid_constant__ AttnBatch ab, int splits) {
    const int h = blockIdx.x, b = blockIdx.y, prob = blockIdx.z;
    const AttnProblem& P = ab.p[prob];
    const int H = ab.H;
    const int64_t u0 = ((int64_t)prob * ab.batch + b) * splits;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, ab.part_ml[((u0 + s) * H + h) * 2]);
    float L = 0.0f;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
        for (int s = 0; s < splits; ++s) {
            const float m = ab.part_ml[((u0 + s) * H + h) * 2];
            const float l = ab.part_ml[((u0 + s) * H + h) * 2 + 1];
            if (m == -INFINITY || l == 0.0f) continue;
            const float f = expf(m - M);
            L += l * f;
            const float* po = ab.part_o + ((u0 + s) * H + h) * D;
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = fmaf(f, po[threadIdx.x + 128 * i], acc[i]);
        }
    }
    float* o = P.out + ((int64_t)b * H + h) * D;
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) o[threadIdx.x + 128 * i] = acc[i] * inv;
}

int sm_count_attn() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

}  // namespace

// Splits of the item tiles per (problem, sequence): enough units to fill the
// SMs when the batch is small, none when there are already plenty.
int attn_mma_splits(int n_problems, int batch, int Kmax) {
    const int tiles = (Kmax + WIN + kT - 1) / kT;
    const int pairs = n_problems * batch;
    const int want = (sm_count_attn() + pairs - 1) / pairs;
    return std::max(1, std::min(tiles, want));
}

bool attn_mma_supported(const AttnBatch& ab) { return ab.H >= 1 && ab.H <= kHp; }

size_t attn_mma_workspace_bytes(int n_problems, int batch, int H, int Kmax) {
    const int splits = attn_mma_splits(n_problems, batch, Kmax);
    if (splits == 1) return 0;
    const size_t units = (size_t)n_problems * batch * splits;
    return units * H * D * sizeof(float) + units * H * 2 * sizeof(float);
}

cudaError_t launch_attn_mma(const AttnBatch& ab_in, cudaStream_t st, cudaEvent_t* ev) {
    AttnBatch ab = ab_in;
    const int splits = attn_mma_splits(ab.n, ab.batch, ab.Kmax);
    const int tiles = (ab.Kmax + WIN + kT - 1) / kT;
    const int tps = (tiles + splits - 1) / splits;
    if (splits > 1) {
        const size_t units = (size_t)ab.n * ab.batch * splits;
        ab.part_ml = ab.part_o + units * ab.H * D;
    }
    const size_t smem = sizeof(Smem) + 1024;
    static const bool attr = [smem] {
        cudaFuncSetAttribute(k_attn_mma, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        return true;
    }();
    (void)attr;
    k_attn_mma<<<ab.n * ab.batch * splits, kThreads, smem, st>>>(ab, splits, tps);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (ev) cudaEventRecord(ev[0], st);
    if (splits > 1) {
        dim3 g(ab.H, ab.batch, ab.n);
        k_attn_mma_combine<<<g, 128, 0, st>>>(ab, splits);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess && ev) cudaEventRecord(ev[1], st);
    return e;
}

}  // namespace csa2
