// Device-side codecs and shared definitions of the CSA2 kernels (sm_100a).
//
// Every operation whose floating-point result decides a stored code uses an
// explicitly rounded intrinsic (__fmul_rn, __fmaf_rn, __fdiv_rn, ...) so that
// the compiler can neither contract nor reorder it: the packed cache is a pure
// function of the inputs, bit for bit.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "../../include/csa2.h"

namespace csa2 {

constexpr int D = 512;
constexpr int DI = 128;
constexpr int WIN = 128;
constexpr int PAGE = 64;
constexpr int MCB = 256;  // main code bytes per entry
constexpr int MSB = 32;   // main scale bytes per entry
constexpr int ICB = 64;   // indexer code bytes per entry
constexpr int ISB = 4;    // indexer scale bytes per entry

// ---------------------------------------------------------------- E2M1

// E2M1 code (nearest, ties to the even code, saturating at 6, sign kept) of v.
// The seven decision points are the midpoints between the eight magnitudes
// 0, .5, 1, 1.5, 2, 3, 4, 6; at a midpoint the even code wins, which makes
// the comparison strict (>) where the lower neighbour is even and non-strict
// (>=) where the upper neighbour is even.
__device__ __forceinline__ uint32_t e2m1_encode(float v) {
    float a = fabsf(v);
    uint32_t c = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) +
                 (a >= 3.5f) + (a > 5.0f);
    return c | ((__float_as_uint(v) >> 28) & 8u);
}

// Magnitude table of the 16 codes (sign in bit 3).
__device__ __forceinline__ float e2m1_decode(uint32_t code) {
    // 0, .5, 1, 1.5, 2, 3, 4, 6 as fp32 bit patterns: exponent field only
    // differs, mantissa is 0 or 0.5.
    const uint32_t m = code & 7u;
    float mag;
    if (m < 2)
        mag = 0.5f * (float)m;
    else
        mag = __uint_as_float(((126u + (m >> 1)) << 23) | ((m & 1u) << 22));
    return (code & 8u) ? -mag : mag;
}

// ---------------------------------------------------------------- E4M3

// Nearest-even E4M3 with saturation to +-448 (hardware cvt, sm_89+).
__device__ __forceinline__ uint32_t e4m3_encode(float v) {
    return (uint32_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

// Two E4M3 codes (low byte = first channel) -> fp16x2 bits (exact: every E4M3
// value is an fp16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t two) {
    uint32_t out;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(out) : "r"(two));
    return out;
}

// Exact fp32 value of a non-negative E4M3 code (the scales are never negative).
__device__ __forceinline__ float e4m3_decode_pos(uint32_t code) {
    const uint32_t e = (code >> 3) & 15u, m = code & 7u;
    if (e == 0) return __fmul_rn((float)m, 0.001953125f);  // m * 2^-9
    return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// ---------------------------------------------------------------- E8M0 / MX

// floor(log2(a)) for a finite a > 0, from the fp32 bits.
__device__ __forceinline__ int floor_log2_pos(float a) {
    uint32_t u = __float_as_uint(a);
    uint32_t be = u >> 23;
    if (be) return (int)be - 127;
    return (31 - __clz((int)u)) - 149;  // subnormal: m * 2^-149
}

// 2^k as fp32 for k in [-126, 127].
__device__ __forceinline__ float pow2i(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }

// OCP MX shared exponent for FP4 elements: floor(log2 amax) - 2, in [-127, 127].
__device__ __forceinline__ int mx_shared_exp(float amax) {
    int x = floor_log2_pos(amax) - 2;
    return x < -127 ? -127 : (x > 127 ? 127 : x);
}

// ---------------------------------------------------------------- fixed exp

// The cache write's fp32 exponential: Cody & Waite reduction by ln 2 (head
// with 15 significant bits so n * head is exact, plus a tail), degree-7
// Taylor polynomial of e^r in Horner form with fused multiply-adds, scaling by
// 2^n as two exact power-of-two factors.  Every step is one correctly rounded
// IEEE operation, so any implementation of this definition gives the same bits.
__device__ __forceinline__ float spec_exp(float x) {
    const float log2e = 1.44269502162933349609375f;
    const float ln2_hi = 0.693145751953125f;
    const float ln2_lo = 1.42860682030941723212e-6f;
    x = x > 89.0f ? 89.0f : x;
    x = x < -104.0f ? -104.0f : x;
    const float n = rintf(__fmul_rn(x, log2e));
    float r = __fmaf_rn(-n, ln2_hi, x);
    r = __fmaf_rn(-n, ln2_lo, r);
    float p = __fdiv_rn(1.0f, 5040.0f);
    p = __fmaf_rn(p, r, __fdiv_rn(1.0f, 720.0f));
    p = __fmaf_rn(p, r, __fdiv_rn(1.0f, 120.0f));
    p = __fmaf_rn(p, r, __fdiv_rn(1.0f, 24.0f));
    p = __fmaf_rn(p, r, __fdiv_rn(1.0f, 6.0f));
    p = __fmaf_rn(p, r, 0.5f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    const int ni = (int)n;
    const int n1 = ni / 2, n2 = ni - n1;
    return __fmul_rn(__fmul_rn(p, pow2i(n1)), pow2i(n2));
}

// ---------------------------------------------------------------- misc

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
    return __uint_as_float((uint32_t)b << 16);
}

// Order-preserving map fp32 -> uint32 (larger float <=> larger key).
__device__ __forceinline__ uint32_t f32_order_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float order_key_f32(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Device view of one cache (plain values, passed by value to kernels).
struct CacheView {
    uint8_t* main_codes;
    uint8_t* main_scales;
    uint8_t* idx_codes;
    uint8_t* idx_scales;
    const int32_t* page_table;
    int32_t* n_entries;
    float* pend_x;
    float* pend_g;
    int32_t* pend_valid;
    uint32_t* status;
    int32_t batch, max_pages, num_pages, ratio;
};

inline CacheView view_of(const csa2_cache& c) {
    return CacheView{c.main_codes, c.main_scales, c.idx_codes, c.idx_scales, c.page_table,
                     c.n_entries,  c.pend_x,      c.pend_g,    c.pend_valid, c.status,
                     c.batch,      c.max_pages,   c.num_pages, c.ratio};
}

// Physical page of logical entry e of sequence b, or -1 (and a status bit)
// when the page table points outside the pool.
__device__ __forceinline__ int page_of(const CacheView& c, int b, int e) {
    int p = c.page_table[(int64_t)b * c.max_pages + e / PAGE];
    if (p < 0 || p >= c.num_pages) {
        atomicOr(c.status, CSA2_DEVERR_PAGE);
        return -1;
    }
    return p;
}

// Entry count of sequence b clamped to the table's capacity.
__device__ __forceinline__ int entries_of(const CacheView& c, int b) {
    int n = c.n_entries[b];
    int cap = c.max_pages * PAGE;
    if (n < 0 || n > cap) {
        atomicOr(c.status, CSA2_DEVERR_COUNT);
        n = n < 0 ? 0 : cap;
    }
    return n;
}

}  // namespace csa2
