// moe_common.cuh -- device helpers shared by the MoE kernels (CUDA side only).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/moe_api.h"

namespace moe {

constexpr int kWarp = 32;
constexpr int kGroup = 64;      // quantisation group along the input dimension
constexpr int kRowBlock = 32;   // rows per tiled block (one per lane)
constexpr int kChunkCols = 32;  // columns per 16-byte chunk of 4-bit codes
constexpr int kMaxK = 32;
constexpr int kMaxE = 1024;

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
    return __uint_as_float(bits16 << 16);
}

// fp64 -> bf16 bits, round to nearest even in a single rounding.  The value
// is first narrowed to fp32 with round-to-odd (truncate, then set the last
// bit if anything was dropped), which keeps enough information for the
// following round-to-nearest-even to bf16 to be correctly rounded (Boldo and
// Melquiond, "Emulation of FMA and correctly rounded sums: proved algorithms
// using rounding to odd", IEEE TC 2008): fp32 carries 16 more bits than bf16.
__device__ __forceinline__ uint16_t f64_to_bf16_bits(double x) {
    float t = __double2float_rz(x);
    uint32_t u = __float_as_uint(t);
    if ((double)t != x && (u & 0x7f800000u) != 0x7f800000u) u |= 1u;
    return __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(u)));
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Block-wide sum; every thread gets the result.  `red` needs blockDim/32 slots.
template <typename T>
__device__ __forceinline__ T block_sum(T v, T *red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[wid] = v;
    __syncthreads();
    T s = T(0);
    for (int i = 0; i < nw; ++i) s += red[i];  // fixed order: deterministic
    return s;
}

// ---------------------------------------------------------------------------
// 4-bit code decoding for the dequant-GEMV.
//
// For a packed word holding codes q_0..q_7 (q_j in bits 4j..4j+3), build for
// each j the fp32 value f_j = 1 + q_j * c_j, exactly, by OR-ing the code into
// the fraction of 1.0f at bits 16..19 (c = 2^-7) or 12..15 (c = 2^-11).  With
// the input pre-scaled as x'_j = x_j / c_j,
//     sum_j f_j * x'_j = sum_j x'_j + sum_j q_j * x_j,
// so one FMA per code accumulates q*x, and the per-chunk constant sum_j x'_j
// is subtracted once.  c_j depends only on j = column % 8:
//     j : 0     1      2     3      4     5      6     7
//     c : 2^-7  2^-11  2^-7  2^-11  2^-7  2^-11  2^-7  2^-7
// ---------------------------------------------------------------------------
__host__ __device__ constexpr float code_prescale(int j) {
    return (j == 1 || j == 3 || j == 5) ? 2048.0f : 128.0f;
}

struct Decoded8 {
    float f[8];
};

__device__ __forceinline__ Decoded8 decode_word(uint32_t w) {
    constexpr uint32_t kOne = 0x3f800000u;
    const uint32_t w8 = w << 8, w16 = w << 16, v8 = w >> 8, v12 = w >> 12;
    Decoded8 d;
    d.f[0] = __uint_as_float((w16 & 0x000f0000u) | kOne);
    d.f[1] = __uint_as_float((w8 & 0x0000f000u) | kOne);
    d.f[2] = __uint_as_float((w8 & 0x000f0000u) | kOne);
    d.f[3] = __uint_as_float((w & 0x0000f000u) | kOne);
    d.f[4] = __uint_as_float((w & 0x000f0000u) | kOne);
    d.f[5] = __uint_as_float((v8 & 0x0000f000u) | kOne);
    d.f[6] = __uint_as_float((v8 & 0x000f0000u) | kOne);
    d.f[7] = __uint_as_float((v12 & 0x000f0000u) | kOne);
    return d;
}

// Two fp32 FMAs in one packed instruction (sm_100): (a.x*b.x + c.x, a.y*b.y + c.y).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    unsigned long long ra, rb, rc, rd;
    ra = (unsigned long long)__float_as_uint(a.x) | ((unsigned long long)__float_as_uint(a.y) << 32);
    rb = (unsigned long long)__float_as_uint(b.x) | ((unsigned long long)__float_as_uint(b.y) << 32);
    rc = (unsigned long long)__float_as_uint(c.x) | ((unsigned long long)__float_as_uint(c.y) << 32);
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
    return make_float2(__uint_as_float((uint32_t)rd), __uint_as_float((uint32_t)(rd >> 32)));
}

// 16 bytes = 32 codes of one row against 32 pre-scaled inputs (two float4 x
// 4).  Returns sum_j f_j * x'_j accumulated as two interleaved partial sums.
__device__ __forceinline__ float dot_chunk(const uint4 q, const float4 *xp) {
    float2 acc = make_float2(0.f, 0.f);
    const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const Decoded8 d = decode_word(words[i]);
        const float4 xa = xp[2 * i], xb = xp[2 * i + 1];
        acc = ffma2(make_float2(d.f[0], d.f[1]), make_float2(xa.x, xa.y), acc);
        acc = ffma2(make_float2(d.f[2], d.f[3]), make_float2(xa.z, xa.w), acc);
        acc = ffma2(make_float2(d.f[4], d.f[5]), make_float2(xb.x, xb.y), acc);
        acc = ffma2(make_float2(d.f[6], d.f[7]), make_float2(xb.z, xb.w), acc);
    }
    return acc.x + acc.y;
}

__device__ __forceinline__ uint4 ldg_nc_v4(const uint32_t *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t ldg_nc_u32(const uint32_t *p) {
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
    return g / (1.0f + expf(-g)) * u;
}

}  // namespace moe
