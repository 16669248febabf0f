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

// fp32 -> bf16 bits, round to nearest even, with integer operations only
// (keeps the conversion off the special-function pipe).  Finite inputs.
__device__ __forceinline__ uint32_t f32_to_bf16_bits_alu(float x) {
    const uint32_t u = __float_as_uint(x);
    return (u + 0x7fffu + ((u >> 16) & 1u)) >> 16;
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
// 4-bit code decoding for the dequant-GEMV ("subnormal" decode).
//
// A packed word holds codes q_0..q_7, q_j in bits 4j..4j+3.  With every other
// bit cleared, the word read as an fp32 is exactly q_j * 2^(4j - 149): a
// subnormal for j <= 4, and for j = 5 still q * 2^-129 because the code's top
// bit then lands in the exponent's lowest bit, where the smallest normal
// numbers continue the subnormal spacing (2^-126 + f * 2^-149).  Codes 6 and 7
// would land in the exponent proper, so they are first shifted down by 12
// bits, to the positions of codes 3 and 4.  One AND per code (plus one shift
// per word) therefore yields an fp32 proportional to the code, and with the
// input pre-scaled by 2^(100 - 4p) (p = the position the code is read at) the
// product with the code is exactly q * x * 2^-49 -- no offset, no
// cancellation.  Accumulated sums are multiplied back by 2^49 once per group.
// fp32 subnormals are handled at full speed by FFMA (no flush-to-zero: the
// library is built without fast-math).
// ---------------------------------------------------------------------------
constexpr float kCodeUnscale = 0x1p49f;

__host__ __device__ constexpr int code_pos(int j) { return j < 6 ? j : j - 3; }

// 2^(100 - 4 * code_pos(j)): built from its exponent field, so that a
// runtime j costs a few integer operations and no table or branch.
__host__ __device__ inline float code_prescale(int j) {
    const unsigned e = 127u + 100u - 4u * (unsigned)code_pos(j & 7);
#ifdef __CUDA_ARCH__
    return __uint_as_float(e << 23);
#else
    union { unsigned u; float f; } v{e << 23};
    return v.f;
#endif
}

// 1 / code_prescale(j) = 2^(4 * code_pos(j) - 100), exact.
__host__ __device__ inline float code_unprescale(int j) {
    const unsigned e = 127u - 100u + 4u * (unsigned)code_pos(j & 7);
#ifdef __CUDA_ARCH__
    return __uint_as_float(e << 23);
#else
    union { unsigned u; float f; } v{e << 23};
    return v.f;
#endif
}

struct Decoded8 {
    float f[8];
};

__device__ __forceinline__ Decoded8 decode_word(uint32_t w) {
    const uint32_t v = w >> 12;
    Decoded8 d;
    d.f[0] = __uint_as_float(w & 0x0000000fu);
    d.f[1] = __uint_as_float(w & 0x000000f0u);
    d.f[2] = __uint_as_float(w & 0x00000f00u);
    d.f[3] = __uint_as_float(w & 0x0000f000u);
    d.f[4] = __uint_as_float(w & 0x000f0000u);
    d.f[5] = __uint_as_float(w & 0x00f00000u);
    d.f[6] = __uint_as_float(v & 0x0000f000u);
    d.f[7] = __uint_as_float(v & 0x000f0000u);
    return d;
}

// Two fp32 FMAs in one packed instruction (sm_100): (a.x*b.x + c.x, a.y*b.y + c.y).
// The register pairs are formed inside the asm so the compiler can allocate
// them as pairs.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    asm("{\n .reg .b64 ra, rb, rc;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n mov.b64 rc, {%0, %1};\n"
        " fma.rn.f32x2 rc, ra, rb, rc;\n mov.b64 {%0, %1}, rc;\n}"
        : "+f"(c.x), "+f"(c.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return c;
}

// One word (8 codes) against 8 pre-scaled inputs, into two packed accumulators.
__device__ __forceinline__ void dot_word(uint32_t w, const float *xp, float2 &a0, float2 &a1) {
    const Decoded8 d = decode_word(w);
    const float4 xa = reinterpret_cast<const float4 *>(xp)[0], xb = reinterpret_cast<const float4 *>(xp)[1];
    a0 = ffma2(make_float2(d.f[0], d.f[1]), make_float2(xa.x, xa.y), a0);
    a1 = ffma2(make_float2(d.f[2], d.f[3]), make_float2(xa.z, xa.w), a1);
    a0 = ffma2(make_float2(d.f[4], d.f[5]), make_float2(xb.x, xb.y), a0);
    a1 = ffma2(make_float2(d.f[6], d.f[7]), make_float2(xb.z, xb.w), a1);
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
