// Device helpers shared by the kernels of libmoe.so (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

constexpr unsigned kFull = 0xffffffffu;

// First error wins; the word is read and cleared by moe_get_status().
__device__ __forceinline__ void latch_status(int *status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// fp32 -> bf16 bits, round to nearest even, on the integer pipe: finite
// values round as the IEEE conversion does (overflow goes to infinity); a NaN
// becomes the canonical bf16 NaN 0x7fff.
__device__ __forceinline__ uint32_t bf16_bits_rn(float f)
{
    const uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return 0x7fffu;
    return (u + 0x7fffu + ((u >> 16) & 1u)) >> 16;
}

// Two fp32 -> packed bf16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// 8 bf16 (one 16-byte vector) -> 8 floats.
__device__ __forceinline__ void unpack8(const uint4 &u, float *v)
{
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x);
    v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z);
    v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}

__device__ __forceinline__ uint4 pack8(const float *v)
{
    return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                      pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

// Two fp32 -> two e4m3fn codes (lo in byte 0), round to nearest even,
// saturating to +-448 (the hardware conversion).
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi)
{
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return (uint32_t)r;
}

// Scale of a block: fp32(amax / 448), IEEE division.
__device__ __forceinline__ float block_scale(float amax) { return __fdiv_rn(amax, 448.0f); }

// (d0, d1) = (a0 * b0 + c0, a1 * b1 + c1) on two fp32 lanes at once (packed
// f32x2), each rounded once to nearest even
__device__ __forceinline__ void ffma2x(float &d0, float &d1, float a0, float a1, float b0, float b1, float c0,
                                       float c1)
{
    asm("{\n\t.reg .b64 a, b, c, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "mov.b64 c, {%6, %7};\n\tfma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

// (a0, a1) += (p0 * s0, p1 * s1), packed f32x2, each rounded once
__device__ __forceinline__ void ffma2(float &a0, float &a1, float p0, float p1, float s0, float s1)
{
    asm("{\n\t.reg .b64 a, p, q;\n\tmov.b64 a, {%0, %1};\n\tmov.b64 p, {%2, %3};\n\t"
        "mov.b64 q, {%4, %5};\n\tfma.rn.f32x2 a, p, q, a;\n\tmov.b64 {%0, %1}, a;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "f"(p0), "f"(p1), "f"(s0), "f"(s1));
}

// (r0, r1) = (a0 * b0, a1 * b1), packed f32x2, each rounded once
__device__ __forceinline__ void fmul2(float &r0, float &r1, float a0, float a1, float b0, float b1)
{
    asm("{\n\t.reg .b64 a, b, r;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "mul.rn.f32x2 r, a, b;\n\tmov.b64 {%0, %1}, r;\n\t}"
        : "=f"(r0), "=f"(r1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// The e4m3 codes of the correctly rounded quotients RN_fp32(x / s), without a
// divide per element: Markstein's correction of a quotient by a correctly
// rounded reciprocal (P. Markstein, "Computation of elementary functions on
// the IBM RISC System/6000 processor", IBM J. Res. Develop. 34(1), 1990):
//   r = RN(1/s),  q0 = RN(x r),  e = x - q0 s (one FMA, exact),  q = RN(q0 + e r).
// Every quantiser here feeds it bf16 values x with |x| <= amax, amax a bf16
// value and s = RN(amax / 448).  On that domain q = RN(x / s) whenever
// |x / s| >= 2^-12, and below that both round to a zero code (with x's sign);
// an exhaustive host check over every bf16 x against every bf16 amax mantissa,
// across the exponent range, found no other case.  Scales below 2^-90 (r above
// 2^90) and non-finite scales take IEEE division instead, out of line.
// Each step runs on two elements at once (packed f32x2) with -r in place of r:
// the chain then computes -q0, e and -q, exactly the negatives (rounding to
// nearest is symmetric), so a zero quotient comes out with the sign opposite
// to x's; the four codes' sign bits are flipped together at the end.
template <int n>
struct Floats {
    float v[n];
};

template <int n>
__device__ __noinline__ Floats<n> quotients_exact(Floats<n> x, float s)
{
    Floats<n> q;
#pragma unroll
    for (int i = 0; i < n; ++i) q.v[i] = __fdiv_rn(x.v[i], s);
    return q;
}

// w[i] = codes of v[4i .. 4i+3] (element 4i + j in byte j); s > 0.
template <int n>
__device__ __forceinline__ void e4m3_codes(const float *v, float s, uint32_t *w)
{
    static_assert(n % 4 == 0, "groups of four");
    const float r = __frcp_rn(s);
    if (!(r <= 0x1p90f) || r == 0.0f) {  // s below about 2^-90 (or not finite): IEEE division, out of line
        Floats<n> x;
#pragma unroll
        for (int i = 0; i < n; ++i) x.v[i] = v[i];
        const Floats<n> q = quotients_exact<n>(x, s);
#pragma unroll
        for (int i = 0; i < n / 4; ++i)
            w[i] = e4m3x2(q.v[4 * i], q.v[4 * i + 1]) | (e4m3x2(q.v[4 * i + 2], q.v[4 * i + 3]) << 16);
        return;
    }
    const float nr = -r;
#pragma unroll
    for (int i = 0; i < n / 4; ++i) {
        const float *x = v + 4 * i;
        float a0, a1, a2, a3, e0, e1, e2, e3, q0, q1, q2, q3;
        fmul2(a0, a1, x[0], x[1], nr, nr);             // -q0
        fmul2(a2, a3, x[2], x[3], nr, nr);
        ffma2x(e0, e1, a0, a1, s, s, x[0], x[1]);      // x - q0 s
        ffma2x(e2, e3, a2, a3, s, s, x[2], x[3]);
        ffma2x(q0, q1, e0, e1, nr, nr, a0, a1);        // -(q0 + e r)
        ffma2x(q2, q3, e2, e3, nr, nr, a2, a3);
        w[i] = (e4m3x2(q0, q1) | (e4m3x2(q2, q3) << 16)) ^ 0x80808080u;
    }
}

// Sixteen codes; a zero scale gives zero codes.
__device__ __forceinline__ uint4 quant16(const float *v, float s)
{
    if (s == 0.0f) return make_uint4(0, 0, 0, 0);
    uint32_t w[4];
    e4m3_codes<16>(v, s, w);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Four codes (element i in byte i); a zero scale gives zero codes.
__device__ __forceinline__ uint32_t quant4(const float *v, float s)
{
    if (s == 0.0f) return 0u;
    uint32_t w;
    e4m3_codes<4>(v, s, &w);
    return w;
}

__device__ __forceinline__ uint2 quant8(const float *v, float s)
{
    if (s == 0.0f) return make_uint2(0, 0);
    uint32_t w[2];
    e4m3_codes<8>(v, s, w);
    return make_uint2(w[0], w[1]);
}

// sigmoid(g) for the SiLU gate, fast intrinsics (h and its gradient are
// compared within a tolerance, not bit for bit).  exp(80) < 2^126 keeps the
// fast division in range; below g = -80 the sigmoid is 0 in fp32 anyway.
__device__ __forceinline__ float sigmoid_fast(float g)
{
    return __fdividef(1.0f, 1.0f + __expf(-fmaxf(g, -80.0f)));
}

__device__ __forceinline__ float absmax8(const float *v, float m)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
    return m;
}

}  // namespace moe

#include "launch.h"
