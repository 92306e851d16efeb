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

// The e4m3 code of the correctly rounded quotient q = RN_fp32(x / s),
// without a divide per element and without a branch.
//
// With r = RN(1/s), q' = RN(x * r) = (x/s)(1 + d), |d| < 3 * 2^-24, so q' is
// within 3 fp32 ulps of q.  Let M be the e4m3 rounding midpoint of the bracket
// [V_j, V_j+1) of e4m3 values that holds q'.  In e4m3's normal range M has
// q''s sign, exponent and top three mantissa bits, then a 1 (20 low mantissa
// bits 0x80000).  Below 2^-6 (e4m3's subnormal grid, step 2^-9) the midpoints
// are the odd multiples of 2^-10: adding 2^-6 with rounding toward zero maps
// q' into [2^-6, 2^-5), whose brackets are the same 2^-9 steps (the boundaries
// are representable, so the truncated sum lies in the exact sum's bracket).
//
// q rounds like M's neighbours: q > M iff x/s > M + u/2, q < M iff x/s <
// M - u/2, else q == M (u = fp32 ulp of M; M has 4 significant bits, so its
// last fp32 mantissa bit is 0 and ties at M +- u/2 round to M; the one
// midpoint that is a power of two, 2^-10, ties down to code 0 either way).
// The test compares e = fma(-M, s, |x|) with c = s * u/2 (exact: a power-of-two
// multiple of s):
//   - when q' is within 4 ulps of M, x - M*s is a small multiple of the grid
//     of M*s (at most 11 significant bits), so e is that difference exactly;
//   - otherwise |x/s - M| > 1 ulp of M (1.5 * 2^-29 below 2^-6), so |x - M*s|
//     > 2c and the rounded e falls on the same side of +-c as the exact one.
// The element then converts through M or its fp32 neighbour on the decided
// side, which e4m3 rounds like q.  Scales below 2^-90 use IEEE division:
// from there up, c (>= s * 2^-34) and the grid of M*s (>= 2^-126 for M >=
// 2^-10) stay in fp32's normal range, so neither is rounded.
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

// Values whose e4m3 conversion equals that of fp32(v[i] / s), s != 0.
template <int n>
__device__ __forceinline__ void quotients(const float *v, float s, float *q)
{
    const float r = __frcp_rn(s);
    if (!(r <= 0x1p90f)) {  // s below about 2^-90: IEEE division, out of line
        Floats<n> x;
#pragma unroll
        for (int i = 0; i < n; ++i) x.v[i] = v[i];
        const Floats<n> e = quotients_exact<n>(x, s);
#pragma unroll
        for (int i = 0; i < n; ++i) q[i] = e.v[i];
        return;
    }
    const float s24 = s * 0x1p-24f;  // u/2 * s = s24 * 2^exponent(M), exact
#pragma unroll
    for (int i = 0; i < n; ++i) {
        const float qp = __fmul_rn(v[i], r);
        const uint32_t b = __float_as_uint(qp) & 0x7fffffffu;
        const bool sub = b < 0x3c800000u;
        const uint32_t y = sub ? __float_as_uint(__fadd_rz(__uint_as_float(b), 0x1p-6f)) : b;
        const float My = __uint_as_float((y & 0xfff00000u) | 0x00080000u);
        const float M = sub ? __fsub_rn(My, 0x1p-6f) : My;
        const float c = __fmul_rn(s24, __uint_as_float(__float_as_uint(M) & 0x7f800000u));
        const float e = __fmaf_rn(-M, s, fabsf(v[i]));
        const uint32_t mb = __float_as_uint(M) + (e > c ? 1u : 0u) - (e < -c ? 1u : 0u);
        q[i] = __uint_as_float(mb | (__float_as_uint(qp) & 0x80000000u));
    }
}

// Sixteen codes; a zero scale gives zero codes.
__device__ __forceinline__ uint4 quant16(const float *v, float s)
{
    if (s == 0.0f) return make_uint4(0, 0, 0, 0);
    float q[16];
    quotients<16>(v, s, q);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = e4m3x2(q[4 * i], q[4 * i + 1]) | (e4m3x2(q[4 * i + 2], q[4 * i + 3]) << 16);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Four codes (element i in byte i); a zero scale gives zero codes.
__device__ __forceinline__ uint32_t quant4(const float *v, float s)
{
    if (s == 0.0f) return 0u;
    float q[4];
    quotients<4>(v, s, q);
    return e4m3x2(q[0], q[1]) | (e4m3x2(q[2], q[3]) << 16);
}

__device__ __forceinline__ uint2 quant8(const float *v, float s)
{
    if (s == 0.0f) return make_uint2(0, 0);
    float q[8];
    quotients<8>(v, s, q);
    return make_uint2(e4m3x2(q[0], q[1]) | (e4m3x2(q[2], q[3]) << 16),
                      e4m3x2(q[4], q[5]) | (e4m3x2(q[6], q[7]) << 16));
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

// Launchers (host side, one per kernel family), defined in the .cu files.
namespace moe {
// Counts one kernel launch (or one launch recorded into a stream capture);
// read by moe_kernel_launches().
void count_launch();
int launch_route_topk(const float *z, int T, int E, int k, int32_t *idx, float *w, cudaStream_t s);
int launch_route_replay(const int32_t *P, int layer, int T, int E, int k, const float *w_in,
                        const float *z, int32_t *idx, float *w, int *status, cudaStream_t s);
int launch_permute_index(const int32_t *idx, int T, int k, int E, int align, int32_t *counts,
                         int32_t *offsets, int32_t *pos, int32_t *src_idx, int64_t R_cap,
                         void *ws, int *status, cudaStream_t s);
size_t permute_ws_bytes(int T, int k, int E);
int launch_quant_1x128(const uint16_t *in, int64_t ld, int64_t rows, int64_t cols,
                       const int32_t *pos, int k, uint8_t *q, int64_t ldq, float *sc,
                       int64_t ld_s, cudaStream_t s);
int launch_dispatch_quant(const uint16_t *x, int64_t T, int64_t D, const int32_t *pos, int k, uint8_t *xq,
                          float *xs, int64_t R_cap, const int32_t *counts, const int32_t *offsets, int E,
                          cudaStream_t s);
int launch_quant_rows128(const uint16_t *in, int64_t ld, const int32_t *src_idx, int k,
                         int64_t rows, int64_t cols, int64_t ld_rows, uint8_t *qT, float *sT,
                         cudaStream_t s);
int launch_pad_rows(const int32_t *counts, const int32_t *offsets, int E, int64_t cols,
                    int64_t R_cap, uint8_t *q, float *sc, uint16_t *bf, cudaStream_t s);
int launch_quant_128x128(const uint16_t *in, int64_t rows, int64_t cols, int64_t ld, int experts,
                         int64_t in_expert_stride, int rb_mul, int rb_add, uint8_t *q,
                         int64_t q_expert_stride, float *sc, int64_t s_expert_stride, uint8_t *qT,
                         int64_t qT_ld, int64_t qT_expert_stride, float *sT, int64_t sT_ld,
                         int64_t sT_expert_stride, cudaStream_t s);
size_t router_bwd_ws_bytes(int T, int D, int E);
int launch_router_logits(const uint16_t *x, const uint16_t *w_r, int T, int D, int E, float *z, int *status,
                         uint64_t budget, cudaStream_t s);
int launch_capture(const int32_t *idx, int T, int k, int layer, int32_t *payload, cudaStream_t s);
int launch_router_bwd(const float *dz, const uint16_t *x, const uint16_t *w_r, int T, int D, int E,
                      const uint16_t *dx_in, uint16_t *dx, float *dw_r, void *ws, cudaStream_t s);
int launch_quant_nvfp4(const uint16_t *in, int64_t rows, int64_t cols, int64_t ld, uint8_t *q, uint8_t *sf,
                       float *amax, float *s_g, int sms, cudaStream_t s);
int launch_combine(const uint16_t *Y, const float *w, const int32_t *pos, int T, int D, int k,
                   uint16_t *y, cudaStream_t s);
int launch_combine_bwd(const uint16_t *dy, const uint16_t *Y, const float *w, const int32_t *pos,
                       const int32_t *idx, int T, int D, int k, int E, int64_t R_cap,
                       uint8_t *dYq, float *dYs, uint16_t *dYb, float *d_w, float *d_logits,
                       cudaStream_t s);
}  // namespace moe
