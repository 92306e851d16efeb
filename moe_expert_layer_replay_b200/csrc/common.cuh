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

__device__ __forceinline__ uint32_t bf16_bits_rn(float f)
{
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    return bf16_bits_rn(lo) | (bf16_bits_rn(hi) << 16);
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

// Four codes of fp32(v / s), s != 0.
__device__ __forceinline__ uint32_t quant4(const float *v, float s)
{
    return e4m3x2(__fdiv_rn(v[0], s), __fdiv_rn(v[1], s)) |
           (e4m3x2(__fdiv_rn(v[2], s), __fdiv_rn(v[3], s)) << 16);
}

// Sixteen codes; a zero scale gives zero codes.
__device__ __forceinline__ uint4 quant16(const float *v, float s)
{
    if (s == 0.0f) return make_uint4(0, 0, 0, 0);
    return make_uint4(quant4(v, s), quant4(v + 4, s), quant4(v + 8, s), quant4(v + 12, s));
}

__device__ __forceinline__ uint2 quant8(const float *v, float s)
{
    if (s == 0.0f) return make_uint2(0, 0);
    return make_uint2(quant4(v, s), quant4(v + 4, s));
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
int launch_combine(const uint16_t *Y, const float *w, const int32_t *pos, int T, int D, int k,
                   uint16_t *y, cudaStream_t s);
int launch_combine_bwd(const uint16_t *dy, const uint16_t *Y, const float *w, const int32_t *pos,
                       const int32_t *idx, int T, int D, int k, int E, int64_t R_cap,
                       uint8_t *dYq, float *dYs, uint16_t *dYb, float *d_w, float *d_logits,
                       cudaStream_t s);
}  // namespace moe
