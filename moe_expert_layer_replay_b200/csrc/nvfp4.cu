// NVFP4 block quantisation: e2m1 elements in 16-element blocks along a row,
// an e4m3 scale per block and an fp32 scale per tensor (NVIDIA's NVFP4; the
// format Blackwell's tensor cores take with hardware block scales, named as
// future work in "RL at 1T scale: prime-rl performance deep dive", §Future
// work).
//
// Rule (every step IEEE fp32, rounding to nearest even):
//   amax_t = max |x| over the tensor; s_g = 2688 / amax_t (1 if amax_t = 0);
//   per block: s_b = amax_b / 6; S8 = e4m3 satfinite (s_b * s_g); S_b = value of S8;
//   codes: 0 if S_b = 0, else e2m1 satfinite (x * (s_g / S_b)).
// Two launches: the tensor amax (a max is order-free: every block folds its
// maximum into one word with an integer atomicMax on the non-negative float
// bits), then one thread per 16-element block.
#include "common.cuh"

namespace moe {
namespace nvfp4 {

// Eight fp32 -> eight e2m1 codes, element i in bits 4i..4i+3 (round to
// nearest even, saturate to +-6: the hardware conversion).
__device__ __forceinline__ uint32_t e2m1x8(const float *v)
{
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// The value of an e4m3 code (exact: e4m3 values are fp16 values).
__device__ __forceinline__ float e4m3_value(uint32_t code)
{
    uint32_t h2;
    asm("{\n\t.reg .b16 c;\n\tcvt.u16.u32 c, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}" : "=r"(h2) : "r"(code));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu)));
}

__device__ __forceinline__ float tensor_scale(float amax) { return amax > 0.0f ? __fdiv_rn(2688.0f, amax) : 1.0f; }

__global__ void __launch_bounds__(256) amax_kernel(const uint16_t *__restrict__ in, int64_t rows, int64_t cols,
                                                   int64_t ld, float *__restrict__ amax)
{
    __shared__ float wmax[8];
    const int64_t per_row = cols / 8;   // 16-byte pieces
    const int64_t n = rows * per_row;
    float m = 0.0f;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / per_row, c = (i - r * per_row) * 8;
        float v[8];
        unpack8(*reinterpret_cast<const uint4 *>(in + r * ld + c), v);
        m = absmax8(v, m);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < 8; ++w) m = fmaxf(m, wmax[w]);
        atomicMax(reinterpret_cast<int *>(amax), __float_as_int(m));
    }
}

// The block-scaled MMA's scale layouts (as tcgen05.cp 128x256b copies them
// into TMEM, four copies of every scale, one per TMEM lane quarter).  A 4096-
// byte block holds, for TMEM lane l (0..127) and half h, the 16 bytes of
// "line" l % 32 of one 128-row, 64-element atom (row 32 r1 + l % 32, group j
// at byte 4 r1 + j), at (l >> 3) * 256 + h * 128 + (l & 7) * 16: 8-row core
// matrices, the two halves 128 bytes apart, row groups 256 bytes apart.
//   A side: block (row block rb, K-step pair kp) at (rb * cols/128 + kp) *
//           4096, half h = K step 2 kp + h;
//   B side: block (row-block pair rbp, K step ks) at (rbp * cols/64 + ks) *
//           4096, half h = row block 2 rbp + h.
// Byte offset of the copy for lane quarter q of the scale of (row r, group b).
__device__ __forceinline__ int64_t sf_mma_offset(int64_t r, int64_t b, int64_t cols, bool b_side, int q)
{
    const int64_t rb = r >> 7, rr = r & 127, ks = b >> 2, j = b & 3;
    const int64_t l = 32 * q + (rr & 31), byte = ((rr >> 5) << 2) + j;
    const int64_t blk = b_side ? ((rb >> 1) * (cols / 64) + ks) : (rb * (cols / 128) + (ks >> 1));
    const int64_t h = b_side ? (rb & 1) : (ks & 1);
    return (blk << 12) + ((l >> 3) << 8) + (h << 7) + ((l & 7) << 4) + byte;
}

__global__ void __launch_bounds__(256) quant_kernel(const uint16_t *__restrict__ in, int64_t rows, int64_t cols,
                                                    int64_t ld, const float *__restrict__ amax,
                                                    uint8_t *__restrict__ q, uint8_t *__restrict__ sf, int sf_layout,
                                                    float *__restrict__ s_g_out)
{
    const float s_g = tensor_scale(*amax);
    if (blockIdx.x == 0 && threadIdx.x == 0) *s_g_out = s_g;
    const int64_t nb = cols / 16;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows * nb) return;
    const int64_t r = i / nb, b = i - r * nb;
    const uint16_t *src = in + r * ld + 16 * b;
    float v[16];
    unpack8(*reinterpret_cast<const uint4 *>(src), v);
    unpack8(*reinterpret_cast<const uint4 *>(src + 8), v + 8);
    const float s_b = __fdiv_rn(absmax8(v + 8, absmax8(v, 0.0f)), 6.0f);
    const uint32_t code = e4m3x2(__fmul_rn(s_b, s_g), 0.0f) & 0xffu;   // the low element's code
    const float S_b = e4m3_value(code);
    uint2 out = make_uint2(0, 0);
    if (S_b > 0.0f) {
        const float inv = __fdiv_rn(s_g, S_b);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = __fmul_rn(v[j], inv);
        out = make_uint2(e2m1x8(v), e2m1x8(v + 8));
    }
    *reinterpret_cast<uint2 *>(q + r * (cols / 2) + 8 * b) = out;
    if (sf_layout == 0) {
        sf[r * nb + b] = (uint8_t)code;
    } else {
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) sf[sf_mma_offset(r, b, cols, sf_layout == 2, qq)] = (uint8_t)code;
    }
}

}  // namespace nvfp4

int launch_quant_nvfp4(const uint16_t *in, int64_t rows, int64_t cols, int64_t ld, uint8_t *q, uint8_t *sf,
                       int sf_layout, float *amax, float *s_g, int sms, cudaStream_t s)
{
    if (cudaMemsetAsync(amax, 0, sizeof(float), s) != cudaSuccess) return MOE_ERR_CUDA;
    if (rows > 0) {
        const int64_t pieces = rows * (cols / 8);
        const int64_t want = (pieces + 255) / 256;
        const unsigned grid = (unsigned)(want < 8 * (int64_t)sms ? want : 8 * (int64_t)sms);
        nvfp4::amax_kernel<<<grid, 256, 0, s>>>(in, rows, cols, ld, amax);
        count_launch();
    }
    const int64_t blocks = rows * (cols / 16);
    nvfp4::quant_kernel<<<(unsigned)((blocks + 255) / 256 > 0 ? (blocks + 255) / 256 : 1), 256, 0, s>>>(
        in, rows, cols, ld, amax, q, sf, sf_layout, s_g);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
