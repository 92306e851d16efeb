// Block-scaled FP8 quantisers ("RL at 1T scale: prime-rl performance deep
// dive", §FP8 Training: block-scaled FP8 as proposed by DeepSeek-V3) and the
// fused quantise-and-dispatch of a4.
//
// Rule for every block: amax = max |x| (exact, from bf16); scale =
// fp32(amax / 448) by IEEE division; code = cvt.rn.satfinite.e4m3(fp32(x /
// scale)) by IEEE division; a zero scale gives zero codes.  All kernels are
// HBM-bound moves: 16-byte vector loads and stores, one pass over the input.
#include "common.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// 1x128 blocks along a row, optionally scattered to k permuted rows.
// One warp per input row; lane l covers 16 columns of each 512-column step,
// so 8 lanes make one 128-block (amax by a 3-step xor butterfly).  The loads
// of up to four steps (2048 columns) are issued before any is used.
// Destination rows: pos == nullptr -> the row itself (k must be 1);
// otherwise row t goes to pos[t*k + j] for each j with pos >= 0.
// Codes q[p*ldq + c], scales sc[(c/128)*ld_s + p].
// kPad (dispatch): E * kPadWarps further warps zero the padding rows of the
// permuted layout, [offsets[e] + counts[e], offsets[e+1]) for each expert e,
// codes and scales, so the padded tiles of the grouped GEMMs read zeros.
// ---------------------------------------------------------------------------
constexpr int kPadWarps = 8;

template <bool kPad>
__global__ void __launch_bounds__(256) quant_1x128_kernel(const uint16_t *__restrict__ in, int64_t ld,
                                                          int64_t rows, int64_t cols,
                                                          const int32_t *__restrict__ pos, int k,
                                                          uint8_t *__restrict__ q, int64_t ldq,
                                                          float *__restrict__ sc, int64_t ld_s,
                                                          const int32_t *__restrict__ counts,
                                                          const int32_t *__restrict__ offsets, int E)
{
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= rows) {
        if (!kPad) return;
        const int64_t g = t - rows;
        const int e = (int)(g / kPadWarps), w = (int)(g % kPadWarps);
        if (e >= E) return;
        const int64_t r1 = offsets[e + 1];
        for (int64_t r = (int64_t)offsets[e] + counts[e] + w; r < r1; r += kPadWarps) {
            for (int64_t c = lane * 16; c < cols; c += 512)
                *reinterpret_cast<uint4 *>(q + r * ldq + c) = make_uint4(0, 0, 0, 0);
            for (int64_t kb = lane; kb < cols / 128; kb += 32) sc[kb * ld_s + r] = 0.0f;
        }
        return;
    }
    int my_pos = -1;
    if (pos) {
        if (lane < k) my_pos = pos[t * k + lane];
    } else if (lane == 0) {
        my_pos = (int)t;
    }
    const int kk = pos ? k : 1;
    const uint16_t *row = in + t * ld;
    for (int64_t g0 = 0; g0 < cols; g0 += 2048) {
        uint4 buf[8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t c = g0 + 512 * u + lane * 16;
            if (c < cols) {
                buf[2 * u] = *reinterpret_cast<const uint4 *>(row + c);
                buf[2 * u + 1] = *reinterpret_cast<const uint4 *>(row + c + 8);
            } else {
                buf[2 * u] = buf[2 * u + 1] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (g0 + 512 * u >= cols) break;  // warp-uniform
            const int64_t c = g0 + 512 * u + lane * 16;
            const bool act = c < cols;
            float v[16];
            unpack8(buf[2 * u], v);
            unpack8(buf[2 * u + 1], v + 8);
            float amax = act ? absmax8(v + 8, absmax8(v, 0.0f)) : 0.0f;
            amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
            amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 4));
            const float s = block_scale(amax);
            uint4 codes = make_uint4(0, 0, 0, 0);
            if (act) codes = quant16(v, s);
            const int64_t kb = c / 128;
            for (int j = 0; j < kk; ++j) {
                const int p = __shfl_sync(kFull, my_pos, j);
                if (p >= 0 && act) {
                    *reinterpret_cast<uint4 *>(q + (int64_t)p * ldq + c) = codes;
                    if ((lane & 7) == 0) sc[kb * ld_s + p] = s;
                }
            }
        }
    }
}

int launch_quant_1x128(const uint16_t *in, int64_t ld, int64_t rows, int64_t cols,
                       const int32_t *pos, int k, uint8_t *q, int64_t ldq, float *sc,
                       int64_t ld_s, cudaStream_t s)
{
    if (rows == 0) return MOE_OK;
    int64_t blocks = (rows + 7) / 8;
    quant_1x128_kernel<false><<<(unsigned)blocks, 256, 0, s>>>(in, ld, rows, cols, pos, k, q, ldq, sc, ld_s,
                                                               nullptr, nullptr, 0);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_dispatch_quant(const uint16_t *x, int64_t T, int64_t D, const int32_t *pos, int k, uint8_t *xq,
                          float *xs, int64_t R_cap, const int32_t *counts, const int32_t *offsets, int E,
                          cudaStream_t s)
{
    if (T == 0) return MOE_OK;  // no routed rows: every segment is empty, nothing to pad
    const int64_t warps = T + (int64_t)E * kPadWarps;
    quant_1x128_kernel<true><<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(x, D, T, D, pos, k, xq, D, xs, R_cap,
                                                                        counts, offsets, E);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// 128x1 blocks (128 rows of one column), written transposed:
//   qT[c*ld_rows + r], sT[(r/128)*cols + c].
// Row r of the source is in[r*ld], or, when src_idx != nullptr, the token row
// in[(src_idx[r]/k)*ld] (a zero row for src_idx[r] < 0): the gather that
// makes the permuted activation rows without materialising them.
// Block = 128 rows x 64 columns; 256 threads: thread (col = tid%64,
// part = tid/64) reduces 32 rows of its column and writes 32 codes.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quant_rows128_kernel(const uint16_t *__restrict__ in, int64_t ld,
                                                            const int32_t *__restrict__ src_idx, int k,
                                                            int64_t rows, int64_t cols, int64_t ld_rows,
                                                            uint8_t *__restrict__ qT,
                                                            float *__restrict__ sT)
{
    // bf16 tile, rows of 64 columns + 8 pad (144 B: 16-byte aligned rows, and a
    // warp's 32 consecutive columns of one row are 64 contiguous bytes)
    __shared__ __align__(16) uint16_t tile[128][72];
    __shared__ float part_max[4][64];
    const int tid = threadIdx.x;
    const int64_t r0 = (int64_t)blockIdx.x * 128;
    const int64_t c0 = (int64_t)blockIdx.y * 64;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        int idx = it * 256 + tid;  // 1024 16-byte pieces: 128 rows x 8
        int r = idx >> 3, cc = (idx & 7) * 8;
        int64_t gr = r0 + r;
        const uint16_t *src = nullptr;
        if (gr < rows) {
            if (src_idx) {
                int si = src_idx[gr];
                if (si >= 0) src = in + (int64_t)(si / k) * ld;
            } else {
                src = in + gr * ld;
            }
        }
        uint4 v = make_uint4(0, 0, 0, 0);
        if (src && c0 + cc < cols) v = *reinterpret_cast<const uint4 *>(src + c0 + cc);
        *reinterpret_cast<uint4 *>(&tile[r][cc]) = v;
    }
    __syncthreads();
    const int col = tid & 63, part = tid >> 6;
    float v[32];  // this thread's 32 rows of its column
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        v[i] = __uint_as_float((uint32_t)tile[part * 32 + i][col] << 16);
        amax = fmaxf(amax, fabsf(v[i]));
    }
    part_max[part][col] = amax;
    __syncthreads();
    amax = fmaxf(fmaxf(part_max[0][col], part_max[1][col]), fmaxf(part_max[2][col], part_max[3][col]));
    const float s = block_scale(amax);
    const int64_t gc = c0 + col;
    if (gc >= cols) return;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int64_t rr = r0 + part * 32 + h * 16;
        const uint4 codes = quant16(v + 16 * h, s);
        if (rr < rows) *reinterpret_cast<uint4 *>(qT + gc * ld_rows + rr) = codes;
    }
    if (part == 0) sT[(r0 / 128) * cols + gc] = s;
}

int launch_quant_rows128(const uint16_t *in, int64_t ld, const int32_t *src_idx, int k,
                         int64_t rows, int64_t cols, int64_t ld_rows, uint8_t *qT, float *sT,
                         cudaStream_t s)
{
    if (rows == 0 || cols == 0) return MOE_OK;
    dim3 grid((unsigned)((rows + 127) / 128), (unsigned)((cols + 63) / 64));
    quant_rows128_kernel<<<grid, 256, 0, s>>>(in, ld, src_idx, k, rows, cols, ld_rows, qT, sT);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Padding rows [offsets[e] + counts[e], offsets[e+1]) of a permuted 1x128
// matrix: zero codes (and bf16 copy) and zero scales.  One block per expert.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) pad_rows_kernel(const int32_t *__restrict__ counts,
                                                       const int32_t *__restrict__ offsets,
                                                       int64_t cols, int64_t R_cap,
                                                       uint8_t *__restrict__ q,
                                                       float *__restrict__ sc,
                                                       uint16_t *__restrict__ bf)
{
    const int e = blockIdx.x;
    const int64_t r0 = (int64_t)offsets[e] + counts[e], r1 = offsets[e + 1];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int64_t r = r0 + wid; r < r1; r += 8) {
        for (int64_t c = lane * 16; c < cols; c += 512) {
            if (q) *reinterpret_cast<uint4 *>(q + r * cols + c) = z;
            if (bf) {
                *reinterpret_cast<uint4 *>(bf + r * cols + c) = z;
                *reinterpret_cast<uint4 *>(bf + r * cols + c + 8) = z;
            }
        }
        if (sc)
            for (int64_t kb = lane; kb < cols / 128; kb += 32) sc[kb * R_cap + r] = 0.0f;
    }
}

int launch_pad_rows(const int32_t *counts, const int32_t *offsets, int E, int64_t cols,
                    int64_t R_cap, uint8_t *q, float *sc, uint16_t *bf, cudaStream_t s)
{
    if (E == 0) return MOE_OK;
    pad_rows_kernel<<<E, 256, 0, s>>>(counts, offsets, cols, R_cap, q, sc, bf);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// 128x128 blocks of a stack of matrices in[e] = in + e*in_expert_stride,
// [rows][cols] with row stride ld.  One block per (column block, row block,
// expert); 256 threads, each converting 8 contiguous elements of 8 rows.
// Output row block of source row block rb is rb*rb_mul + rb_add (this lays
// gate and up out interleaved by 128-row blocks).
//   q  [e]: codes at (dst row, c), row stride cols;
//   sc [e]: scale at dst_rb * nbc + cb;
//   qT [e] (nullable): codes of the transpose at (c, dst row), row stride qT_ld;
//   sT [e]: scale at cb * sT_ld + dst_rb.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quant_128x128_kernel(
    const uint16_t *__restrict__ in, int64_t rows, int64_t cols, int64_t ld, int64_t in_es,
    int rb_mul, int rb_add, uint8_t *__restrict__ q, int64_t q_es, float *__restrict__ sc,
    int64_t s_es, uint8_t *__restrict__ qT, int64_t qT_ld, int64_t qT_es, float *__restrict__ sT,
    int64_t sT_ld, int64_t sT_es)
{
    __shared__ float warp_max[8];
    __shared__ uint8_t codes_s[128][144];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t cb = blockIdx.x, rb = blockIdx.y, e = blockIdx.z;
    const int64_t nbc = (cols + 127) / 128;
    const uint16_t *src = in + e * in_es;
    const int cc = (tid & 15) * 8;   // column within the block
    const int rr0 = tid >> 4;        // rows rr0, rr0+16, ...
    float v[8][8];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int64_t r = rb * 128 + rr0 + 16 * i, c = cb * 128 + cc;
        if (r < rows && c < cols) {
            unpack8(*reinterpret_cast<const uint4 *>(src + r * ld + c), v[i]);
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) v[i][j] = 0.0f;
        }
        amax = absmax8(v[i], amax);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, off));
    if (lane == 0) warp_max[wid] = amax;
    __syncthreads();
    amax = warp_max[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, warp_max[i]);
    const float s = block_scale(amax);
    const int64_t drb = rb * rb_mul + rb_add;
    uint8_t *qe = q + e * q_es;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint2 c8 = quant8(v[i], s);
        int64_t r = rb * 128 + rr0 + 16 * i, c = cb * 128 + cc;
        if (r < rows && c < cols) *reinterpret_cast<uint2 *>(qe + (drb * 128 + rr0 + 16 * i) * cols + c) = c8;
        *reinterpret_cast<uint2 *>(&codes_s[rr0 + 16 * i][cc]) = c8;
    }
    if (tid == 0) sc[e * s_es + drb * nbc + cb] = s;
    if (!qT) return;
    __syncthreads();
    // transposed: tile column c -> 128 bytes of qT row (cb*128 + c); each
    // thread assembles 16 codes (rows 16*h .. 16*h+15) of one column.  A warp
    // takes 32 consecutive columns of the same rows (no shared-memory bank
    // conflicts: the rows 16 apart of one column would share a bank).
    uint8_t *qTe = qT + e * qT_es;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int c = tid & 127, h = 2 * it + (tid >> 7);  // 128 columns x 8 pieces
        uint32_t w[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            w[b] = (uint32_t)codes_s[16 * h + 4 * b][c] | ((uint32_t)codes_s[16 * h + 4 * b + 1][c] << 8) |
                   ((uint32_t)codes_s[16 * h + 4 * b + 2][c] << 16) |
                   ((uint32_t)codes_s[16 * h + 4 * b + 3][c] << 24);
        }
        int64_t gc = cb * 128 + c, gr = rb * 128 + 16 * h;
        if (gc < cols && gr < rows)
            *reinterpret_cast<uint4 *>(qTe + gc * qT_ld + drb * 128 + 16 * h) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (tid == 0) sT[e * sT_es + cb * sT_ld + drb] = s;
}

int launch_quant_128x128(const uint16_t *in, int64_t rows, int64_t cols, int64_t ld, int experts,
                         int64_t in_expert_stride, int rb_mul, int rb_add, uint8_t *q,
                         int64_t q_expert_stride, float *sc, int64_t s_expert_stride, uint8_t *qT,
                         int64_t qT_ld, int64_t qT_expert_stride, float *sT, int64_t sT_ld,
                         int64_t sT_expert_stride, cudaStream_t s)
{
    if (rows == 0 || cols == 0 || experts == 0) return MOE_OK;
    dim3 grid((unsigned)((cols + 127) / 128), (unsigned)((rows + 127) / 128), (unsigned)experts);
    quant_128x128_kernel<<<grid, 256, 0, s>>>(in, rows, cols, ld, in_expert_stride, rb_mul, rb_add, q,
                                              q_expert_stride, sc, s_expert_stride, qT, qT_ld,
                                              qT_expert_stride, sT, sT_ld, sT_expert_stride);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
