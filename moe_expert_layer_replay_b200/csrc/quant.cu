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
// Tiles of 128 rows x 64 columns; a persistent grid sized to the blocks the
// SMs hold at once.  Each block keeps the copies of its next two tiles in
// flight (cp.async into a three-slot ring in shared memory, 16 bytes a copy,
// zero-filled for missing rows) while it quantises the current one.  256
// threads: thread (col = tid%64, part = tid/64) reduces 32 rows of its column
// and writes 32 codes.  Row blocks vary fastest, so the blocks in flight
// share their column block: their codes fill whole lines of the transposed
// output, and, gathering, the token rows they read stay in L2 for the k
// permuted rows that repeat them.
// ---------------------------------------------------------------------------
constexpr int kR128Pad = 72;   // bf16 per tile row: 144 B, 16-byte aligned rows
constexpr int kR128Slots = 3;
constexpr int kR128Smem = kR128Slots * 128 * kR128Pad * 2;

__device__ __forceinline__ void cp_async16_zfill(void *dst, const void *src, uint32_t bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit_group() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int n>
__device__ __forceinline__ void cp_async_wait_groups() { asm volatile("cp.async.wait_group %0;" ::"n"(n) : "memory"); }

__global__ void __launch_bounds__(256, 4) quant_rows128_kernel(const uint16_t *__restrict__ in, int64_t ld,
                                                            const int32_t *__restrict__ src_idx, int k,
                                                            int64_t rows, int64_t cols, int64_t ld_rows,
                                                            uint8_t *__restrict__ qT,
                                                            float *__restrict__ sT)
{
    extern __shared__ __align__(16) uint16_t ring[];   // [kR128Slots][128][kR128Pad]
    __shared__ float part_max[4][64];
    const int tid = threadIdx.x;
    const int64_t ntr = (rows + 127) / 128, ntiles = ntr * ((cols + 63) / 64);
    // the source row of each of this thread's four pieces of tile t (-1: zeros);
    // gathering, the indices are loaded one tile ahead of their copies, so the
    // copies never wait for them
    auto rows_of = [&](int64_t t, int32_t *src_row) {
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int64_t gr = (t % ntr) * 128 + ((it * 256 + tid) >> 3);
            int32_t sr = -1;
            if (t < ntiles && gr < rows) {
                if (src_idx) {
                    const int si = src_idx[gr];
                    sr = si >= 0 ? si / k : -1;
                } else {
                    sr = (int32_t)gr;
                }
            }
            src_row[it] = sr;
        }
    };
    // the copies of tile t into ring slot `slot` (one commit group; none past the end)
    auto issue = [&](int64_t t, int slot, const int32_t *src_row) {
        if (t < ntiles) {
            const int64_t c0 = (t / ntr) * 64;
            uint16_t *tile = ring + slot * 128 * kR128Pad;
#pragma unroll
            for (int it = 0; it < 4; ++it) {
                const int idx = it * 256 + tid;  // 1024 16-byte pieces: 128 rows x 8
                const int r = idx >> 3, cc = (idx & 7) * 8;
                const bool ok = src_row[it] >= 0 && c0 + cc < cols;
                // (no bytes are read from the base address when zero-filling)
                cp_async16_zfill(tile + r * kR128Pad + cc, ok ? in + (int64_t)src_row[it] * ld + c0 + cc : in,
                                 ok ? 16u : 0u);
            }
        }
        cp_async_commit_group();   // (an empty group past the end keeps the count)
    };
    const int64_t G = gridDim.x;
    // 32-byte code stores need a 32-byte aligned output and row stride
    const bool wide = ((reinterpret_cast<uintptr_t>(qT) | (uintptr_t)ld_rows) & 31) == 0;
    int slot = 0;
    int32_t rw[4], nxt[4];
    rows_of(blockIdx.x, rw);
    issue(blockIdx.x, 0, rw);
    rows_of(blockIdx.x + G, rw);
    issue(blockIdx.x + G, 1, rw);
    rows_of(blockIdx.x + 2 * G, nxt);
    for (int64_t t = blockIdx.x; t < ntiles; t += G) {
        issue(t + 2 * G, (slot + 2) % kR128Slots, nxt);
        rows_of(t + 3 * G, nxt);
        cp_async_wait_groups<2>();   // tile t has landed
        __syncthreads();
        const uint16_t *tile = ring + slot * 128 * kR128Pad;
        const int64_t r0 = (t % ntr) * 128, c0 = (t / ntr) * 64;
        const int col = tid & 63, part = tid >> 6;
        float v[32];  // this thread's 32 rows of its column
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            v[i] = __uint_as_float((uint32_t)tile[(part * 32 + i) * kR128Pad + col] << 16);
            amax = fmaxf(amax, fabsf(v[i]));
        }
        part_max[part][col] = amax;
        __syncthreads();
        amax = fmaxf(fmaxf(part_max[0][col], part_max[1][col]), fmaxf(part_max[2][col], part_max[3][col]));
        const float s = block_scale(amax);
        const int64_t gc = c0 + col;
        if (gc < cols) {
            const int64_t rr = r0 + part * 32;
            const uint4 q0 = quant16(v, s), q1 = quant16(v + 16, s);
            uint8_t *dst = qT + gc * ld_rows + rr;
            if (wide && rr + 32 <= rows) {   // the column's 32 codes in one 32-byte store
                asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(q0.x),
                             "r"(q0.y), "r"(q0.z), "r"(q0.w), "r"(q1.x), "r"(q1.y), "r"(q1.z), "r"(q1.w)
                             : "memory");
            } else {
                if (rr < rows) *reinterpret_cast<uint4 *>(dst) = q0;
                if (rr + 16 < rows) *reinterpret_cast<uint4 *>(dst + 16) = q1;
            }
            if (part == 0) sT[(r0 / 128) * cols + gc] = s;
        }
        __syncthreads();  // this slot and part_max are read before they are refilled
        slot = (slot + 1) % kR128Slots;
    }
    cp_async_wait_groups<0>();   // (only empty groups remain; none outlives the block)
}

int launch_quant_rows128(const uint16_t *in, int64_t ld, const int32_t *src_idx, int k,
                         int64_t rows, int64_t cols, int64_t ld_rows, uint8_t *qT, float *sT,
                         cudaStream_t s)
{
    if (rows == 0 || cols == 0) return MOE_OK;
    if (rows > INT32_MAX) return MOE_ERR_UNSUPPORTED;   // row indices are 32-bit in the kernel
    static int per_sm = 0, sms = 0;   // per process: the device and the kernel's resources are fixed
    if (per_sm == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaFuncSetAttribute(quant_rows128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kR128Smem) !=
                cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_rows128_kernel, 256, kR128Smem) !=
                cudaSuccess ||
            per_sm <= 0)
            return MOE_ERR_CUDA;
    }
    const int64_t ntiles = ((rows + 127) / 128) * ((cols + 63) / 64);
    const int64_t grid = ntiles < (int64_t)per_sm * sms ? ntiles : (int64_t)per_sm * sms;
    quant_rows128_kernel<<<(unsigned)grid, 256, kR128Smem, s>>>(in, ld, src_idx, k, rows, cols, ld_rows, qT, sT);
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
// The block is staged in shared memory by cp.async (no values held in
// registers while the copies fly), so several blocks per SM keep copies in
// flight.
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
    // the bf16 block (rows of 136: 272 B, 16-byte aligned), later reused for
    // its codes (rows of 144 B) once every thread holds its own in registers
    __shared__ __align__(16) uint16_t tile[128][136];
    __shared__ float warp_max[8];
    uint8_t(*codes_s)[144] = reinterpret_cast<uint8_t(*)[144]>(&tile[0][0]);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int64_t cb = blockIdx.x, rb = blockIdx.y, e = blockIdx.z;
    const int64_t nbc = (cols + 127) / 128;
    const uint16_t *src = in + e * in_es;
    // the whole block into shared memory at once: eight 16-byte copies per
    // thread in flight, none held in registers (zero-filled past the edges)
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        const int idx = it * 256 + tid;  // 2048 pieces: 128 rows x 16
        const int r = idx >> 4, c = (idx & 15) * 8;
        const int64_t gr = rb * 128 + r, gc = cb * 128 + c;
        const bool in_range = gr < rows && gc < cols;
        cp_async16_zfill(&tile[r][c], in_range ? src + gr * ld + gc : src, in_range ? 16u : 0u);
    }
    cp_async_commit_group();
    cp_async_wait_groups<0>();
    __syncthreads();
    const int cc = (tid & 15) * 8;   // column within the block
    const int rr0 = tid >> 4;        // rows rr0, rr0+16, ...
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float v[8];
        unpack8(*reinterpret_cast<const uint4 *>(&tile[rr0 + 16 * i][cc]), v);
        amax = absmax8(v, amax);
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
    uint2 c8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float v[8];
        unpack8(*reinterpret_cast<const uint4 *>(&tile[rr0 + 16 * i][cc]), v);
        c8[i] = quant8(v, s);
        const int64_t r = rb * 128 + rr0 + 16 * i, c = cb * 128 + cc;
        if (r < rows && c < cols) *reinterpret_cast<uint2 *>(qe + (drb * 128 + rr0 + 16 * i) * cols + c) = c8[i];
    }
    if (tid == 0) sc[e * s_es + drb * nbc + cb] = s;
    if (!qT) return;
    __syncthreads();   // every thread has read its bf16 values: the tile takes the codes
#pragma unroll
    for (int i = 0; i < 8; ++i) *reinterpret_cast<uint2 *>(&codes_s[rr0 + 16 * i][cc]) = c8[i];
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
