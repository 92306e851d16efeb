// a8 weighted combine, b1 combine backward, b3 unpermute-reduce.
//
// Combine is the per-layer gather of each token's expert outputs ("prime-rl
// 0.6.0 løfter trillion-parameter RL ...", §Drift og omkostninger i
// realiteten; "RL at 1T scale ...", §Parallelism/EP).  It is written as a
// gather over pos[t][j] (not a scatter-add), so each output element is summed
// by one thread in a fixed slot order: deterministic without atomics.
#include "common.cuh"

namespace moe {

// One warp per token; lane l covers 8 columns of each 256-column step.
// y[t] = bf16(sum_j w[t][j] * Y[pos[t][j]]) in fp32, j ascending.
// scale_by_w = false gives the plain sum (unpermute-reduce of dX).
template <bool kWeighted>
__global__ void __launch_bounds__(256) gather_reduce_kernel(const uint16_t *__restrict__ Y,
                                                            const float *__restrict__ w,
                                                            const int32_t *__restrict__ pos, int T,
                                                            int D, int k, uint16_t *__restrict__ y)
{
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    int my_pos = -1;
    float my_w = 0.0f;
    if (lane < k) {
        my_pos = pos[t * k + lane];
        if (kWeighted) my_w = w[t * k + lane];
    }
    for (int c0 = 0; c0 < D; c0 += 256) {
        const int c = c0 + lane * 8;
        const bool act = c < D;
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        for (int j0 = 0; j0 < k; j0 += 4) {
            uint4 rv[4];
            float wj[4];
            bool ok[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                int j = j0 + u;
                int p = __shfl_sync(kFull, my_pos, j & 31);
                wj[u] = __shfl_sync(kFull, my_w, j & 31);
                ok[u] = act && j < k && p >= 0;
                if (ok[u]) rv[u] = *reinterpret_cast<const uint4 *>(Y + (int64_t)p * D + c);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (!ok[u]) continue;
                float v[8];
                unpack8(rv[u], v);
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = kWeighted ? fmaf(wj[u], v[i], acc[i]) : acc[i] + v[i];
            }
        }
        if (act) *reinterpret_cast<uint4 *>(y + t * D + c) = pack8(acc);
    }
}

int launch_combine(const uint16_t *Y, const float *w, const int32_t *pos, int T, int D, int k,
                   uint16_t *y, cudaStream_t s)
{
    if (T == 0) return MOE_OK;
    unsigned blocks = (unsigned)((T + 7) / 8);
    if (w)
        gather_reduce_kernel<true><<<blocks, 256, 0, s>>>(Y, w, pos, T, D, k, y);
    else
        gather_reduce_kernel<false><<<blocks, 256, 0, s>>>(Y, nullptr, pos, T, D, k, y);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// b1: one warp per token; lane l covers 16 columns of each 512-column step
// (8 lanes = one 1x128 block of a dY row).
//   dY[pos[t][j]] = bf16(fp32(w[t][j] * dy[t])) -> 1x128 FP8 (+ optional bf16)
//   d_w[t][j] = <dy[t], Y[pos[t][j]]>
//   d_logits[t][e] = w_e (d_w_e - <w, d_w>) on the chosen experts, else 0.
__global__ void __launch_bounds__(256) combine_bwd_kernel(
    const uint16_t *__restrict__ dy, const uint16_t *__restrict__ Y, const float *__restrict__ w,
    const int32_t *__restrict__ pos, const int32_t *__restrict__ idx, int T, int D, int k, int E,
    int64_t R_cap, uint8_t *__restrict__ dYq, float *__restrict__ dYs, uint16_t *__restrict__ dYb,
    float *__restrict__ d_w, float *__restrict__ d_logits)
{
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    int my_pos = -1;
    float my_w = 0.0f;
    if (lane < k) {
        my_pos = pos[t * k + lane];
        my_w = w[t * k + lane];
    }
    float dw_part[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) dw_part[j] = 0.0f;
    for (int c0 = 0; c0 < D; c0 += 512) {
        const int c = c0 + lane * 16;
        const bool act = c < D;
        float g[16];
        if (act) {
            unpack8(*reinterpret_cast<const uint4 *>(dy + t * D + c), g);
            unpack8(*reinterpret_cast<const uint4 *>(dy + t * D + c + 8), g + 8);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) g[i] = 0.0f;
        }
#pragma unroll
        for (int j0 = 0; j0 < 16; j0 += 4) {
            if (j0 >= k) break;
            // the Y rows of up to 4 slots are loaded before any is used
            uint4 yr[4][2];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = j0 + u;
                const int p = __shfl_sync(kFull, my_pos, j & 31);
                yr[u][0] = yr[u][1] = make_uint4(0, 0, 0, 0);
                if (act && j < k && p >= 0) {
                    yr[u][0] = *reinterpret_cast<const uint4 *>(Y + (int64_t)p * D + c);
                    yr[u][1] = *reinterpret_cast<const uint4 *>(Y + (int64_t)p * D + c + 8);
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = j0 + u;
                if (j >= k) break;
                const int p = __shfl_sync(kFull, my_pos, j);
                const float wj = __shfl_sync(kFull, my_w, j);
                float v[16];
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    // the product in fp32, then bf16: the rounding point of a dY row
                    float prod = __fmul_rn(wj, g[i]);
                    v[i] = __uint_as_float(bf16_bits_rn(prod) << 16);
                    amax = fmaxf(amax, fabsf(v[i]));
                }
                amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
                amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
                amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 4));
                const float s = block_scale(amax);
                if (act && p >= 0) {
                    *reinterpret_cast<uint4 *>(dYq + (int64_t)p * D + c) = quant16(v, s);
                    if ((lane & 7) == 0) dYs[(int64_t)(c / 128) * R_cap + p] = s;
                    if (dYb) {
                        *reinterpret_cast<uint4 *>(dYb + (int64_t)p * D + c) = pack8(v);
                        *reinterpret_cast<uint4 *>(dYb + (int64_t)p * D + c + 8) = pack8(v + 8);
                    }
                    float yv[16];
                    unpack8(yr[u][0], yv);
                    unpack8(yr[u][1], yv + 8);
#pragma unroll
                    for (int i = 0; i < 16; ++i) dw_part[j] = fmaf(g[i], yv[i], dw_part[j]);
                }
            }
        }
    }
    float my_dw = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        if (j >= k) break;
        float s = dw_part[j];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(kFull, s, off);
        if (lane == j) my_dw = s;
    }
    if (lane < k) d_w[t * k + lane] = my_dw;
    if (!d_logits) return;
    float inner = 0.0f;
    for (int j = 0; j < k; ++j) inner += __shfl_sync(kFull, my_w, j) * __shfl_sync(kFull, my_dw, j);
    float *dz = d_logits + t * E;
    for (int e = lane; e < E; e += 32) dz[e] = 0.0f;
    __syncwarp();
    if (lane < k) {
        int e = idx[t * k + lane];
        if (e >= 0 && e < E && my_pos >= 0) dz[e] = my_w * (my_dw - inner);
    }
}

int launch_combine_bwd(const uint16_t *dy, const uint16_t *Y, const float *w, const int32_t *pos,
                       const int32_t *idx, int T, int D, int k, int E, int64_t R_cap,
                       uint8_t *dYq, float *dYs, uint16_t *dYb, float *d_w, float *d_logits,
                       cudaStream_t s)
{
    if (T == 0) return MOE_OK;
    combine_bwd_kernel<<<(unsigned)((T + 7) / 8), 256, 0, s>>>(dy, Y, w, pos, idx, T, D, k, E, R_cap,
                                                               dYq, dYs, dYb, d_w, d_logits);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
