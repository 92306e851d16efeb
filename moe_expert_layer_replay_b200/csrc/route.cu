// a1 top-k routing and a2 router replay.
//
// Top-k: each token activates a top-k set of experts ("prime-rl 0.6.0 løfter
// trillion-parameter RL ...", §Drift og omkostninger i realiteten).
// Replay: the routed experts captured at inference, a [num_layers, top_k,
// seq_len] integer payload, are replayed in the trainer ("RL at 1T scale:
// prime-rl performance deep dive", §Router Replay).
#include <math.h>

#include "common.cuh"

namespace moe {

// One warp per token.  Lane l holds logits l, l+32, ... (E <= 256).  Each of
// the k rounds takes the warp-wide best untaken (value desc, index asc) by an
// xor butterfly, which leaves the same winner in every lane.
__global__ void __launch_bounds__(256) route_topk_kernel(const float *__restrict__ z, int T, int E,
                                                         int k, int32_t *__restrict__ idx,
                                                         float *__restrict__ w)
{
    const int lane = threadIdx.x & 31;
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    const float *zt = z + (int64_t)t * E;
    float v[8];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int e = lane + 32 * i;
        v[i] = (e < E) ? zt[e] : -INFINITY;
        if (e >= E) taken |= 1u << i;
    }
    float my_v = -INFINITY;
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            int e = lane + 32 * i;
            bool free_ = !((taken >> i) & 1u);
            if (free_ && (v[i] > bv || (v[i] == bv && e < be))) {
                bv = v[i];
                be = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            float ov = __shfl_xor_sync(kFull, bv, off);
            int oe = __shfl_xor_sync(kFull, be, off);
            if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == j) {
            my_v = bv;
            my_e = be;
        }
    }
    // softmax over the chosen set; the first selection holds the largest logit
    float m = __shfl_sync(kFull, my_v, 0);
    float ex = (lane < k) ? expf(my_v - m) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(kFull, sum, off);
    if (lane < k) {
        idx[(int64_t)t * k + lane] = my_e;
        w[(int64_t)t * k + lane] = ex / sum;
    }
}

// E <= 32: one thread per token with its E logits in registers (16-byte
// loads when E is a multiple of 4); each of the k rounds scans them in index
// order for the best untaken (value desc, index asc), as the warp form does.
__global__ void __launch_bounds__(128) route_topk_small_kernel(const float *__restrict__ z, int T, int E,
                                                               int k, int32_t *__restrict__ idx,
                                                               float *__restrict__ w)
{
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    const float *zt = z + (int64_t)t * E;
    float v[32];
    if ((E & 3) == 0 && (reinterpret_cast<uintptr_t>(z) & 15u) == 0) {
#pragma unroll
        for (int e4 = 0; e4 < 32; e4 += 4) {
            float4 q = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            if (e4 < E) q = *reinterpret_cast<const float4 *>(zt + e4);
            v[e4] = q.x, v[e4 + 1] = q.y, v[e4 + 2] = q.z, v[e4 + 3] = q.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = (e < E) ? zt[e] : -INFINITY;
    }
    uint32_t taken = (E < 32) ? ~((1u << E) - 1u) : 0u;
    float sv[16];
    int se[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        sv[j] = -INFINITY;
        se[j] = 0;
        if (j < k) {
            float bv = -INFINITY;
            int be = 0x7fffffff;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                if (!((taken >> e) & 1u) && (v[e] > bv || (v[e] == bv && e < be))) {
                    bv = v[e];
                    be = e;
                }
            }
            taken |= 1u << (be & 31);
            sv[j] = bv;
            se[j] = be;
        }
    }
    // softmax over the chosen set; the first selection holds the largest logit
    float ex[16], sum = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        ex[j] = (j < k) ? expf(sv[j] - sv[0]) : 0.0f;
        sum += ex[j];
    }
#pragma unroll
    for (int j = 0; j < 16; ++j)
        if (j < k) {
            idx[(int64_t)t * k + j] = se[j];
            w[(int64_t)t * k + j] = ex[j] / sum;
        }
}

// One thread per token.  idx[t][j] = P[(layer*k + j)*T + t] (reads coalesced
// over t).  An entry outside [0,E) or a repeated expert latches
// MOE_ERR_BAD_ROUTING and zeroes the token's weights.
__global__ void __launch_bounds__(64) route_replay_kernel(const int32_t *__restrict__ P, int layer,
                                                           int T, int E, int k,
                                                           const float *__restrict__ w_in,
                                                           const float *__restrict__ z,
                                                           int32_t *__restrict__ idx,
                                                           float *__restrict__ w, int *status)
{
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    int e[16];
    float wi[16];
    bool bad = false;
#pragma unroll
    for (int j = 0; j < 16; ++j) {  // every load first, then the checks and stores
        if (j < k) {
            e[j] = P[((int64_t)layer * k + j) * T + t];
            wi[j] = w_in ? w_in[(int64_t)t * k + j] : 0.0f;
        }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        if (j < k) {
            idx[(int64_t)t * k + j] = e[j];
            bad |= (e[j] < 0) || (e[j] >= E);
        }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j)
#pragma unroll
        for (int jj = j + 1; jj < 16; ++jj)
            if (jj < k) bad |= (e[j] == e[jj]);
    if (bad) {
        latch_status(status, MOE_ERR_BAD_ROUTING);
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < k) w[(int64_t)t * k + j] = 0.0f;
        return;
    }
    if (w_in) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < k) w[(int64_t)t * k + j] = wi[j];
        return;
    }
    const float *zt = z + (int64_t)t * E;
    float zs[16];
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < 16; ++j)
        if (j < k) {
            zs[j] = zt[e[j]];
            m = fmaxf(m, zs[j]);
        }
    float sum = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j)
        if (j < k) {
            zs[j] = expf(zs[j] - m);
            sum += zs[j];
        }
#pragma unroll
    for (int j = 0; j < 16; ++j)
        if (j < k) w[(int64_t)t * k + j] = zs[j] / sum;
}

int launch_route_topk(const float *z, int T, int E, int k, int32_t *idx, float *w, cudaStream_t s)
{
    if (T == 0) return MOE_OK;
    if (E <= 32) {
        route_topk_small_kernel<<<(T + 127) / 128, 128, 0, s>>>(z, T, E, k, idx, w);
        count_launch();
    } else {
        const int blocks = (T + 7) / 8;
        route_topk_kernel<<<blocks, 256, 0, s>>>(z, T, E, k, idx, w);
        count_launch();
    }
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_route_replay(const int32_t *P, int layer, int T, int E, int k, const float *w_in,
                        const float *z, int32_t *idx, float *w, int *status, cudaStream_t s)
{
    if (T == 0) return MOE_OK;
    route_replay_kernel<<<(T + 63) / 64, 64, 0, s>>>(P, layer, T, E, k, w_in, z, idx, w, status);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
