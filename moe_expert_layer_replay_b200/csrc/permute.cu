// a3: per-expert histogram, exclusive scan and stable permutation index.
//
// Dispatch groups each layer's routed token copies by expert ("RL at 1T
// scale: prime-rl performance deep dive", §Wide Expert Parallelism and
// §Parallelism/EP).  Routed entry i = t*k + j goes to row
//     pos[i] = offsets[e] + #{ i' < i : idx[i'] = e },   e = idx[i],
// with every expert's segment padded to a multiple of `align` rows.
//
// Three deterministic passes (no global atomics, so the result never depends
// on scheduling; the rows of src_idx that no entry fills are set to -1 by the
// place pass):
//   count: block b counts its chunk of entries per expert (shared atomics);
//   scan:  per expert, an exclusive scan of the block counts (block bases),
//          totals, then padded offsets;
//   place: block b ranks its chunk in order; within a warp, peers with the
//          same expert are found with match.any and ranked by lane order.
#include "common.cuh"

namespace moe {

constexpr int kChunk = 1024;  // entries per block
constexpr int kPlaceWarps = 8;

size_t permute_ws_bytes(int T, int k, int E)
{
    int64_t n = (int64_t)T * k;
    int64_t nblk = (n + kChunk - 1) / kChunk;
    if (nblk == 0) nblk = 1;
    return (size_t)(2 * nblk * E) * sizeof(int32_t);
}

__global__ void __launch_bounds__(256) perm_count_kernel(const int32_t *__restrict__ idx, int64_t n,
                                                         int E, int32_t *__restrict__ blkcnt)
{
    extern __shared__ int hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    int64_t base = (int64_t)blockIdx.x * kChunk;
    for (int i = threadIdx.x; i < kChunk; i += blockDim.x) {
        int64_t g = base + i;
        if (g < n) {
            int e = idx[g];
            if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) blkcnt[(int64_t)blockIdx.x * E + e] = hist[e];
}

__global__ void __launch_bounds__(256) perm_scan_kernel(const int32_t *__restrict__ blkcnt, int nblk,
                                                        int E, int align,
                                                        int32_t *__restrict__ blkbase,
                                                        int32_t *__restrict__ counts,
                                                        int32_t *__restrict__ offsets)
{
    __shared__ int padded[256];
    int e = threadIdx.x;
    if (e < E) {
        int run = 0;
        for (int b = 0; b < nblk; ++b) {
            blkbase[(int64_t)b * E + e] = run;
            run += blkcnt[(int64_t)b * E + e];
        }
        counts[e] = run;
        padded[e] = (run + align - 1) / align * align;
    }
    __syncthreads();
    if (threadIdx.x < 32) {  // exclusive scan of the padded sizes, 32 experts per step
        const int lane = threadIdx.x;
        int carry = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int v = e0 + lane < E ? padded[e0 + lane] : 0;
            int x = v;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(kFull, x, d);
                if (lane >= d) x += y;
            }
            if (e0 + lane < E) offsets[e0 + lane] = carry + x - v;
            carry += __shfl_sync(kFull, x, 31);
        }
        if (lane == 0) offsets[E] = carry;
    }
}

// kFused (few blocks): the scan pass is done here, by every block for itself:
// per expert the total over all blocks' counts and this block's base, then
// the padded offsets (block 0 stores counts and offsets).  Otherwise counts,
// offsets and bases come from perm_scan_kernel.
template <bool kFused>
__global__ void __launch_bounds__(256) perm_place_kernel(const int32_t *__restrict__ idx, int64_t n,
                                                         int E, int align, int nblk,
                                                         const int32_t *__restrict__ blkcnt,
                                                         const int32_t *__restrict__ blkbase,
                                                         int32_t *__restrict__ offsets,
                                                         int32_t *__restrict__ counts, int64_t R_cap,
                                                         int32_t *__restrict__ pos,
                                                         int32_t *__restrict__ src_idx, int *status)
{
    __shared__ int s_off[257], s_cnt[256], s_base[256];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (kFused) {
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
            int tot = 0, base = 0;
            for (int b = 0; b < nblk; ++b) {
                const int c = blkcnt[(int64_t)b * E + e];
                if (b < (int)blockIdx.x) base += c;
                tot += c;
            }
            s_cnt[e] = tot;
            s_base[e] = base;
        }
        __syncthreads();
        if (wid == 0) {  // exclusive scan of the padded sizes, 32 experts per step
            int carry = 0;
            for (int e0 = 0; e0 < E; e0 += 32) {
                const int e = e0 + lane;
                const int v = e < E ? (s_cnt[e] + align - 1) / align * align : 0;
                int x = v;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const int y = __shfl_up_sync(kFull, x, d);
                    if (lane >= d) x += y;
                }
                if (e < E) s_off[e] = carry + x - v;
                carry += __shfl_sync(kFull, x, 31);
            }
            if (lane == 0) s_off[E] = carry;
        }
        __syncthreads();
        if (blockIdx.x == 0) {
            for (int e = threadIdx.x; e < E; e += blockDim.x) counts[e] = s_cnt[e];
            for (int e = threadIdx.x; e <= E; e += blockDim.x) offsets[e] = s_off[e];
        }
    } else {
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
            s_cnt[e] = counts[e];
            s_base[e] = blkbase[(int64_t)blockIdx.x * E + e];
        }
        for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = offsets[e];
        __syncthreads();
    }
    // rows no entry fills: expert e's padding goes to block e % gridDim.x;
    // the rows past offsets[E] are shared by all blocks
    for (int e = blockIdx.x; e < E; e += gridDim.x)
        for (int64_t r = (int64_t)s_off[e] + s_cnt[e] + threadIdx.x; r < s_off[e + 1]; r += blockDim.x)
            src_idx[r] = -1;
    for (int64_t r = (int64_t)s_off[E] + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < R_cap;
         r += (int64_t)gridDim.x * blockDim.x)
        src_idx[r] = -1;
    if (n == 0) return;
    extern __shared__ int whist[];  // [kPlaceWarps][E]
    for (int i = threadIdx.x; i < kPlaceWarps * E; i += blockDim.x) whist[i] = 0;
    __syncthreads();
    constexpr int sub = kChunk / kPlaceWarps;
    const int64_t s0 = (int64_t)blockIdx.x * kChunk + (int64_t)wid * sub;
    for (int i = lane; i < sub; i += 32) {
        int64_t g = s0 + i;
        if (g < n) {
            int e = idx[g];
            if (e >= 0 && e < E) atomicAdd(&whist[wid * E + e], 1);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = s_off[e] + s_base[e];
        for (int w = 0; w < kPlaceWarps; ++w) {
            int c = whist[w * E + e];
            whist[w * E + e] = run;
            run += c;
        }
    }
    __syncthreads();
    const unsigned lt = (1u << lane) - 1u;
    for (int i0 = 0; i0 < sub; i0 += 32) {
        int64_t g = s0 + i0 + lane;
        bool in = g < n;
        int e = in ? idx[g] : -1;
        bool valid = in && e >= 0 && e < E;
        unsigned peers = __match_any_sync(kFull, valid ? e : -1);
        if (valid) {
            int p = whist[wid * E + e] + __popc(peers & lt);
            pos[g] = p;
            src_idx[p] = (int32_t)g;
        } else if (in) {
            pos[g] = -1;
            latch_status(status, MOE_ERR_BAD_ROUTING);
        }
        __syncwarp();
        if (valid && (peers & lt) == 0) whist[wid * E + e] += __popc(peers);
        __syncwarp();
    }
}

int launch_permute_index(const int32_t *idx, int T, int k, int E, int align, int32_t *counts,
                         int32_t *offsets, int32_t *pos, int32_t *src_idx, int64_t R_cap,
                         void *ws, int *status, cudaStream_t s)
{
    int64_t n = (int64_t)T * k;
    int nblk = (int)((n + kChunk - 1) / kChunk);
    int32_t *blkcnt = (int32_t *)ws;
    int32_t *blkbase = blkcnt + (int64_t)(nblk ? nblk : 1) * E;
    if (nblk > 0) {
        perm_count_kernel<<<nblk, 256, E * sizeof(int), s>>>(idx, n, E, blkcnt);
        count_launch();
    }
    // place also writes -1 to the rows of src_idx that no entry fills; with
    // few blocks it does the scan pass itself (one launch less)
    const int pblk = nblk > 0 ? nblk : 1;
    const size_t psmem = kPlaceWarps * E * sizeof(int);
    if (nblk <= 64) {
        perm_place_kernel<true><<<pblk, 32 * kPlaceWarps, psmem, s>>>(idx, n, E, align, nblk, blkcnt, blkbase,
                                                                     offsets, counts, R_cap, pos, src_idx, status);
        count_launch();
    } else {
        perm_scan_kernel<<<1, 256, 0, s>>>(blkcnt, nblk, E, align, blkbase, counts, offsets);
        count_launch();
        perm_place_kernel<false><<<pblk, 32 * kPlaceWarps, psmem, s>>>(idx, n, E, align, nblk, blkcnt, blkbase,
                                                                      offsets, counts, R_cap, pos, src_idx, status);
        count_launch();
    }
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
