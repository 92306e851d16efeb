// Router of the MoE layer and the capture of its decisions.
//
// The router is the linear gate before the top-k: logits z = x W_r^T over the
// E experts, then the top-k of each token ("prime-rl 0.6.0 løfter
// trillion-parameter RL ...", §Drift og omkostninger i realiteten).  Router
// replay records, per layer, the experts chosen at inference as an integer
// [num_layers, top_k, seq_len] tensor that the trainer replays ("RL at 1T
// scale: prime-rl performance deep dive", §Router Replay); the capture kernel
// below writes that record.
//
// Logits: a dense bf16 contraction (K = d_model) with a small N (E experts),
// on the tensor cores (tcgen05.mma kind::f16, fp32 accumulators in TMEM).
// One persistent CTA per SM, 256 threads:
//   warp 0     TMA producer: per 64-element K block, the 128-token x box
//              (128 rows x 128 B) and the W_r box (N rows x 128 B), both
//              128-byte swizzled, into a ring of stages;
//   warp 1     allocates TMEM (two N-column accumulators) and issues
//              M=128 x N x K=16 MMAs, four per K block;
//   warps 4-7  epilogue: thread = token; reads its N logits from TMEM and
//              writes the row of z; the buffer then goes back to the MMA,
//              which is already on the next tile.
// N = E rounded up to 16 (rows of W_r past E are read as zeros by TMA).
// The kernel streams x once: it is HBM-bound (E FLOP per byte of x); W_r is
// re-read from L2 for every tile.  The top-k of z then runs as in
// moe_route_topk.
//
// Backward (CUDA cores, fp32): dx[t] = bf16(fp32(dx_in[t]) + sum_e dz[t][e]
// W_r[e]) with W_r staged in shared memory per 256-column slice; dW_r[e] +=
// sum_t dz[t][e] x[t] as per-chunk partial sums in the caller's workspace,
// reduced in a fixed chunk order (deterministic, no atomics).
#include "sm100.cuh"

namespace moe {
namespace router {

using namespace sm100;

constexpr int BM = 128;             // tokens per tile
constexpr int X_BYTES = BM * 128;   // one K block of the x tile: 128 rows x 64 bf16
constexpr int NUM_THREADS = 256;
constexpr int EPI_WARP0 = 4;
constexpr int MAX_STAGES = 8;
constexpr int SMEM_RING = 200 * 1024;

struct Args {
    int T, D, E, N;    // N = E rounded up to 16
    int stages, stage_bytes;
    uint32_t tmem_cols;
    float *z;
    int *status;
    uint64_t budget;
};

__device__ __forceinline__ uint32_t idesc_bf16(int N)
{
    // D fp32, A and B bf16, both K-major, N, M = 128
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accum)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(accum));
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
router_logits_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, const Args p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    __shared__ __align__(8) uint64_t bars[2 * MAX_STAGES + 5];
    __shared__ uint32_t tmem_slot;
    __shared__ volatile int abort_flag;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = smem_u32(&bars[0]);
    const uint32_t bar_empty = bar_full + 8 * MAX_STAGES;
    const uint32_t bar_tfull = bar_empty + 8 * MAX_STAGES;   // [2]
    const uint32_t bar_tempty = bar_tfull + 16;              // [2]
    const uint32_t bar_drain = bar_tempty + 16;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = (p.T + BM - 1) / BM;
    const int KB = p.D / 64;
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, 4);   // one arrival per epilogue warp
        }
        mbar_init(bar_drain, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                     "r"(p.tmem_cols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;

    if (warp == 0) {
        if (lane == 0) {   // ------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0, pend = 0, pend_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                for (int kb = 0; kb < KB; ++kb) {
                    if (!wait_bounded(bar_empty + 8 * stage, phase ^ 1, p.budget, &abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = bar_full + 8 * stage;
                    const uint32_t dX = sbase + stage * p.stage_bytes, dW = dX + X_BYTES;
                    mbar_arrive_expect_tx(fb, p.stage_bytes);
                    tma_load_2d(dX, &tmX, kb * 64, t * BM, fb);
                    tma_load_2d(dW, &tmW, kb * 64, 0, fb);
                    pend |= 1u << stage;
                    pend_phase = (pend_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            if (!ok)   // loads still in flight land before the CTA exits
                for (int s = 0; s < p.stages; ++s)
                    if (pend & (1u << s)) wait_drain(bar_full + 8 * s, (pend_phase >> s) & 1u);
        }
    } else if (warp == 1) {
        if (lane == 0) {   // -------------------------------------- MMA issuer
            const uint32_t idesc = idesc_bf16(p.N);
            int stage = 0, buf = 0;
            uint32_t phase = 0, bphase = 0;
            bool ok = true, issued = false;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                if (!wait_bounded(bar_tempty + 8 * buf, bphase ^ 1, p.budget, &abort_flag, p.status)) break;
                tc_fence_after();
                const uint32_t dtm = tmem_base + (uint32_t)(buf * p.N);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!wait_bounded(bar_full + 8 * stage, phase, p.budget, &abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t aX = sbase + stage * p.stage_bytes, aW = aX + X_BYTES;
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                        mma_bf16(dtm, sdesc(aX + 32 * k4), sdesc(aW + 32 * k4), idesc, (kb | k4) ? 1u : 0u);
                    issued = true;
                    mma_commit(bar_empty + 8 * stage);
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                mma_commit(bar_tfull + 8 * buf);
                buf ^= 1;
                if (buf == 0) bphase ^= 1;
            }
            if (issued) {
                mma_commit(bar_drain);
                wait_drain(bar_drain, 0);
            }
        }
    } else if (warp >= EPI_WARP0) {   // ---------------------------- epilogue
        const int q = warp & 3;
        const int row = 32 * q + lane;
        const uint32_t lane_addr = tmem_base + ((uint32_t)(32 * q) << 16);
        int buf = 0;
        uint32_t bphase = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
            if (!warp_wait_bounded(bar_tfull + 8 * buf, bphase, p.budget, &abort_flag, p.status)) break;
            tc_fence_after();
            const int64_t tok = (int64_t)t * BM + row;
            float *zr = p.z + tok * p.E;
            for (int c0 = 0; c0 < p.N; c0 += 16) {
                uint32_t r[16];
                MOE_TMEM_LD16(lane_addr + (uint32_t)(buf * p.N + c0), r);
                tmem_wait_ld();
                if (tok < p.T) {
                    if ((p.E & 3) == 0) {
#pragma unroll
                        for (int i = 0; i < 16; i += 4)
                            if (c0 + i < p.E)
                                *reinterpret_cast<float4 *>(zr + c0 + i) =
                                    make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]),
                                                __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c0 + i < p.E) zr[c0 + i] = __uint_as_float(r[i]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_tempty + 8 * buf);
            buf ^= 1;
            if (buf == 0) bphase ^= 1;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(p.tmem_cols));
}

// payload[(layer*k + j)*T + t] = idx[t*k + j]: one thread per token; the
// stores of each slot j are coalesced over t.
__global__ void __launch_bounds__(256) capture_kernel(const int32_t *__restrict__ idx, int T, int k, int layer,
                                                      int32_t *__restrict__ payload)
{
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    int e[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
        if (j < k) e[j] = idx[(int64_t)t * k + j];
#pragma unroll
    for (int j = 0; j < 16; ++j)
        if (j < k) payload[((int64_t)layer * k + j) * T + t] = e[j];
}

// dx: block = 256 columns (128 threads x 2) of a chunk of tokens.  W_r's
// columns of the slice sit in shared memory as bf16 pairs; each token's dz
// row is staged in shared memory and read as a broadcast.
constexpr int DX_TOK = 32;   // tokens per block
__global__ void __launch_bounds__(128) router_dx_kernel(const float *__restrict__ dz, const uint16_t *__restrict__ Wr,
                                                        const uint16_t *__restrict__ dx_in, int T, int D, int E,
                                                        uint16_t *__restrict__ dx)
{
    extern __shared__ uint32_t wsm[];            // [E][128] bf16 pairs, then dz rows [DX_TOK][E]
    float *dzs = reinterpret_cast<float *>(wsm + E * 128);
    const int tid = threadIdx.x;
    const int64_t c = (int64_t)blockIdx.x * 256 + 2 * tid;   // this thread's two columns
    const int64_t t0 = (int64_t)blockIdx.y * DX_TOK;
    const int ntok = (int)min((int64_t)DX_TOK, (int64_t)T - t0);
    for (int e = 0; e < E; ++e)
        wsm[e * 128 + tid] = c < D ? *reinterpret_cast<const uint32_t *>(Wr + (int64_t)e * D + c) : 0u;
    for (int i = tid; i < ntok * E; i += 128) dzs[i] = dz[t0 * E + i];
    __syncthreads();
    if (c >= D) return;
    for (int i = 0; i < ntok; ++i) {
        float a0 = 0.0f, a1 = 0.0f;
        for (int e = 0; e < E; ++e) {
            const float g = dzs[i * E + e];
            const uint32_t w2 = wsm[e * 128 + tid];
            a0 = fmaf(g, bf16_lo(w2), a0);
            a1 = fmaf(g, bf16_hi(w2), a1);
        }
        const int64_t o = (t0 + i) * D + c;
        if (dx_in) {
            const uint32_t x2 = *reinterpret_cast<const uint32_t *>(dx_in + o);
            a0 += bf16_lo(x2);
            a1 += bf16_hi(x2);
        }
        *reinterpret_cast<uint32_t *>(dx + o) = pack_bf16x2(a0, a1);
    }
}

// dW_r partials: block = 256 columns (128 threads x 2) x a chunk of tokens x
// a group of up to 32 experts; part[chunk][e][d] = sum over the chunk's
// tokens of dz[t][e] * x[t][d], tokens in order.
constexpr int DW_TOK = 256;   // tokens per chunk
__global__ void __launch_bounds__(128) router_dw_part_kernel(const float *__restrict__ dz,
                                                             const uint16_t *__restrict__ x, int T, int D, int E,
                                                             float *__restrict__ part)
{
    __shared__ float dzs[DW_TOK][33];
    const int tid = threadIdx.x;
    const int64_t c = (int64_t)blockIdx.x * 256 + 2 * tid;
    const int64_t t0 = (int64_t)blockIdx.y * DW_TOK;
    const int e0 = blockIdx.z * 32;
    const int ne = min(32, E - e0);
    const int ntok = (int)min((int64_t)DW_TOK, (int64_t)T - t0);
    for (int i = tid; i < ntok * 32; i += 128) {
        const int tt = i >> 5, e = i & 31;
        dzs[tt][e] = e < ne ? dz[(t0 + tt) * E + e0 + e] : 0.0f;
    }
    __syncthreads();
    if (c >= D) return;
    float a0[32], a1[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) a0[e] = a1[e] = 0.0f;
    for (int i = 0; i < ntok; ++i) {
        const uint32_t x2 = *reinterpret_cast<const uint32_t *>(x + (t0 + i) * D + c);
        const float x0 = bf16_lo(x2), x1 = bf16_hi(x2);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const float g = dzs[i][e];
            a0[e] = fmaf(g, x0, a0[e]);
            a1[e] = fmaf(g, x1, a1[e]);
        }
    }
    float *o = part + ((int64_t)blockIdx.y * E + e0) * D + c;
    for (int e = 0; e < ne; ++e) *reinterpret_cast<float2 *>(o + (int64_t)e * D) = make_float2(a0[e], a1[e]);
}

// dW_r[e][d] += sum over chunks (in order) of part[chunk][e][d].
__global__ void __launch_bounds__(256) router_dw_reduce_kernel(const float *__restrict__ part, int64_t ED,
                                                               int nchunk, float *__restrict__ dw)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= ED) return;
    float s = 0.0f;
    for (int c = 0; c < nchunk; ++c) s += part[(int64_t)c * ED + i];
    dw[i] += s;
}

}  // namespace router

// ------------------------------------------------------------------ host ----
size_t router_bwd_ws_bytes(int T, int D, int E)
{
    const int64_t nchunk = ((int64_t)T + router::DW_TOK - 1) / router::DW_TOK;
    return (size_t)(nchunk > 0 ? nchunk : 1) * E * D * sizeof(float);
}

int launch_router_logits(const uint16_t *x, const uint16_t *w_r, int T, int D, int E, float *z, int *status,
                         uint64_t budget, cudaStream_t s)
{
    using namespace router;
    if (T == 0) return MOE_OK;
    Args a{};
    a.T = T;
    a.D = D;
    a.E = E;
    a.N = (E + 15) / 16 * 16;
    a.stage_bytes = X_BYTES + a.N * 128;
    a.stages = min(MAX_STAGES, SMEM_RING / a.stage_bytes);
    uint32_t cols = 32;
    while (cols < (uint32_t)(2 * a.N)) cols <<= 1;
    a.tmem_cols = cols;
    a.z = z;
    a.status = status;
    a.budget = budget;
    CUtensorMap mX, mW;
    if (!make_map_bf16(&mX, x, D, T, BM) || !make_map_bf16(&mW, w_r, D, E, a.N)) return MOE_ERR_CUDA;
    const int smem = 1024 + a.stages * a.stage_bytes;
    if (cudaFuncSetAttribute(router_logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return MOE_ERR_CUDA;
    const int ntiles = (T + BM - 1) / BM;
    router_logits_kernel<<<min(ntiles, sm_count()), NUM_THREADS, smem, s>>>(mX, mW, a);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_capture(const int32_t *idx, int T, int k, int layer, int32_t *payload, cudaStream_t s)
{
    if (T == 0) return MOE_OK;
    router::capture_kernel<<<(T + 255) / 256, 256, 0, s>>>(idx, T, k, layer, payload);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_router_bwd(const float *dz, const uint16_t *x, const uint16_t *w_r, int T, int D, int E,
                      const uint16_t *dx_in, uint16_t *dx, float *dw_r, void *ws, cudaStream_t s)
{
    using namespace router;
    if (T == 0) return MOE_OK;
    if (dx) {
        const int smem = E * 128 * 4 + DX_TOK * E * 4;
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(router_dx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return MOE_ERR_CUDA;
        dim3 grid((unsigned)((D + 255) / 256), (unsigned)((T + DX_TOK - 1) / DX_TOK));
        router_dx_kernel<<<grid, 128, smem, s>>>(dz, w_r, dx_in, T, D, E, dx);
        count_launch();
        if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (dw_r) {
        const int nchunk = (T + DW_TOK - 1) / DW_TOK;
        float *part = static_cast<float *>(ws);
        dim3 grid((unsigned)((D + 255) / 256), (unsigned)nchunk, (unsigned)((E + 31) / 32));
        router_dw_part_kernel<<<grid, 128, 0, s>>>(dz, x, T, D, E, part);
        count_launch();
        const int64_t ED = (int64_t)E * D;
        router_dw_reduce_kernel<<<(unsigned)((ED + 255) / 256), 256, 0, s>>>(part, ED, nchunk, dw_r);
        count_launch();
        if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

}  // namespace moe
