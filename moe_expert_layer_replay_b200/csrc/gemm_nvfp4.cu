// Grouped NVFP4 GEMM on sm_100a tensor cores with the hardware block scales
// (tcgen05.mma kind::mxf4nvf4, block16: e2m1 operands, one ue4m3 scale per 16
// elements along K).  NVFP4 training and inference on Blackwell are named as
// future work in "RL at 1T scale: prime-rl performance deep dive", §Future
// work; this is the expert GEMM in that format.
//
//   out[r][n] = sum_k value(A)[r][k] * value(B_e)[n][k],  r in segment e,
//   value(X)[i][k] = e2m1(code) * value(S8[i][k/16]) / s_g(X)
//
// Unlike the block-scaled FP8 GEMM (arbitrary fp32 scales, promoted per K
// block by the epilogue), the 16-element scales ride in the MMA itself, so
// the accumulator stays in TMEM over the whole K and the epilogue runs once
// per tile: multiply by 1 / (s_g(A) s_g(B_e)) and store fp32.
//
// Design (one persistent CTA per SM, 12 warps):
//   warp 0     TMA producer: per 256-element K block, A (128 rows x 128 B),
//              B (256 rows x 128 B), both 128-byte swizzled, and the scale
//              factors of both (one bulk copy each) into a 3-stage ring;
//   warp 1     allocates 512 TMEM columns; lane 0 copies each K block's
//              scale factors from shared memory into TMEM (six tcgen05.cp
//              128x256b) and issues four MMAs (M=128, N=256, K=64);
//   warps 4-11 epilogue (TMEM lane quarter warp % 4, column half (warp - 4) / 4).
// TMEM: the accumulator in columns 0-255; scale-factor slot s (one per ring
// stage) in columns 256 + 48 s: A's four K steps (4 columns each), then B's
// (8 columns each: rows 0-127, then rows 128-255).
//
// Scale layout the MMA reads (one K step, one 128-row block): TMEM lane
// 32 q + r0 (every q), four columns, column r1 byte j = the scale of row
// 32 r1 + r0, group j.  The global and shared images (moe.h, MOE_NVFP4_SF_MMA_A
// / _B) hold those lanes' bytes already replicated, as 4096-byte blocks of two
// such atoms that one tcgen05.cp 128x256b moves into 8 columns: for A a pair
// of K steps (SFA of step ks at 4 ks), for B the two 128-row blocks of one K
// step (SFB of step ks at 8 ks).  A copy instruction costs about 60 cycles of
// the MMA thread whatever its size (measured: twelve 32x128b.warpx4 copies of
// the compact atoms took 720 cycles per K block, six 128x256b 340), so the
// fourfold replication in memory buys half the copies.
//
// Every mbarrier wait is bounded; on expiry the kernel latches
// MOE_ERR_TIMEOUT, drains what it issued, frees TMEM and returns.
#include "sm100.cuh"

namespace moe {

namespace nvfp4g {

using namespace sm100;

constexpr int BM = 128, BN = 256;
constexpr int KB_ELEMS = 256;   // e2m1 elements of K per stage (128 bytes per row)
constexpr int KB_BYTES = KB_ELEMS / 2;
constexpr int STAGES = 3;
constexpr int NUM_THREADS = 384;
constexpr int EPI_WARP0 = 4;
constexpr uint32_t TMEM_COLS = 512;
constexpr int A_BYTES = BM * KB_BYTES;        // 16 KB
constexpr int B_BYTES = BN * KB_BYTES;        // 32 KB
constexpr int SF_BLOCK = 4096;                // one tcgen05.cp 128x256b source (two atoms, x4 lanes)
constexpr int SFA_BYTES = 2 * SF_BLOCK;       // two K-step pairs
constexpr int SFB_BYTES = 4 * SF_BLOCK;       // four K steps, both row blocks
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int OFF_BAR = STAGES * STAGE_BYTES;
constexpr int OFF_TMEM_SLOT = OFF_BAR + (2 * STAGES + 3) * 8;
constexpr int OFF_ABORT = OFF_TMEM_SLOT + 4;
constexpr int OFF_OFFSETS = OFF_BAR + 128;
constexpr int MAX_SEG = 256;
constexpr int SMEM_BYTES = 1024 + OFF_OFFSETS + 4 * (MAX_SEG + 1);
constexpr uint32_t SF_COL0 = 256, SF_SLOT_COLS = 48;
static_assert(STAGE_BYTES % 1024 == 0 && A_BYTES % 1024 == 0, "1024-aligned operand tiles");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(SF_COL0 + STAGES * SF_SLOT_COLS <= TMEM_COLS, "TMEM budget");
static_assert(OFF_ABORT + 4 <= OFF_OFFSETS, "barrier area");

// Instruction descriptor, kind::mxf4nvf4: A and B e2m1 (format 1), K-major,
// N = 256 (bits 17-22: N/8), scale format ue4m3 (bit 23 = 0), M = 128 (bits
// 24-28: M/16), dense K = 64, both scale-factor ids 0.
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void mma_nvf4(uint32_t d, uint64_t a, uint64_t b, uint32_t sfa, uint32_t sfb,
                                         uint32_t accum)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(IDESC), "r"(sfa), "r"(sfb), "r"(accum));
}

// Shared-memory descriptor of one 4096-byte scale block for tcgen05.cp
// 128x256b: K-major, no swizzle, 8-row core matrices of 16-byte rows; the two
// 16-byte halves of a lane's 32 bytes 128 bytes apart (leading byte offset),
// row groups 256 bytes apart (stride byte offset).
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(128 >> 4) << 16;   // leading byte offset
    d |= (uint64_t)(256 >> 4) << 32;   // stride byte offset
    d |= (uint64_t)1 << 46;            // descriptor version
    return d;                          // layout type 0: no swizzle
}

__device__ __forceinline__ void sf_copy(uint32_t taddr, uint64_t desc)
{
    asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

struct Args {
    const int32_t *offsets;   // [n_seg + 1], 128-aligned
    int n_seg;
    int N, K;                 // output columns (% 256 == 0), reduction length (% 256 == 0)
    const uint8_t *sfa;       // A scales, blocks [R_cap/128][K/128][4096]
    const uint8_t *sfb;       // B scales, blocks [n_seg*N/256][K/64][4096]
    const float *a_sg;        // A's tensor scale (one float)
    const float *b_sg;        // each segment's B tensor scale [n_seg]
    float *out;               // [R_cap][N]
    int *status;
    uint64_t budget;
};

struct Tile {
    int e, m0, n0;
};

__device__ __forceinline__ Tile tile_of(int t, const Args &p, const int *offs_s)
{
    const int NT = p.N / BN;
    Tile x;
    const int mt = t / NT;
    x.n0 = (t - mt * NT) * BN;
    x.m0 = mt * BM;
    int lo = 0, hi = p.n_seg - 1;   // last segment with offs[e] <= m0
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offs_s[mid] <= x.m0) lo = mid; else hi = mid - 1;
    }
    x.e = lo;
    return x;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const Args p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + OFF_BAR;        // [STAGES]
    const uint32_t bar_empty = bar_full + STAGES * 8;  // [STAGES]
    const uint32_t bar_tfull = bar_empty + STAGES * 8;
    const uint32_t bar_tempty = bar_tfull + 8;
    const uint32_t bar_drain = bar_tempty + 8;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_ABORT);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_TMEM_SLOT);
    int *offs_s = reinterpret_cast<int *>(smem + OFF_OFFSETS);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    for (int i = threadIdx.x; i <= p.n_seg; i += blockDim.x) offs_s[i] = p.offsets[i];
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        mbar_init(bar_tfull, 1);
        mbar_init(bar_tempty, 8);   // the eight epilogue warps
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int ntiles = (offs_s[p.n_seg] / BM) * (p.N / BN);
    const int KB = p.K / KB_ELEMS, KS = p.K / 64;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer ----
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, pend = 0, pend_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                const Tile x = tile_of(t, p, offs_s);
                const int brow = x.e * p.N + x.n0;
                const uint8_t *sfa = p.sfa + ((int64_t)(x.m0 / 128) * (KS / 2)) * SF_BLOCK;
                const uint8_t *sfb = p.sfb + ((int64_t)(brow / 256) * KS) * SF_BLOCK;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!wait_bounded(bar_empty + 8 * stage, phase ^ 1, p.budget, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    pend &= ~(1u << stage);
                    const uint32_t fb = bar_full + 8 * stage;
                    const uint32_t dA = sbase + stage * STAGE_BYTES, dB = dA + A_BYTES;
                    const uint32_t dSA = dB + B_BYTES, dSB = dSA + SFA_BYTES;
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    tma_load_2d(dA, &tmA, kb * KB_BYTES, x.m0, fb);
                    tma_load_2d(dB, &tmB, kb * KB_BYTES, brow, fb);
                    bulk_g2s(dSA, sfa + (int64_t)2 * kb * SF_BLOCK, SFA_BYTES, fb);
                    bulk_g2s(dSB, sfb + (int64_t)4 * kb * SF_BLOCK, SFB_BYTES, fb);
                    pend |= 1u << stage;
                    pend_phase = (pend_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            if (!ok)
                for (int s = 0; s < STAGES; ++s)
                    if (pend & (1u << s)) wait_drain(bar_full + 8 * s, (pend_phase >> s) & 1u);
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ----
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, tphase = 0;
            bool ok = true, issued = false;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                // the epilogue has drained the accumulator of the previous tile
                if (!wait_bounded(bar_tempty, tphase ^ 1, p.budget, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                tphase ^= 1;
                tc_fence_after();
                for (int kb = 0; kb < KB; ++kb) {
                    if (!wait_bounded(bar_full + 8 * stage, phase, p.budget, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t dA = sbase + stage * STAGE_BYTES, dB = dA + A_BYTES;
                    const uint32_t dSA = dB + B_BYTES, dSB = dSA + SFA_BYTES;
                    const uint32_t sf = tmem_base + SF_COL0 + SF_SLOT_COLS * (uint32_t)stage;
                    sf_copy(sf, sf_desc(dSA));
                    sf_copy(sf + 8, sf_desc(dSA + SF_BLOCK));
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) sf_copy(sf + 16 + 8 * ks, sf_desc(dSB + ks * SF_BLOCK));
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_nvf4(tmem_base, sdesc(dA + 32 * ks), sdesc(dB + 32 * ks), sf + 4 * ks, sf + 16 + 8 * ks,
                                 (kb | ks) != 0 ? 1u : 0u);
                    mma_commit(bar_empty + 8 * stage);   // the stage and its scale slot are free
                    issued = true;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (ok) mma_commit(bar_tfull);   // the tile's accumulator is complete
            }
            if (issued) {
                mma_commit(bar_drain);
                wait_drain(bar_drain, 0);
            }
        }
    } else if (warp >= EPI_WARP0) {
        // --------------------------------------------------- epilogue ----
        const int q = warp & 3, h = (warp - EPI_WARP0) >> 2;   // lane quarter, column half
        const int row = 32 * q + lane;
        const uint32_t lane_addr = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(128 * h);
        uint32_t tphase = 0;
        const float a_sg = *p.a_sg;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
            const Tile x = tile_of(t, p, offs_s);
            if (!warp_wait_bounded(bar_tfull, tphase, p.budget, abort_flag, p.status)) break;
            tphase ^= 1;
            tc_fence_after();
            const float inv = __fdiv_rn(1.0f, a_sg * p.b_sg[x.e]);
            float *o = p.out + ((int64_t)x.m0 + row) * p.N + x.n0 + 128 * h;
            // the warp's 128 columns read at once, the accumulator handed back to
            // the next tile's MMAs, then scaled and stored (the stores no longer
            // hold the tensor core: measured, 6.7k cycles per tile with reads and
            // stores interleaved)
            uint32_t r[128];
#pragma unroll
            for (int j = 0; j < 8; ++j) MOE_TMEM_LD16(lane_addr + (uint32_t)(16 * j), (r + 16 * j));
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_tempty);
#pragma unroll
            for (int i = 0; i < 128; i += 4) {
                float4 v;
                v.x = __uint_as_float(r[i]) * inv;
                v.y = __uint_as_float(r[i + 1]) * inv;
                v.z = __uint_as_float(r[i + 2]) * inv;
                v.w = __uint_as_float(r[i + 3]) * inv;
                *reinterpret_cast<float4 *>(o + i) = v;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS));
}

}  // namespace nvfp4g

int launch_gemm_nvfp4(int64_t R_cap, int N, int K, int n_seg, const int32_t *offsets, const uint8_t *a,
                      const uint8_t *sfa, const float *a_sg, const uint8_t *b, const uint8_t *sfb,
                      const float *b_sg, float *out, int *status, uint64_t budget, cudaStream_t s)
{
    using namespace nvfp4g;
    CUtensorMap mA, mB;
    if (!sm100::make_map(&mA, a, (uint64_t)K / 2, (uint64_t)R_cap, BM) ||
        !sm100::make_map(&mB, b, (uint64_t)K / 2, (uint64_t)n_seg * N, BN))
        return MOE_ERR_CUDA;
    Args args{};
    args.offsets = offsets;
    args.n_seg = n_seg;
    args.N = N;
    args.K = K;
    args.sfa = sfa;
    args.sfb = sfb;
    args.a_sg = a_sg;
    args.b_sg = b_sg;
    args.out = out;
    args.status = status;
    args.budget = budget;
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(gemm_nvfp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
        configured = true;
    }
    gemm_nvfp4_kernel<<<sm100::sm_count(), NUM_THREADS, SMEM_BYTES, s>>>(mA, mB, args);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
