// Grouped block-scaled FP8 GEMMs of the expert FFN on sm_100a tensor cores
// (a6 gate/up + SiLU + h-quant, a7 down, b2 dgrad down + SiLU backward,
// b3 dgrad gate/up, b4 wgrad).  Block-scaled FP8 as proposed by DeepSeek-V3
// is what the trainer runs ("RL at 1T scale: prime-rl performance deep
// dive", §FP8 Training).
//
// Design (one persistent CTA per SM, 12 warps = 3 warpgroups):
//   warp 0     TMA producer: 128-byte-swizzled tiles of A (128 x 128 B) and
//              B (256 x 128 B) per 128-deep K block into a 4-stage ring;
//   warp 1     allocates 512 TMEM columns; lane 0 issues tcgen05.mma
//              (kind::f8f6f4, e4m3 x e4m3 -> fp32, M=128, N=256, K=32) x4
//              per K block into one of two 256-column TMEM accumulators;
//   warps 2-3  idle (they complete warpgroup 0, which gives its registers
//              to the epilogue: setmaxnreg 40 here, 232 in warpgroups 1-2;
//              128*40 + 256*232 = 384*168, the launch allocation);
//   warps 4-11 epilogue: per K block, read the accumulator with tcgen05.ld,
//              multiply by that block's scales (row scale x weight-block
//              scale; per-column for wgrad) and add into fp32 registers; the
//              freed TMEM buffer is handed back while the MMA fills the
//              other.  After the last K block: the fused output step (TMA
//              stores of bf16 rows or h codes; 32-byte stores of the
//              SiLU-backward outputs; L2 reductions into dW for wgrad).
//              Rows mode reads TMEM in the 32x32b shape (a thread = a row),
//              wgrad in the 16x256b shape (a thread = 4 rows x 32 columns,
//              fewer column scales per thread).
// 2-SM variant (rows mode): clusters of two CTAs on two SMs; the leader issues
// tcgen05.mma.cta_group::2 with M = 256 (each CTA's own 128 rows of A) and
// N = 128, each K block as two column halves into separate 128-column TMEM
// slots (four slots in all).  The epilogue warpgroup of one half releases its
// slot while the other half's MMAs still run, so the MMA-to-release round trip
// has three half-K-blocks of MMA work to hide behind instead of one K block.
// Each CTA loads its own operand rows (no multicast); per SM and K block the
// shared memory moves 32 KB of TMA writes and 48 KB of MMA reads instead of
// 48 + 48 KB in the one-SM tile.
// The scales are arbitrary fp32 (amax/448), so they cannot ride in the
// hardware block-scaled MMA (which takes power-of-two UE8M0 scales); each
// K block's partial product is promoted in fp32 instead.
//
// Tile spaces:
//   rows mode (a6, a7, b2, b3): one tile = 128 permuted rows (always inside
//   one expert: segments are 128-aligned) x 256 output columns; K = D, I or
//   2I.  The number of row tiles, offsets[E]/128, is read on the device.
//   wgrad mode (b4): one tile = (expert, 128 rows of dW, 256 columns of dW);
//   K runs over the expert's permuted rows.
//
// Every mbarrier wait is bounded; on expiry the kernel latches
// MOE_ERR_TIMEOUT, drains the copies and MMAs it issued, frees TMEM and exits.
#include "sm100.cuh"

namespace moe {

namespace gemm {

constexpr int BM = 128, BN = 256, BK = 128;
constexpr int A_BYTES = BM * BK;
constexpr int NUM_THREADS = 384;
constexpr int EPI_WARP0 = 4;
constexpr int EPI_THREADS = 256;
constexpr uint32_t TMEM_COLS = 512;
constexpr int WS_FLOATS = 128 + 256;
constexpr int SC_SLOTS = 8;
constexpr int TSTORE_BUF = 32 * 64;

// Shared memory of one variant (kPair: the 2-SM MMA, where each CTA of a pair
// holds its own 128 rows of A and half of B):
//   operand ring [STAGES][A tile | B tile] | barriers (full[STAGES],
//   empty[STAGES], tfull[2], tempty[2], drain, epi) | tmem slot | abort flag |
//   offsets[257] | (kPair) pair-tile prefix sums[257] | then, 1024-aligned, a
//   region whose use depends on the epilogue:
//   SILU   amax exchange [2][2][128] fp32 | h-code store buffers [8 warps][32 rows][64 B]
//   BF16   output store buffers [8 warps][2][32 rows][64 B]
//   WGRAD  scale ring [SC_SLOTS][128 row + 256 column] fp32 with its own
//          full/empty barriers (filled by the producer, released by the
//          epilogue warps), deeper than the operand ring
//   DSILU  unused
// Store buffers are read by TMA stores (32 rows x 64 bytes boxes; bf16 boxes under
// the 64-byte swizzle, code boxes plain).
template <bool kPair, int kEpi = 0>
struct Lay {
    // the 2-SM bf16 output keeps four store boxes per warp (below) in place of
    // the ring's fifth stage
    static constexpr int STAGES = kPair ? (kEpi == 1 ? 4 : 5) : 4;
    static constexpr int BF16_BUFS = kPair ? 4 : 2;   // store boxes per epilogue warp (bf16 output)
    static constexpr int B_BYTES = (kPair ? BN / 2 : BN) * BK;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
    static constexpr int OFF_TMEM_SLOT = OFF_BAR + 24 * 8;
    static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 4;
    static constexpr int OFF_OFFSETS = OFF_BAR + 256;
    static constexpr int OFF_PAIRS = OFF_OFFSETS + 1040;
    static constexpr int OFF_DEFXY = OFF_PAIRS + (kPair ? 1040 : 0);   // SILU: [8 warps][2] ints
    static constexpr int OFF_EPI = (OFF_DEFXY + 64 + 1023) / 1024 * 1024;
    static constexpr int OFF_AMAX = OFF_EPI;
    static constexpr int OFF_WS = OFF_EPI;
    static constexpr int OFF_WS_BAR = OFF_WS + SC_SLOTS * WS_FLOATS * 4;  // sfull[SC_SLOTS], sempty[SC_SLOTS]
    static constexpr int OFF_TSTORE_SILU = OFF_EPI + 2 * 2 * 128 * 4;
    static constexpr int OFF_TSTORE_BF16 = OFF_EPI;
    // pair mode, SILU: each epilogue thread's 64 h values (bf16) wait here for
    // their quantisation, which runs during the next tile's K loop; rows of
    // 128 h values padded to 272 bytes (16-byte accesses free of bank conflicts)
    static constexpr int HSTAGE_ROW = 272;
    static constexpr int OFF_HSTAGE = OFF_TSTORE_SILU + 8 * TSTORE_BUF;
};

enum Epi { EPI_SILU = 0, EPI_BF16 = 1, EPI_DSILU = 2, EPI_WGRAD = 3 };

template <int kEpi, bool kPair = false>
constexpr int smem_bytes()
{
    using L = Lay<kPair, kEpi>;
    return 1024 + (kEpi == EPI_SILU   ? L::OFF_TSTORE_SILU + 8 * TSTORE_BUF + (kPair ? 128 * L::HSTAGE_ROW : 0)
                   : kEpi == EPI_BF16 ? L::OFF_TSTORE_BF16 + 8 * L::BF16_BUFS * TSTORE_BUF
                   : kEpi == EPI_WGRAD ? L::OFF_WS_BAR + 2 * SC_SLOTS * 8
                                       : L::OFF_EPI);  // + alignment slack
}
static_assert(smem_bytes<EPI_SILU>() <= 232448 && smem_bytes<EPI_BF16>() <= 232448 &&
                  smem_bytes<EPI_WGRAD>() <= 232448 && smem_bytes<EPI_DSILU>() <= 232448 &&
                  smem_bytes<EPI_SILU, true>() <= 232448 && smem_bytes<EPI_BF16, true>() <= 232448 &&
                  smem_bytes<EPI_DSILU, true>() <= 232448,
              "shared memory budget");
static_assert(EPI_BF16 == 1, "Lay's bf16 layout");
static_assert(Lay<false>::OFF_DEFXY + 64 <= Lay<false>::OFF_EPI && Lay<true>::OFF_DEFXY + 64 <= Lay<true>::OFF_EPI,
              "deferred-store coordinates below the epilogue region");
static_assert(Lay<false>::OFF_EPI == 198656, "the one-SM layout is unchanged");

struct Args {
    const int32_t *offsets;
    int E;   // row segments (rows mode) or experts (wgrad mode)
    int ew;  // rows mode: segment v uses the weights of expert v % ew
    int64_t R_cap;
    int M;  // wgrad: rows of dW (D or 2I)
    int N;  // output columns
    int K;  // rows mode: reduction length
    const float *sa;
    const float *sb;
    const uint16_t *aux;
    uint8_t *out_q;
    float *out_s;
    uint16_t *out_bf16;
    float *out_f32;
    int *status;
    uint64_t budget;
    // gather (a6 only): A rows come from the token-row codes a_rows [T][K],
    // row r of the permuted layout being token src_idx[r] / k (no row for
    // src_idx < 0); row scales sa[kb * T + token]
    const uint8_t *a_rows;
    const int32_t *src_idx;
    int k;
    int T;
};

// ----------------------------------------------------------------- PTX ----
using namespace sm100;

// Instruction descriptor, kind::f8f6f4: D fp32, A and B e4m3, both K-major,
// N = 256, M = 128.
constexpr uint32_t IDESC = (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void mma_f8(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t accum)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(IDESC), "r"(accum));
}

// The 2-SM MMA (cta_group::2): M = 256 over the CTA pair (128 rows of A in
// each CTA's shared memory at the same offset), N = 128: each CTA supplies 64
// rows of B from the same offset, the leader's give D columns 0-63 and the
// peer's columns 64-127; D lands in each CTA's TMEM (its own 128 rows).
// Issued by the leader CTA only, twice per K block (the two column halves of
// the 256-column tile, each into its own TMEM slot).
constexpr int BN_HALF = BN / 2;
constexpr uint32_t IDESC_PAIR = (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(BN_HALF >> 3) << 17) |
                                ((uint32_t)(2 * BM >> 4) << 24);

__device__ __forceinline__ void mma_f8_pair(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t accum)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(IDESC_PAIR), "r"(accum));
}

// Arrives once, when the leader's MMAs issued so far are done, on the barrier
// at this offset in each CTA of the pair.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"((uint16_t)3)
        : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// shared::cluster address of the same shared-memory offset in CTA `rank`
__device__ __forceinline__ uint32_t peer_addr(uint32_t a, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// arrive on an mbarrier given by its shared::cluster address (any CTA of the
// cluster).  The arriving thread's TMEM reads have completed (tcgen05.wait::ld)
// and are fenced (tcgen05.fence::before_thread_sync); nothing else needs to be
// made visible to the peer, so the arrive keeps the default CTA-scope order.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}

// TMA tile load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (shared::cluster address).  No
// multicast: every CTA loads its own bytes.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int32_t c0, int32_t c1,
                                                 uint32_t bar_cluster)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}

// Four rows (row coordinates r0..r3, the same 128-byte column window c0) of a
// tensor whose map has a one-row box, into four consecutive 128-byte rows of
// shared memory (128-byte swizzled like any TMA tile).
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap *map, int32_t c0, int32_t r0,
                                            int32_t r1, int32_t r2, int32_t r3, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
        : "memory");
}

// ------------------------------------------------------------ schedule ----
struct Tile {
    int e;      // expert
    int m0;     // first row (rows mode: permuted row; wgrad: row of dW)
    int n0;     // first output column
    int nt;     // column-tile index
    int kb0;    // first K block
    int kb1;    // one past the last K block
    bool valid; // this CTA's rows belong to the tile (a pair's second half may not)
};

// Pair mode: segment v of 128-row tiles mt_v = (offs[v+1] - offs[v]) / 128 has
// ceil(mt_v / 2) pair tiles; pps[v] counts them before segment v.
template <bool kWgrad, bool kPair>
__device__ __forceinline__ int num_tiles(const Args &p, const int *offs_s, const int *pps_s)
{
    const int NT = (p.N + BN - 1) / BN;
    if (kWgrad) return p.E * (p.M / BM) * NT;
    if (kPair) return pps_s[p.E] * NT;
    return (offs_s[p.E] / BM) * NT;
}

template <bool kWgrad, bool kPair = false>
__device__ __forceinline__ Tile tile_of(int t, const Args &p, const int *offs_s, const int *pps_s = nullptr,
                                        uint32_t rank = 0)
{
    const int NT = (p.N + BN - 1) / BN;
    Tile x;
    x.valid = true;
    if (kWgrad) {
        const int MT = p.M / BM;
        x.e = t / (MT * NT);
        int rem = t - x.e * MT * NT;
        int mt = rem / NT;
        x.nt = rem - mt * NT;
        x.m0 = mt * BM;
        x.n0 = x.nt * BN;
        x.kb0 = offs_s[x.e] / BK;
        x.kb1 = offs_s[x.e + 1] / BK;
    } else if (kPair) {
        const int pt = t / NT;
        x.nt = t - pt * NT;
        x.n0 = x.nt * BN;
        int lo = 0, hi = p.E - 1;  // last v with pps[v] <= pt
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (pps_s[mid] <= pt) lo = mid; else hi = mid - 1;
        }
        const int base = offs_s[lo] + 2 * BM * (pt - pps_s[lo]);
        x.m0 = base + BM * (int)rank;
        x.valid = x.m0 < offs_s[lo + 1];
        x.e = lo < p.ew ? lo : lo % p.ew;
        x.kb0 = 0;
        x.kb1 = p.K / BK;
    } else {
        int mt = t / NT;
        x.nt = t - mt * NT;
        x.m0 = mt * BM;
        x.n0 = x.nt * BN;
        int lo = 0, hi = p.E - 1;  // last e with offs[e] <= m0
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (offs_s[mid] <= x.m0) lo = mid; else hi = mid - 1;
        }
        x.e = lo < p.ew ? lo : lo % p.ew;   // the weights' expert
        x.kb0 = 0;
        x.kb1 = p.K / BK;
    }
    return x;
}

// Byte offset of 16-byte chunk c of row r in a bf16 TMA store box of 64-byte
// rows under the 64-byte swizzle (the chunk index XOR bits 1-2 of the row): the
// 32 lanes of a warp writing one chunk of their own rows then spread over all
// eight 16-byte bank groups instead of two.  Boxes start on 1024-byte
// boundaries, so the pattern lines up with the address bits TMA swizzles.
// (Measured on the down GEMM: output step 3.4k -> 2.9k cycles per tile.  The
// h-code boxes of the gate/up GEMM stay unswizzled: there it measured no
// better.)
__device__ __forceinline__ int box_off(int r, int c) { return r * 64 + ((c ^ ((r >> 1) & 3)) << 4); }

// 32-byte global accesses (sm_100 vector width); the address must be 32-byte aligned.
__device__ __forceinline__ void ld_global_32B(const void *src, uint4 *v)
{
    asm volatile("ld.global.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v[0].x), "=r"(v[0].y), "=r"(v[0].z), "=r"(v[0].w), "=r"(v[1].x), "=r"(v[1].y), "=r"(v[1].z),
                   "=r"(v[1].w)
                 : "l"(src));
}
__device__ __forceinline__ void st_global_32B(void *dst, const uint4 &a, const uint4 &b)
{
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(a.x), "r"(a.y), "r"(a.z),
                 "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
                 : "memory");
}

// --------------------------------------------------------------- kernel ----
template <int kEpi, bool kGather = false, bool kPair = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const Args p)
{
    constexpr bool kWgrad = (kEpi == EPI_WGRAD);
    static_assert(!(kPair && (kWgrad || kGather)), "the 2-SM variant covers the rows-mode GEMMs");
    using L = Lay<kPair, kEpi>;
    constexpr int STAGES = L::STAGES, STAGE_BYTES = L::STAGE_BYTES;
    constexpr int OFF_BAR = L::OFF_BAR, OFF_ABORT = L::OFF_ABORT, OFF_TMEM_SLOT = L::OFF_TMEM_SLOT;
    constexpr int OFF_OFFSETS = L::OFF_OFFSETS, OFF_AMAX = L::OFF_AMAX, OFF_WS = L::OFF_WS;
    constexpr int OFF_WS_BAR = L::OFF_WS_BAR, OFF_TSTORE_SILU = L::OFF_TSTORE_SILU;
    constexpr int OFF_TSTORE_BF16 = L::OFF_TSTORE_BF16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar_full = sbase + OFF_BAR;           // [STAGES]
    const uint32_t bar_empty = bar_full + STAGES * 8;     // [STAGES]
    // TMEM slots: two 256-column buffers; in pair mode each buffer is two
    // 128-column slots (one per MMA column half), slot 2 * buffer + half
    constexpr int NQ = kPair ? 4 : 2;
    static_assert(2 * STAGES * 8 + 2 * NQ * 8 + 16 <= OFF_TMEM_SLOT - OFF_BAR, "barrier area");
    const uint32_t bar_tfull = bar_empty + STAGES * 8;    // [NQ]
    const uint32_t bar_tempty = bar_tfull + NQ * 8;       // [NQ]
    const uint32_t bar_drain = bar_tempty + NQ * 8;
    const uint32_t bar_epi = bar_drain + 8;  // the 256 epilogue threads meet here
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_ABORT);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_TMEM_SLOT);
    int *offs_s = reinterpret_cast<int *>(smem + OFF_OFFSETS);
    int *pps_s = reinterpret_cast<int *>(smem + L::OFF_PAIRS);        // pair mode: [E+1]
    float *amax_s = reinterpret_cast<float *>(smem + OFF_AMAX);       // [2][2][128]
    float *wscale = reinterpret_cast<float *>(smem + OFF_WS);          // wgrad: [SC_SLOTS][WS_FLOATS]
    const uint32_t bar_sfull = sbase + OFF_WS_BAR;                     // wgrad: [SC_SLOTS]
    const uint32_t bar_sempty = bar_sfull + SC_SLOTS * 8;              // wgrad: [SC_SLOTS]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // pair mode: CTA `rank` of the pair (0 leads: it issues the MMAs and
    // holds the barriers the pair's loads and TMEM releases count on); the
    // pairs walk the tiles together
    const uint32_t rank = kPair ? cluster_rank() : 0;
    const int t_first = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int t_step = kPair ? (int)(gridDim.x >> 1) : (int)gridDim.x;

    for (int i = threadIdx.x; i <= p.E; i += blockDim.x) offs_s[i] = p.offsets[i];
    if (kPair) {
        __syncthreads();
        if (threadIdx.x == 0) {
            int acc = 0;
            for (int v = 0; v < p.E; ++v) {
                pps_s[v] = acc;
                acc += ((offs_s[v + 1] - offs_s[v]) / BM + 1) / 2;
            }
            pps_s[p.E] = acc;
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            // gathering: the B load's arrival and the 64 gathering threads' cp.async arrivals
            mbar_init(bar_full + 8 * s, kGather ? 65 : 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        if (kWgrad)
            for (int s = 0; s < SC_SLOTS; ++s) {
                mbar_init(bar_sfull + 8 * s, 1);
                mbar_init(bar_sempty + 8 * s, EPI_THREADS / 32);
            }
        // a slot is released by the epilogue warps that read it: all eight
        // (one SM), or one warpgroup in each CTA of the pair (2 x 4)
        for (int b = 0; b < NQ; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, EPI_THREADS / 32);
        }
        mbar_init(bar_drain, 1);
        mbar_init(bar_epi, EPI_THREADS);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        if (kPair) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                         "r"(TMEM_COLS));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                         "r"(TMEM_COLS));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        }
    }
    tc_fence_before();
    __syncthreads();
    if (kPair) cluster_sync_all();   // both CTAs' barriers exist before either signals the other's
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int ntiles = num_tiles<kWgrad, kPair>(p, offs_s, pps_s);
    // the leader's barriers as the pair addresses them
    const uint32_t lead_full = kPair ? peer_addr(bar_full, 0) : bar_full;
    const uint32_t lead_tempty = kPair ? peer_addr(bar_tempty, 0) : bar_tempty;

    if (warp < EPI_WARP0) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");
      if (kGather && (warp == 0 || warp >= 2)) {
        // ------------------------------------------ producer, gathering ----
        // The A rows of each K block come from the token-row codes along two
        // paths at once (each alone kept the tensor core waiting longer): warp 0
        // loads tile rows 0-63 with TMA tile::gather4 (lanes 0-15, four rows
        // each) and B with a TMA tile load (lane 0); warps 2-3 copy tile rows
        // 64-127 with cp.async, one row per thread, 16 bytes a copy, into the
        // same 128-byte-swizzled layout (a row with no token reads zeros).  The stage's full barrier counts the TMA bytes
        // and lane 0's arrival plus the 64 threads' cp.async arrivals
        // (cp.async.mbarrier.arrive.noinc).
        const bool tma_side = warp == 0;
        int stage = 0;
        uint32_t phase = 0;
        uint32_t pend = 0, pend_phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const Tile x = tile_of<false>(t, p, offs_s);
            int tok[4] = {-1, -1, -1, -1};
            if (tma_side) {
                if (lane < 16)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int si = p.src_idx[x.m0 + 4 * lane + i];
                        tok[i] = si >= 0 ? si / p.k : p.T;   // row T is out of range: zeros
                    }
            } else {
                const int si = p.src_idx[x.m0 + 64 + 32 * (warp - 2) + lane];
                tok[0] = si >= 0 ? si / p.k : -1;
            }
            for (int kb = x.kb0; kb < x.kb1; ++kb) {
                if (!warp_wait_bounded(bar_empty + 8 * stage, phase ^ 1, p.budget, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                pend &= ~(1u << stage);
                const uint32_t fb = bar_full + 8 * stage;
                const uint32_t dA = sbase + stage * STAGE_BYTES, dB = dA + A_BYTES;
                if (tma_side) {
                    if (lane == 0) {
                        mbar_arrive_expect_tx(fb, L::B_BYTES + A_BYTES / 2);
                        tma_load_2d(dB, &tmB, kb * BK, x.e * p.N + x.n0, fb);
                    }
                    __syncwarp();
                    if (lane < 16) tma_gather4(dA + 512 * lane, &tmA, kb * BK, tok[0], tok[1], tok[2], tok[3], fb);
                } else {
                    const int r = 64 + 32 * (warp - 2) + lane;
                    const uint8_t *src = tok[0] >= 0 ? p.a_rows + (int64_t)tok[0] * p.K + kb * BK : p.a_rows;
                    const uint32_t bytes = tok[0] >= 0 ? 16u : 0u;
#pragma unroll
                    for (int c = 0; c < BK / 16; ++c)
                        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                                         dA + r * BK + ((c ^ (r & 7)) << 4)),
                                     "l"(src + 16 * c), "r"(bytes)
                                     : "memory");
                    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(fb) : "memory");
                }
                pend |= 1u << stage;
                pend_phase = (pend_phase & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");   // no copy of this thread outlives the CTA
        if (!ok && tma_side && lane == 0)
            for (int s = 0; s < STAGES; ++s)
                if (pend & (1u << s)) wait_drain(bar_full + 8 * s, (pend_phase >> s) & 1u);
      } else if (warp == 0) {
        // ------------------------------------------------ TMA producer ----
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t pend = 0, pend_phase = 0;  // loads issued, not yet seen consumed
            int sslot = 0;                      // wgrad scale ring
            uint32_t sphase = 0, spend = 0, spend_phase = 0;
            bool ok = true;
            for (int t = t_first; t < ntiles && ok; t += t_step) {
                const Tile x = tile_of<kWgrad, kPair>(t, p, offs_s, pps_s, rank);
                for (int kb = x.kb0; kb < x.kb1; ++kb) {
                    if (!wait_bounded(bar_empty + 8 * stage, phase ^ 1, p.budget, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
                    pend &= ~(1u << stage);
                    const uint32_t fb = bar_full + 8 * stage;
                    const uint32_t dA = sbase + stage * STAGE_BYTES, dB = dA + A_BYTES;
                    if (kWgrad) {
                        // the K block's scales into the next slot of the scale ring
                        if (!wait_bounded(bar_sempty + 8 * sslot, sphase ^ 1, p.budget, abort_flag, p.status)) {
                            ok = false;
                            break;
                        }
                        spend &= ~(1u << sslot);
                        const int ncols = min(BN, p.N - x.n0);  // 128 or 256 (N is a multiple of 128)
                        const uint32_t ws = smem_u32(wscale + sslot * WS_FLOATS), sfb = bar_sfull + 8 * sslot;
                        mbar_arrive_expect_tx(sfb, 4 * (BM + ncols));
                        bulk_g2s(ws, p.sa + (int64_t)kb * p.M + x.m0, 4 * BM, sfb);
                        bulk_g2s(ws + 4 * BM, p.sb + (int64_t)kb * p.N + x.n0, 4 * ncols, sfb);
                        spend |= 1u << sslot;
                        spend_phase = (spend_phase & ~(1u << sslot)) | (sphase << sslot);
                        if (++sslot == SC_SLOTS) {
                            sslot = 0;
                            sphase ^= 1;
                        }
                        mbar_arrive_expect_tx(fb, STAGE_BYTES);
                        tma_load_2d(dA, &tmA, kb * BK, x.m0, fb);
                        tma_load_2d(dB, &tmB, kb * BK, x.n0, fb);
                    } else if (kPair) {
                        // this CTA's 128 rows of A and 128 rows of B; both CTAs'
                        // bytes complete on the leader's full barrier.  B rows
                        // 64h..64h+63 of this CTA feed column half h of the MMA:
                        // SILU, tile rows 128 * rank + [0, 128) (the leader the
                        // gate block, the peer the up block: each half gets 64
                        // gate and the matching 64 up columns); otherwise tile
                        // rows 128h + 64 * rank + [0, 64) (half h = output
                        // columns 128h .. 128h + 127, in order)
                        const uint32_t lfb = lead_full + 8 * stage;
                        const int brow = x.e * p.N + x.n0;
                        if (rank == 0) mbar_arrive_expect_tx(fb, 2 * STAGE_BYTES);
                        tma_load_2d_pair(dA, &tmA, kb * BK, x.m0, lfb);
                        if (kEpi == EPI_SILU) {
                            tma_load_2d_pair(dB, &tmB, kb * BK, brow + BN_HALF * (int)rank, lfb);
                        } else {
                            tma_load_2d_pair(dB, &tmB, kb * BK, brow + 64 * (int)rank, lfb);
                            tma_load_2d_pair(dB + L::B_BYTES / 2, &tmB, kb * BK, brow + BN_HALF + 64 * (int)rank,
                                             lfb);
                        }
                    } else {
                        mbar_arrive_expect_tx(fb, STAGE_BYTES);
                        tma_load_2d(dA, &tmA, kb * BK, x.m0, fb);
                        tma_load_2d(dB, &tmB, kb * BK, x.e * p.N + x.n0, fb);
                    }
                    pend |= 1u << stage;
                    pend_phase = (pend_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // (pair mode: the peer's loads complete on the leader's barriers;
            // the leader's drain waits for the stages it announced, and the
            // pair leaves together after the closing cluster barrier)
            if (!ok && rank == 0) {
                for (int s = 0; s < STAGES; ++s)
                    if (pend & (1u << s)) wait_drain(bar_full + 8 * s, (pend_phase >> s) & 1u);
                if (kWgrad)
                    for (int s = 0; s < SC_SLOTS; ++s)
                        if (spend & (1u << s)) wait_drain(bar_sfull + 8 * s, (spend_phase >> s) & 1u);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ----
        // (pair mode: the leader only; its MMAs span both CTAs)
        if (lane == 0 && rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int buf = 0;
            uint32_t bphase = 0;
            bool ok = true, issued = false;
            for (int t = t_first; t < ntiles && ok; t += t_step) {
                const Tile x = tile_of<kWgrad, kPair>(t, p, offs_s, pps_s, rank);
                for (int kb = x.kb0; kb < x.kb1; ++kb) {
                    if (kPair) {
                        // two column halves, each into its own slot as soon as
                        // that slot is free (the epilogue warpgroup of half 0
                        // releases it while half 1's MMAs still run)
                        if (!wait_bounded(bar_full + 8 * stage, phase, p.budget, abort_flag, p.status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t aA = sbase + stage * STAGE_BYTES, aB = aA + A_BYTES;
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int slot = 2 * buf + hh;
                            if (!wait_bounded(bar_tempty + 8 * slot, bphase ^ 1, p.budget, abort_flag, p.status)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            const uint32_t dtm = tmem_base + (uint32_t)(buf * BN + hh * BN_HALF);
                            const uint32_t bB = aB + (uint32_t)(hh * (L::B_BYTES / 2));
#pragma unroll
                            for (int k4 = 0; k4 < BK / 32; ++k4)
                                mma_f8_pair(dtm, sdesc(aA + 32 * k4), sdesc(bB + 32 * k4), k4 > 0 ? 1u : 0u);
                            mma_commit_pair(bar_tfull + 8 * slot);    // both CTAs' warpgroup hh may read
                            issued = true;
                        }
                        if (!ok) break;
                        mma_commit_pair(bar_empty + 8 * stage);       // both CTAs' stage is free
                    } else {
                        if (!wait_bounded(bar_tempty + 8 * buf, bphase ^ 1, p.budget, abort_flag, p.status)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        if (!wait_bounded(bar_full + 8 * stage, phase, p.budget, abort_flag, p.status)) {
                            ok = false;
                            break;
                        }
                        // (gathering: A was written by cp.async, through the generic
                        // proxy; the MMA reads it through the async proxy)
                        if (kGather) fence_proxy_async_smem();
                        tc_fence_after();
                        const uint32_t aA = sbase + stage * STAGE_BYTES, aB = aA + A_BYTES;
                        const uint32_t dtm = tmem_base + (uint32_t)(buf * BN);
#pragma unroll
                        for (int k4 = 0; k4 < BK / 32; ++k4)
                            mma_f8(dtm, sdesc(aA + 32 * k4), sdesc(aB + 32 * k4), k4 > 0 ? 1u : 0u);
                        mma_commit(bar_empty + 8 * stage);
                        mma_commit(bar_tfull + 8 * buf);
                        issued = true;
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                    buf ^= 1;
                    if (buf == 0) bphase ^= 1;
                }
            }
            if (issued) {
                if (kPair)
                    mma_commit_pair(bar_drain);
                else
                    mma_commit(bar_drain);
                wait_drain(bar_drain, 0);
            }
        }
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 232;");
        // --------------------------------------------------- epilogue ----
        const int ew = warp - EPI_WARP0;     // 0..7
        const int q = warp & 3;              // TMEM lane quarter of this warp
        const int h = ew >> 2;               // column half
        const int row = 32 * q + lane;       // row within the tile
        const uint32_t lane_addr = tmem_base + ((uint32_t)(32 * q) << 16);
        const int KB = p.K / BK, NB = p.N / BK;
        int buf = 0;
        uint32_t bphase = 0;
        int wstage = 0;  // wgrad: scale-ring slot of the current K block
        uint32_t wphase = 0;
        int tcount = 0;
        bool ok = true;
        uint32_t ephase = 0;
        // all epilogue threads meet; bounded, so an aborting CTA cannot hang here
        auto epi_sync = [&]() -> bool {
            mbar_arrive(bar_epi);
            bool r = wait_bounded(bar_epi, ephase, p.budget, abort_flag, p.status);
            ephase ^= 1;
            return r;
        };
        // SILU, 2-SM layout: the h codes of a tile are made during the next
        // tile's K loop, four per thread after each K block (the scale is known
        // by then); the h values wait in this thread's own slot of a
        // shared-memory staging area.  (In the one-SM kernel the state this
        // keeps live through the K loop cost register spills there that slowed
        // it by a third; its codes are made at once.)
        constexpr bool kDefer = kEpi == EPI_SILU && kPair;
        constexpr bool defer_on = kDefer;
        int def_left = 0;           // h values of the deferred tile still to quantise
        float def_s = 0.0f;
        // the deferred tile's store coordinates (column, first row), per warp, kept in
        // shared memory: the K loop's registers are all taken
        int *def_xy = reinterpret_cast<int *>(smem + L::OFF_DEFXY) + 2 * ew;
        const uint8_t *def_src = nullptr;   // this thread's 64 h values (bf16) of the deferred tile
        uint2 def_next = make_uint2(0, 0);  // the next four, loaded one step ahead
        uint8_t *hst = smem + L::OFF_HSTAGE + row * L::HSTAGE_ROW + 128 * h;   // 2-SM staging slot
        uint8_t *box = smem + OFF_TSTORE_SILU + ew * TSTORE_BUF;              // this warp's code box
        auto defer_step = [&]() {
            if (!kDefer || def_left == 0) return;   // warp-uniform
            const int i0 = 64 - def_left;
            if (i0 == 0) {
                if (lane == 0) bulk_wait_read<0>();   // the box's previous store has read it
                __syncwarp();
            }
            const uint2 hv = def_next;
            if (i0 + 4 < 64) def_next = *reinterpret_cast<const uint2 *>(def_src + 2 * (i0 + 4));
            const float v[4] = {bf16_lo(hv.x), bf16_hi(hv.x), bf16_lo(hv.y), bf16_hi(hv.y)};
            *reinterpret_cast<uint32_t *>(box + lane * 64 + i0) = quant4(v, def_s);
            def_left -= 4;
            if (def_left == 0) {
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmC, smem_u32(box), def_xy[0], def_xy[1] + 32 * q);
                    bulk_commit();
                }
            }
        };
        for (int t = t_first; t < ntiles && ok; t += t_step, ++tcount) {
            const Tile x = tile_of<kWgrad, kPair>(t, p, offs_s, pps_s, rank);
            if (kWgrad && x.kb1 == x.kb0) continue;
            float acc[128];
#pragma unroll
            for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
            // Scales of K block kb.  Rows mode: plain loads two K blocks ahead
            // into registers (row scale, weight-block scale(s)).  Wgrad: the
            // producer bulk-copies them into the scale ring, up to SC_SLOTS K
            // blocks ahead; each warp releases a slot after reading it.
            int tok_r = 0;
            if (kGather) {
                const int si = p.src_idx[x.m0 + row];
                tok_r = si >= 0 ? si / p.k : -1;
            }
            auto load_rows = [&](int kb, float &a, float &b0, float &b1) {
                if (kGather)
                    a = tok_r >= 0 ? p.sa[(int64_t)kb * p.T + tok_r] : 0.0f;
                else   // (a pair's idle half may lie past the last row)
                    a = x.valid ? p.sa[(int64_t)kb * p.R_cap + x.m0 + row] : 0.0f;
                const int64_t sbrow = (int64_t)x.e * NB + 2 * x.nt;
                if (kEpi == EPI_SILU) {
                    b0 = p.sb[sbrow * KB + kb];        // gate block
                    b1 = p.sb[(sbrow + 1) * KB + kb];  // up block
                } else {
                    b0 = (2 * x.nt + h < NB) ? p.sb[(sbrow + h) * KB + kb] : 0.0f;
                    b1 = b0;
                }
            };
            if (kEpi == EPI_DSILU && x.valid && (2 * x.nt + h) * 128 < p.N) {
                // the saved g, u this thread reads after the last K block: to L2 now
                const uint16_t *gu = p.aux + ((int64_t)x.m0 + row) * 2 * (int64_t)p.N + (int64_t)(2 * x.nt + h) * 256;
#pragma unroll
                for (int j = 0; j < 4; ++j) asm volatile("prefetch.global.L2 [%0];" ::"l"(gu + 64 * j));
            }
            float c_a = 0.f, c_b0 = 0.f, c_b1 = 0.f, n_a = 0.f, n_b0 = 0.f, n_b1 = 0.f;
            if (!kWgrad) {
                load_rows(x.kb0, c_a, c_b0, c_b1);
                if (x.kb0 + 1 < x.kb1) load_rows(x.kb0 + 1, n_a, n_b0, n_b1);
            }
            for (int kb = x.kb0; kb < x.kb1; ++kb) {
                const float *d = wscale + wstage * WS_FLOATS;
                float s0, s1;   // rows mode: row scale x weight-block scale(s)
                float sa4[4];   // wgrad: the row scales of this thread's four rows (see below)
                if (kWgrad) {
                    if (!warp_wait_bounded(bar_sfull + 8 * wstage, wphase, p.budget, abort_flag, p.status)) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) sa4[i] = d[32 * q + (lane >> 2) + 8 * i];
                    s0 = s1 = 0.0f;
                } else {
                    s0 = c_a * c_b0;
                    s1 = c_a * c_b1;
                    c_a = n_a, c_b0 = n_b0, c_b1 = n_b1;
                    if (kb + 2 < x.kb1) load_rows(kb + 2, n_a, n_b0, n_b1);
                }
                const int slot = kPair ? 2 * buf + h : buf;   // this warpgroup's TMEM slot
                if (!warp_wait_bounded(bar_tfull + 8 * slot, bphase, p.budget, abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t cbase = lane_addr + (uint32_t)(buf * BN);
                // TMEM column of chunk c (32 columns) of this warp's share: one
                // SM, SILU: gate columns 64h.. then up columns 128 + 64h..; 2-SM:
                // the warpgroup's own 128-column slot (SILU: 64 gate, 64 up)
                auto col_of = [&](int c) -> uint32_t {
                    if (kEpi == EPI_SILU && !kPair) return (c < 2) ? (64 * h + 32 * c) : (128 + 64 * h + 32 * (c - 2));
                    return 128 * h + 32 * c;
                };
                // TMEM reads in 16-column pieces, four per wait (64 registers in
                // flight); the slot goes back to the MMA as soon as the last piece
                // has landed, before its FMAs.  (Measured against 32-column loads
                // two per wait, and against loads one chunk ahead of the FMAs: the
                // MMA of the next K block, running meanwhile, finished sooner.)
                auto release = [&]() {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if (kPair)
                            mbar_arrive_cluster(lead_tempty + 8 * slot);
                        else
                            mbar_arrive(bar_tempty + 8 * slot);
                    }
                };
                uint32_t rr[64];
                if (kWgrad) {
                    // The 16x256b shape, 32 columns of this warp's half at a time,
                    // lanes 0-15 then 16-31 of its quarter: this thread holds rows
                    // 32q + lane/4 + 8i (i = 0..3) x the column pairs
                    // 8j + 2(lane%4), +1, so it needs 32 column scales per K block
                    // instead of 128 (fewer shared loads).  Each column pair's two
                    // scales come in one 8-byte shared load (the four lanes of a row
                    // group read 32 contiguous bytes); the scale products sa * sb[n]
                    // run on two lanes at once (the same fp32 products as two scalar
                    // multiplies).
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const uint32_t cb = cbase + 128 * h + 32 * g;
                        MOE_TMEM_LD_16x256b_X4(cb, rr);
                        MOE_TMEM_LD_16x256b_X4(cb + (16u << 16), rr + 16);
                        tmem_wait_ld();
                        if (g == 3) release();
                        const float *cs = d + BM + 128 * h + 32 * g + 2 * (lane & 3);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float2 c2 = *reinterpret_cast<const float2 *>(cs + 8 * j);
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const uint32_t *cur = rr + 16 * (i >> 1) + 4 * j + 2 * (i & 1);
                                float p0, p1;
                                fmul2(p0, p1, sa4[i], sa4[i], c2.x, c2.y);
                                float *a = acc + 2 * (16 * i + 4 * g + j);
                                ffma2(a[0], a[1], __uint_as_float(cur[0]), __uint_as_float(cur[1]), p0, p1);
                            }
                        }
                    }
                } else {
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int c16 = 4 * g + j;
                            MOE_TMEM_LD16(cbase + col_of(c16 >> 1) + 16 * (c16 & 1), rr + 16 * j);
                        }
                        tmem_wait_ld();
                        if (g == 1) release();
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int c16 = 4 * g + j;
                            const uint32_t *cur = rr + 16 * j;
                            const float sc = (kEpi == EPI_SILU && c16 >= 4) ? s1 : s0;
#pragma unroll
                            for (int i = 0; i < 16; i += 2)
                                ffma2(acc[16 * c16 + i], acc[16 * c16 + i + 1], __uint_as_float(cur[i]),
                                      __uint_as_float(cur[i + 1]), sc, sc);
                        }
                    }
                }
                if (kWgrad) {  // this warp has read the slot's scales
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_sempty + 8 * wstage);
                    if (++wstage == SC_SLOTS) {
                        wstage = 0;
                        wphase ^= 1;
                    }
                }
                defer_step();
                buf ^= 1;
                if (buf == 0) bphase ^= 1;
            }
            cp_async_wait<0>();
            if (!ok) break;
            if (kPair && !x.valid) continue;   // the idle half of a pair: nothing to write
            const int64_t r = (int64_t)x.m0 + row;
            // ------------------------------------------- fused outputs ----
            if (kEpi == EPI_SILU) {
                // acc[0..63] = g, acc[64..127] = u of I-columns nt*128 + 64h + i
                const int64_t I = p.N / 2;
                const int64_t icol = (int64_t)x.nt * 128 + 64 * h;
                float amax = 0.0f;
#pragma unroll
                for (int i0 = 0; i0 < 64; i0 += 8) {
                    if (p.aux && (i0 & 8) == 0) {   // g and u rows (training), 32-byte pieces
                        uint16_t *gu = const_cast<uint16_t *>(p.aux) + r * p.N + x.n0 + 64 * h + i0;
                        st_global_32B(gu, pack8(&acc[i0]), pack8(&acc[i0 + 8]));
                        st_global_32B(gu + 128, pack8(&acc[64 + i0]), pack8(&acc[64 + i0 + 8]));
                    }
#pragma unroll
                    for (int i = i0; i < i0 + 8; ++i) {
                        const float g = acc[i], u = acc[64 + i];
                        const float sg = g * sigmoid_fast(g);
                        const float hv = __uint_as_float(bf16_bits_rn(sg * u) << 16);
                        acc[i] = hv;
                        amax = fmaxf(amax, fabsf(hv));
                    }
                }
                float *ax = amax_s + (tcount & 1) * 256;
                ax[h * 128 + row] = amax;
                if (!epi_sync()) break;
                amax = fmaxf(ax[row], ax[128 + row]);
                const float s = block_scale(amax);
                if (defer_on) {
                    while (def_left > 0) defer_step();   // a short tile: the previous codes first
                    // the h row to the staging slot, read back by the deferred steps
                    uint8_t *dst = hst;
#pragma unroll
                    for (int i0 = 0; i0 < 64; i0 += 8) *reinterpret_cast<uint4 *>(dst + 2 * i0) = pack8(&acc[i0]);
                    def_src = dst;
                    def_next = *reinterpret_cast<const uint2 *>(dst);
                    def_left = 64;
                    def_s = s;
                    if (lane == 0) {
                        def_xy[0] = (int)icol;
                        def_xy[1] = x.m0;
                    }
                } else {
                    // this warp's 32 rows x 64 codes leave through one TMA store
                    uint8_t *sb = box;
                    if (lane == 0) bulk_wait_read<0>();  // the previous tile's store has read sb
                    __syncwarp();
#pragma unroll
                    for (int i0 = 0; i0 < 64; i0 += 16)
                        *reinterpret_cast<uint4 *>(sb + lane * 64 + i0) = quant16(&acc[i0], s);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmC, smem_u32(sb), (int32_t)icol, x.m0 + 32 * q);
                        bulk_commit();
                    }
                }
                if (h == 0) p.out_s[(int64_t)x.nt * p.R_cap + r] = s;
                if (p.out_bf16) {
                    uint16_t *hb = p.out_bf16 + r * I + icol;
#pragma unroll
                    for (int i0 = 0; i0 < 64; i0 += 16) st_global_32B(hb + i0, pack8(&acc[i0]), pack8(&acc[i0 + 8]));
                }
            } else if (kEpi == EPI_BF16) {
                // 32-column chunks through per-warp smem buffers (two, or one per
                // chunk in the 2-SM layout), written to global memory by TMA
                // stores that run while the warp moves on
                constexpr int NB = L::BF16_BUFS;
                const int64_t c0 = (int64_t)x.n0 + 128 * h;
                if (c0 < p.N) {
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        uint8_t *buf = smem + OFF_TSTORE_BF16 + (ew * NB + (ch % NB)) * TSTORE_BUF;
                        if (NB == 2) {
                            if (lane == 0) bulk_wait_read<1>();  // the store that last read buf is done
                        } else if (ch == 0) {
                            if (lane == 0) bulk_wait_read<0>();  // the previous tile's four stores have read theirs
                        }
                        __syncwarp();
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            *reinterpret_cast<uint4 *>(buf + box_off(lane, j)) = pack8(&acc[32 * ch + 8 * j]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tmC, smem_u32(buf), (int32_t)(c0 + 32 * ch), x.m0 + 32 * q);
                            bulk_commit();
                        }
                    }
                }
            } else if (kEpi == EPI_DSILU) {
                // acc = dH of I-block nb = 2nt + h; its gate/up columns in the
                // interleaved 2I space are gc = 2nb*128 and uc = gc + 128.
                //   dg = dH u s (1 + g (1 - s)), du = dH g s, s = sigmoid(g),
                // each rounded to bf16, stored, and quantised 1x128 (one block
                // each).  Two fully unrolled passes: pass 1 makes dg, du, stores
                // their bf16 rows and takes the block maxima, keeping the bf16
                // pairs in registers (they take the places of the accumulators
                // they replace); pass 2 makes the codes from those registers.
                const int nb = 2 * x.nt + h;
                if (nb * 128 < p.N) {
                    const int64_t N2 = 2 * (int64_t)p.N;
                    const int64_t gc = (int64_t)(2 * nb) * 128, uc = gc + 128;
                    // 32-byte accesses (each lane reads or writes its own row, so
                    // a warp's access touches 32 rows: wider pieces mean fewer of
                    // them)
                    const uint16_t *gu = p.aux + r * N2;
                    uint16_t *ob = p.out_bf16 + r * N2;
                    uint8_t *oq = p.out_q + r * N2;
                    float amax_g = 0.0f, amax_u = 0.0f;
                    uint4 bg[16], bu[16];   // bf16 dg, du of columns 8j .. 8j + 7
                    // g, u loaded two steps ahead of their use (the accesses are
                    // ordered asm, so a load written after a store stays after it)
                    uint4 gwb[3][2], uwb[3][2];
                    ld_global_32B(gu + gc, gwb[0]);
                    ld_global_32B(gu + uc, uwb[0]);
                    ld_global_32B(gu + gc + 16, gwb[1]);
                    ld_global_32B(gu + uc + 16, uwb[1]);
#pragma unroll
                    for (int j = 0; j < 16; j += 2) {
                        if (j + 4 < 16) {
                            ld_global_32B(gu + gc + 8 * (j + 4), gwb[((j >> 1) + 2) % 3]);
                            ld_global_32B(gu + uc + 8 * (j + 4), uwb[((j >> 1) + 2) % 3]);
                        }
                        const uint4 *gw = gwb[(j >> 1) % 3], *uw = uwb[(j >> 1) % 3];
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            float g[8], u[8], dg[8], du[8];
                            unpack8(gw[hh], g);
                            unpack8(uw[hh], u);
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float d = acc[8 * (j + hh) + i];
                                const float sg = sigmoid_fast(g[i]);
                                dg[i] = __uint_as_float(bf16_bits_rn(d * u[i] * sg * (1.0f + g[i] * (1.0f - sg))) << 16);
                                du[i] = __uint_as_float(bf16_bits_rn(d * g[i] * sg) << 16);
                            }
                            amax_g = absmax8(dg, amax_g);
                            amax_u = absmax8(du, amax_u);
                            bg[j + hh] = pack8(dg);
                            bu[j + hh] = pack8(du);
                        }
                        st_global_32B(ob + gc + 8 * j, bg[j], bg[j + 1]);
                        st_global_32B(ob + uc + 8 * j, bu[j], bu[j + 1]);
                    }
                    const float sgs = block_scale(amax_g), sus = block_scale(amax_u);
#pragma unroll
                    for (int j = 0; j < 16; j += 4) {
                        uint4 cg[2], cu[2];
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            float dg[16], du[16];
                            unpack8(bg[j + 2 * hh], dg);
                            unpack8(bg[j + 2 * hh + 1], dg + 8);
                            unpack8(bu[j + 2 * hh], du);
                            unpack8(bu[j + 2 * hh + 1], du + 8);
                            cg[hh] = quant16(dg, sgs);
                            cu[hh] = quant16(du, sus);
                        }
                        st_global_32B(oq + gc + 8 * j, cg[0], cg[1]);
                        st_global_32B(oq + uc + 8 * j, cu[0], cu[1]);
                    }
                    p.out_s[(int64_t)(2 * nb) * p.R_cap + r] = sgs;
                    p.out_s[(int64_t)(2 * nb + 1) * p.R_cap + r] = sus;
                }
            } else {  // EPI_WGRAD: dW[e][m][n] += acc
                // The adds run in L2 (vector reductions, no value comes back), so
                // the next tile's K loop starts without waiting for dW to arrive.
                // One CTA owns each dW tile, so every element gets exactly one add
                // per launch: the result does not depend on timing.
                // acc[2 (16i + jj) + e] = dW row 32q + lane/4 + 8i, column
                // 128h + 8jj + 2(lane%4) + e of the tile
                const int64_t c0 = (int64_t)x.n0 + 128 * h;
                // Lanes 2l and 2l+1 hold neighbouring column pairs; one exchange
                // per two column groups gives the even lane four columns of group
                // 2m and the odd lane four of group 2m+1, each added with one
                // 16-byte reduction.
                if (c0 < p.N) {
                    const bool odd = lane & 1;
                    float *o = p.out_f32 + ((int64_t)x.e * p.M + x.m0 + 32 * q + (lane >> 2)) * p.N + c0 +
                               2 * (lane & 3) + (odd ? 6 : 0);
                    const int64_t step = 8 * (int64_t)p.N;   // 8 rows down
#pragma unroll
                    for (int i = 0; i < 4; ++i, o += step) {
#pragma unroll
                        for (int m = 0; m < 8; ++m) {
                            const float *a = acc + 2 * (16 * i + 2 * m);   // group 2m, then 2m+1
                            const float s0 = odd ? a[0] : a[2], s1 = odd ? a[1] : a[3];
                            // (volatile: kept in order with the reductions, so the
                            // exchanges are not all hoisted ahead of them)
                            float r0, r1;
                            asm volatile("shfl.sync.bfly.b32 %0, %1, 1, 0x1f, 0xffffffff;" : "=f"(r0) : "f"(s0));
                            asm volatile("shfl.sync.bfly.b32 %0, %1, 1, 0x1f, 0xffffffff;" : "=f"(r1) : "f"(s1));
                            const float v0 = odd ? r0 : a[0], v1 = odd ? r1 : a[1];
                            const float v2 = odd ? a[2] : r0, v3 = odd ? a[3] : r1;
                            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(o + 16 * m), "f"(v0),
                                         "f"(v1), "f"(v2), "f"(v3)
                                         : "memory");
                        }
                    }
                }
            }
        }
        if (ok)
            while (def_left > 0) defer_step();   // the last tile's codes
        cp_async_wait<0>();  // no copy into shared memory outlives the CTA
        if ((kEpi == EPI_SILU || kEpi == EPI_BF16) && lane == 0) bulk_wait_all();  // every TMA store has completed
    }
    tc_fence_before();
    __syncthreads();
    if (kPair) {
        // After a timeout the peer may still have loads in flight that only the
        // leader's barriers count: give them time to land before the pair
        // leaves (loads finish in microseconds; this waits about a millisecond).
        if (*abort_flag) {
            const long long t0 = clock64();
            while (clock64() - t0 < (1ll << 21)) {
            }
        }
        cluster_sync_all();   // neither CTA frees its TMEM while the pair's MMAs may run
    }
    tc_fence_after();
    if (warp == 1) {
        if (kPair)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS));
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS));
    }
}

}  // namespace gemm

// ------------------------------------------------------------------ host ----
using namespace sm100;

// Rows-mode GEMM kernel: 1-SM (0), 2-SM (1) or chosen per call (-1).
static int g_variant = 0;
void set_gemm_variant(int v) { g_variant = v; }
static int g_pair_clusters = 0;   // clusters of the last 2-SM launch
int pair_clusters() { return g_pair_clusters; }

template <int kEpi, bool kGather = false, bool kPair = false>
static int launch_one(const CUtensorMap &a, const CUtensorMap &b, const CUtensorMap &c, const gemm::Args &args,
                      int grid, cudaStream_t s)
{
    auto kern = gemm::grouped_gemm_kernel<kEpi, kGather, kPair>;
    constexpr int smem = gemm::smem_bytes<kEpi, kPair>();
    static bool configured = false;  // per process; attribute is per function
    if (!configured) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return MOE_ERR_CUDA;
        configured = true;
    }
    if (kPair) {   // clusters of two CTAs (one pair of SMs), as many as can be resident at once
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(grid & ~1));
        cfg.blockDim = dim3(gemm::NUM_THREADS);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        static int max_clusters = 0;   // per process: the device and the kernel's resources are fixed
        if (max_clusters == 0) {
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, (void *)kern, &cfg) != cudaSuccess || n <= 0) return MOE_ERR_CUDA;
            max_clusters = n;
        }
        // the tiles are dealt out statically by cluster index: every cluster
        // must be resident at the same time
        cfg.gridDim = dim3((unsigned)(2 * (grid / 2 < max_clusters ? grid / 2 : max_clusters)));
        g_pair_clusters = (int)(cfg.gridDim.x / 2);
        if (cudaLaunchKernelEx(&cfg, kern, a, b, c, args) != cudaSuccess) return MOE_ERR_CUDA;
    } else {
        kern<<<grid, gemm::NUM_THREADS, smem, s>>>(a, b, c, args);
    }
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}


// The 2-SM variant computes whole pairs of 128-row tiles; a segment with an
// odd number of tiles leaves one half of its last pair idle.  It pays when
// those idle halves (at most one per segment) are a small share of the rows.
static bool use_pair(int n_seg, int64_t R_cap)
{
    if (g_variant >= 0) return g_variant == 1;
    return (int64_t)n_seg * gemm::BM * 32 <= R_cap;
}

int launch_grouped_gemm(int op, const moe_dims &d, int64_t R_cap, const int32_t *offsets, int n_seg,
                        const moe_gemm_args &g, int *status, uint64_t budget, cudaStream_t s)
{
    gemm::Args a{};
    a.offsets = offsets;
    a.E = n_seg;
    a.ew = d.E;
    a.R_cap = R_cap;
    a.sa = g.sa;
    a.sb = g.sb;
    a.aux = g.aux;
    a.out_q = g.out_q;
    a.out_s = g.out_s;
    a.out_bf16 = g.out_bf16;
    a.out_f32 = g.out_f32;
    a.status = status;
    a.budget = budget;
    CUtensorMap mA, mB;
    const int64_t D = d.D, I = d.I, E = d.E;
    bool ok = true;
    switch (op) {
    case MOE_GEMM_GATEUP_SILU:
        a.N = (int)(2 * I); a.K = (int)D;
        ok = make_map(&mA, g.a, D, R_cap, 128) && make_map(&mB, g.b, D, E * 2 * I, 256);
        break;
    case MOE_GEMM_DOWN:
        a.N = (int)D; a.K = (int)I;
        ok = make_map(&mA, g.a, I, R_cap, 128) && make_map(&mB, g.b, I, E * D, 256);
        break;
    case MOE_GEMM_DGRAD_DOWN_SILU:
        a.N = (int)I; a.K = (int)D;
        ok = make_map(&mA, g.a, D, R_cap, 128) && make_map(&mB, g.b, D, E * I, 256);
        break;
    case MOE_GEMM_DGRAD_GATEUP:
        a.N = (int)D; a.K = (int)(2 * I);
        ok = make_map(&mA, g.a, 2 * I, R_cap, 128) && make_map(&mB, g.b, 2 * I, E * D, 256);
        break;
    case MOE_GEMM_WGRAD_DOWN:
        a.M = (int)D; a.N = (int)I;
        ok = make_map(&mA, g.a, R_cap, D, 128) && make_map(&mB, g.b, R_cap, I, 256);
        break;
    case MOE_GEMM_WGRAD_GATEUP:
        a.M = (int)(2 * I); a.N = (int)D;
        ok = make_map(&mA, g.a, R_cap, 2 * I, 128) && make_map(&mB, g.b, R_cap, D, 256);
        break;
    default:
        return MOE_ERR_INVALID_ARG;
    }
    if (!ok) return MOE_ERR_CUDA;
    CUtensorMap mC = mA;  // output map of the epilogues that store through TMA
    if (op == MOE_GEMM_GATEUP_SILU) ok = make_store_map(&mC, g.out_q, a.N / 2, R_cap, 1);
    if (op == MOE_GEMM_DOWN || op == MOE_GEMM_DGRAD_GATEUP) ok = make_store_map(&mC, g.out_bf16, a.N, R_cap, 2);
    if (!ok) return MOE_ERR_CUDA;
    const int grid = sm_count();
    if (op != MOE_GEMM_WGRAD_DOWN && op != MOE_GEMM_WGRAD_GATEUP && use_pair(n_seg, R_cap)) {
        // each CTA loads 128 rows of the 256-row B tile: one 128-row box (gate/up)
        // or two 64-row boxes (the other GEMMs)
        const int64_t Kc = a.K, Nrows = (op == MOE_GEMM_GATEUP_SILU ? 2 * I : op == MOE_GEMM_DGRAD_DOWN_SILU ? I : D);
        if (!make_map(&mB, g.b, Kc, E * Nrows, op == MOE_GEMM_GATEUP_SILU ? 128 : 64)) return MOE_ERR_CUDA;
        switch (op) {
        case MOE_GEMM_GATEUP_SILU: return launch_one<gemm::EPI_SILU, false, true>(mA, mB, mC, a, grid, s);
        case MOE_GEMM_DOWN:
        case MOE_GEMM_DGRAD_GATEUP: return launch_one<gemm::EPI_BF16, false, true>(mA, mB, mC, a, grid, s);
        default: return launch_one<gemm::EPI_DSILU, false, true>(mA, mB, mC, a, grid, s);
        }
    }
    switch (op) {
    case MOE_GEMM_GATEUP_SILU: return launch_one<gemm::EPI_SILU>(mA, mB, mC, a, grid, s);
    case MOE_GEMM_DOWN:
    case MOE_GEMM_DGRAD_GATEUP: return launch_one<gemm::EPI_BF16>(mA, mB, mC, a, grid, s);
    case MOE_GEMM_DGRAD_DOWN_SILU: return launch_one<gemm::EPI_DSILU>(mA, mB, mC, a, grid, s);
    default: return launch_one<gemm::EPI_WGRAD>(mA, mB, mC, a, grid, s);
    }
}

// a6 with its A operand gathered from the token rows: codes xq_tok [T][D]
// (g.a) and 1x128 scales [D/128][T] (g.sa); permuted row r is token
// src_idx[r] / k.  The producer gathers half of the A rows with TMA
// tile::gather4 (the tensor map has one-row boxes) and half with cp.async.
int launch_gateup_gather(const moe_dims &d, int64_t R_cap, const int32_t *offsets, const int32_t *src_idx,
                         const moe_gemm_args &g, int *status, uint64_t budget, cudaStream_t s)
{
    gemm::Args a{};
    a.offsets = offsets;
    a.E = d.E;
    a.ew = d.E;
    a.R_cap = R_cap;
    a.sa = g.sa;
    a.sb = g.sb;
    a.aux = g.aux;
    a.out_q = g.out_q;
    a.out_s = g.out_s;
    a.out_bf16 = g.out_bf16;
    a.status = status;
    a.budget = budget;
    a.a_rows = g.a;
    a.src_idx = src_idx;
    a.k = d.k;
    a.T = d.T;
    const int64_t D = d.D, I = d.I, E = d.E;
    a.N = (int)(2 * I);
    a.K = (int)D;
    CUtensorMap mA, mB, mC;
    if (!make_map(&mA, g.a, D, d.T, 1) || !make_map(&mB, g.b, D, E * 2 * I, 256) ||
        !make_store_map(&mC, g.out_q, I, R_cap, 1))
        return MOE_ERR_CUDA;
    return launch_one<gemm::EPI_SILU, true>(mA, mB, mC, a, sm_count(), s);
}

}  // namespace moe
