/*
 * moe.h — C ABI of the B200 (sm_100a) MoE expert-layer library (libmoe.so).
 *
 * The layer: top-k routing of each token to experts, or replay of routing
 * captured at inference; a stable dispatch of the routed copies grouped by
 * expert; block-scaled FP8 (e4m3) quantisation in the DeepSeek-V3 style;
 * grouped FP8 GEMMs of the SiLU-gated expert FFN; a weighted combine; and the
 * backward of all of it.
 *
 * Sources (page titles and sections of the material this library follows):
 *  [P1] "prime-rl 0.6.0 løfter trillion-parameter RL på lange SWE-flow",
 *       §Drift og omkostninger i realiteten — each token activates a top-k set
 *       of experts; dispatch/combine happen in every layer.
 *  [P4] "RL at 1T scale: prime-rl performance deep dive" —
 *       §Router Replay: routing decisions made at inference are captured and
 *       replayed in the trainer; the payload has shape
 *       [num_layers, top_k, seq_len] and is handled as an opaque tensor;
 *       §Wide Expert Parallelism, §Parallelism/EP: per-layer dispatch and
 *       combine of tokens to experts;
 *       §FP8 Training: block-scaled FP8 as proposed by DeepSeek-V3.
 *
 * Conventions (all entry points):
 *  - Every pointer argument is caller-owned DEVICE memory unless stated; the
 *    library allocates nothing.  bf16 tensors are passed as uint16_t bit
 *    patterns.  All matrices are row-major.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 *  - Calls are asynchronous on `stream` and return a moe_status for the
 *    host-side checks (arguments, launch).  Errors found on the device
 *    (bad replay entries, timeouts) are latched in a per-device status word
 *    read by moe_get_status().
 *  - No call aborts the process or throws.
 *
 * Data layouts (T tokens, D model dim, I expert FFN dim, E experts, k top-k):
 *  - routed entry i = t*k + j (token t, slot j);
 *  - R_cap = moe_rows_capacity(dims): bound on the permuted (padded) rows;
 *    every permuted-row buffer has R_cap rows;
 *  - 1x128 FP8 of a [rows, C] matrix: codes [rows][C]; scales "K-block
 *    major" [C/128][ld_rows] (scale of row r, column block b at b*ld_rows+r);
 *  - 128x1 FP8 (blocks of 128 rows in one column) of a [rows, C] matrix is
 *    stored transposed: codes [C][ld_rows], scales [ld_rows/128][C];
 *  - 128x128 FP8 of a weight [N, K]: codes [N][K], scales [N/128][K/128].
 *  - Scale of a block = fp32(amax / 448) (IEEE fp32 division); code =
 *    e4m3fn(round-nearest-even, saturate to +-448)(fp32(x / scale));
 *    a block with amax 0 has scale 0 and codes 0x00.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer */
    MOE_ERR_UNSUPPORTED = 2, /* D or I not a multiple of 128, E > 256, k > E, k > 16 */
    MOE_ERR_CUDA = 3,        /* a CUDA call or launch failed */
    MOE_ERR_BAD_ROUTING = 4, /* device: replay/permute saw an expert outside [0,E) or a repeat */
    MOE_ERR_TIMEOUT = 5      /* device: a bounded wait inside a kernel ran out */
} moe_status;

/* Problem sizes.  align = 1 or 128: each expert's row segment is padded to a
 * multiple of `align` rows (128 for everything that feeds the GEMMs). */
typedef struct {
    int32_t T, D, I, E, k, align;
} moe_dims;

/* Bound on the permuted rows: T*k + E*(align-1), rounded up to 128. */
int64_t moe_rows_capacity(const moe_dims *dims);

/* Bytes of caller-provided scratch `ws` for moe_permute. */
size_t moe_permute_workspace_size(const moe_dims *dims);

const char *moe_strerror(int status);

/* Synchronises `stream`, then reads and clears the device status word of the
 * current device into *out (MOE_OK if no kernel latched an error). */
int moe_get_status(void *stream, int *out);

/* Bound (in SM clock cycles) on every spin-wait inside the GEMM kernels;
 * 0 restores the default (about 2^32 cycles).  On expiry the kernel
 * latches MOE_ERR_TIMEOUT, drains its own copies and MMAs, frees its tensor
 * memory and returns. */
void moe_set_wait_budget(uint64_t cycles);

/* Number of kernels this library has launched in this process, counting a
 * launch recorded into a stream capture once (a graph replay launches them
 * again without calling into the library).  For accounting only. */
uint64_t moe_kernel_launches(void);

/* Which kernel runs the rows-mode grouped GEMMs (GATEUP_SILU, DOWN,
 * DGRAD_DOWN_SILU, DGRAD_GATEUP): 0 = one SM per 128 x 256 tile (the
 * default), 1 = the 2-SM MMA (a pair of SMs per 256 x 256 tile, each loading
 * half of the weight tile, each K block issued as two 128-column halves),
 * -1 = chosen per call from the shapes.  Results are the same bit for bit;
 * the choice is per process.  Returns MOE_ERR_INVALID_ARG for any other
 * value. */
int moe_set_gemm_variant(int variant);

/* Clusters (CTA pairs) of the last 2-SM GEMM launch: the pairs the device can
 * hold at once, at most half the SMs (0 before any 2-SM launch).  For
 * accounting only. */
int moe_gemm_pair_clusters(void);

/* ------------------------------------------------------------------------ */
/* a1  Top-k routing  [P1 §Drift og omkostninger i realiteten]               */
/* ------------------------------------------------------------------------ */
/* logits fp32 [T][E] -> idx int32 [T][k], w fp32 [T][k].
 * Chooses the k largest logits (compared as fp32; equal logits: lower expert
 * index first), slots in descending logit order; w = softmax of the chosen
 * logits (= softmax over all E renormalised over the chosen set).
 * Logits may be -inf; NaN is not allowed.  E <= 256, k <= min(E, 16). */
int moe_route_topk(const float *logits, const moe_dims *dims, int32_t *idx, float *w,
                   void *stream);

/* ------------------------------------------------------------------------ */
/* Router and capture of its decisions  [P1 §Drift og omkostninger;          */
/* P4 §Router Replay]                                                        */
/* ------------------------------------------------------------------------ */
/* The router is the linear gate before the top-k: x bf16 [T][D], w_r bf16
 * [E][D] -> z fp32 [T][E], z[t][e] = sum_d x[t][d] w_r[e][d] (bf16 products
 * accumulated in fp32 on the tensor cores; the order of the additions is the
 * hardware's).  With idx and w non-NULL (both or neither) it then chooses
 * idx/w from z exactly as moe_route_topk does.  D % 128 == 0, E <= 256;
 * x, w_r and z 16-byte aligned. */
int moe_router_fwd(const uint16_t *x, const uint16_t *w_r, const moe_dims *dims, float *z, int32_t *idx,
                   float *w, void *stream);

/* Capture: writes the routing decisions of one layer into the replay
 * payload, payload[layer][j][t] = idx[t][j] (int32 [L][k][T], element
 * (l,j,t) at (l*k+j)*T+t: the layout moe_route_replay reads).  Other layers'
 * slices are untouched. */
int moe_capture_payload(const int32_t *idx, const moe_dims *dims, int32_t L, int32_t layer, int32_t *payload,
                        void *stream);

/* Bytes of caller-provided scratch for moe_router_bwd's weight gradient. */
size_t moe_router_bwd_workspace_size(const moe_dims *dims);

/* Router backward from the logit gradient dz fp32 [T][E] (moe_combine_bwd's
 * d_logits):
 *   dx bf16 [T][D] (nullable: skipped) = bf16(fp32(dx_in[t][d]) +
 *        sum_e dz[t][e] w_r[e][d]), sum in fp32, e ascending; dx_in nullable
 *        (0) and may equal dx (the router's share added in place);
 *   dw_r fp32 [E][D] (nullable: skipped) += sum_t dz[t][e] x[t][d]: fp32
 *        partial sums over 256-token chunks (tokens in order) in ws, then
 *        added chunk by chunk in order (deterministic).
 * ws: moe_router_bwd_workspace_size() bytes, 16-byte aligned (only for dw_r). */
int moe_router_bwd(const float *dz, const uint16_t *x, const uint16_t *w_r, const moe_dims *dims,
                   const uint16_t *dx_in, uint16_t *dx, float *dw_r, void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------ */
/* a2  Router replay  [P4 §Router Replay]                                    */
/* ------------------------------------------------------------------------ */
/* payload int32 [L][k][T] (element (l,j,t) at (l*k+j)*T+t) ->
 * idx[t][j] = payload[layer][j][t].  Weights: w_in [T][k] copied when non-NULL,
 * else softmax of the trainer logits [T][E] over the replayed set.  Exactly
 * one of w_in / logits must be non-NULL (when T > 0; T = 0 does nothing and
 * checks no array pointer).  An entry outside [0,E) or an expert
 * repeated within a token latches MOE_ERR_BAD_ROUTING; that token's weights
 * are 0 and its idx entries are copied as given (moe_permute drops entries
 * outside [0,E)). */
int moe_route_replay(const int32_t *payload, int32_t L, int32_t layer, const moe_dims *dims,
                     const float *w_in, const float *logits, int32_t *idx, float *w,
                     void *stream);

/* ------------------------------------------------------------------------ */
/* a3+a4  Permute, with the fused 1x128 quantise-and-dispatch                */
/*        [P4 §Wide Expert Parallelism, §Parallelism/EP; §FP8 Training]      */
/* ------------------------------------------------------------------------ */
/* idx [T][k] ->
 *   counts [E]        routed entries per expert (the per-expert load);
 *   offsets [E+1]     offsets[0] = 0, offsets[e+1] = offsets[e] + roundup(counts[e], align);
 *   pos [T][k]        permuted row of entry i: offsets[e] + #{i' < i : idx[i'] = e}
 *                     (stable), -1 for an entry outside [0,E);
 *   src_idx [R_cap]   routed entry i = t*k+j held by each permuted row, -1 for
 *                     padding rows and rows >= offsets[E].
 * With x (bf16 [T][D]) non-NULL, also dispatches x in FP8:
 *   xq [R_cap][D] e4m3, xs [D/128][R_cap] fp32 (both or neither): 1x128
 *   blocks of row pos[t][j] are those of x[t]; padding rows get codes 0 and
 *   scale 0 (NULL when the gate/up GEMM gathers the token rows itself,
 *   moe_gateup_gather_fp8);
 *   xqT [D][R_cap], xsT [R_cap/128][D] (both nullable, align must be 128;
 *   with T > 0 they need x): 128x1 blocks of the permuted rows, for the
 *   weight gradient.  With T = 0 there is no row to dispatch and x may be
 *   NULL (an empty array).
 * ws: moe_permute_workspace_size() bytes of scratch (16-byte aligned). */
int moe_permute(const int32_t *idx, const moe_dims *dims, int32_t *counts, int32_t *offsets,
                int32_t *pos, int32_t *src_idx, const uint16_t *x, uint8_t *xq, float *xs,
                uint8_t *xqT, float *xsT, void *ws, size_t ws_bytes, void *stream);

/* moe_permute without the caller-provided scratch, for callers that cannot
 * allocate device memory (an engine step that has reserved all of HBM and
 * forbids allocation while it runs; a plugin or custom-op host that passes
 * only input and output tensors).  The pages have no counterpart: this is an
 * interface variant, not a step of the method.  Same outputs as moe_permute
 * without the 128x1 outputs.  The scratch is a fixed 1 MiB array inside the
 * library, one per device that loads it, held until the process exits; a
 * problem needing more (moe_permute_workspace_size() > 1 MiB) returns
 * MOE_ERR_UNSUPPORTED.  The first call on a device looks up the array's
 * address (make it before any stream capture); calls overlapping on the GPU
 * share the array and race; entries outside [0,E) are dropped (pos = -1) but
 * not reported through moe_get_status().  The address is kept for the life of
 * the process: after cudaDeviceReset() on a device, do not call this entry
 * point on that device again in the same process. */
int moe_permute_noalloc(const int32_t *idx, const moe_dims *dims, int32_t *counts, int32_t *offsets,
                        int32_t *pos, int32_t *src_idx, const uint16_t *x, uint8_t *xq, float *xs,
                        void *stream);

/* ------------------------------------------------------------------------ */
/* Block-scaled FP8 quantiser  [P4 §FP8 Training]                            */
/* ------------------------------------------------------------------------ */
/* in: bf16 [rows][cols], row stride ld elements (ld % 8 == 0, cols % 16 == 0).
 * (blk_r, blk_c) = (1,128): q [rows][cols], s [ceil(cols/128)][rows];
 *                  (128,1): q [cols][rows] (transposed), s [ceil(rows/128)][cols],
 *                           rows % 16 == 0;
 *                (128,128): q [rows][cols], s [ceil(rows/128)][ceil(cols/128)], and
 *                           optionally qT [cols][rows], sT [ceil(cols/128)][ceil(rows/128)]
 *                           (the quantisation of the transpose; rows % 16 == 0).
 * Edge blocks cover only the elements that exist. */
int moe_quant_fp8_block(const uint16_t *in, int64_t rows, int64_t cols, int64_t ld,
                        int32_t blk_r, int32_t blk_c, uint8_t *q, float *s, uint8_t *qT,
                        float *sT, void *stream);

/* NVFP4 block quantisation (the Blackwell 4-bit format named as future work
 * in [P4 §Future work]) of in bf16 [rows][cols] (row stride ld elements,
 * ld % 8 == 0, cols % 16 == 0, in 16-byte aligned, q 8-byte aligned):
 *   amax (one float)  max |x| over the tensor;
 *   s_g  (one float)  tensor scale fp32(2688 / amax) (1 if amax = 0);
 *   sf                e4m3 block-scale codes e4m3(RNE, satfinite)(
 *                     fp32(fp32(amax_b / 6) * s_g)), amax_b over 16 elements,
 *                     laid out by sf_layout:
 *                       MOE_NVFP4_SF_ROWS   [rows][cols/16];
 *                       MOE_NVFP4_SF_MMA_A  the NVFP4 GEMM's A-side layout
 *                         (rows % 128 == 0, cols % 128 == 0), 4 * rows * cols/16 bytes;
 *                       MOE_NVFP4_SF_MMA_B  its B-side layout (rows % 256 == 0,
 *                         cols % 64 == 0), 4 * rows * cols/16 bytes.
 *                     Both store every scale four times, the image that
 *                     tcgen05.cp 128x256b copies into TMEM lanes 0-127: a
 *                     4096-byte block holds, for lane l and half h, the scales
 *                     of rows 32 r1 + l % 32 (r1 = 0..3) of one 128-row block for
 *                     one 64-column step (row 32 r1 + l % 32, group j at byte
 *                     4 r1 + j of the 16) at (l >> 3) * 256 + h * 128 + (l & 7) * 16.
 *                     A: block (row block rb, step pair kp) at (rb * cols/128 + kp)
 *                     * 4096, h = step 2 kp + h.  B: block (row-block pair rbp,
 *                     step ks) at (rbp * cols/64 + ks) * 4096, h = row block
 *                     2 rbp + h;
 *   q  [rows][cols/2] e2m1 codes, two per byte (element 2i in the low
 *                     nibble): 0 where the block scale is 0, else e2m1(RNE,
 *                     satfinite)(fp32(x * fp32(s_g / value(sf)))).
 * Value of an element: e2m1(q) * value(sf) / s_g.  amax and s_g are device
 * words the call writes (amax is zeroed first, then accumulated).
 * MOE_ERR_INVALID_ARG for an unknown layout or shapes the layout excludes. */
#define MOE_NVFP4_SF_ROWS 0
#define MOE_NVFP4_SF_MMA_A 1
#define MOE_NVFP4_SF_MMA_B 2
int moe_quant_nvfp4(const uint16_t *in, int64_t rows, int64_t cols, int64_t ld, uint8_t *q, uint8_t *sf,
                    int32_t sf_layout, float *amax, float *s_g, void *stream);

/* NVFP4 grouped GEMM [P4 §Future work: NVFP4 on Blackwell], on the tensor
 * cores' block-scaled MMA (kind::mxf4nvf4, 16-element ue4m3 scales):
 *   out[r][n] = sum_k value(A)[r][k] * value(B_e)[n][k]   for r in segment e,
 * segments [offsets[e], offsets[e+1]) of the rows, 128-aligned (n_seg <= 256;
 * offsets on the device, read there).  Operands as moe_quant_nvfp4 makes
 * them:
 *   a    [rows_cap][K/2] packed e2m1 codes;  sfa  A's scales, MOE_NVFP4_SF_MMA_A;
 *   a_sg A's tensor scale (device float);
 *   b    [n_seg][N][K/2] codes of each segment's B;  sfb  their scales,
 *        MOE_NVFP4_SF_MMA_B over the n_seg * N rows;
 *   b_sg [n_seg] tensor scales of the B's (device);
 *   out  [rows_cap][N] fp32, rows past offsets[n_seg] untouched.
 * N % 256 == 0, K % 256 == 0, rows_cap % 128 == 0; pointers 16-byte aligned
 * (MOE_ERR_INVALID_ARG otherwise).  The accumulation is fp32 over exact
 * products; the result is scaled by 1 / (a_sg * b_sg[e]). */
int moe_gemm_nvfp4(int64_t rows_cap, int32_t N, int32_t K, int32_t n_seg, const int32_t *offsets,
                   const uint8_t *a, const uint8_t *sfa, const float *a_sg, const uint8_t *b, const uint8_t *sfb,
                   const float *b_sg, float *out, void *stream);

/* Expert weights (a5): 128x128 FP8 of W_gate, W_up [E][I][D] and W_down [E][D][I].
 *   wgu_q [E][2I][D], wgu_s [E][2I/128][D/128]: gate and up interleaved by
 *        128-row blocks (block 2b = gate rows 128b.., block 2b+1 = up rows 128b..);
 *   wd_q [E][D][I], wd_s [E][D/128][I/128];
 *   for the backward (all four nullable together):
 *   wguT_q [E][D][2I], wguT_s [E][D/128][2I/128]  (transpose of wgu);
 *   wdT_q [E][I][D],   wdT_s [E][I/128][D/128]    (transpose of wd). */
int moe_quant_weights(const uint16_t *w_gate, const uint16_t *w_up, const uint16_t *w_down,
                      const moe_dims *dims, uint8_t *wgu_q, float *wgu_s, uint8_t *wd_q,
                      float *wd_s, uint8_t *wguT_q, float *wguT_s, uint8_t *wdT_q,
                      float *wdT_s, void *stream);

/* ------------------------------------------------------------------------ */
/* a6/a7/b2/b3/b4  Grouped block-scaled FP8 GEMMs on tcgen05  [P4 §FP8 Training] */
/* ------------------------------------------------------------------------ */
enum {
    MOE_GEMM_GATEUP_SILU = 0,    /* a6 */
    MOE_GEMM_DOWN = 1,           /* a7 */
    MOE_GEMM_DGRAD_DOWN_SILU = 2,/* b2 */
    MOE_GEMM_DGRAD_GATEUP = 3,   /* b3 */
    MOE_GEMM_WGRAD_DOWN = 4,     /* b4 */
    MOE_GEMM_WGRAD_GATEUP = 5    /* b4 */
};

/* Operands of moe_grouped_gemm_fp8.  For row r of expert e (offsets[e] <= r <
 * offsets[e+1]) and 1x128 operand scales sa (K-block major, ld R_cap):
 *
 * GATEUP_SILU: a = xq [R_cap][D], sa = xs; b = wgu_q, sb = wgu_s.
 *   g, u = sum over 128-blocks kb of sa[kb][r] * sb[e][n/128][kb] * (a . b)_kb (fp32);
 *   h = bf16(silu(g) * u); out_q = hq [R_cap][I] e4m3, out_s = hs [I/128][R_cap]
 *   (1x128 of h).  Nullable: out_bf16 = h [R_cap][I] bf16;
 *   aux = gu [R_cap][2I] bf16 (g, u saved in wgu's interleaved column order).
 * DOWN: a = hq, sa = hs; b = wd_q, sb = wd_s; out_bf16 = Y [R_cap][D] bf16.
 * DGRAD_DOWN_SILU: a = dYq [R_cap][D], sa = dYs; b = wdT_q, sb = wdT_s;
 *   aux = gu (saved by GATEUP_SILU);  dH = dY . W_down;
 *   dg = dH*u*s*(1+g*(1-s)), du = dH*silu(g), s = sigmoid(g);
 *   out_bf16 = dGU [R_cap][2I] bf16 (interleaved like wgu; required: the
 *   codes are made from it); out_q = dGUq [R_cap][2I] e4m3, out_s = dGUs
 *   [2I/128][R_cap] (1x128 of dGU).
 * DGRAD_GATEUP: a = dGUq, sa = dGUs; b = wguT_q, sb = wguT_s;
 *   out_bf16 = dX [R_cap][D] bf16 (rows in permuted order).
 * WGRAD_DOWN:   a = dYqT [D][R_cap], sa = dYsT [R_cap/128][D];
 *               b = hqT [I][R_cap], sb = hsT [R_cap/128][I];
 *               out_f32 = dWd [E][D][I] fp32, out += sum over the expert's rows.
 * WGRAD_GATEUP: a = dGUqT [2I][R_cap], sa = dGUsT [R_cap/128][2I];
 *               b = xqT [D][R_cap], sb = xsT [R_cap/128][D];
 *               out_f32 = dWgu [E][2I][D] fp32 (interleaved rows), +=.
 * The WGRAD ops add into dW with fp32 reductions in L2 (round to nearest;
 * a subnormal sum may be flushed to zero); each element gets one add per
 * call, so the result does not depend on timing.
 * All code/matrix pointers must be 16-byte aligned; for the WGRAD ops the
 * scale arrays sa and sb too; 32-byte aligned: aux and out_bf16 of
 * GATEUP_SILU, and aux, out_bf16 and out_q of DGRAD_DOWN_SILU (their rows
 * are written or read in 32-byte pieces). */
typedef struct {
    const uint8_t *a;
    const float *sa;
    const uint8_t *b;
    const float *sb;
    const uint16_t *aux;
    uint8_t *out_q;
    float *out_s;
    uint16_t *out_bf16;
    float *out_f32;
} moe_gemm_args;

int moe_grouped_gemm_fp8(int32_t op, const moe_dims *dims, const int32_t *offsets,
                         const moe_gemm_args *args, void *stream);

/* a4+a6 without the permuted copy of the activations: GATEUP_SILU whose A
 * operand is gathered from the token rows by the GEMM's loads (half of each
 * tile's rows by TMA tile::gather4, half by cp.async), so the dispatch writes
 * no R x D FP8 copy.  args->a =
 * codes [T][D] and args->sa = scales [D/128][T] of the 1x128 quantisation of
 * x itself (moe_quant_fp8_block(x, T, D, D, 1, 128, ...)); permuted row r
 * is token src_idx[r] / k (src_idx from moe_permute), a row with src_idx < 0
 * is zero.  Every other operand and every output is that of GATEUP_SILU, so
 * the results equal those of moe_permute's dispatch followed by
 * moe_grouped_gemm_fp8(GATEUP_SILU) [P1 §Drift og omkostninger: the
 * dispatch/combine cost of every layer]. */
int moe_gateup_gather_fp8(const moe_dims *dims, const int32_t *offsets, const int32_t *src_idx,
                          const moe_gemm_args *args, void *stream);

/* The same GEMMs (rows-mode ops only: GATEUP_SILU, DOWN, DGRAD_DOWN_SILU,
 * DGRAD_GATEUP) over n_seg 128-aligned row segments offsets[0..n_seg] that
 * are not one per expert: segment v uses the weights of expert v % dims->E
 * (dims->E experts in the weight arrays; n_seg a multiple of it, <= 256).
 * rows_cap (a multiple of 128) replaces moe_rows_capacity(dims) as the row
 * count of every row-indexed operand and the leading dimension of the 1x128
 * scale arrays; dims->T and dims->k are not used.  This is the layout an
 * expert-parallel rank receives: one segment per (source rank, local expert)
 * [P4 §Parallelism/EP, §Wide Expert Parallelism]. */
int moe_grouped_gemm_fp8_seg(int32_t op, const moe_dims *dims, int64_t rows_cap, const int32_t *offsets,
                             int32_t n_seg, const moe_gemm_args *args, void *stream);

/* ------------------------------------------------------------------------ */
/* a8  Weighted combine  [P1 §Drift og omkostninger; P4 §Parallelism/EP]     */
/* ------------------------------------------------------------------------ */
/* y[t] = bf16( sum_{j=0..k-1} w[t][j] * Y[pos[t][j]] ), fp32, j ascending;
 * entries with pos < 0 are skipped.  Y [R_cap][D] bf16, y [T][D] bf16. */
int moe_combine(const uint16_t *Y, const float *w, const int32_t *pos, const moe_dims *dims,
                uint16_t *y, void *stream);

/* ------------------------------------------------------------------------ */
/* b1  Combine backward  [P4 §FP8 Training]                                  */
/* ------------------------------------------------------------------------ */
/* dy [T][D] bf16, Y [R_cap][D] bf16, w, pos, idx [T][k] ->
 *   dYq [R_cap][D] e4m3, dYs [D/128][R_cap]: 1x128 of the rows
 *        dY[pos[t][j]] = bf16(fp32(w[t][j] * dy[t])), padding rows 0;
 *   dY_bf16 [R_cap][D] (nullable): those rows in bf16;
 *   d_w [T][k] = <dy[t], Y[pos[t][j]]> (fp32);
 *   d_logits [T][E] (nullable; w must be the softmax over the chosen set):
 *        w_j * (d_w_j - sum_i w_i d_w_i) at the chosen experts, 0 elsewhere.
 * counts and offsets (from moe_permute) locate the padding rows, which are
 * written as zeros (codes, scales and dY_bf16). */
int moe_combine_bwd(const uint16_t *dy, const uint16_t *Y, const float *w, const int32_t *pos,
                    const int32_t *idx, const int32_t *counts, const int32_t *offsets,
                    const moe_dims *dims,
                    uint8_t *dYq, float *dYs, uint16_t *dY_bf16, float *d_w, float *d_logits,
                    void *stream);

/* b3  dx[t] = bf16( sum_j dX[pos[t][j]] ), fp32, j ascending. */
int moe_unpermute_reduce(const uint16_t *dX, const int32_t *pos, const moe_dims *dims,
                         uint16_t *dx, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
