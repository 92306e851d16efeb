/*
 * CPU oracle for the MoE expert layer — TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, the smoke check and the CPU-baseline leg of the benchmark load
 * this library.  It shares no code with the CUDA path: no headers, tables,
 * helpers or generators.  Everything here is plain C over host arrays, with
 * fp64 accumulation, written to be read against the method's definition:
 *
 *  - top-k routing of each token to a set of experts
 *      ("prime-rl 0.6.0 løfter trillion-parameter RL ...", §Drift og omkostninger i realiteten);
 *  - router replay: the routing captured at inference, a [num_layers, top_k, seq_len]
 *    integer payload, is replayed in the trainer
 *      ("RL at 1T scale: prime-rl performance deep dive", §Router Replay);
 *  - block-scaled FP8 in the style of DeepSeek-V3 (e4m3 codes, fp32 scale per block)
 *      ("RL at 1T scale ...", §FP8 Training);
 *  - dispatch and combine of tokens per layer
 *      ("RL at 1T scale ...", §Wide Expert Parallelism and §Parallelism/EP).
 *
 * Points the pages leave open are fixed by these readings (each one is listed
 * in the design notes of the repository):
 *  - scale s = fp32(amax / 448) by IEEE fp32 division; code = e4m3fn(RNE,
 *    saturate-to-finite)(fp32(x / s)) by IEEE fp32 division;
 *  - a block whose amax is 0 has s = 0 and all codes 0x00; otherwise the sign
 *    of zero is kept (-0 -> 0x80);
 *  - routing: softmax over all experts in fp64, the k largest fp32 logits are
 *    selected (equal logits: lower expert index first; slot order = descending
 *    logit), weights = p_S / sum(p_S);
 *  - payload element (l, j, t) sits at (l*k + j)*T + t (row-major, seq fastest);
 *  - permute: stable counting sort by expert in flat order t*k + j, each
 *    expert's segment padded to a multiple of `align` rows.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC.
 * (No contraction, no fast-math: every fp32 divide below is IEEE.)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------- */
/* Scalar codecs                                                             */
/* ------------------------------------------------------------------------- */

static float bf16_bits_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a double to the nearest bf16 (ties to even), directly from fp64.
 * bf16 = 1 sign, 8 exponent, 7 stored mantissa bits; same exponent range as
 * fp32, so subnormals are multiples of 2^-133 below 2^-126. */
uint16_t orc_bf16_from_double(double v)
{
    if (isnan(v)) return 0x7FC0;
    const double max_finite = ldexp(255.0, 120); /* (2 - 2^-7) * 2^127 */
    double a = fabs(v);
    double q;
    if (a == 0.0) {
        q = 0.0;
    } else if (a < ldexp(1.0, -126)) {
        q = rint(ldexp(a, 133)) * ldexp(1.0, -133);
    } else {
        int ex;
        frexp(a, &ex);                      /* a in [2^(ex-1), 2^ex) */
        double quantum = ldexp(1.0, ex - 8); /* 8 significant bits */
        q = rint(a / quantum) * quantum;     /* rint: ties to even */
    }
    float f = (q > max_finite) ? INFINITY : (float)q; /* exact: q fits bf16 */
    if (signbit(v)) f = -f;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* Value of an e4m3fn code: 1 sign, 4 exponent (bias 7), 3 mantissa bits;
 * exponent field 0 is subnormal (m * 2^-9); 0x7F / 0xFF are NaN. */
double orc_e4m3_to_double(uint8_t c)
{
    int e = (c >> 3) & 0xF, m = c & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m, -9);
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return (c & 0x80) ? -mag : mag;
}

/* fp32 -> e4m3fn, round to nearest (ties to even), saturating to +-448. */
uint8_t orc_e4m3_from_float(float vf)
{
    double v = vf;
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a > 448.0) return sign | 0x7E; /* saturate to the largest finite */
    double q;
    if (a < ldexp(1.0, -6)) {
        q = rint(a * 512.0) / 512.0; /* subnormal grid: multiples of 2^-9 */
    } else {
        int ex;
        frexp(a, &ex);                      /* a in [2^(ex-1), 2^ex) */
        double quantum = ldexp(1.0, ex - 4); /* 4 significant bits */
        q = rint(a / quantum) * quantum;
    }
    if (q == 0.0) return sign;
    int ex;
    frexp(q, &ex);
    int e_unb = ex - 1; /* q in [2^e_unb, 2^(e_unb+1)) */
    if (e_unb < -6) return sign | (uint8_t)(int)(q * 512.0);
    int mant = (int)((ldexp(q, -e_unb) - 1.0) * 8.0);
    return sign | (uint8_t)(((e_unb + 7) << 3) | mant);
}

void orc_bf16_round_array(const double *in, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_from_double(in[i]);
}

void orc_e4m3_encode_array(const float *in, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_from_float(in[i]);
}

void orc_e4m3_decode_array(const uint8_t *in, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_to_double(in[i]);
}

/* ------------------------------------------------------------------------- */
/* Block-scaled FP8 quantisation ("RL at 1T scale ...", §FP8 Training)        */
/* ------------------------------------------------------------------------- */

/* x: bf16 bits, `rows` x `cols`, row stride `ld` elements.  Blocks are
 * br x bc (1x128 activations, 128x128 weights, 128x1 along rows); a block at
 * the bottom or right edge covers only the elements that exist.
 * q:  codes, rows x cols, row-major (natural layout).
 * s:  scale grid ceil(rows/br) x ceil(cols/bc), row-major (natural layout).
 * For each block: amax = max |x| (exact, from bf16); s = fp32(amax / 448);
 * q = e4m3(fp32(x / s)); s == 0 gives q = 0x00. */
void orc_quant_block(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                     int br, int bc, uint8_t *q, float *s)
{
    int64_t nbr = (rows + br - 1) / br, nbc = (cols + bc - 1) / bc;
#pragma omp parallel for schedule(static)
    for (int64_t bi = 0; bi < nbr; ++bi) {
        for (int64_t bj = 0; bj < nbc; ++bj) {
            int64_t r0 = bi * br, r1 = r0 + br < rows ? r0 + br : rows;
            int64_t c0 = bj * bc, c1 = c0 + bc < cols ? c0 + bc : cols;
            float amax = 0.0f;
            for (int64_t r = r0; r < r1; ++r)
                for (int64_t c = c0; c < c1; ++c) {
                    float a = fabsf(bf16_bits_to_float(x[r * ld + c]));
                    if (a > amax) amax = a;
                }
            float sc = amax / 448.0f;
            s[bi * nbc + bj] = sc;
            for (int64_t r = r0; r < r1; ++r)
                for (int64_t c = c0; c < c1; ++c) {
                    float xv = bf16_bits_to_float(x[r * ld + c]);
                    q[r * cols + c] = (sc == 0.0f) ? 0x00 : orc_e4m3_from_float(xv / sc);
                }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Routing                                                                   */
/* ------------------------------------------------------------------------- */

/* Softmax of the token's E logits in fp64, then renormalised over the chosen
 * set S: w_j = p[S_j] / sum_i p[S_i]. */
static void weights_over_set(const float *z, int E, const int32_t *S, int k, float *w)
{
    double m = -INFINITY;
    for (int e = 0; e < E; ++e)
        if (z[e] > m) m = z[e];
    double *p = (double *)malloc(sizeof(double) * (size_t)E);
    double Z = 0.0;
    for (int e = 0; e < E; ++e) {
        p[e] = exp((double)z[e] - m);
        Z += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= Z;
    double sumS = 0.0;
    for (int j = 0; j < k; ++j) sumS += p[S[j]];
    for (int j = 0; j < k; ++j) w[j] = (float)(p[S[j]] / sumS);
    free(p);
}

/* Top-k routing ("prime-rl 0.6.0 ...", §Drift og omkostninger i realiteten:
 * each token activates a top-k set of experts).  z: fp32 [T][E].
 * idx [T][k]: the k largest logits, compared as fp32; equal logits go to the
 * lower expert index; slots ordered by descending logit.  w [T][k] fp32. */
void orc_route_topk(const float *z, int64_t T, int E, int k, int32_t *idx, float *w)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const float *zt = z + t * E;
        char *chosen = (char *)calloc((size_t)E, 1);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (chosen[e]) continue;
                if (best < 0 || zt[e] > zt[best]) best = e; /* strict: ties keep lower index */
            }
            chosen[best] = 1;
            idx[t * k + j] = best;
        }
        weights_over_set(zt, E, idx + t * k, k, w + t * k);
        free(chosen);
    }
}

/* Router replay ("RL at 1T scale ...", §Router Replay): the payload holds the
 * routed experts of every layer as int32 [L][k][T]; layer `layer` is read back
 * as idx[t][j] = P[(layer*k + j)*T + t].  Weights: w_in [T][k] copied when
 * given, else softmax of the trainer's logits z [T][E] renormalised over the
 * replayed set.  Returns 0, or 4 when an entry is outside [0, E) or a token
 * repeats an expert; such a token gets weight 0 in every slot. */
int orc_route_replay(const int32_t *P, int L, int layer, int64_t T, int E, int k,
                     const float *w_in, const float *z, int32_t *idx, float *w)
{
    int status = 0;
    (void)L;
    for (int64_t t = 0; t < T; ++t) {
        int bad = 0;
        for (int j = 0; j < k; ++j) {
            int32_t e = P[((int64_t)layer * k + j) * T + t];
            idx[t * k + j] = e;
            if (e < 0 || e >= E) bad = 1;
        }
        for (int j = 0; j < k; ++j)
            for (int jj = j + 1; jj < k; ++jj)
                if (idx[t * k + j] == idx[t * k + jj]) bad = 1;
        if (bad) {
            status = 4;
            for (int j = 0; j < k; ++j) w[t * k + j] = 0.0f;
            continue;
        }
        if (w_in) {
            for (int j = 0; j < k; ++j) w[t * k + j] = w_in[t * k + j];
        } else {
            weights_over_set(z + t * E, E, idx + t * k, k, w + t * k);
        }
    }
    return status;
}

/* ------------------------------------------------------------------------- */
/* Permute / dispatch grouping                                               */
/* ------------------------------------------------------------------------- */

/* Stable counting sort of the routed entries i = t*k + j by expert.
 * counts[e] = #entries of e;  offsets[0] = 0, offsets[e+1] = offsets[e] +
 * roundup(counts[e], align);  pos[i] = offsets[e] + #{i' < i : idx[i'] = e};
 * src[r] = i for the row r = pos[i], -1 for every other row of [0, rows_cap).
 * Entries outside [0, E) get pos = -1 and are not counted. */
void orc_permute(const int32_t *idx, int64_t T, int k, int E, int align,
                 int32_t *counts, int32_t *offsets, int32_t *pos, int32_t *src,
                 int64_t rows_cap)
{
    int64_t n = T * k;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t i = 0; i < n; ++i)
        if (idx[i] >= 0 && idx[i] < E) counts[idx[i]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + (counts[e] + align - 1) / align * align;
    for (int64_t r = 0; r < rows_cap; ++r) src[r] = -1;
    int32_t *fill = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    for (int64_t i = 0; i < n; ++i) {
        int32_t e = idx[i];
        if (e < 0 || e >= E) {
            pos[i] = -1;
            continue;
        }
        pos[i] = offsets[e] + fill[e]++;
        src[pos[i]] = (int32_t)i;
    }
    free(fill);
}

/* ------------------------------------------------------------------------- */
/* fp64 contractions over dequantised operands                               */
/* ------------------------------------------------------------------------- */

/* A weight operand: E stacked matrices [E][nr][nc], either as e4m3 codes with
 * a 128x128 scale grid per expert ([E][ceil(nr/128)][ceil(nc/128)]), or as
 * fp64 values (f != NULL; used by the unquantised reference checks). */
typedef struct {
    const uint8_t *q;
    const float *s;
    const double *f;
    int64_t nr, nc;
} orc_wmat;

/* Values of all 256 codes, filled once from orc_e4m3_to_double (a lookup
 * instead of a decode per element; identical values). */
static double e4m3_value[256];
static int e4m3_value_ready = 0;

static void e4m3_table_init(void)
{
    if (e4m3_value_ready) return;
    for (int c = 0; c < 256; ++c) e4m3_value[c] = orc_e4m3_to_double((uint8_t)c);
    e4m3_value_ready = 1;
}

static double wmat_get(const orc_wmat *W, int64_t e, int64_t r, int64_t c)
{
    if (W->f) return W->f[(e * W->nr + r) * W->nc + c];
    int64_t gbr = (W->nr + 127) / 128, gbc = (W->nc + 127) / 128;
    double sc = W->s[(e * gbr + r / 128) * gbc + c / 128];
    return e4m3_value[W->q[(e * W->nr + r) * W->nc + c]] * sc;
}

/* out[i][n] = sum_c A[i][c] * W[e_i][n][c]           (trans = 0; W is [N][K])
 * out[i][n] = sum_c A[i][c] * W[e_i][c][n]           (trans = 1; W is [K][N])
 * A: fp64 [n_rows][K]; expert[i] selects the expert of row i (rows with
 * expert < 0 give zeros).  Sum in ascending c, fp64. */
void orc_rowdot(const double *A, int64_t n_rows, const int32_t *expert, int E,
                const uint8_t *Wq, const float *Ws, const double *Wf,
                int64_t w_nr, int64_t w_nc, int trans, double *out)
{
    orc_wmat W = {Wq, Ws, Wf, w_nr, w_nc};
    int64_t K = trans ? w_nr : w_nc, N = trans ? w_nc : w_nr;
    e4m3_table_init();
    for (int64_t i = 0; i < n_rows * N; ++i) out[i] = 0.0;
    for (int e = 0; e < E; ++e) {
        int64_t cnt = 0;
        for (int64_t i = 0; i < n_rows; ++i) cnt += (expert[i] == e);
        if (!cnt) continue;
        /* dequantise expert e once, as [N][K] */
        double *Wd = (double *)malloc(sizeof(double) * (size_t)(N * K));
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; ++n)
            for (int64_t c = 0; c < K; ++c)
                Wd[n * K + c] = trans ? wmat_get(&W, e, c, n) : wmat_get(&W, e, n, c);
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            const double *wr = Wd + n * K;
            for (int64_t i = 0; i < n_rows; ++i) {
                if (expert[i] != e) continue;
                const double *ar = A + i * K;
                double acc = 0.0;
                for (int64_t c = 0; c < K; ++c) acc += ar[c] * wr[c];
                out[i * N + n] = acc;
            }
        }
        free(Wd);
    }
}

/* Weight gradient of one expert: out[m][n] = sum_r A[r][m] * B[r][n] over the
 * expert's rows r = 0..R-1 (ascending), fp64.  A [R][lda] uses columns
 * m0..m0+M-1, B [R][ldb] columns n0..n0+N-1; out is [M][N]. */
void orc_wgrad(const double *A, int64_t lda, int64_t m0, int64_t M,
               const double *B, int64_t ldb, int64_t n0, int64_t N, int64_t R,
               double *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t r = 0; r < R; ++r) acc += A[r * lda + m0 + m] * B[r * ldb + n0 + n];
            out[m * N + n] = acc;
        }
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
