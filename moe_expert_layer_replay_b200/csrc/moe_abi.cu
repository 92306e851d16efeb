// C ABI of libmoe.so: argument checks, the device status word, and the
// launch sequence of each entry point.  Declarations and contracts are in
// include/moe.h.
#include <stdio.h>

#include <atomic>

#include "common.cuh"

namespace moe {
int launch_grouped_gemm(int op, const moe_dims &d, int64_t R_cap, const int32_t *offsets, int n_seg,
                        const moe_gemm_args &g, int *status, uint64_t budget, cudaStream_t s);
void set_gemm_variant(int v);
int pair_clusters();
int launch_gateup_gather(const moe_dims &d, int64_t R_cap, const int32_t *offsets, const int32_t *src_idx,
                         const moe_gemm_args &g, int *status, uint64_t budget, cudaStream_t s);
}

// Latched device status word (one per device that loads the library).
static __device__ int g_moe_status;

namespace {
std::atomic<uint64_t> g_launches{0};
}

void moe::count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {

constexpr int kMaxDevices = 64;
int *g_status_ptr[kMaxDevices];
uint64_t g_wait_budget = 0;  // 0 = default

cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool aligned8(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

// Device address of the status word for the current device (looked up once
// per device, with that device current).
int *status_ptr()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_moe_status) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<int *>(p);
    }
    return g_status_ptr[dev];
}

uint64_t wait_budget() { return g_wait_budget ? g_wait_budget : (1ull << 32); }

int check_dims(const moe_dims *d, bool need_gemm_shapes)
{
    if (!d) return MOE_ERR_INVALID_ARG;
    if (d->T < 0 || d->D <= 0 || d->E <= 0 || d->k <= 0) return MOE_ERR_INVALID_ARG;
    if (d->align != 1 && d->align != 128) return MOE_ERR_INVALID_ARG;
    if (d->E > 256 || d->k > 16 || d->k > d->E) return MOE_ERR_UNSUPPORTED;
    if (d->D % 128) return MOE_ERR_UNSUPPORTED;
    if (need_gemm_shapes && (d->I <= 0 || d->I % 128 || d->align != 128)) return MOE_ERR_UNSUPPORTED;
    if ((int64_t)d->T * d->k > (int64_t)1 << 30) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}


}  // namespace

extern "C" {

int64_t moe_rows_capacity(const moe_dims *d)
{
    if (!d) return 0;
    int64_t r = (int64_t)d->T * d->k + (int64_t)d->E * (d->align - 1);
    return (r + 127) / 128 * 128;
}

size_t moe_permute_workspace_size(const moe_dims *d)
{
    if (!d) return 0;
    return moe::permute_ws_bytes(d->T, d->k, d->E);
}

const char *moe_strerror(int status)
{
    switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported sizes";
    case MOE_ERR_CUDA: return "CUDA call or launch failed";
    case MOE_ERR_BAD_ROUTING: return "routing entry outside [0, E) or repeated expert";
    case MOE_ERR_TIMEOUT: return "bounded wait inside a kernel ran out";
    default: return "unknown status";
    }
}

int moe_get_status(void *stream, int *out)
{
    if (!out) return MOE_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    int *p = status_ptr();
    if (!p) return MOE_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemset(p, 0, sizeof v) != cudaSuccess) return MOE_ERR_CUDA;
    *out = v;
    return MOE_OK;
}

void moe_set_wait_budget(uint64_t cycles) { g_wait_budget = cycles; }

uint64_t moe_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

int moe_set_gemm_variant(int variant)
{
    if (variant < -1 || variant > 1) return MOE_ERR_INVALID_ARG;
    moe::set_gemm_variant(variant);
    return MOE_OK;
}

int moe_gemm_pair_clusters(void) { return moe::pair_clusters(); }

int moe_route_topk(const float *logits, const moe_dims *d, int32_t *idx, float *w, void *stream)
{
    int st = check_dims(d, false);
    if (st) return st;
    if (d->T > 0 && (!logits || !idx || !w)) return MOE_ERR_INVALID_ARG;
    return moe::launch_route_topk(logits, d->T, d->E, d->k, idx, w, as_stream(stream));
}

int moe_route_replay(const int32_t *payload, int32_t L, int32_t layer, const moe_dims *d,
                     const float *w_in, const float *logits, int32_t *idx, float *w, void *stream)
{
    int st = check_dims(d, false);
    if (st) return st;
    if (L <= 0 || layer < 0 || layer >= L) return MOE_ERR_INVALID_ARG;
    if (d->T == 0) return MOE_OK;  // nothing to replay (empty arrays may be null)
    if ((w_in == nullptr) == (logits == nullptr)) return MOE_ERR_INVALID_ARG;
    if (!payload || !idx || !w) return MOE_ERR_INVALID_ARG;
    int *sp = status_ptr();
    if (!sp) return MOE_ERR_CUDA;
    return moe::launch_route_replay(payload, layer, d->T, d->E, d->k, w_in, logits, idx, w, sp,
                                    as_stream(stream));
}

int moe_router_fwd(const uint16_t *x, const uint16_t *w_r, const moe_dims *d, float *z, int32_t *idx, float *w,
                   void *stream)
{
    int st = check_dims(d, false);
    if (st) return st;
    if (d->T == 0) return MOE_OK;
    if (!x || !w_r || !z || !aligned16(x) || !aligned16(w_r) || !aligned16(z)) return MOE_ERR_INVALID_ARG;
    if ((idx == nullptr) != (w == nullptr)) return MOE_ERR_INVALID_ARG;
    int *sp = status_ptr();
    if (!sp) return MOE_ERR_CUDA;
    cudaStream_t s = as_stream(stream);
    st = moe::launch_router_logits(x, w_r, d->T, d->D, d->E, z, sp, wait_budget(), s);
    if (st || !idx) return st;
    return moe::launch_route_topk(z, d->T, d->E, d->k, idx, w, s);
}

int moe_capture_payload(const int32_t *idx, const moe_dims *d, int32_t L, int32_t layer, int32_t *payload,
                        void *stream)
{
    int st = check_dims(d, false);
    if (st) return st;
    if (L <= 0 || layer < 0 || layer >= L) return MOE_ERR_INVALID_ARG;
    if (d->T == 0) return MOE_OK;
    if (!idx || !payload) return MOE_ERR_INVALID_ARG;
    return moe::launch_capture(idx, d->T, d->k, layer, payload, as_stream(stream));
}

size_t moe_router_bwd_workspace_size(const moe_dims *d)
{
    if (!d || d->T < 0 || d->D <= 0 || d->E <= 0) return 0;
    return moe::router_bwd_ws_bytes(d->T, d->D, d->E);
}

int moe_router_bwd(const float *dz, const uint16_t *x, const uint16_t *w_r, const moe_dims *d,
                   const uint16_t *dx_in, uint16_t *dx, float *dw_r, void *ws, size_t ws_bytes, void *stream)
{
    int st = check_dims(d, false);
    if (st) return st;
    if (d->T == 0) return MOE_OK;
    if (!dz) return MOE_ERR_INVALID_ARG;
    if (dx && (!w_r || !aligned4(w_r) || !aligned4(dx) || (dx_in && !aligned4(dx_in)))) return MOE_ERR_INVALID_ARG;
    if (dw_r && (!x || !aligned4(x) || !aligned8(dw_r) || !ws || ws_bytes < moe_router_bwd_workspace_size(d) ||
                 !aligned16(ws)))
        return MOE_ERR_INVALID_ARG;
    return moe::launch_router_bwd(dz, x, w_r, d->T, d->D, d->E, dx_in, dx, dw_r, ws, as_stream(stream));
}

int moe_permute(const int32_t *idx, const moe_dims *d, int32_t *counts, int32_t *offsets,
                int32_t *pos, int32_t *src_idx, const uint16_t *x, uint8_t *xq, float *xs,
                uint8_t *xqT, float *xsT, void *ws, size_t ws_bytes, void *stream)
{
    int st = check_dims(d, false);
    if (st) return st;
    if (!counts || !offsets || !src_idx || !ws) return MOE_ERR_INVALID_ARG;
    if (d->T > 0 && (!idx || !pos)) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_permute_workspace_size(d) || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
    if ((xq == nullptr) != (xs == nullptr) || (xq && !x && d->T > 0)) return MOE_ERR_INVALID_ARG;
    if (x && (!aligned16(x) || (xq && (!aligned16(xq) || !aligned4(xs))))) return MOE_ERR_INVALID_ARG;
    if ((xqT == nullptr) != (xsT == nullptr)) return MOE_ERR_INVALID_ARG;
    if (xqT && ((d->T > 0 && !x) || d->align != 128 || !aligned16(xqT))) return MOE_ERR_INVALID_ARG;
    int *sp = status_ptr();
    if (!sp) return MOE_ERR_CUDA;
    cudaStream_t s = as_stream(stream);
    const int64_t R_cap = moe_rows_capacity(d);
    st = moe::launch_permute_index(idx, d->T, d->k, d->E, d->align, counts, offsets, pos, src_idx,
                                   R_cap, ws, sp, s);
    if (st || !x) return st;
    if (xq) st = moe::launch_dispatch_quant(x, d->T, d->D, pos, d->k, xq, xs, R_cap, counts, offsets, d->E, s);
    if (st || !xqT) return st;
    return moe::launch_quant_rows128(x, d->D, src_idx, d->k, R_cap, d->D, R_cap, xqT, xsT, s);
}

int moe_quant_fp8_block(const uint16_t *in, int64_t rows, int64_t cols, int64_t ld, int32_t br,
                        int32_t bc, uint8_t *q, float *s, uint8_t *qT, float *sT, void *stream)
{
    if (rows < 0 || cols <= 0 || cols % 16 || ld < cols || ld % 8) return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (!in || !aligned16(in)) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    if (br == 1 && bc == 128) {
        if (!q || !s || qT || sT || !aligned16(q) || !aligned4(s)) return MOE_ERR_INVALID_ARG;
        return moe::launch_quant_1x128(in, ld, rows, cols, nullptr, 1, q, cols, s, rows, st);
    }
    if (br == 128 && bc == 1) {
        if (!q || !s || qT || sT || rows % 16 || !aligned16(q) || !aligned4(s)) return MOE_ERR_INVALID_ARG;
        return moe::launch_quant_rows128(in, ld, nullptr, 1, rows, cols, rows, q, s, st);
    }
    if (br == 128 && bc == 128) {
        if (!q || !s || !aligned16(q) || !aligned4(s)) return MOE_ERR_INVALID_ARG;
        if ((qT == nullptr) != (sT == nullptr)) return MOE_ERR_INVALID_ARG;
        if (qT && (rows % 16 || !aligned16(qT))) return MOE_ERR_INVALID_ARG;
        const int64_t nbr = (rows + 127) / 128;
        return moe::launch_quant_128x128(in, rows, cols, ld, 1, 0, 1, 0, q, 0, s, 0, qT, rows, 0, sT, nbr,
                                         0, st);
    }
    return MOE_ERR_UNSUPPORTED;
}

int moe_quant_nvfp4(const uint16_t *in, int64_t rows, int64_t cols, int64_t ld, uint8_t *q, uint8_t *sf,
                    int32_t sf_layout, float *amax, float *s_g, void *stream)
{
    if (rows < 0 || cols <= 0 || cols % 16 || ld < cols || ld % 8) return MOE_ERR_INVALID_ARG;
    if (sf_layout != MOE_NVFP4_SF_ROWS && sf_layout != MOE_NVFP4_SF_MMA_A && sf_layout != MOE_NVFP4_SF_MMA_B)
        return MOE_ERR_INVALID_ARG;
    if (sf_layout == MOE_NVFP4_SF_MMA_A && (rows % 128 || cols % 128)) return MOE_ERR_INVALID_ARG;
    if (sf_layout == MOE_NVFP4_SF_MMA_B && (rows % 256 || cols % 64)) return MOE_ERR_INVALID_ARG;
    if (!amax || !s_g || !aligned4(amax) || !aligned4(s_g)) return MOE_ERR_INVALID_ARG;
    if (rows > 0 && (!in || !q || !sf || !aligned16(in) || !aligned8(q))) return MOE_ERR_INVALID_ARG;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return moe::launch_quant_nvfp4(in, rows, cols, ld, q, sf, sf_layout, amax, s_g, sms, as_stream(stream));
}

int moe_gemm_nvfp4(int64_t rows_cap, int32_t N, int32_t K, int32_t n_seg, const int32_t *offsets,
                   const uint8_t *a, const uint8_t *sfa, const float *a_sg, const uint8_t *b, const uint8_t *sfb,
                   const float *b_sg, float *out, void *stream)
{
    if (rows_cap < 0 || rows_cap % 128 || N <= 0 || N % 256 || K <= 0 || K % 256 || n_seg <= 0 || n_seg > 256)
        return MOE_ERR_INVALID_ARG;
    if (!offsets || !a || !sfa || !a_sg || !b || !sfb || !b_sg || !out) return MOE_ERR_INVALID_ARG;
    for (const void *p : {(const void *)a, (const void *)sfa, (const void *)b, (const void *)sfb, (const void *)out})
        if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
    if (!aligned4(a_sg) || !aligned4(b_sg)) return MOE_ERR_INVALID_ARG;
    if (rows_cap == 0) return MOE_OK;
    int *sp = status_ptr();
    if (!sp) return MOE_ERR_CUDA;
    return moe::launch_gemm_nvfp4(rows_cap, N, K, n_seg, offsets, a, sfa, a_sg, b, sfb, b_sg, out, sp,
                                  wait_budget(), as_stream(stream));
}

int moe_quant_weights(const uint16_t *w_gate, const uint16_t *w_up, const uint16_t *w_down,
                      const moe_dims *d, uint8_t *wgu_q, float *wgu_s, uint8_t *wd_q, float *wd_s,
                      uint8_t *wguT_q, float *wguT_s, uint8_t *wdT_q, float *wdT_s, void *stream)
{
    if (!d || d->E <= 0 || d->E > 256 || d->D <= 0 || d->I <= 0) return MOE_ERR_INVALID_ARG;
    if (d->D % 128 || d->I % 128) return MOE_ERR_UNSUPPORTED;
    if (!w_gate || !w_up || !w_down || !wgu_q || !wgu_s || !wd_q || !wd_s) return MOE_ERR_INVALID_ARG;
    const bool T_ = wguT_q || wguT_s || wdT_q || wdT_s;
    if (T_ && !(wguT_q && wguT_s && wdT_q && wdT_s)) return MOE_ERR_INVALID_ARG;
    for (const void *p : {(const void *)w_gate, (const void *)w_up, (const void *)w_down, (const void *)wgu_q,
                          (const void *)wd_q})
        if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
    if (T_ && (!aligned16(wguT_q) || !aligned16(wdT_q))) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    const int64_t E = d->E, D = d->D, I = d->I;
    const int64_t nD = D / 128, nI = I / 128;
    int st;
    // gate -> row blocks 2b, up -> 2b+1 of the [2I][D] stack
    for (int part = 0; part < 2; ++part) {
        const uint16_t *src = part == 0 ? w_gate : w_up;
        st = moe::launch_quant_128x128(src, I, D, D, (int)E, I * D, 2, part, wgu_q, 2 * I * D, wgu_s,
                                       2 * nI * nD, wguT_q, 2 * I, D * 2 * I, wguT_s, 2 * nI, nD * 2 * nI, s);
        if (st) return st;
    }
    return moe::launch_quant_128x128(w_down, D, I, I, (int)E, D * I, 1, 0, wd_q, D * I, wd_s, nD * nI, wdT_q, D,
                                     I * D, wdT_s, nD, nI * nD, s);
}

namespace {
int check_gemm_args(int32_t op, const moe_gemm_args *g)
{
    if (!g || !g->a || !g->sa || !g->b || !g->sb) return MOE_ERR_INVALID_ARG;
    if (!aligned16(g->a) || !aligned16(g->b)) return MOE_ERR_INVALID_ARG;
    switch (op) {
    case MOE_GEMM_GATEUP_SILU:
        if (!g->out_q || !g->out_s || !aligned16(g->out_q)) return MOE_ERR_INVALID_ARG;
        // g, u and h rows leave in 32-byte pieces
        if ((g->aux && !aligned32(g->aux)) || (g->out_bf16 && !aligned32(g->out_bf16))) return MOE_ERR_INVALID_ARG;
        break;
    case MOE_GEMM_DOWN:
    case MOE_GEMM_DGRAD_GATEUP:
        if (!g->out_bf16 || !aligned16(g->out_bf16)) return MOE_ERR_INVALID_ARG;
        break;
    case MOE_GEMM_DGRAD_DOWN_SILU:  // the output step moves 32-byte pieces of aux, out_bf16 and out_q
        if (!g->aux || !g->out_q || !g->out_s || !g->out_bf16 || !aligned32(g->aux) || !aligned32(g->out_q) ||
            !aligned32(g->out_bf16))
            return MOE_ERR_INVALID_ARG;
        break;
    case MOE_GEMM_WGRAD_DOWN:
    case MOE_GEMM_WGRAD_GATEUP:  // the scale rows are bulk-copied: 16-byte alignment
        if (!g->out_f32 || !aligned16(g->out_f32) || !aligned16(g->sa) || !aligned16(g->sb))
            return MOE_ERR_INVALID_ARG;
        break;
    default:
        return MOE_ERR_INVALID_ARG;
    }
    return MOE_OK;
}
}  // namespace

int moe_grouped_gemm_fp8(int32_t op, const moe_dims *d, const int32_t *offsets, const moe_gemm_args *g,
                         void *stream)
{
    int st = check_dims(d, true);
    if (st) return st;
    if (!offsets) return MOE_ERR_INVALID_ARG;
    st = check_gemm_args(op, g);
    if (st) return st;
    int *sp = status_ptr();
    if (!sp) return MOE_ERR_CUDA;
    return moe::launch_grouped_gemm(op, *d, moe_rows_capacity(d), offsets, d->E, *g, sp, wait_budget(),
                                    as_stream(stream));
}

int moe_gateup_gather_fp8(const moe_dims *d, const int32_t *offsets, const int32_t *src_idx,
                          const moe_gemm_args *g, void *stream)
{
    int st = check_dims(d, true);
    if (st) return st;
    if (!offsets || !src_idx) return MOE_ERR_INVALID_ARG;
    st = check_gemm_args(MOE_GEMM_GATEUP_SILU, g);
    if (st) return st;
    if (d->T == 0) return MOE_OK;   // no token: every segment is empty
    int *sp = status_ptr();
    if (!sp) return MOE_ERR_CUDA;
    return moe::launch_gateup_gather(*d, moe_rows_capacity(d), offsets, src_idx, *g, sp, wait_budget(),
                                     as_stream(stream));
}

int moe_grouped_gemm_fp8_seg(int32_t op, const moe_dims *d, int64_t rows_cap, const int32_t *offsets, int32_t n_seg,
                             const moe_gemm_args *g, void *stream)
{
    int st = check_dims(d, true);
    if (st) return st;
    if (op != MOE_GEMM_GATEUP_SILU && op != MOE_GEMM_DOWN && op != MOE_GEMM_DGRAD_DOWN_SILU &&
        op != MOE_GEMM_DGRAD_GATEUP)
        return MOE_ERR_INVALID_ARG;
    if (!offsets || rows_cap < 0 || rows_cap % 128 || n_seg <= 0 || n_seg > 256 || n_seg % d->E)
        return MOE_ERR_INVALID_ARG;
    st = check_gemm_args(op, g);
    if (st) return st;
    int *sp = status_ptr();
    if (!sp) return MOE_ERR_CUDA;
    return moe::launch_grouped_gemm(op, *d, rows_cap, offsets, n_seg, *g, sp, wait_budget(), as_stream(stream));
}

int moe_combine(const uint16_t *Y, const float *w, const int32_t *pos, const moe_dims *d, uint16_t *y,
                void *stream)
{
    int st = check_dims(d, false);
    if (st) return st;
    if (d->T == 0) return MOE_OK;
    if (!Y || !w || !pos || !y || !aligned16(Y) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
    return moe::launch_combine(Y, w, pos, d->T, d->D, d->k, y, as_stream(stream));
}

int moe_combine_bwd(const uint16_t *dy, const uint16_t *Y, const float *w, const int32_t *pos,
                    const int32_t *idx, const int32_t *counts, const int32_t *offsets, const moe_dims *d,
                    uint8_t *dYq, float *dYs, uint16_t *dY_bf16, float *d_w, float *d_logits, void *stream)
{
    int st = check_dims(d, false);
    if (st) return st;
    if (!counts || !offsets || !dYq || !dYs) return MOE_ERR_INVALID_ARG;
    if (d->T > 0 && (!dy || !Y || !w || !pos || !idx || !d_w)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(dYq) || (dy && !aligned16(dy)) || (Y && !aligned16(Y)) ||
        (dY_bf16 && !aligned16(dY_bf16)))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    const int64_t R_cap = moe_rows_capacity(d);
    st = moe::launch_combine_bwd(dy, Y, w, pos, idx, d->T, d->D, d->k, d->E, R_cap, dYq, dYs, dY_bf16, d_w,
                                 d_logits, s);
    if (st) return st;
    return moe::launch_pad_rows(counts, offsets, d->E, d->D, R_cap, dYq, dYs, dY_bf16, s);
}

int moe_unpermute_reduce(const uint16_t *dX, const int32_t *pos, const moe_dims *d, uint16_t *dx, void *stream)
{
    int st = check_dims(d, false);
    if (st) return st;
    if (d->T == 0) return MOE_OK;
    if (!dX || !pos || !dx || !aligned16(dX) || !aligned16(dx)) return MOE_ERR_INVALID_ARG;
    return moe::launch_combine(dX, nullptr, pos, d->T, d->D, d->k, dx, as_stream(stream));
}

}  // extern "C"
