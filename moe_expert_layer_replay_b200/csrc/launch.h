// Host-side launchers of libmoe.so's kernels (one per kernel family), defined
// in the .cu files and called by the C ABI in moe_abi.cu.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {
// Counts one kernel launch (or one launch recorded into a stream capture);
// read by moe_kernel_launches().
void count_launch();
int launch_route_topk(const float *z, int T, int E, int k, int32_t *idx, float *w, cudaStream_t s);
int launch_route_replay(const int32_t *P, int layer, int T, int E, int k, const float *w_in,
                        const float *z, int32_t *idx, float *w, int *status, cudaStream_t s);
int launch_permute_index(const int32_t *idx, int T, int k, int E, int align, int32_t *counts,
                         int32_t *offsets, int32_t *pos, int32_t *src_idx, int64_t R_cap,
                         void *ws, int *status, cudaStream_t s);
size_t permute_ws_bytes(int T, int k, int E);
int launch_quant_1x128(const uint16_t *in, int64_t ld, int64_t rows, int64_t cols,
                       const int32_t *pos, int k, uint8_t *q, int64_t ldq, float *sc,
                       int64_t ld_s, cudaStream_t s);
int launch_dispatch_quant(const uint16_t *x, int64_t T, int64_t D, const int32_t *pos, int k, uint8_t *xq,
                          float *xs, int64_t R_cap, const int32_t *counts, const int32_t *offsets, int E,
                          cudaStream_t s);
int launch_quant_rows128(const uint16_t *in, int64_t ld, const int32_t *src_idx, int k,
                         int64_t rows, int64_t cols, int64_t ld_rows, uint8_t *qT, float *sT,
                         cudaStream_t s);
int launch_pad_rows(const int32_t *counts, const int32_t *offsets, int E, int64_t cols,
                    int64_t R_cap, uint8_t *q, float *sc, uint16_t *bf, cudaStream_t s);
int launch_quant_128x128(const uint16_t *in, int64_t rows, int64_t cols, int64_t ld, int experts,
                         int64_t in_expert_stride, int rb_mul, int rb_add, uint8_t *q,
                         int64_t q_expert_stride, float *sc, int64_t s_expert_stride, uint8_t *qT,
                         int64_t qT_ld, int64_t qT_expert_stride, float *sT, int64_t sT_ld,
                         int64_t sT_expert_stride, cudaStream_t s);
size_t router_bwd_ws_bytes(int T, int D, int E);
int launch_router_logits(const uint16_t *x, const uint16_t *w_r, int T, int D, int E, float *z, int *status,
                         uint64_t budget, cudaStream_t s);
int launch_capture(const int32_t *idx, int T, int k, int layer, int32_t *payload, cudaStream_t s);
int launch_router_bwd(const float *dz, const uint16_t *x, const uint16_t *w_r, int T, int D, int E,
                      const uint16_t *dx_in, uint16_t *dx, float *dw_r, void *ws, cudaStream_t s);
int launch_quant_nvfp4(const uint16_t *in, int64_t rows, int64_t cols, int64_t ld, uint8_t *q, uint8_t *sf,
                       int sf_layout, float *amax, float *s_g, int sms, cudaStream_t s);
int launch_gemm_nvfp4(int64_t R_cap, int N, int K, int n_seg, const int32_t *offsets, const uint8_t *a,
                      const uint8_t *sfa, const float *a_sg, const uint8_t *b, const uint8_t *sfb,
                      const float *b_sg, float *out, int *status, uint64_t budget, cudaStream_t s);
int launch_combine(const uint16_t *Y, const float *w, const int32_t *pos, int T, int D, int k,
                   uint16_t *y, cudaStream_t s);
int launch_combine_bwd(const uint16_t *dy, const uint16_t *Y, const float *w, const int32_t *pos,
                       const int32_t *idx, int T, int D, int k, int E, int64_t R_cap,
                       uint8_t *dYq, float *dYs, uint16_t *dYb, float *d_w, float *d_logits,
                       cudaStream_t s);
}  // namespace moe
