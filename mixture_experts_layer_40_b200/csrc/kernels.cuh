// Launchers of the MoE kernels (each defined in its own .cu file) and the
// host helpers they share.
#pragma once

#include "common.cuh"
#include "host_util.h"

namespace moe {

// Rows of the grouped expert GEMMs (see moe_expert_up / moe_expert_down).
struct GroupedGemm {
  int32_t H, I, n_groups;
  const int32_t* group_rows;   // device [n_groups]
  const int32_t* group_start;  // device [n_groups]
  int64_t rows;
  uint32_t* status;
};

// 2-D uint8 tensor map over a row-major [rows, inner] buffer, box of
// box_inner bytes x box_rows rows, 128-byte swizzle (host side).
cudaError_t make_tmap_u8(CUtensorMap* map, const void* base, int64_t inner, int64_t rows,
                         int box_inner, int box_rows);

// fp32 [rows, inner] row-major; the swizzle span is the box row (box_inner * 4
// bytes: 32, 64 or 128)
cudaError_t make_tmap_f32(CUtensorMap* map, const void* base, int64_t inner, int64_t rows,
                          int box_inner, int box_rows);
// bf16 tensor map over [depth, rows, inner] (depth 1: 2-D), box of box_inner
// elements x box_rows rows x box_depth; 64-byte swizzle for 32-element box
// rows, 128-byte swizzle otherwise (host side).
cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int64_t inner, int64_t rows,
                           int64_t depth, int box_inner, int box_rows, int box_depth = 1);

// The sizes every entry point accepts (see moe_shape in moe_capi.h).
bool shape_ok(const moe_shape& s);

cudaError_t launch_quantize_1x128(const void* x, int64_t rows, int64_t cols, uint8_t* q,
                                  float* scales, cudaStream_t stream, int sm_count);
cudaError_t launch_quantize_128x128(const float* w, int64_t rows, int64_t cols, uint8_t* q,
                                    float* scales, cudaStream_t stream);

// Router: gate logits (fp32 SIMT GEMM), then sigmoid, biased top-K (node-
// limited to the M best of G expert groups when G > 1), gates and counts
// (counts must be zero on entry; null: not counted).
cudaError_t launch_router(const void* x, const float* gate_w, const float* bias, int T, int H,
                          int N, int K, int G, int M, float* logits, int32_t* ids, float* gates,
                          int32_t* counts, uint32_t* status, cudaStream_t stream, int sm_count);

// Router on tensor cores: splits the fp32 centroids into three bf16 terms in
// `wsplit` (router_split_bytes), computes the logits with BF16 tcgen05 MMAs
// and fp32 accumulation, then the same top-K as launch_router (for large T
// at N = 256 and K <= 8 inside the logits kernel's epilogue; the logits are
// written in every case). splitk_scratch (splitk_bytes, 16-byte aligned; may
// be NULL): room for partial logits, so that batches too small to fill the
// GPU with whole-depth tiles split the reduction over several CTAs.
// presplit: the three terms made earlier (launch_split_gate); NULL: split
// into wsplit first.
size_t router_split_bytes(int N, int H);
// Bytes of partial logits launch_router_tc needs as splitk_scratch to split
// the reduction for this shape (0: no split). With less it computes the
// logits with whole-depth tiles, whose fp32 sums round differently.
size_t router_splitk_bytes(int64_t T, int N, int H);
cudaError_t launch_split_gate(const float* gate_w, int N, int H, __nv_bfloat16* wsplit,
                              cudaStream_t stream, int sm_count);
cudaError_t launch_router_tc(const void* x, const float* gate_w, const float* bias, int T, int H,
                             int N, int K, int G, int M, __nv_bfloat16* wsplit, float* logits,
                             int32_t* ids, float* gates, int32_t* counts, uint32_t* status,
                             cudaStream_t stream, int sm_count,
                             const __nv_bfloat16* presplit = nullptr,
                             float* splitk_scratch = nullptr, size_t splitk_bytes = 0);

// Backward of the expert path (backward.cu).
cudaError_t launch_transpose_blocks(const uint8_t* w, const float* s, int64_t groups, int64_t rows,
                                    int64_t cols, uint8_t* wt, float* st, cudaStream_t stream);
cudaError_t launch_dy_rows_quantize(const void* dy, const float* gates, int T, int H, int K,
                                    const int32_t* token_row, int64_t routed_cap, uint8_t* q,
                                    float* qs, float* row_gate, uint32_t* status,
                                    cudaStream_t stream, int sm_count);
// Column-tile (128 GEMM rows x 1 channel) quantisation of a weight-gradient
// operand, transposed to [C, R]; source 0: gate * dy rows, 1: x rows, 2: h
// from [G|U], 3: [dG|dU] from [G|U] and dh.
cudaError_t launch_quantize_cols(int source, const int32_t* row_token, int64_t routed_cap, int T,
                                 const float* row_gate, const void* src, const float* gu,
                                 const float* dh, int64_t R, int C, int I, uint8_t* codes,
                                 float* scales, bool b_operand, cudaStream_t stream);
// Per-expert weight gradients C_g [M, N] = A_g . B_g^T over each expert's
// GEMM rows, operands transposed [M|N, R] (wgrad.cu).
cudaError_t launch_wgrad(const int32_t* group_rows, const int32_t* group_start, int n_groups,
                         int M, int N, int64_t gemm_rows, const uint8_t* a_t, const float* a_s,
                         const uint8_t* b_t, const float* b_inv, float* c, uint32_t* status,
                         cudaStream_t stream, int sm_count);
cudaError_t launch_swiglu_backward(const float* gu, const float* dh, int64_t rows, int I,
                                   uint8_t* q, float* qs, cudaStream_t stream, int sm_count);
cudaError_t launch_gate_grad(const void* dy, const __nv_bfloat16* y_rows, const int32_t* token_row, int T,
                             int H, int K, int64_t routed_cap, float* dgates, uint32_t* status,
                             cudaStream_t stream, int sm_count);

// Sequence-wise balance statistics from the router's logits and top-K ids
// (f, P [S, N], loss [S]); scratch of balance_scratch_bytes(T, N) bytes.
size_t balance_scratch_bytes(int64_t T, int64_t N);
cudaError_t launch_balance_stats(const float* logits, const int32_t* ids, int T, int N, int K,
                                 int seq_len, float alpha, uint8_t* scratch, float* f, float* P,
                                 float* loss, cudaStream_t stream);

// Permutation: per-chunk ranks and counts, a scan of the counts into group
// tables and per-chunk base rows, and the stable placement of the (token,
// slot) pairs into expert-major GEMM rows. Slots whose id is negative are
// skipped (their token_row entries are left as they are); `pairs` is the
// number of slots with an id, checked against the counts. With count_out the
// per-expert counts are written from the chunks' histograms, else they are
// read and checked against them. `hist` is scratch of
// permute_scratch_bytes(T, N) bytes.
size_t permute_scratch_bytes(int64_t T, int N);
cudaError_t launch_permute(const int32_t* ids, int32_t* counts, bool count_out, int T, int N,
                           int K, int64_t pairs, int64_t routed_cap, int32_t* hist,
                           int32_t* offsets, int32_t* group_rows, int32_t* row_start,
                           int32_t* row_token, int32_t* token_row, uint32_t* status,
                           cudaStream_t stream, int sm_count);
// 1x128 quantisation of x written to each token's shared-expert row
// (routed_cap + t) and to its K routed rows token_row[t, k].
cudaError_t launch_quantize_scatter(const void* x, int T, int H, int K, const int32_t* token_row,
                                    int64_t routed_cap, uint8_t* a_q, float* a_s,
                                    uint32_t* status, cudaStream_t stream, int sm_count);

cudaError_t launch_expert_up(const GroupedGemm& gg, const uint8_t* a_q, const float* a_s,
                             const uint8_t* w13, const float* s13, uint8_t* h_q, float* h_s,
                             cudaStream_t stream, int sm_count);
// Down GEMM with fp32 output rows (the backward's GEMMs; the accumulation
// pin) and with bf16 output rows (the layer's expert outputs).
cudaError_t launch_expert_down(const GroupedGemm& gg, const uint8_t* h_q, const float* h_s,
                               const uint8_t* w2, const float* s2, float* y,
                               cudaStream_t stream, int sm_count);
cudaError_t launch_expert_down_bf16(const GroupedGemm& gg, const uint8_t* h_q, const float* h_s,
                                    const uint8_t* w2, const float* s2, __nv_bfloat16* y,
                                    cudaStream_t stream, int sm_count);

// Combine of the layer (bf16 expert rows) and of the backward's input
// gradients (fp32 rows): y[t] = row[shared] + sum_k g[t,k] row[token_row[t,k]]
// in fp32, slots by ascending expert id, one rounding to bf16 (gates null:
// every weight 1).
cudaError_t launch_combine(const __nv_bfloat16* y_rows, const int32_t* ids, const float* gates,
                           const int32_t* token_row, int T, int H, int K, int64_t routed_cap,
                           int64_t rows_total, __nv_bfloat16* y, uint32_t* status,
                           cudaStream_t stream);
cudaError_t launch_combine(const float* y_rows, const int32_t* ids, const float* gates,
                           const int32_t* token_row, int T, int H, int K, int64_t routed_cap,
                           int64_t rows_total, __nv_bfloat16* y, uint32_t* status,
                           cudaStream_t stream);

cudaError_t launch_update_bias(float* bias, const int32_t* counts, int N, int T, int K,
                               float gamma, cudaStream_t stream);

}  // namespace moe
