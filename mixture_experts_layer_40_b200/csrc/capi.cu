// C ABI entry points (declared in include/moe_capi.h): argument checks,
// workspace layout, tensor maps, and the launch sequence of the forward.
#include <algorithm>
#include <mutex>

#include "host_util.h"
#include "kernels.cuh"

namespace moe {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(p);
    }
  });
  return fn;
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev] = n;
  }
  return cached[dev];
}



void layout_of(const moe_shape& s, moe_ws_layout* L) {
  const int64_t T = s.T, H = s.H, N = s.N, K = s.K, I = s.I;
  L->routed_cap = round_up(T * K + N * (kTile - 1), kTile);
  L->rows_total = L->routed_cap + round_up(T, kTile);
  Carver carve;
  auto take = [&](size_t bytes) { return carve.take(bytes); };
  L->status = take(16);
  L->counts = take(N * 4);
  L->offsets = take((N + 1) * 4);
  L->group_rows = take((N + 1) * 4);
  L->row_start = take((N + 1) * 4);
  L->row_token = take((size_t)L->routed_cap * 4);
  L->token_row = take((size_t)(T * K) * 4);
  L->topk_ids = take((size_t)(T * K) * 4);
  L->topk_gates = take((size_t)(T * K) * 4);
  L->logits = take((size_t)(T * N) * 4);
  // the router's partial logits live here until the rows are written
  L->a_q = take(std::max((size_t)L->rows_total * H, router_splitk_bytes(T, (int)N, (int)H)));
  L->a_s = take((size_t)L->rows_total * (H / kTile) * 4);
  L->h_q = take((size_t)L->rows_total * I);
  L->h_s = take((size_t)L->rows_total * (I / kTile) * 4);
  L->y_rows = take((size_t)L->rows_total * H * 2);
  L->gate_split = take(router_split_bytes((int)N, (int)H));
  L->bal_scratch = take(balance_scratch_bytes(T, N));
  L->perm_scratch = take(permute_scratch_bytes(T, (int)N));
  L->total = carve.off;
}


}  // namespace

bool shape_ok(const moe_shape& s) {
  return s.T >= 0 && s.H >= 256 && s.H % 256 == 0 && s.I >= 128 && s.I % 128 == 0 && s.N >= 16 &&
         s.N <= 1024 && s.N % 16 == 0 && s.K >= 1 && s.K <= s.N && s.K <= 16 &&
         (int64_t)s.T * s.K < (1ll << 31) && (int64_t)s.T * s.N < (1ll << 31) &&
         (s.G == 0 || (s.G >= 1 && s.G <= 32 && s.N % s.G == 0 && s.M >= 1 && s.M <= s.G &&
                       s.K % s.M == 0 && s.K / s.M <= s.N / s.G));
}

cudaError_t make_tmap_u8(CUtensorMap* map, const void* base, int64_t inner, int64_t rows,
                         int box_inner, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)(rows > 0 ? rows : 1)};
  const cuuint64_t strides[1] = {(cuuint64_t)inner};
  const cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_f32(CUtensorMap* map, const void* base, int64_t inner, int64_t rows,
                          int box_inner, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)(rows > 0 ? rows : 1)};
  const cuuint64_t strides[1] = {(cuuint64_t)inner * 4};
  const cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        box_inner * 4 == 32    ? CU_TENSOR_MAP_SWIZZLE_32B
                        : box_inner * 4 == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
                                               : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int64_t inner, int64_t rows,
                           int64_t depth, int box_inner, int box_rows, int box_depth) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)(rows > 0 ? rows : 1),
                              (cuuint64_t)(depth > 0 ? depth : 1)};
  const cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)(inner * 2 * (rows > 0 ? rows : 1))};
  const cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows,
                             (cuuint32_t)(box_depth > 0 ? box_depth : 1)};
  const cuuint32_t estr[3] = {1, 1, 1};
  const cuuint32_t rank = depth > 1 ? 3 : 2;
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        box_inner * 2 == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                            : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace moe

using namespace moe;

extern "C" {

int moe_device_sm_count(void) { return sm_count(); }

int moe_quantize_1x128(const void* x, int64_t rows, int64_t cols, uint8_t* q, float* scales,
                       void* stream) {
  if (rows < 0 || cols <= 0 || cols % kTile != 0) return MOE_ERR_SHAPE;
  if (rows == 0) return MOE_OK;  // nothing to do; empty tensors may carry NULL
  if (x == nullptr || q == nullptr || scales == nullptr) return MOE_ERR_NULL;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(scales, 4)) return MOE_ERR_ALIGN;
  return cuda_status(launch_quantize_1x128(x, rows, cols, q, scales,
                                           static_cast<cudaStream_t>(stream), sm_count()));
}

int moe_quantize_128x128(const float* w, int64_t rows, int64_t cols, uint8_t* q, float* scales,
                         void* stream) {
  if (w == nullptr || q == nullptr || scales == nullptr) return MOE_ERR_NULL;
  if (rows <= 0 || cols <= 0 || rows % kTile != 0 || cols % kTile != 0) return MOE_ERR_SHAPE;
  if (rows / kTile > 65535) return MOE_ERR_SHAPE;
  if (!aligned(w, 16) || !aligned(q, 16) || !aligned(scales, 4)) return MOE_ERR_ALIGN;
  return cuda_status(
      launch_quantize_128x128(w, rows, cols, q, scales, static_cast<cudaStream_t>(stream)));
}

int moe_split_gate(const float* gate_w, int32_t N, int32_t H, void* gate_split, void* stream) {
  if (!gate_w || !gate_split) return MOE_ERR_NULL;
  if (N < 1 || H < 1) return MOE_ERR_SHAPE;
  if (!aligned(gate_w, 16) || !aligned(gate_split, 16)) return MOE_ERR_ALIGN;
  return cuda_status(launch_split_gate(gate_w, N, H, static_cast<__nv_bfloat16*>(gate_split),
                                       static_cast<cudaStream_t>(stream), sm_count()));
}

size_t moe_workspace_size(moe_shape sh) {
  if (!shape_ok(sh)) return 0;
  moe_ws_layout L;
  layout_of(sh, &L);
  return L.total;
}

int moe_workspace_layout(moe_shape sh, moe_ws_layout* out) {
  if (out == nullptr) return MOE_ERR_NULL;
  if (!shape_ok(sh)) return MOE_ERR_SHAPE;
  layout_of(sh, out);
  return MOE_OK;
}

int moe_route(moe_shape sh, const float* gate_w, const void* x, const float* bias,
              int32_t* topk_ids, float* topk_gates, int32_t* counts, void* ws, size_t ws_bytes,
              void* stream) {
  if (!shape_ok(sh)) return MOE_ERR_SHAPE;
  if (sh.T == 0) {  // an empty batch: only the counts are cleared
    if (!counts) return MOE_ERR_NULL;
    return cuda_status(
        cudaMemsetAsync(counts, 0, (size_t)sh.N * 4, static_cast<cudaStream_t>(stream)));
  }
  if (!gate_w || !x || !bias || !topk_ids || !topk_gates || !counts || !ws) return MOE_ERR_NULL;
  if (!aligned(x, 16) || !aligned(gate_w, 16) || !aligned(ws, 256)) return MOE_ERR_ALIGN;
  moe_ws_layout L;
  layout_of(sh, &L);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  NvtxRange range("moe_route");
  uint32_t* status = at<uint32_t>(ws, L.status);
  cudaError_t e = cudaMemsetAsync(status, 0, 4, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(counts, 0, (size_t)sh.N * 4, s);
  if (e == cudaSuccess)
    e = launch_router_tc(x, gate_w, bias, sh.T, sh.H, sh.N, sh.K, sh.G, sh.M,
                         at<__nv_bfloat16>(ws, L.gate_split), at<float>(ws, L.logits), topk_ids,
                         topk_gates, counts, status, s, sm_count(), nullptr,
                         at<float>(ws, L.a_q), (size_t)L.rows_total * sh.H);
  return cuda_status(e);
}

int moe_balance_stats(moe_shape sh, int32_t seq_len, float alpha, void* ws, size_t ws_bytes,
                      const int32_t* topk_ids, float* f, float* P, float* loss, void* stream) {
  if (!shape_ok(sh) || seq_len < 1) return MOE_ERR_SHAPE;
  if (sh.T == 0) return MOE_OK;  // no sequences
  if (!ws || !topk_ids || !f || !P || !loss) return MOE_ERR_NULL;
  if (!aligned(ws, 256)) return MOE_ERR_ALIGN;
  moe_ws_layout L;
  layout_of(sh, &L);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  return cuda_status(launch_balance_stats(at<float>(ws, L.logits), topk_ids, sh.T, sh.N, sh.K,
                                          seq_len, alpha, at<uint8_t>(ws, L.bal_scratch), f, P,
                                          loss, static_cast<cudaStream_t>(stream)));
}

static int forward_impl(moe_shape sh, const moe_weights* w, const void* x, const float* bias,
                        void* y, int32_t* topk_ids_opt, float* topk_gates_opt, int32_t* counts_opt,
                        void* ws, size_t ws_bytes, void* stream, void* const* events) {
  if (!shape_ok(sh)) return MOE_ERR_SHAPE;
  if (sh.T == 0) {
    // an empty batch: nothing to compute; the status word and the counts
    // (for moe_update_bias, which then leaves the bias unchanged) are cleared
    if (!ws) return MOE_ERR_NULL;
    if (!aligned(ws, 256)) return MOE_ERR_ALIGN;
    moe_ws_layout L;
    layout_of(sh, &L);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(at<uint32_t>(ws, L.status), 0, 4, s);
    int32_t* counts = counts_opt ? counts_opt : at<int32_t>(ws, L.counts);
    if (e == cudaSuccess) e = cudaMemsetAsync(counts, 0, (size_t)sh.N * 4, s);
    for (int i = 0; events != nullptr && i < MOE_TRACE_EVENTS && e == cudaSuccess; ++i)
      e = cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s);
    return cuda_status(e);
  }
  if (!w || !x || !bias || !y || !ws) return MOE_ERR_NULL;
  if (!w->gate_w || !w->w13 || !w->s13 || !w->w2 || !w->s2) return MOE_ERR_NULL;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(w->gate_w, 16) || !aligned(w->w13, 16) ||
      !aligned(w->w2, 16) || !aligned(ws, 256) || !aligned(w->gate_split, 16))
    return MOE_ERR_ALIGN;
  moe_ws_layout L;
  layout_of(sh, &L);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = sm_count();
  uint32_t* status = at<uint32_t>(ws, L.status);
  int32_t* ids = topk_ids_opt ? topk_ids_opt : at<int32_t>(ws, L.topk_ids);
  float* gates = topk_gates_opt ? topk_gates_opt : at<float>(ws, L.topk_gates);
  int32_t* counts = counts_opt ? counts_opt : at<int32_t>(ws, L.counts);
  uint8_t* a_q = at<uint8_t>(ws, L.a_q);
  float* a_s = at<float>(ws, L.a_s);

  // optional stage events: recorded before each of the 6 stages and at the
  // end; an NVTX range per stage in any case
  static const char* const kStageNames[MOE_TRACE_EVENTS - 1] = {
      "moe_forward/route", "moe_forward/permute", "moe_forward/quantize",
      "moe_forward/expert_up", "moe_forward/expert_down", "moe_forward/combine"};
  NvtxRange whole("moe_forward");
  bool in_range = false;
  auto mark = [&](int i, cudaError_t e) {
    if (in_range) nvtxRangePop();
    in_range = i < MOE_TRACE_EVENTS - 1;
    if (in_range) nvtxRangePushA(kStageNames[i]);
    if (events != nullptr && e == cudaSuccess)
      return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s);
    return e;
  };
  cudaError_t e = mark(0, cudaSuccess);
  if (e == cudaSuccess) e = cudaMemsetAsync(status, 0, 4, s);
  // a2-a5: gate logits, sigmoid, biased top-K, gates (from bf16 x)
  if (e == cudaSuccess)
    e = launch_router_tc(x, w->gate_w, bias, sh.T, sh.H, sh.N, sh.K, sh.G, sh.M,
                         at<__nv_bfloat16>(ws, L.gate_split), at<float>(ws, L.logits), ids, gates,
                         nullptr, status, s, sms,
                         static_cast<const __nv_bfloat16*>(w->gate_split),
                         // the activation rows are written after the routing:
                         // their region holds the partial logits meanwhile
                         reinterpret_cast<float*>(a_q), (size_t)L.rows_total * sh.H);
  e = mark(1, e);
  // a6-a7: counts from per-chunk histograms, offsets, stable expert-major
  // placement of the (token, slot) pairs
  if (e == cudaSuccess)
    e = launch_permute(ids, counts, true, sh.T, sh.N, sh.K, (int64_t)sh.T * sh.K, L.routed_cap,
                       at<int32_t>(ws, L.perm_scratch), at<int32_t>(ws, L.offsets),
                       at<int32_t>(ws, L.group_rows), at<int32_t>(ws, L.row_start),
                       at<int32_t>(ws, L.row_token), at<int32_t>(ws, L.token_row), status, s,
                       sms);
  e = mark(2, e);
  // a1 (+ a7's row copies): x -> 1x128 codes and scales, written to the
  // token's shared-expert row and its K routed rows
  if (e == cudaSuccess)
    e = launch_quantize_scatter(x, sh.T, sh.H, sh.K, at<int32_t>(ws, L.token_row), L.routed_cap,
                                a_q, a_s, status, s, sms);
  GroupedGemm gg{sh.H, sh.I, sh.N + 1, at<int32_t>(ws, L.group_rows), at<int32_t>(ws, L.row_start),
                 L.rows_total, status};
  e = mark(3, e);
  // a8: up/gate GEMM + SwiGLU + 1x128 re-quantisation
  if (e == cudaSuccess)
    e = launch_expert_up(gg, a_q, a_s, w->w13, w->s13, at<uint8_t>(ws, L.h_q), at<float>(ws, L.h_s),
                         s, sms);
  e = mark(4, e);
  // a9: down GEMM -> bf16 expert outputs
  if (e == cudaSuccess)
    e = launch_expert_down_bf16(gg, at<uint8_t>(ws, L.h_q), at<float>(ws, L.h_s), w->w2, w->s2,
                                at<__nv_bfloat16>(ws, L.y_rows), s, sms);
  e = mark(5, e);
  // a10: weighted combine with the shared expert
  if (e == cudaSuccess)
    e = launch_combine(at<__nv_bfloat16>(ws, L.y_rows), ids, gates, at<int32_t>(ws, L.token_row),
                       sh.T, sh.H, sh.K, L.routed_cap, L.rows_total,
                       static_cast<__nv_bfloat16*>(y), status, s);
  e = mark(6, e);
  return cuda_status(e);
}

int moe_forward(moe_shape sh, const moe_weights* w, const void* x, const float* bias, void* y,
                int32_t* topk_ids_opt, float* topk_gates_opt, int32_t* counts_opt, void* ws,
                size_t ws_bytes, void* stream) {
  return forward_impl(sh, w, x, bias, y, topk_ids_opt, topk_gates_opt, counts_opt, ws, ws_bytes,
                      stream, nullptr);
}

int moe_forward_traced(moe_shape sh, const moe_weights* w, const void* x, const float* bias,
                       void* y, int32_t* topk_ids_opt, float* topk_gates_opt, int32_t* counts_opt,
                       void* ws, size_t ws_bytes, void* stream, void* const* events,
                       int32_t n_events) {
  if (events == nullptr || n_events < MOE_TRACE_EVENTS) return MOE_ERR_NULL;
  for (int i = 0; i < MOE_TRACE_EVENTS; ++i)
    if (events[i] == nullptr) return MOE_ERR_NULL;
  return forward_impl(sh, w, x, bias, y, topk_ids_opt, topk_gates_opt, counts_opt, ws, ws_bytes,
                      stream, events);
}


int moe_update_bias(float* bias, const int32_t* counts, int32_t N, int32_t T, int32_t K,
                    float gamma, void* stream) {
  if (!bias || !counts) return MOE_ERR_NULL;
  if (N < 1 || T < 0 || K < 1) return MOE_ERR_SHAPE;
  return cuda_status(launch_update_bias(bias, counts, N, T, K, gamma, static_cast<cudaStream_t>(stream)));
}

static int expert_args_ok(int32_t H, int32_t I, int32_t n_groups, const int32_t* gr,
                          const int32_t* gs, int64_t rows) {
  if (H < 256 || H % 256 != 0 || I < 128 || I % 128 != 0) return MOE_ERR_SHAPE;
  if (n_groups < 1 || n_groups > 1025 || rows < 0 || rows >= (1ll << 31)) return MOE_ERR_SHAPE;
  if (!gr || !gs) return MOE_ERR_NULL;
  return MOE_OK;
}

int moe_expert_up(int32_t H, int32_t I, int32_t n_groups, const int32_t* group_rows,
                  const int32_t* group_start, int64_t rows, const uint8_t* a_q, const float* a_s,
                  const uint8_t* w13, const float* s13, uint8_t* h_q, float* h_s,
                  uint32_t* status_ws, void* stream) {
  const int r = expert_args_ok(H, I, n_groups, group_rows, group_start, rows);
  if (r != MOE_OK) return r;
  if (!a_q || !a_s || !w13 || !s13 || !h_q || !h_s) return MOE_ERR_NULL;
  if (!aligned(a_q, 16) || !aligned(w13, 16) || !aligned(h_q, 16)) return MOE_ERR_ALIGN;
  GroupedGemm gg{H, I, n_groups, group_rows, group_start, rows, status_ws};
  return cuda_status(launch_expert_up(gg, a_q, a_s, w13, s13, h_q, h_s,
                                      static_cast<cudaStream_t>(stream), sm_count()));
}

int moe_expert_down(int32_t H, int32_t I, int32_t n_groups, const int32_t* group_rows,
                    const int32_t* group_start, int64_t rows, const uint8_t* h_q,
                    const float* h_s, const uint8_t* w2, const float* s2, void* y_rows,
                    uint32_t* status_ws, void* stream) {
  const int r = expert_args_ok(H, I, n_groups, group_rows, group_start, rows);
  if (r != MOE_OK) return r;
  if (!h_q || !h_s || !w2 || !s2 || !y_rows) return MOE_ERR_NULL;
  if (!aligned(h_q, 16) || !aligned(w2, 16) || !aligned(y_rows, 16)) return MOE_ERR_ALIGN;
  GroupedGemm gg{H, I, n_groups, group_rows, group_start, rows, status_ws};
  return cuda_status(launch_expert_down(gg, h_q, h_s, w2, s2, static_cast<float*>(y_rows),
                                        static_cast<cudaStream_t>(stream), sm_count()));
}

int moe_expert_down_bf16(int32_t H, int32_t I, int32_t n_groups, const int32_t* group_rows,
                         const int32_t* group_start, int64_t rows, const uint8_t* h_q,
                         const float* h_s, const uint8_t* w2, const float* s2, void* y_rows,
                         uint32_t* status_ws, void* stream) {
  const int r = expert_args_ok(H, I, n_groups, group_rows, group_start, rows);
  if (r != MOE_OK) return r;
  if (!h_q || !h_s || !w2 || !s2 || !y_rows) return MOE_ERR_NULL;
  if (!aligned(h_q, 16) || !aligned(w2, 16) || !aligned(y_rows, 16)) return MOE_ERR_ALIGN;
  GroupedGemm gg{H, I, n_groups, group_rows, group_start, rows, status_ws};
  return cuda_status(launch_expert_down_bf16(gg, h_q, h_s, w2, s2,
                                             static_cast<__nv_bfloat16*>(y_rows),
                                             static_cast<cudaStream_t>(stream), sm_count()));
}

int moe_transpose_weights(moe_shape sh, const moe_weights* w, uint8_t* w13t, float* s13t,
                          uint8_t* w2t, float* s2t, void* stream) {
  if (!shape_ok(sh)) return MOE_ERR_SHAPE;
  if (!w || !w->w13 || !w->s13 || !w->w2 || !w->s2) return MOE_ERR_NULL;
  if (!w13t || !s13t || !w2t || !s2t) return MOE_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t E = sh.N + 1, H = sh.H, I = sh.I;
  cudaError_t e = launch_transpose_blocks(w->w13, w->s13, E, 2 * I, H, w13t, s13t, s);
  if (e == cudaSuccess) e = launch_transpose_blocks(w->w2, w->s2, E, H, I, w2t, s2t, s);
  return cuda_status(e);
}

}  // extern "C"

namespace moe {
namespace {

struct BackwardLayout {
  size_t dy_q, dy_s, gu, dh, dgu_q, dgu_s, dx_rows;
  // weight gradients: row gates and the column-tile operands
  size_t row_gate, dyt_q, dyt_s, ht_q, ht_inv, dgut_q, dgut_s, xt_q, xt_inv;
  size_t total;
};

BackwardLayout backward_layout(const moe_shape& sh) {
  moe_ws_layout L;
  layout_of(sh, &L);
  const size_t R = (size_t)L.rows_total, H = sh.H, I = sh.I;
  BackwardLayout B{};
  Carver carve;
  auto take = [&](size_t bytes) { return carve.take(bytes); };
  B.dy_q = take(R * H);
  B.dy_s = take(R * (H / kTile) * 4);
  B.gu = take(R * 2 * I * 4);
  B.dh = take(R * I * 4);
  B.dgu_q = take(R * 2 * I);
  B.dgu_s = take(R * (2 * I / kTile) * 4);
  B.dx_rows = take(R * H * 4);
  B.row_gate = take(R * 4);
  B.dyt_q = take(H * R);
  B.dyt_s = take(H * (R / kTile) * 4);
  B.ht_q = take(I * R);
  B.ht_inv = take((R / kTile) * I * 4);
  B.dgut_q = take(2 * I * R);
  B.dgut_s = take(2 * I * (R / kTile) * 4);
  B.xt_q = take(H * R);
  B.xt_inv = take((R / kTile) * H * 4);
  B.total = carve.off;
  return B;
}

bool backward_shape_ok(const moe_shape& sh) { return shape_ok(sh) && sh.I % 256 == 0; }

}  // namespace
}  // namespace moe

extern "C" {

size_t moe_backward_workspace_size(moe_shape sh) {
  if (!backward_shape_ok(sh)) return 0;
  return backward_layout(sh).total;
}

int moe_backward(moe_shape sh, const moe_weights* w, const moe_weights* wt,
                 const int32_t* topk_ids, const float* topk_gates, const void* x, const void* dy,
                 void* ws, size_t ws_bytes, void* bws, size_t bws_bytes, void* dx, float* dgates,
                 float* dw13, float* dw2, void* stream) {
  if (!backward_shape_ok(sh)) return MOE_ERR_SHAPE;
  if (!w || !wt || !ws || !bws) return MOE_ERR_NULL;
  moe_ws_layout L;
  layout_of(sh, &L);
  const BackwardLayout B = backward_layout(sh);
  if (ws_bytes < L.total || bws_bytes < B.total) return MOE_ERR_WORKSPACE;
  if (!aligned(ws, 256) || !aligned(bws, 256)) return MOE_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = at<uint32_t>(ws, L.status);
  if (sh.T == 0) return cuda_status(cudaMemsetAsync(status, 0, 4, s));
  if (!topk_ids || !topk_gates || !dy || !dx || !dgates) return MOE_ERR_NULL;
  if (!w->w13 || !w->s13 || !wt->w13 || !wt->s13 || !wt->w2 || !wt->s2) return MOE_ERR_NULL;
  if (!aligned(dy, 16) || !aligned(dx, 16) || !aligned(w->w13, 16) || !aligned(wt->w13, 16) ||
      !aligned(wt->w2, 16))
    return MOE_ERR_ALIGN;
  const int sms = sm_count();
  NvtxRange range("moe_backward");
  const int32_t* token_row = at<int32_t>(ws, L.token_row);
  const __nv_bfloat16* y_rows = at<__nv_bfloat16>(ws, L.y_rows);
  float* dx_rows = at<float>(bws, B.dx_rows);
  cudaError_t e = cudaMemsetAsync(status, 0, 4, s);
  // gate gradients from the forward's bf16 expert output rows
  if (e == cudaSuccess)
    e = launch_gate_grad(dy, y_rows, token_row, sh.T, sh.H, sh.K, L.routed_cap, dgates, status, s,
                         sms);
  // dY rows: g dy (routed), dy (shared), 1x128 along H
  const bool wgrad = dw13 != nullptr && dw2 != nullptr;
  if (wgrad && (!x || !aligned(dw13, 16) || !aligned(dw2, 16))) return MOE_ERR_NULL;
  if (e == cudaSuccess && wgrad)
    e = cudaMemsetAsync(at<float>(bws, B.row_gate), 0, (size_t)L.rows_total * 4, s);
  if (e == cudaSuccess)
    e = launch_dy_rows_quantize(dy, topk_gates, sh.T, sh.H, sh.K, token_row, L.routed_cap,
                                at<uint8_t>(bws, B.dy_q), at<float>(bws, B.dy_s),
                                wgrad ? at<float>(bws, B.row_gate) : nullptr, status, s, sms);
  const int32_t* gr = at<int32_t>(ws, L.group_rows);
  const int32_t* gs = at<int32_t>(ws, L.row_start);
  // [G | U] recomputed from the forward's x rows: fp32 [rows, 2I]
  if (e == cudaSuccess) {
    GroupedGemm gg{2 * sh.I, sh.H, sh.N + 1, gr, gs, L.rows_total, status};
    e = launch_expert_down(gg, at<uint8_t>(ws, L.a_q), at<float>(ws, L.a_s), w->w13, w->s13,
                           at<float>(bws, B.gu), s, sms);
  }
  // Dgrad of the down projection: dh = dY . W2, fp32 [rows, I]
  if (e == cudaSuccess) {
    GroupedGemm gg{sh.I, sh.H, sh.N + 1, gr, gs, L.rows_total, status};
    e = launch_expert_down(gg, at<uint8_t>(bws, B.dy_q), at<float>(bws, B.dy_s), wt->w2, wt->s2,
                           at<float>(bws, B.dh), s, sms);
  }
  // SwiGLU backward, [dG | dU] 1x128 in w13's row order
  if (e == cudaSuccess)
    e = launch_swiglu_backward(at<float>(bws, B.gu), at<float>(bws, B.dh), L.rows_total, sh.I,
                               at<uint8_t>(bws, B.dgu_q), at<float>(bws, B.dgu_s), s, sms);
  // Dgrad of the up/gate projection: dX rows = [dG | dU] . W13, fp32 [rows, H]
  if (e == cudaSuccess) {
    GroupedGemm gg{sh.H, 2 * sh.I, sh.N + 1, gr, gs, L.rows_total, status};
    e = launch_expert_down(gg, at<uint8_t>(bws, B.dgu_q), at<float>(bws, B.dgu_s), wt->w13,
                           wt->s13, dx_rows, s, sms);
  }
  // dx[t] = the token's K + 1 row gradients, fixed order, one bf16 rounding
  if (e == cudaSuccess)
    e = launch_combine(dx_rows, topk_ids, nullptr, token_row, sh.T, sh.H, sh.K, L.routed_cap,
                       L.rows_total, static_cast<__nv_bfloat16*>(dx), status, s);
  if (!wgrad || e != cudaSuccess) return cuda_status(e);
  // Wgrad: operands in column tiles (128 rows x 1 channel), transposed
  const int32_t* row_token = at<int32_t>(ws, L.row_token);
  const int64_t R = L.rows_total;
  const float* rg = at<float>(bws, B.row_gate);
  const float* gu = at<float>(bws, B.gu);
  const int64_t cap = L.routed_cap;
  uint8_t* b8 = static_cast<uint8_t*>(bws);
  e = launch_quantize_cols(0, row_token, cap, sh.T, rg, dy, nullptr, nullptr, R, sh.H, sh.I,
                           b8 + B.dyt_q, at<float>(bws, B.dyt_s), false, s);
  if (e == cudaSuccess)
    e = launch_quantize_cols(2, row_token, cap, sh.T, rg, nullptr, gu, nullptr, R, sh.I, sh.I,
                             b8 + B.ht_q, at<float>(bws, B.ht_inv), true, s);
  if (e == cudaSuccess)
    e = launch_quantize_cols(3, row_token, cap, sh.T, rg, nullptr, gu, at<float>(bws, B.dh), R,
                             2 * sh.I, sh.I, b8 + B.dgut_q, at<float>(bws, B.dgut_s), false, s);
  if (e == cudaSuccess)
    e = launch_quantize_cols(1, row_token, cap, sh.T, rg, x, nullptr, nullptr, R, sh.H, sh.I,
                             b8 + B.xt_q, at<float>(bws, B.xt_inv), true, s);
  // dW2_e [H, I] = dY_e^T . h_e;  dW13_e [2I, H] = [dG|dU]_e^T . x_e
  if (e == cudaSuccess)
    e = launch_wgrad(gr, gs, sh.N + 1, sh.H, sh.I, R, at<uint8_t>(bws, B.dyt_q),
                     at<float>(bws, B.dyt_s), at<uint8_t>(bws, B.ht_q), at<float>(bws, B.ht_inv),
                     dw2, status, s, sms);
  if (e == cudaSuccess)
    e = launch_wgrad(gr, gs, sh.N + 1, 2 * sh.I, sh.H, R, at<uint8_t>(bws, B.dgut_q),
                     at<float>(bws, B.dgut_s), at<uint8_t>(bws, B.xt_q), at<float>(bws, B.xt_inv),
                     dw13, status, s, sms);
  return cuda_status(e);
}

int moe_get_status(void* ws, void* stream) {
  if (!ws) return MOE_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, ws, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemset(ws, 0, 4) != cudaSuccess) return MOE_ERR_CUDA;
  if (word & kStatusTimeout) return MOE_ERR_TIMEOUT;
  if (word & kStatusBounds) return MOE_ERR_BOUNDS;
  return MOE_OK;
}

}  // extern "C"
