// Expert parallelism: the layer split over W ranks (one GPU each), routed
// experts sharded contiguously (rank d holds experts [d N/W, (d+1) N/W)), the
// shared expert and the gate replicated. "DeepSeek-V3: Auxiliary-Loss-Free MoE
// Load Balancing, ..." section V ("Training at Scale", "Custom all-to-all
// kernels"): a token is sent once to each rank that holds one of its experts
// and reaches all of its experts there; dispatch, expert MLP and combine are
// separate steps so the exchange can overlap other work. "DeepSeek-V3,
// explained", recipe step 8: 64-way expert parallelism.
//
// Per step, on every rank (the exchanges between the steps belong to the
// caller: two all-to-alls with row counts known from send_counts):
//   dispatch (source) : route its own tokens, plan the send rows (rank-major,
//                       token ascending, one row per (token, rank) that holds
//                       one of its experts), quantise x 1x128 once into the
//                       send rows and into its shared-expert GEMM rows
//   shared   (source) : the shared expert on its own tokens, bf16 rows
//   experts  (dest)   : received rows -> expert-major GEMM rows of its local
//                       experts -> grouped FP8 up/down GEMMs (bf16 expert
//                       outputs) -> per received row, the gate-weighted sum
//                       over its local experts (fp32, ascending expert id)
//   combine  (source) : y_t = shared_t + sum over ranks (ascending) of the
//                       returned partial sums, rounded once to bf16
// Every slot and row is fixed by the data, so results do not depend on timing.
//
// Two ways to move the rows. All-to-all mode: dispatch fills a local send
// buffer (destination-major) and the caller exchanges it, and later the
// partial sums, with all-to-alls. Peer mode: dispatch stores each row straight
// into its destination's receive buffer (one segment of T_cap rows per
// source) and the reduction stores each partial sum straight into its
// source's return buffer, through device pointers to the other ranks' memory;
// the caller only places a barrier after each of the two phases. Both modes
// use the same plan, the same packed rows and the same sums, so they give the
// same bits.
#include "block_scan.cuh"
#include "host_util.h"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kMaxRanks = 16;
constexpr int kMaxK = 16;


bool ep_ok(const moe_shape& sh, int W) {
  if (!shape_ok(sh) || W < 1 || W > kMaxRanks || sh.N % W != 0) return false;
  const int El = sh.N / W;
  return El >= 16 && El % 16 == 0;
}

// Bytes of one packed dispatch row: codes [H] u8, scales [H/128] f32, local
// expert ids [K] i32 (-1: not on this rank), gates [K] f32; 16-byte multiple.
int64_t row_bytes_of(const moe_shape& sh) {
  return round_up((int64_t)sh.H + 4 * (sh.H / kTile) + 8 * (int64_t)sh.K, 16);
}
__host__ __device__ inline int64_t meta_offset(int H) { return (int64_t)H + 4 * (int64_t)(H / kTile); }

struct SourceLayout {
  int64_t rows;  // shared-expert GEMM rows (T rounded up to 128)
  size_t status, counts, topk_ids, topk_gates, logits, gate_split, send_slot, grp, plan, dest_off;
  size_t send_counts;
  size_t a_q, a_s, h_q, h_s, y_shared, splitk, total;
};

SourceLayout source_layout(const moe_shape& sh, int W) {
  const int64_t T = sh.T, H = sh.H, N = sh.N, K = sh.K, I = sh.I;
  SourceLayout L{};
  L.rows = round_up(T, kTile);
  Carver carve;
  auto take = [&](size_t bytes) { return carve.take(bytes); };
  L.status = take(16);
  L.counts = take(N * 4);
  L.topk_ids = take((size_t)(T * K) * 4);
  L.topk_gates = take((size_t)(T * K) * 4);
  L.logits = take((size_t)(T * N) * 4);
  L.gate_split = take(router_split_bytes((int)N, (int)H));
  L.send_slot = take((size_t)(T * W) * 4);
  L.grp = take(2 * 4);
  L.plan = take((size_t)2 * ((T + 1023) / 1024) * W * 4);  // per-chunk rows and pairs
  L.dest_off = take((size_t)W * 4);
  L.send_counts = take((size_t)W * 2 * 4);
  L.a_q = take((size_t)(L.rows * H));
  L.a_s = take((size_t)(L.rows * (H / kTile)) * 4);
  L.h_q = take((size_t)(L.rows * I));
  L.h_s = take((size_t)(L.rows * (I / kTile)) * 4);
  L.y_shared = take((size_t)(L.rows * H) * 2);
  // the router's partial logits, so that the dispatch routes the rank's
  // tokens exactly as the one-GPU layer does
  L.splitk = take(router_splitk_bytes(T, (int)N, (int)H));
  L.total = carve.off;
  return L;
}

struct ExpertLayout {
  int64_t routed_cap;
  size_t status, counts, offsets, group_rows, row_start, ids, gates, token_row, row_token;
  size_t a_q, a_s, h_q, h_s, y_rows, perm_scratch, total;
};

ExpertLayout expert_layout(const moe_shape& sh, int W, int64_t R, int64_t pairs) {
  const int64_t El = sh.N / W, H = sh.H, K = sh.K, I = sh.I;
  ExpertLayout L{};
  L.routed_cap = round_up(pairs + El * (kTile - 1), kTile);
  Carver carve;
  auto take = [&](size_t bytes) { return carve.take(bytes); };
  L.status = take(16);
  L.counts = take(El * 4);
  L.offsets = take((El + 1) * 4);
  L.group_rows = take((El + 1) * 4);
  L.row_start = take((El + 1) * 4);
  L.ids = take((size_t)(R * K) * 4);
  L.gates = take((size_t)(R * K) * 4);
  L.token_row = take((size_t)(R * K) * 4);
  L.row_token = take((size_t)L.routed_cap * 4);
  L.a_q = take((size_t)L.routed_cap * H);
  L.a_s = take((size_t)L.routed_cap * (H / kTile) * 4);
  L.h_q = take((size_t)L.routed_cap * I);
  L.h_s = take((size_t)L.routed_cap * (I / kTile) * 4);
  L.y_rows = take((size_t)L.routed_cap * H * 2);
  L.perm_scratch = take(permute_scratch_bytes(R, (int)El));
  L.total = carve.off;
  return L;
}

// Sum of one int per thread over the block; red: shared int[32].
MOE_DEV int block_sum(int v, int* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  int r = 0;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) r += red[i];
  __syncthreads();
  return r;
}

// Where the rows of one source go. Row `local` (0-based among the rows for
// destination d, tokens ascending) lives
//   all-to-all mode: in this rank's send buffer at row dest_off[d] + local
//                    (destination-major; send_cap rows);
//   peer mode:       in rank d's receive buffer at row peer_row0 + local,
//                    written directly over NVLink (peer_row0 = this rank's
//                    segment, rank * T_cap).
struct SendRows {
  uint8_t* send;
  int64_t send_cap;
  uint8_t* const* peer;  // device array [W] of receive buffers; null: all-to-all mode
  int64_t peer_row0;
  int64_t row_bytes;
};

// Dispatch plan, in chunks of kPlanChunk tokens (one thread per token).
// ep_count_kernel, one CTA per chunk: per destination rank d, the chunk's
// tokens bound for d (rows) and its (token, slot) pairs for d.
// ep_slot_kernel, one CTA per (chunk, d): the chunk's first row for d is d's
// rows in earlier chunks; a block scan numbers the chunk's tokens for d in
// token order, and each row gets its local ids and gates. Positions come from
// scans only, never from atomics.
constexpr int kPlanChunk = 1024;

__global__ void __launch_bounds__(kPlanChunk) ep_count_kernel(
    const int32_t* __restrict__ ids, int T, int K, int N, int W, int32_t* __restrict__ chunk_rows,
    int32_t* __restrict__ chunk_pairs, uint32_t* __restrict__ status) {
  __shared__ int red[32];
  const int c = blockIdx.x;
  const int t = c * kPlanChunk + threadIdx.x;
  const int El = N / W;
  uint32_t mask = 0;
  int np[kMaxRanks];
#pragma unroll
  for (int d = 0; d < kMaxRanks; ++d) np[d] = 0;
  if (t < T) {
    for (int k = 0; k < K; ++k) {
      const int e = __ldg(ids + (int64_t)t * K + k);
      if (e < 0 || e >= N) {
        flag_status(status, kStatusBounds);
        continue;
      }
      const int r = e / El;
      mask |= 1u << r;
#pragma unroll
      for (int d = 0; d < kMaxRanks; ++d) np[d] += (r == d);
    }
  }
#pragma unroll
  for (int d = 0; d < kMaxRanks; ++d) {
    if (d < W) {  // the same for the whole block, so the barriers inside are safe
      const int rows = __syncthreads_count((mask >> d) & 1u);
      const int pairs = block_sum(np[d], red);
      if (threadIdx.x == 0) {
        chunk_rows[c * W + d] = rows;
        chunk_pairs[c * W + d] = pairs;
      }
    }
  }
}

// Also writes, from CTA (0, d): dest_off[d] (the rows of lower destinations),
// send_counts[2d] and [2d+1] (rows and pairs for d), and in peer mode d's
// count of rows from this rank, peer_counts[d][rank].
__global__ void __launch_bounds__(kPlanChunk) ep_slot_kernel(
    const int32_t* __restrict__ ids, const float* __restrict__ gates, int T, int K, int N, int W,
    int H, int rank, int n_chunks, const int32_t* __restrict__ chunk_rows,
    const int32_t* __restrict__ chunk_pairs, SendRows dst, int32_t* const* peer_counts,
    int32_t* __restrict__ send_slot, int32_t* __restrict__ dest_off,
    int32_t* __restrict__ send_counts, int32_t* __restrict__ grp, uint32_t* __restrict__ status) {
  __shared__ int sums[33];
  __shared__ int64_t s_before;  // rows of lower destinations
  __shared__ int64_t s_local;   // d's rows in earlier chunks
  const int c = blockIdx.x, d = blockIdx.y;
  const int El = N / W;
  if (threadIdx.x == 0) {
    int64_t before = 0, local = 0;
    for (int cc = 0; cc < n_chunks; ++cc)
      for (int dd = 0; dd < d; ++dd) before += chunk_rows[cc * W + dd];
    for (int cc = 0; cc < c; ++cc) local += chunk_rows[cc * W + d];
    s_before = before;
    s_local = local;
    if (c == 0) {
      int rows = 0, pairs = 0;
      for (int cc = 0; cc < n_chunks; ++cc) {
        rows += chunk_rows[cc * W + d];
        pairs += chunk_pairs[cc * W + d];
      }
      dest_off[d] = (int32_t)before;
      send_counts[2 * d] = rows;
      send_counts[2 * d + 1] = pairs;
      if (dst.peer != nullptr) {
        peer_counts[d][rank] = rows;
        __threadfence_system();
      }
      if (d == 0) {  // the shared expert's single GEMM group: rows [0, T)
        grp[0] = T;
        grp[1] = 0;
      }
    }
  }
  const int t = c * kPlanChunk + threadIdx.x;
  bool sel = false;
  if (t < T) {
    for (int k = 0; k < K; ++k) {
      const int e = __ldg(ids + (int64_t)t * K + k);
      sel |= (e >= 0 && e < N && e / El == d);
    }
  }
  int total;
  const int pos = block_scan_flag(sel, sums, &total);  // synchronises: s_before/s_local visible
  if (threadIdx.x == 0 && total != chunk_rows[c * W + d]) flag_status(status, kStatusBounds);
  if (t >= T) return;
  int32_t slot = -1;
  if (sel) {
    const int64_t local = s_local + pos;
    uint8_t* row = nullptr;
    if (dst.peer != nullptr) {
      row = dst.peer[d] + (dst.peer_row0 + local) * dst.row_bytes;
    } else if (s_before + local < dst.send_cap) {
      row = dst.send + (s_before + local) * dst.row_bytes;
    } else {
      flag_status(status, kStatusBounds);
    }
    if (row != nullptr) {
      slot = (int32_t)local;
      uint8_t* meta = row + meta_offset(H);
      int32_t* lid = reinterpret_cast<int32_t*>(meta);
      float* g = reinterpret_cast<float*>(meta) + K;
      for (int k = 0; k < K; ++k) {
        const int e = __ldg(ids + (int64_t)t * K + k);
        const bool here = e >= 0 && e < N && e / El == d;
        lid[k] = here ? e - d * El : -1;
        g[k] = here ? __ldg(gates + (int64_t)t * K + k) : 0.0f;
      }
      if (dst.peer != nullptr) __threadfence_system();
    }
  }
  send_slot[(int64_t)t * W + d] = slot;
}

// x -> 1x128 E4M3 codes and scales, written to the token's shared-expert row
// t and to its rows for each destination d with send_slot[t, d] >= 0 (at
// most W <= 16). 8 threads per tile, 16 elements each; lane k of a tile's 8
// threads holds the slots of ranks k and k + 8.
__global__ void __launch_bounds__(256) ep_pack_kernel(const uint4* __restrict__ x, int T, int H,
                                                      int W, const int32_t* __restrict__ send_slot,
                                                      const int32_t* __restrict__ dest_off,
                                                      SendRows dst, uint8_t* __restrict__ a_q,
                                                      float* __restrict__ a_s) {
  const int sub = threadIdx.x & 7;
  const int tiles_per_row = H / kTile;
  const int64_t n_tiles = (int64_t)T * tiles_per_row;
  // the whole CTA iterates together so that every shuffle is warp-convergent
  for (int64_t base = (int64_t)blockIdx.x * 32; base < n_tiles; base += (int64_t)gridDim.x * 32) {
    const int64_t tile = base + (threadIdx.x >> 3);
    const bool live = tile < n_tiles;
    const int64_t t = live ? tile / tiles_per_row : 0;
    const int c = live ? (int)(tile - t * tiles_per_row) : 0;
    const uint4 v0 = live ? __ldcs(x + tile * 16 + 2 * sub) : make_uint4(0, 0, 0, 0);
    const uint4 v1 = live ? __ldcs(x + tile * 16 + 2 * sub + 1) : make_uint4(0, 0, 0, 0);
    const int slot_a = (live && sub < W) ? __ldg(send_slot + t * W + sub) : -1;
    const int slot_b = (live && sub + 8 < W) ? __ldg(send_slot + t * W + sub + 8) : -1;
    float f[16] = {bf16_lo(v0.x), bf16_hi(v0.x), bf16_lo(v0.y), bf16_hi(v0.y),
                   bf16_lo(v0.z), bf16_hi(v0.z), bf16_lo(v0.w), bf16_hi(v0.w),
                   bf16_lo(v1.x), bf16_hi(v1.x), bf16_lo(v1.y), bf16_hi(v1.y),
                   bf16_lo(v1.z), bf16_hi(v1.z), bf16_lo(v1.w), bf16_hi(v1.w)};
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = tile_scale(amax);
    uint4 out;
    out.x = e4m3x4(__fmul_rn(f[0], s), __fmul_rn(f[1], s), __fmul_rn(f[2], s), __fmul_rn(f[3], s));
    out.y = e4m3x4(__fmul_rn(f[4], s), __fmul_rn(f[5], s), __fmul_rn(f[6], s), __fmul_rn(f[7], s));
    out.z = e4m3x4(__fmul_rn(f[8], s), __fmul_rn(f[9], s), __fmul_rn(f[10], s), __fmul_rn(f[11], s));
    out.w = e4m3x4(__fmul_rn(f[12], s), __fmul_rn(f[13], s), __fmul_rn(f[14], s), __fmul_rn(f[15], s));
    if (live) {
      reinterpret_cast<uint4*>(a_q + t * H + (int64_t)c * kTile)[sub] = out;
      if (sub == 0) a_s[t * tiles_per_row + c] = s;
    }
    for (int d = 0; d < W; ++d) {
      const int sa = __shfl_sync(0xffffffffu, slot_a, d & 7, 8);
      const int sb = __shfl_sync(0xffffffffu, slot_b, d & 7, 8);
      const int local = d < 8 ? sa : sb;
      if (live && local >= 0) {
        uint8_t* row = dst.peer != nullptr
                           ? dst.peer[d] + (dst.peer_row0 + local) * dst.row_bytes
                           : dst.send + ((int64_t)__ldg(dest_off + d) + local) * dst.row_bytes;
        reinterpret_cast<uint4*>(row + (int64_t)c * kTile)[sub] = out;
        if (sub == 0) reinterpret_cast<float*>(row + H)[c] = s;
      }
    }
  }
  if (dst.peer != nullptr) __threadfence_system();
}

// Received rows: local ids and gates into dense [R, K] arrays, counts per
// local expert (counts zero on entry). With seg_rows > 0 the R rows are W
// segments of seg_rows rows, one per source, of which the first
// seg_counts[s] are valid; the other rows get no slot (id -1).
__global__ void __launch_bounds__(256) ep_recv_index_kernel(
    const uint8_t* __restrict__ recv, int64_t R, int K, int H, int64_t row_bytes, int El,
    int64_t seg_rows, const int32_t* __restrict__ seg_counts, int32_t* __restrict__ ids,
    float* __restrict__ gates, int32_t* __restrict__ counts, uint32_t* __restrict__ status) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= R * K) return;
  const int64_t j = i / K;
  const int k = (int)(i - j * K);
  if (seg_rows > 0) {
    const int64_t s = j / seg_rows;
    const int64_t n = __ldg(seg_counts + s);
    if (n < 0 || n > seg_rows) flag_status(status, kStatusBounds);
    if (j - s * seg_rows >= n) {
      ids[i] = -1;
      gates[i] = 0.0f;
      return;
    }
  }
  const uint8_t* meta = recv + j * row_bytes + meta_offset(H);
  int lid = reinterpret_cast<const int32_t*>(meta)[k];
  const float g = reinterpret_cast<const float*>(meta)[K + k];
  if (lid < -1 || lid >= El) {
    flag_status(status, kStatusBounds);
    lid = -1;
  }
  ids[i] = lid;
  gates[i] = g;
  if (lid >= 0) atomicAdd(counts + lid, 1);
}

// Codes and scales of received row j copied to its GEMM rows token_row[j, k]
// (slots without a row are skipped; rows without any are not read). 8
// threads per 128-byte tile.
__global__ void __launch_bounds__(256) ep_gather_rows_kernel(
    const uint8_t* __restrict__ recv, int64_t R, int H, int K, int64_t row_bytes,
    const int32_t* __restrict__ token_row, int64_t routed_cap, uint8_t* __restrict__ a_q,
    float* __restrict__ a_s, uint32_t* __restrict__ status) {
  const int sub = threadIdx.x & 7;
  const int tiles_per_row = H / kTile;
  const int64_t n_tiles = R * tiles_per_row;
  for (int64_t base = (int64_t)blockIdx.x * 32; base < n_tiles; base += (int64_t)gridDim.x * 32) {
    const int64_t tile = base + (threadIdx.x >> 3);
    if (tile >= n_tiles) continue;  // no shuffles below
    const int64_t j = tile / tiles_per_row;
    const int c = (int)(tile - j * tiles_per_row);
    bool any = false;
    for (int k = 0; k < K; ++k) any |= __ldg(token_row + j * K + k) >= 0;
    if (!any) continue;
    const uint8_t* row = recv + j * row_bytes;
    const uint4 v = reinterpret_cast<const uint4*>(row + (int64_t)c * kTile)[sub];
    const float s = reinterpret_cast<const float*>(row + H)[c];
    for (int k = 0; k < K; ++k) {
      const int64_t r = __ldg(token_row + j * K + k);
      if (r < 0) continue;
      if (r >= routed_cap) {
        if (sub == 0) flag_status(status, kStatusBounds);
        continue;
      }
      reinterpret_cast<uint4*>(a_q + r * H + (int64_t)c * kTile)[sub] = v;
      if (sub == 0) a_s[r * tiles_per_row + c] = s;
    }
  }
}

// 8 consecutive bf16 row elements as fp32 (streamed: each is read once)
MOE_DEV void load8_bf16(const __nv_bfloat16* p, int64_t c, float (&v)[8]) {
  const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p) + c);
  v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
  v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}

// Per received row: the sum over its local slots, by ascending expert id, of
// g * Y[row], fp32 (the rank's share of the token's combine). Written to
// out[j] (all-to-all mode), or in peer mode straight into the source's
// return buffer: row j = s seg_rows + i goes to peer_ret[s] at row
// rank * seg_rows + i; rows without a slot are not written. Each thread
// takes 8 columns at a time and puts up to four rows' loads in flight
// before their adds, which keep the ascending order.
__global__ void __launch_bounds__(128) ep_reduce_kernel(
    const __nv_bfloat16* __restrict__ y_rows, const int32_t* __restrict__ ids,
    const float* __restrict__ gates, const int32_t* __restrict__ token_row, int H, int K,
    int64_t routed_cap, float* __restrict__ out, float* const* peer_ret, int rank,
    int64_t seg_rows, uint32_t* __restrict__ status) {
  __shared__ int64_t s_row[kMaxK];
  __shared__ float s_gate[kMaxK];
  __shared__ int s_n;
  const int64_t j = blockIdx.x;
  // slot k (thread k) goes to position = the number of the row's local slots
  // with a lower expert id (a token's experts are distinct); slots of other
  // ranks' experts (id < 0) are skipped, rows out of range dropped and flagged
  if (threadIdx.x < K) {
    const int k = threadIdx.x;
    const int e = ids[j * K + k];
    int64_t r = -1;
    float g = 0.0f;
    bool ok = false;
    if (e >= 0) {
      r = token_row[j * K + k];
      ok = r >= 0 && r < routed_cap;
      if (!ok) flag_status(status, kStatusBounds);
      g = gates[j * K + k];
    }
    const unsigned mask = (1u << K) - 1u;
    int pos = 0;
    for (int i = 0; i < K; ++i) {
      const int ei = __shfl_sync(mask, e, i);
      const bool oki = __shfl_sync(mask, ok, i);
      pos += (oki && ei < e) ? 1 : 0;
    }
    const int n_ok = __popc(__ballot_sync(mask, ok));
    if (ok) {
      s_row[pos] = r * H;
      s_gate[pos] = g;
    }
    if (k == 0) s_n = n_ok;
  }
  __syncthreads();
  const int n = s_n;
  float* dst_row = out + j * H;
  if (peer_ret != nullptr) {
    if (n == 0) return;  // a row without a slot: an unused row of its segment
    const int64_t s = j / seg_rows;
    dst_row = peer_ret[s] + ((int64_t)rank * seg_rows + (j - s * seg_rows)) * H;
  }
  float4* o = reinterpret_cast<float4*>(dst_row);
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    float acc[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    int k = 0;
    for (; k + 4 <= n; k += 4) {
      float f[4][8];
#pragma unroll
      for (int q = 0; q < 4; ++q) load8_bf16(y_rows + s_row[k + q], c, f[q]);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float g = s_gate[k + q];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(g, f[q][i], acc[i]);
      }
    }
    for (; k < n; ++k) {
      float f[8];
      load8_bf16(y_rows + s_row[k], c, f);
      const float g = s_gate[k];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(g, f[i], acc[i]);
    }
    o[2 * c] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    o[2 * c + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  if (peer_ret != nullptr) __threadfence_system();
}

// y_t = shared_t + the returned partial sums of t's rows, ranks ascending,
// fp32, one rounding to bf16. The row for (t, d) with local position l is
// ret[dest_off[d] + l] (all-to-all mode) or ret[d seg_rows + l] (peer mode,
// seg_rows > 0).
__global__ void __launch_bounds__(128) ep_combine_kernel(
    const __nv_bfloat16* __restrict__ y_shared, const float* __restrict__ ret,
    const int32_t* __restrict__ send_slot, const int32_t* __restrict__ dest_off, int H, int W,
    int64_t ret_rows, int64_t seg_rows, __nv_bfloat16* __restrict__ y,
    uint32_t* __restrict__ status) {
  __shared__ int64_t s_slot[kMaxRanks];
  __shared__ int s_n;
  const int64_t t = blockIdx.x;
  if (threadIdx.x == 0) {
    int n = 0;
    for (int d = 0; d < W; ++d) {
      const int64_t local = send_slot[t * W + d];
      if (local < 0) continue;
      const int64_t r = seg_rows > 0 ? d * seg_rows + local : (int64_t)dest_off[d] + local;
      if (r >= ret_rows || (seg_rows > 0 && local >= seg_rows)) {
        flag_status(status, kStatusBounds);
        continue;
      }
      s_slot[n++] = r;
    }
    s_n = n;
  }
  __syncthreads();
  const int n = s_n;
  const uint4* ys = reinterpret_cast<const uint4*>(y_shared + t * H);
  uint4* out = reinterpret_cast<uint4*>(y + t * H);
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    const uint4 v = __ldcs(ys + c);
    float acc[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                    bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    for (int i = 0; i < n; ++i) {
      const float4* p = reinterpret_cast<const float4*>(ret + s_slot[i] * H);
      const float4 u0 = __ldcs(p + 2 * c), u1 = __ldcs(p + 2 * c + 1);
      acc[0] += u0.x;
      acc[1] += u0.y;
      acc[2] += u0.z;
      acc[3] += u0.w;
      acc[4] += u1.x;
      acc[5] += u1.y;
      acc[6] += u1.z;
      acc[7] += u1.w;
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    out[c] = o;
  }
}

unsigned tile_grid(int64_t n_tiles) {
  int64_t blocks = (n_tiles + 31) / 32;
  const int64_t cap = (int64_t)moe_device_sm_count() * 8;
  if (cap > 0 && blocks > cap) blocks = cap;
  return (unsigned)(blocks > 0 ? blocks : 1);
}

// T = 0 in peer mode: this rank sends nothing this step, which its
// destinations learn from a zero count.
__global__ void ep_zero_counts_kernel(int32_t* const* peer_counts, int W, int rank) {
  const int d = threadIdx.x;
  if (d < W) peer_counts[d][rank] = 0;
  __threadfence_system();
}

int dispatch_impl(const moe_shape& sh, int W, int rank, const float* gate_w,
                  const void* gate_split, const void* x,
                  const float* bias, int32_t* topk_ids_opt, float* topk_gates_opt,
                  int32_t* counts_opt, SendRows dst, int32_t* const* peer_counts,
                  int32_t* send_counts_opt, void* ws, size_t ws_bytes, cudaStream_t s) {
  if (!ws) return MOE_ERR_NULL;
  if (!aligned(ws, 256)) return MOE_ERR_ALIGN;
  const SourceLayout L = source_layout(sh, W);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (!aligned(gate_split, 16)) return MOE_ERR_ALIGN;
  uint32_t* status = at<uint32_t>(ws, L.status);
  int32_t* counts = counts_opt ? counts_opt : at<int32_t>(ws, L.counts);
  int32_t* send_counts = send_counts_opt ? send_counts_opt : at<int32_t>(ws, L.send_counts);
  cudaError_t e = cudaMemsetAsync(status, 0, 4, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(counts, 0, (size_t)sh.N * 4, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(send_counts, 0, (size_t)W * 2 * 4, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (sh.T == 0) {
    if (dst.peer != nullptr) {
      ep_zero_counts_kernel<<<1, 32, 0, s>>>(peer_counts, W, rank);
      e = cudaGetLastError();
    }
    return cuda_status(e);
  }
  if (!gate_w || !x || !bias) return MOE_ERR_NULL;
  if (!aligned(x, 16) || !aligned(gate_w, 16)) return MOE_ERR_ALIGN;
  const int sms = moe_device_sm_count();
  int32_t* ids = topk_ids_opt ? topk_ids_opt : at<int32_t>(ws, L.topk_ids);
  float* gates = topk_gates_opt ? topk_gates_opt : at<float>(ws, L.topk_gates);
  e = launch_router_tc(x, gate_w, bias, sh.T, sh.H, sh.N, sh.K, sh.G, sh.M,
                       at<__nv_bfloat16>(ws, L.gate_split), at<float>(ws, L.logits), ids, gates,
                       counts, status, s, sms, static_cast<const __nv_bfloat16*>(gate_split),
                       at<float>(ws, L.splitk),
                       router_splitk_bytes(sh.T, sh.N, sh.H));
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  int32_t* send_slot = at<int32_t>(ws, L.send_slot);
  int32_t* dest_off = at<int32_t>(ws, L.dest_off);
  const int n_chunks = (sh.T + kPlanChunk - 1) / kPlanChunk;
  int32_t* chunk_rows = at<int32_t>(ws, L.plan);
  int32_t* chunk_pairs = chunk_rows + (size_t)n_chunks * W;
  ep_count_kernel<<<n_chunks, kPlanChunk, 0, s>>>(ids, sh.T, sh.K, sh.N, W, chunk_rows,
                                                  chunk_pairs, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  ep_slot_kernel<<<dim3(n_chunks, W), kPlanChunk, 0, s>>>(
      ids, gates, sh.T, sh.K, sh.N, W, sh.H, rank, n_chunks, chunk_rows, chunk_pairs, dst,
      peer_counts, send_slot, dest_off, send_counts, at<int32_t>(ws, L.grp), status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  const int64_t n_tiles = (int64_t)sh.T * (sh.H / kTile);
  ep_pack_kernel<<<tile_grid(n_tiles), 256, 0, s>>>(reinterpret_cast<const uint4*>(x), sh.T, sh.H,
                                                    W, send_slot, dest_off, dst,
                                                    at<uint8_t>(ws, L.a_q), at<float>(ws, L.a_s));
  return cuda_status(cudaGetLastError());
}

// The receiver's steps for R rows (seg_rows > 0: W source segments of
// seg_rows rows with seg_counts valid each; pairs < 0: not checked).
int experts_impl(const moe_shape& sh, int W, const moe_weights* w_local, const uint8_t* recv,
                 int64_t R, int64_t pairs, int64_t pairs_cap, int64_t seg_rows,
                 const int32_t* seg_counts, float* out, float* const* peer_ret, int rank,
                 void* ws, size_t ws_bytes, cudaStream_t s) {
  if (!ws) return MOE_ERR_NULL;
  if (!aligned(ws, 256)) return MOE_ERR_ALIGN;
  const ExpertLayout L = expert_layout(sh, W, R, pairs_cap);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  uint32_t* status = at<uint32_t>(ws, L.status);
  cudaError_t e = cudaMemsetAsync(status, 0, 4, s);
  if (R == 0 || e != cudaSuccess) return cuda_status(e);
  if (!w_local || !w_local->w13 || !w_local->s13 || !w_local->w2 || !w_local->s2 || !recv)
    return MOE_ERR_NULL;
  if (!aligned(w_local->w13, 16) || !aligned(w_local->w2, 16) || !aligned(recv, 16) ||
      !aligned(out, 16))
    return MOE_ERR_ALIGN;
  const int sms = moe_device_sm_count();
  const int El = sh.N / W;
  const int64_t rb = row_bytes_of(sh);
  int32_t* counts = at<int32_t>(ws, L.counts);
  int32_t* ids = at<int32_t>(ws, L.ids);
  float* gates = at<float>(ws, L.gates);
  int32_t* token_row = at<int32_t>(ws, L.token_row);
  e = cudaMemsetAsync(counts, 0, (size_t)El * 4, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(token_row, 0xFF, (size_t)(R * sh.K) * 4, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  const int64_t n_idx = R * sh.K;
  ep_recv_index_kernel<<<(unsigned)((n_idx + 255) / 256), 256, 0, s>>>(
      recv, R, sh.K, sh.H, rb, El, seg_rows, seg_counts, ids, gates, counts, status);
  e = cudaGetLastError();
  if (e == cudaSuccess)
    e = launch_permute(ids, counts, false, (int)R, El, sh.K, pairs, L.routed_cap,
                       at<int32_t>(ws, L.perm_scratch), at<int32_t>(ws, L.offsets),
                       at<int32_t>(ws, L.group_rows), at<int32_t>(ws, L.row_start),
                       at<int32_t>(ws, L.row_token), token_row, status, s, sms);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  const int64_t n_tiles = R * (sh.H / kTile);
  ep_gather_rows_kernel<<<tile_grid(n_tiles), 256, 0, s>>>(recv, R, sh.H, sh.K, rb, token_row,
                                                           L.routed_cap, at<uint8_t>(ws, L.a_q),
                                                           at<float>(ws, L.a_s), status);
  e = cudaGetLastError();
  GroupedGemm gg{sh.H, sh.I, El, at<int32_t>(ws, L.group_rows), at<int32_t>(ws, L.row_start),
                 L.routed_cap, status};
  if (e == cudaSuccess)
    e = launch_expert_up(gg, at<uint8_t>(ws, L.a_q), at<float>(ws, L.a_s), w_local->w13,
                         w_local->s13, at<uint8_t>(ws, L.h_q), at<float>(ws, L.h_s), s, sms);
  if (e == cudaSuccess)
    e = launch_expert_down_bf16(gg, at<uint8_t>(ws, L.h_q), at<float>(ws, L.h_s), w_local->w2,
                                w_local->s2, at<__nv_bfloat16>(ws, L.y_rows), s, sms);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  ep_reduce_kernel<<<(unsigned)R, 128, 0, s>>>(at<__nv_bfloat16>(ws, L.y_rows), ids, gates, token_row,
                                               sh.H, sh.K, L.routed_cap, out, peer_ret, rank,
                                               seg_rows, status);
  return cuda_status(cudaGetLastError());
}

int combine_impl(const moe_shape& sh, int W, const float* ret, int64_t ret_rows, int64_t seg_rows,
                 void* ws, size_t ws_bytes, void* y, cudaStream_t s) {
  if (!ws) return MOE_ERR_NULL;
  if (!aligned(ws, 256)) return MOE_ERR_ALIGN;
  const SourceLayout L = source_layout(sh, W);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (sh.T == 0) return MOE_OK;
  if (!y || (ret_rows > 0 && !ret)) return MOE_ERR_NULL;
  if (!aligned(y, 16) || !aligned(ret, 16)) return MOE_ERR_ALIGN;
  ep_combine_kernel<<<(unsigned)sh.T, 128, 0, s>>>(
      at<__nv_bfloat16>(ws, L.y_shared), ret, at<int32_t>(ws, L.send_slot), at<int32_t>(ws, L.dest_off),
      sh.H, W, ret_rows, seg_rows, static_cast<__nv_bfloat16*>(y), at<uint32_t>(ws, L.status));
  return cuda_status(cudaGetLastError());
}

// Peer mode sizes: W segments of T_cap rows, each row with at most min(K, El) slots.
bool peer_ok(const moe_shape& sh, int W, int rank, int64_t T_cap) {
  return ep_ok(sh, W) && rank >= 0 && rank < W && T_cap >= 1 && sh.T <= T_cap &&
         (int64_t)W * T_cap * sh.K < (1ll << 31);
}
int64_t peer_pairs_cap(const moe_shape& sh, int W, int64_t T_cap) {
  return (int64_t)W * T_cap * std::min<int64_t>(sh.K, sh.N / W);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

int64_t moe_ep_row_bytes(moe_shape sh) { return shape_ok(sh) ? row_bytes_of(sh) : 0; }

size_t moe_ep_dispatch_workspace_size(moe_shape sh, int32_t W) {
  return ep_ok(sh, W) ? source_layout(sh, W).total : 0;
}

size_t moe_ep_expert_workspace_size(moe_shape sh, int32_t W, int64_t R, int64_t pairs) {
  if (!ep_ok(sh, W) || R < 0 || pairs < 0 || pairs > R * sh.K || R * sh.K >= (1ll << 31))
    return 0;
  return expert_layout(sh, W, R, pairs).total;
}

int moe_ep_dispatch(moe_shape sh, int32_t W, const float* gate_w, const void* gate_split_opt,
                    const void* x, const float* bias,
                    int32_t* topk_ids_opt, float* topk_gates_opt, int32_t* counts_opt,
                    uint8_t* send, int64_t send_cap, int32_t* send_counts, void* ws,
                    size_t ws_bytes, void* stream) {
  if (!ep_ok(sh, W) || send_cap < 0 || send_cap >= (1ll << 31)) return MOE_ERR_SHAPE;
  if (!send_counts) return MOE_ERR_NULL;
  if (sh.T > 0 && !send) return MOE_ERR_NULL;
  if (!aligned(send, 16)) return MOE_ERR_ALIGN;
  SendRows dst{send, send_cap, nullptr, 0, row_bytes_of(sh)};
  return dispatch_impl(sh, W, 0, gate_w, gate_split_opt, x, bias, topk_ids_opt, topk_gates_opt,
                       counts_opt, dst, nullptr, send_counts, ws, ws_bytes,
                       static_cast<cudaStream_t>(stream));
}

int moe_ep_shared(moe_shape sh, int32_t W, const moe_weights* w_local, void* ws, size_t ws_bytes,
                  void* stream) {
  if (!ep_ok(sh, W)) return MOE_ERR_SHAPE;
  if (!ws) return MOE_ERR_NULL;
  if (!aligned(ws, 256)) return MOE_ERR_ALIGN;
  const SourceLayout L = source_layout(sh, W);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (sh.T == 0) return MOE_OK;
  if (!w_local || !w_local->w13 || !w_local->s13 || !w_local->w2 || !w_local->s2)
    return MOE_ERR_NULL;
  if (!aligned(w_local->w13, 16) || !aligned(w_local->w2, 16)) return MOE_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = moe_device_sm_count();
  const int64_t El = sh.N / W, H = sh.H, I = sh.I;
  // the shared expert is the last of the rank's El + 1 weight sets
  const uint8_t* w13 = w_local->w13 + El * 2 * I * H;
  const float* s13 = w_local->s13 + El * (2 * I / kTile) * (H / kTile);
  const uint8_t* w2 = w_local->w2 + El * H * I;
  const float* s2 = w_local->s2 + El * (H / kTile) * (I / kTile);
  const int32_t* grp = at<int32_t>(ws, L.grp);
  GroupedGemm gg{sh.H, sh.I, 1, grp, grp + 1, L.rows, at<uint32_t>(ws, L.status)};
  cudaError_t e = launch_expert_up(gg, at<uint8_t>(ws, L.a_q), at<float>(ws, L.a_s), w13, s13,
                                   at<uint8_t>(ws, L.h_q), at<float>(ws, L.h_s), s, sms);
  if (e == cudaSuccess)
    e = launch_expert_down_bf16(gg, at<uint8_t>(ws, L.h_q), at<float>(ws, L.h_s), w2, s2,
                                at<__nv_bfloat16>(ws, L.y_shared), s, sms);
  return cuda_status(e);
}

int moe_ep_experts(moe_shape sh, int32_t W, const moe_weights* w_local, const uint8_t* recv,
                   int64_t R, int64_t pairs, float* out, void* ws, size_t ws_bytes,
                   void* stream) {
  if (!ep_ok(sh, W) || R < 0 || pairs < 0 || pairs > R * sh.K || R * sh.K >= (1ll << 31))
    return MOE_ERR_SHAPE;
  if (R > 0 && !out) return MOE_ERR_NULL;
  return experts_impl(sh, W, w_local, recv, R, pairs, pairs, 0, nullptr, out, nullptr, 0, ws,
                      ws_bytes, static_cast<cudaStream_t>(stream));
}

int moe_ep_combine(moe_shape sh, int32_t W, const float* ret, int64_t ret_rows, void* ws,
                   size_t ws_bytes, void* y, void* stream) {
  if (!ep_ok(sh, W) || ret_rows < 0) return MOE_ERR_SHAPE;
  return combine_impl(sh, W, ret, ret_rows, 0, ws, ws_bytes, y, static_cast<cudaStream_t>(stream));
}

size_t moe_ep_peer_expert_workspace_size(moe_shape sh, int32_t W, int32_t T_cap) {
  if (!ep_ok(sh, W) || T_cap < 1 || (int64_t)W * T_cap * sh.K >= (1ll << 31)) return 0;
  return expert_layout(sh, W, (int64_t)W * T_cap, peer_pairs_cap(sh, W, T_cap)).total;
}

int moe_ep_dispatch_peer(moe_shape sh, int32_t W, int32_t rank, int32_t T_cap,
                         const float* gate_w, const void* gate_split_opt, const void* x,
                         const float* bias, int32_t* topk_ids_opt, float* topk_gates_opt,
                         int32_t* counts_opt, uint8_t* const* peer_recv,
                         int32_t* const* peer_counts, int32_t* send_counts_opt, void* ws,
                         size_t ws_bytes, void* stream) {
  if (!peer_ok(sh, W, rank, T_cap)) return MOE_ERR_SHAPE;
  if (!peer_recv || !peer_counts) return MOE_ERR_NULL;
  SendRows dst{nullptr, 0, peer_recv, (int64_t)rank * T_cap, row_bytes_of(sh)};
  return dispatch_impl(sh, W, rank, gate_w, gate_split_opt, x, bias, topk_ids_opt,
                       topk_gates_opt, counts_opt, dst, peer_counts, send_counts_opt, ws, ws_bytes,
                       static_cast<cudaStream_t>(stream));
}

int moe_ep_experts_peer(moe_shape sh, int32_t W, int32_t rank, int32_t T_cap,
                        const moe_weights* w_local, const uint8_t* recv,
                        const int32_t* recv_counts, float* const* peer_ret, void* ws,
                        size_t ws_bytes, void* stream) {
  if (!peer_ok(sh, W, rank, T_cap)) return MOE_ERR_SHAPE;
  if (!recv_counts || !peer_ret) return MOE_ERR_NULL;
  const int64_t R = (int64_t)W * T_cap;
  return experts_impl(sh, W, w_local, recv, R, -1, peer_pairs_cap(sh, W, T_cap), T_cap,
                      recv_counts, nullptr, peer_ret, rank, ws, ws_bytes,
                      static_cast<cudaStream_t>(stream));
}

int moe_ep_combine_peer(moe_shape sh, int32_t W, int32_t T_cap, const float* ret, void* ws,
                        size_t ws_bytes, void* y, void* stream) {
  if (!ep_ok(sh, W) || T_cap < 1 || sh.T > T_cap) return MOE_ERR_SHAPE;
  return combine_impl(sh, W, ret, (int64_t)W * T_cap, T_cap, ws, ws_bytes, y,
                      static_cast<cudaStream_t>(stream));
}

}  // extern "C"
