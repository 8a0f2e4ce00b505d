// Internal interface between the C-ABI layer (e4b_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/e4b.h"

namespace e4b {

// Tokens handled by one CTA of the routing kernels.
constexpr int kRouteTokensPerBlock = 64;
// Header ints at the front of the tile list: [0] = m-tiles, [1] = rows used.
constexpr int kTileHeader = 8;

// Tile list layout (int32): header ([0] 128-row m-tiles, [1] rows used,
// [2] 256-row m-units), then (expert, first row) per 128-row m-tile, then the
// experts ordered by descending token count, then (expert, first row, rows)
// per 256-row m-unit (two consecutive m-tiles of one expert; the last unit of
// an expert may hold 128 rows).
inline int64_t mtiles_cap(int64_t N, int E) { return (N + 127) / 128 + E; }
inline int64_t order_offset(int64_t mt_cap) { return kTileHeader + 2 * mt_cap; }
inline int64_t munits_offset(int64_t mt_cap, int E) { return kTileHeader + 2 * mt_cap + E; }
// Then (expert, first row, slots) per 32-slot tile of the weight-streaming
// forward used for decode-sized batches ([3] = their count).
inline int64_t stiles_offset(int64_t mt_cap, int E) { return munits_offset(mt_cap, E) + 3 * mt_cap; }
inline int64_t tiles_cap(int64_t N, int E) { return stiles_offset(mtiles_cap(N, E), E) + 12 * mtiles_cap(N, E); }
// Forward path choice: the weight-streaming kernel when the batch routes few
// slots per expert (decode-sized), the 2-SM training tiles otherwise.
inline bool use_streaming_forward(int64_t N, int E) { return N <= 16 * (int64_t)E; }
inline int64_t rows_cap(int64_t N, int E) { return ((N + (int64_t)E * 127) + 127) / 128 * 128; }
// Upper bound of the 32-slot streaming tiles of N slots over E experts.
inline int64_t stiles_cap(int64_t N, int E) { return (N + 31) / 32 + E; }

// Device counters of the one-launch serving forward (int32, in the workspace after
// the error word, zeroed by the routing launch before it): slots prepped per
// expert [E], gate_up units done per slot tile [st_cap], LoRA-down projection
// done per slot tile [st_cap], slots of a token whose y_perm piece is written
// [T * ceil(H/128)].
inline int64_t serve_cnt_a_offset(int E) { return E; }
inline int64_t serve_pd_offset(int E, int64_t st_cap) { return E + st_cap; }
inline int64_t serve_comb_offset(int E, int64_t st_cap) { return E + 2 * st_cap; }
inline int64_t serve_claim_offset(int E, int64_t st_cap, int T, int H) {
  return E + 2 * st_cap + (int64_t)T * ((H + 127) / 128);
}
// ... and the unit-claim counter.
inline int64_t serve_counters(int E, int64_t st_cap, int T, int H) { return serve_claim_offset(E, st_cap, T, H) + 1; }
// Then (256-byte aligned) float32 shares of the LoRA down projection, one [32, r]
// block per (slot tile, 64-feature gate/up tile).
inline int64_t serve_part_floats(int64_t st_cap, int I, int r) { return st_cap * (I / 64) * 32 * (int64_t)r; }

struct DeviceError;

// Brackets one kernel launch: counts it and, while the profiler is on,
// records CUDA events around it on `stream`.
class LaunchScope {
 public:
  LaunchScope(const char* name, cudaStream_t stream);
  ~LaunchScope();

 private:
  const char* name_;
  cudaStream_t stream_;
  int slot_;
};

// ---- routing (route.cu)
cudaError_t launch_route(const float* logits, const uint16_t* x, int T, int E, int H, int k,
                         int32_t* topk_ids, float* topk_w, int32_t* counts, int32_t* offsets,
                         int32_t* row_of_slot, int32_t* slot_of_row, int32_t* tiles, int64_t mt_cap,
                         uint16_t* x_perm, int64_t rows_cap, int32_t* scratch, int num_sms,
                         cudaStream_t stream);

// Routing tables for the serving forward (no x gather, no padding markers for
// batches of at most kRouteTokensPerBlock tokens, which take one launch).
// `zero`/`n_zero` (optional): int32 counters that the same launch sets to 0 (the
// one-launch serving forward's counters).
cudaError_t launch_route_serve(const float* logits, int T, int E, int H, int k, int32_t* topk_ids, float* topk_w,
                               int32_t* counts, int32_t* offsets, int32_t* row_of_slot, int32_t* slot_of_row,
                               int32_t* tiles, int64_t mt_cap, int64_t rows_cap, int32_t* scratch, int num_sms,
                               cudaStream_t stream, int32_t* zero = nullptr, int64_t n_zero = 0);
// out[row(f)] = bf16(s * src_row(f) . A[e(f)]^T) per routed slot f on the CUDA cores; src_row is the token's
// row (by_token) or the permuted row; copy_dst (optional) receives the source row at the permuted row.
cudaError_t launch_lora_rows(const uint16_t* src, bool by_token, const int32_t* topk_ids, const int32_t* row_of_slot,
                             int N, int k, int K, const uint16_t* A, int r, float s, uint16_t* copy_dst,
                             uint16_t* out, int num_sms, cudaStream_t stream);

// dst[row] = src[token of row] (optionally scaled by the slot's routing weight), zero for padding rows.
cudaError_t launch_gather_rows(const uint16_t* src, const int32_t* slot_of_row, const int32_t* tiles,
                               const float* scale_w, int H, int k, int64_t rows_cap, uint16_t* dst,
                               int num_sms, cudaStream_t stream);

// out[t] = sum_j (w[t,j] or 1) * src_perm[row(t,j)] in float32, rounded once to bf16.
cudaError_t launch_combine(const uint16_t* src_perm, const int32_t* row_of_slot, const float* topk_w, int T,
                           int k, int H, uint16_t* out, int num_sms, cudaStream_t stream);

cudaError_t launch_router_bwd(const uint16_t* dY, const uint16_t* y_perm, const int32_t* row_of_slot,
                              const int32_t* topk_ids, const float* topk_w, int T, int k, int H, int E,
                              float* d_logits, float* dw, int num_sms, cudaStream_t stream);
cudaError_t launch_nf4_quantize(const uint16_t* w, int64_t n, uint8_t* packed, float* absmax, int num_sms,
                                cudaStream_t stream);
cudaError_t launch_nf4_dequant(const uint8_t* packed, const float* absmax, int64_t n, uint16_t* out,
                               int num_sms, cudaStream_t stream);

cudaError_t launch_watchdog(DeviceError* err, long long timeout_ns, cudaStream_t stream);

// ---- grouped GEMMs (gemm.cu, stream.cu)
enum Nf4Mode { kFwdGateUp = 0, kFwdDown = 1, kDgradDown = 2, kDgradGateUp = 3 };

struct Nf4GemmHost {
  int mode;
  int E, H, I, r, r_pad;
  const uint8_t* nf4;      // stored stack [E, rows, cols/2]
  const float* absmax;     // [E, rows, cols/64]
  int stored_rows, stored_cols;
  const uint16_t* act_in;  // A operand [rows_cap, K]
  int K;                   // reduction length
  int n_dim;               // output columns
  const uint16_t* lora_a_rows;  // p or q [rows_cap, r]
  const uint16_t* lora_w;       // LoRA weight used as the B operand of the K = r step
  uint16_t* out0;          // gu | y_perm | dgu | dx_perm
  uint16_t* out1;          // act (forward gate_up) or nullptr
  const uint16_t* aux;     // saved gu (down dgrad) or nullptr
  const int32_t* tiles;
  int64_t rows_cap, mt_cap;
  DeviceError* err;
  long long timeout_ns;
};
cudaError_t launch_nf4_gemm(const Nf4GemmHost& h, int num_sms, cudaStream_t stream);
// Weight-streaming forward (kFwdGateUp / kFwdDown only) for decode-sized batches.
cudaError_t launch_nf4_stream(const Nf4GemmHost& h, int num_sms, cudaStream_t stream);

// The serving forward of a decode-sized batch in one launch (serve.cu): x
// scatter + p_gu, gate_up, p_d, down and the weighted combine.
struct ServeHost {
  int T, k, E, H, I, r, r_pad;
  float s;
  const uint8_t* gate_up_nf4;
  const float* gate_up_absmax;
  const uint8_t* down_nf4;
  const float* down_absmax;
  const uint16_t *A_gu, *B_gu, *A_d, *B_d;
  const uint16_t* x;
  uint16_t *x_perm, *p_gu, *gu, *act, *p_d, *y_perm, *y;
  const int32_t *topk_ids, *row_of_slot, *slot_of_row, *counts, *tiles;
  const float* topk_w;
  int32_t* counters;  // serve_counters(E, st_cap, T, H) ints, zero on entry
  float* pd_part;     // serve_part_floats(st_cap, I, r) floats (no initial contents needed)
  int64_t rows_cap, mt_cap, st_cap;
  DeviceError* err;
  long long timeout_ns;
};
cudaError_t launch_nf4_serve(const ServeHost& h, int num_sms, cudaStream_t stream);

struct LoraProjHost {
  const uint16_t* act_in;  // [rows_cap, K]
  int K;
  const uint16_t* w;       // LoRA factor: A [E, r, K] (k_major) or B [E, K, r] (mn_major)
  bool w_mn_major;
  int E, r, r_pad;
  float scale;
  uint16_t* out;           // [rows_cap, r]
  const int32_t* tiles;
  int64_t rows_cap, mt_cap;
  DeviceError* err;
  long long timeout_ns;
  // launch_gather_proj only: act_in is written as act_in[row] = w(slot) * gather_src[token of row]
  const uint16_t* gather_src;   // [T, K]
  const int32_t* slot_of_row;   // [rows_cap]
  const float* gather_w;        // [T*k] or nullptr
  int k;
};
cudaError_t launch_lora_proj(const LoraProjHost& h, int num_sms, cudaStream_t stream);
// The row gather fused with the projection: writes act_in (the gathered rows) and out.
cudaError_t launch_gather_proj(const LoraProjHost& h, int num_sms, cudaStream_t stream);

struct WgradHost {
  // four products dOut_g[e] = Act_g[e rows]^T * Low_g[e rows]
  const uint16_t* act[4];  // [rows_cap, F_g]
  const uint16_t* low[4];  // [rows_cap, r]
  uint16_t* out[4];        // [E, F_g, r] (transposed = false) or [E, r, F_g] (transposed = true)
  int F[4];
  bool transposed[4];
  int E, r, r_pad;
  const int32_t* counts;
  const int32_t* offsets;
  const int32_t* tiles;
  int64_t rows_cap, mt_cap;
  DeviceError* err;
  long long timeout_ns;
};
cudaError_t launch_wgrad(const WgradHost& h, int num_sms, cudaStream_t stream);

// Tensor maps of the operands (gemm.cu): row-major bf16 [rows, cols], bf16
// stacks [E, rows, cols], byte stacks [E, rows, bytes].
CUtensorMapSwizzle swizzle_for_bytes(int row_bytes);
cudaError_t map_bf16_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                        uint32_t box_rows, CUtensorMapSwizzle swz);
cudaError_t map_bf16_3d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t E,
                        uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz);
cudaError_t map_u8_3d(CUtensorMap* m, const void* base, uint64_t bytes, uint64_t rows, uint64_t E,
                      uint32_t box_bytes, uint32_t box_rows, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_NONE);

// Tensor-map encoding through the driver entry point (no link-time libcuda).
cudaError_t encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                              const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                              CUtensorMapSwizzle swizzle);

}  // namespace e4b
