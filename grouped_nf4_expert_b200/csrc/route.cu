// Routing and permutation kernels: top-k + softmax, expert histogram, prefix
// sums with per-expert padding, the device work list, a deterministic stable
// scatter, row gathers and the weighted un-permute combine; the serving call's
// one-CTA routing and CUDA-core LoRA row projections; the router backward
// (d logits of a trained router); the NF4 quantiser and the dequantisation
// test kernel; the watchdog self-test.
//
// Pages: "How do I QLoRA-train the fused experts of a MoE", section "Which
// project solves it" (grouped execution of the routed experts) and section
// "The abstraction that fails" (router frozen: its logits are inputs).
#include <math.h>

#include "e4b_device.cuh"
#include "e4b_internal.h"

namespace e4b {

// NaN ranks lowest; equal values go to the lower expert id.
__device__ __forceinline__ bool route_better(float av, int ae, float bv, int be) {
  const bool an = isnan(av), bn = isnan(bv);
  if (an || bn) return (an && bn) ? (ae < be) : bn;
  return av > bv || (av == bv && ae < be);
}

// Order-preserving unsigned key of a logit: larger value -> larger key, both
// zeros -> the same key, NaN -> 0 (below every number, whose keys are >= 1).
__device__ __forceinline__ uint32_t route_key(float v) {
  if (isnan(v)) return 0u;
  const uint32_t b = (v == 0.0f) ? 0u : __float_as_uint(v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float route_key_value(uint32_t key) {
  if (key == 0u) return __int_as_float(0x7fc00000);
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// One warp per token: k rounds of a warp-wide argmax over the unpicked
// experts (a max-reduction of the value keys, then a min-reduction of the
// expert ids holding that key: ties go to the lower id), then a softmax over
// the k selected logits.  The CTA also counts the slots it produced per
// expert (order-independent shared counters).
template <int EPL>
__global__ void __launch_bounds__(1024) route_topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                         int32_t* __restrict__ topk_ids,
                                                         float* __restrict__ topk_w,
                                                         int32_t* __restrict__ block_counts) {
  extern __shared__ int s_cnt[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_cnt[e] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const int t0 = blockIdx.x * kRouteTokensPerBlock;
  const int t1 = min(T, t0 + kRouteTokensPerBlock);
  for (int t = t0 + warp; t < t1; t += nwarps) {
    const float* row = logits + (size_t)t * E;
    uint32_t key[EPL];  // 0 once picked or past E (a NaN logit also has key 0, but keeps its id)
    uint32_t live = 0;  // bit i: element i is a real, unpicked expert
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      key[i] = (e < E) ? route_key(__ldg(row + e)) : 0u;
      if (e < E) live |= 1u << i;
    }
    float my_v = 0.0f;
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
      // This lane's best live element: largest key, then lowest id (lowest i).
      uint32_t bk = 0u, bi = 0xffffffffu;
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if ((live & (1u << i)) && (bi == 0xffffffffu || key[i] > bk)) {
          bk = key[i];
          bi = (uint32_t)(lane + 32 * i);
        }
      const uint32_t kmax = __reduce_max_sync(0xffffffffu, bk);
      const uint32_t e_sel = __reduce_min_sync(0xffffffffu, (bk == kmax) ? bi : 0xffffffffu);
      if ((int)(e_sel & 31u) == lane) live &= ~(1u << (e_sel >> 5));
      if (lane == j) {
        my_v = route_key_value(kmax);
        my_e = (int)e_sel;
      }
    }
    const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
    const float z = (lane < k) ? expf(my_v - vmax) : 0.0f;
    float sum = z;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < k) {
      topk_ids[(size_t)t * k + lane] = my_e;
      topk_w[(size_t)t * k + lane] = z / sum;
      atomicAdd(&s_cnt[my_e], 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) block_counts[(size_t)blockIdx.x * E + e] = s_cnt[e];
}

// Block-wide exclusive scan of one int per thread (blockDim.x == 1024).
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = s_warp[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += y;
    }
    s_warp[lane] = w;  // inclusive
  }
  __syncthreads();
  const int before = (warp > 0) ? s_warp[warp - 1] : 0;
  __syncthreads();
  return before + x - v;
}

// One CTA of 1024 threads, one thread per expert: counts, 128-aligned group
// offsets, per-(CTA, expert) scatter bases and the experts in descending-count
// order; then the whole CTA writes the padding markers and the three work
// lists (m-tiles, 256-row m-units, 32-slot streaming tiles) as flat index
// spaces, each entry's expert found by a binary search of the per-expert
// prefix sums, so that no thread walks a heavy expert's entries alone.
__device__ __forceinline__ int owner_of(const int* prefix, int E, int i) {  // last e with prefix[e] <= i
  int lo = 0, hi = E;  // prefix[lo] <= i < prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= i) lo = mid; else hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(1024) route_scan_kernel(const int32_t* __restrict__ block_counts, int nblk,
                                                          int E, int32_t* __restrict__ block_base,
                                                          int32_t* __restrict__ counts,
                                                          int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ slot_of_row,
                                                          int32_t* __restrict__ tiles, int64_t mt_cap) {
  __shared__ int s_warp[32];
  __shared__ int s_cnt[E4B_MAX_EXPERTS];
  __shared__ int s_off[E4B_MAX_EXPERTS];
  __shared__ int s_pmt[E4B_MAX_EXPERTS + 1], s_pmu[E4B_MAX_EXPERTS + 1], s_pst[E4B_MAX_EXPERTS + 1];
  __shared__ int s_ppad[E4B_MAX_EXPERTS + 1];
  const int e = threadIdx.x;
  int cnt = 0;
  if (e < E)
    for (int b = 0; b < nblk; ++b) cnt += block_counts[(size_t)b * E + e];
  const int padded = (cnt + 127) / 128 * 128;
  const int off = block_exclusive_scan(e < E ? padded : 0, s_warp);
  const int mt_off = block_exclusive_scan(e < E ? padded / 128 : 0, s_warp);
  const int n_mu = (padded / 128 + 1) / 2;
  const int mu_off = block_exclusive_scan(e < E ? n_mu : 0, s_warp);
  const int n_st = (cnt + 31) / 32;
  const int st_off = block_exclusive_scan(e < E ? n_st : 0, s_warp);
  const int pad_off = block_exclusive_scan(e < E ? padded - cnt : 0, s_warp);
  if (e < E) {
    s_cnt[e] = cnt;
    s_off[e] = off;
    s_pmt[e] = mt_off;
    s_pmu[e] = mu_off;
    s_pst[e] = st_off;
    s_ppad[e] = pad_off;
    counts[e] = cnt;
    offsets[e] = off;
    int run = off;
    for (int b = 0; b < nblk; ++b) {
      block_base[(size_t)b * E + e] = run;
      run += block_counts[(size_t)b * E + e];
    }
    if (e == E - 1) {
      s_pmt[E] = mt_off + padded / 128;
      s_pmu[E] = mu_off + n_mu;
      s_pst[E] = st_off + n_st;
      s_ppad[E] = pad_off + padded - cnt;
      offsets[E] = off + padded;
      tiles[0] = mt_off + padded / 128;
      tiles[1] = off + padded;
      tiles[2] = mu_off + n_mu;
      tiles[3] = st_off + n_st;
    }
  }
  __syncthreads();
  if (e < E) {
    int rank = 0;
    for (int o = 0; o < E; ++o) rank += (s_cnt[o] > cnt) || (s_cnt[o] == cnt && o < e);
    tiles[kTileHeader + 2 * mt_cap + rank] = e;
  }
  for (int i = threadIdx.x; i < s_ppad[E]; i += blockDim.x) {
    const int x = owner_of(s_ppad, E, i);
    slot_of_row[s_off[x] + s_cnt[x] + (i - s_ppad[x])] = -1;
  }
  for (int i = threadIdx.x; i < s_pmt[E]; i += blockDim.x) {
    const int x = owner_of(s_pmt, E, i);
    tiles[kTileHeader + 2 * i] = x;
    tiles[kTileHeader + 2 * i + 1] = s_off[x] + 128 * (i - s_pmt[x]);
  }
  int32_t* mu = tiles + kTileHeader + 2 * mt_cap + E;
  for (int i = threadIdx.x; i < s_pmu[E]; i += blockDim.x) {
    const int x = owner_of(s_pmu, E, i), q = i - s_pmu[x];
    const int pad_x = (s_cnt[x] + 127) / 128 * 128;
    mu[3 * i] = x;
    mu[3 * i + 1] = s_off[x] + 256 * q;
    mu[3 * i + 2] = min(256, pad_x - 256 * q);
  }
  int32_t* st = tiles + kTileHeader + 2 * mt_cap + E + 3 * mt_cap;
  for (int i = threadIdx.x; i < s_pst[E]; i += blockDim.x) {
    const int x = owner_of(s_pst, E, i), q = i - s_pst[x];
    st[3 * i] = x;
    st[3 * i + 1] = s_off[x] + 32 * q;
    st[3 * i + 2] = min(32, s_cnt[x] - 32 * q);
  }
}

// Stable scatter: one warp walks its CTA's slots in flat order, 32 at a time;
// slots of the same expert inside a step are ranked by lane (match_any), and
// a shared running count per expert carries the rank across steps.  The
// warp's expert ids are loaded before the walk (kRouteTokensPerBlock * k /
// 32 per lane).
constexpr int kRankIdsPerLane = kRouteTokensPerBlock * E4B_MAX_TOP_K / 32;
__global__ void __launch_bounds__(32) route_rank_kernel(const int32_t* __restrict__ topk_ids, int N, int E,
                                                        int slots_per_block,
                                                        const int32_t* __restrict__ block_base,
                                                        int32_t* __restrict__ row_of_slot,
                                                        int32_t* __restrict__ slot_of_row) {
  extern __shared__ int s_run[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_run[e] = block_base[(size_t)blockIdx.x * E + e];
  __syncwarp();
  const int lane = threadIdx.x;
  const int f0 = blockIdx.x * slots_per_block;
  const int f1 = min(N, f0 + slots_per_block);
  const int steps = (f1 - f0 + 31) / 32;  // <= kRankIdsPerLane
  int ids[kRankIdsPerLane];
#pragma unroll
  for (int s = 0; s < kRankIdsPerLane; ++s) {
    const int f = f0 + 32 * s + lane;
    ids[s] = (s < steps && f < f1) ? __ldg(topk_ids + f) : -1;
  }
#pragma unroll
  for (int s = 0; s < kRankIdsPerLane; ++s) {
    if (s >= steps) break;
    const int f = f0 + 32 * s + lane;
    const int e = ids[s];
    const bool valid = e >= 0;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int leader = __ffs(peers) - 1;
    if (valid) {
      const int row = s_run[e] + rank;
      row_of_slot[f] = row;
      slot_of_row[row] = f;
    }
    __syncwarp();
    if (valid && lane == leader) s_run[e] += __popc(peers);
    __syncwarp();
  }
}

// Routing of a batch of at most kRouteTokensPerBlock tokens in one CTA, for
// the serving forward: top-k + softmax per token (as route_topk_kernel), the
// expert counts, 128-aligned group offsets, the weight-streaming tile list
// and the stable slot ranks (row_of_slot, and slot_of_row for the routed
// rows), as route_scan_kernel and route_rank_kernel do, in one launch.  No
// padding markers and no m-tile lists: the serving forward reads neither.  The
// launch also sets `n_zero` ints at `zero` to 0 (the counters of the serving
// launch that follows it).
template <int EPL>
__global__ void __launch_bounds__(1024) route_small_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                          int32_t* __restrict__ topk_ids,
                                                          float* __restrict__ topk_w,
                                                          int32_t* __restrict__ counts,
                                                          int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ row_of_slot,
                                                          int32_t* __restrict__ slot_of_row,
                                                          int32_t* __restrict__ tiles, int64_t st_offset,
                                                          int32_t* __restrict__ zero, int64_t n_zero) {
  for (int64_t z = threadIdx.x; z < n_zero; z += blockDim.x) zero[z] = 0;
  __shared__ int s_cnt[E4B_MAX_EXPERTS];
  __shared__ int s_run[E4B_MAX_EXPERTS];
  __shared__ int s_warp[32];
  __shared__ int s_ids[kRouteTokensPerBlock * E4B_MAX_TOP_K];
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_cnt[e] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  for (int t = warp; t < T; t += nwarps) {
    const float* row = logits + (size_t)t * E;
    uint32_t key[EPL];
    uint32_t live = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      key[i] = (e < E) ? route_key(__ldg(row + e)) : 0u;
      if (e < E) live |= 1u << i;
    }
    float my_v = 0.0f;
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
      uint32_t bk = 0u, bi = 0xffffffffu;
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if ((live & (1u << i)) && (bi == 0xffffffffu || key[i] > bk)) {
          bk = key[i];
          bi = (uint32_t)(lane + 32 * i);
        }
      const uint32_t kmax = __reduce_max_sync(0xffffffffu, bk);
      const uint32_t e_sel = __reduce_min_sync(0xffffffffu, (bk == kmax) ? bi : 0xffffffffu);
      if ((int)(e_sel & 31u) == lane) live &= ~(1u << (e_sel >> 5));
      if (lane == j) {
        my_v = route_key_value(kmax);
        my_e = (int)e_sel;
      }
    }
    const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
    const float z = (lane < k) ? expf(my_v - vmax) : 0.0f;
    float sum = z;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < k) {
      topk_ids[(size_t)t * k + lane] = my_e;
      topk_w[(size_t)t * k + lane] = z / sum;
      s_ids[t * k + lane] = my_e;
      atomicAdd(&s_cnt[my_e], 1);
    }
  }
  __syncthreads();
  // one thread per expert: offsets and streaming tiles
  const int e = threadIdx.x;
  const int cnt = (e < E) ? s_cnt[e] : 0;
  const int padded = (cnt + 127) / 128 * 128;
  const int off = block_exclusive_scan(e < E ? padded : 0, s_warp);
  const int n_st = (cnt + 31) / 32;
  const int st_off = block_exclusive_scan(e < E ? n_st : 0, s_warp);
  if (e < E) {
    counts[e] = cnt;
    offsets[e] = off;
    s_run[e] = off;
    int32_t* st = tiles + st_offset;
    for (int i = 0; i < n_st; ++i) {
      st[3 * (st_off + i)] = e;
      st[3 * (st_off + i) + 1] = off + 32 * i;
      st[3 * (st_off + i) + 2] = min(32, cnt - 32 * i);
    }
    if (e == E - 1) {
      offsets[E] = off + padded;
      tiles[0] = 0;  // no m-tile list
      tiles[1] = off + padded;
      tiles[2] = 0;  // no m-unit list
      tiles[3] = st_off + n_st;
    }
  }
  __syncthreads();
  // stable ranks: warp 0 walks the slots in flat order, 32 at a time
  if (warp == 0) {
    const int N = T * k;
    for (int f0 = 0; f0 < N; f0 += 32) {
      const int f = f0 + lane;
      const int ex = (f < N) ? s_ids[f] : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, ex);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int leader = __ffs(peers) - 1;
      if (ex >= 0) {
        row_of_slot[f] = s_run[ex] + rank;
        slot_of_row[s_run[ex] + rank] = f;
      }
      __syncwarp();
      if (ex >= 0 && lane == leader) s_run[ex] += __popc(peers);
      __syncwarp();
    }
  }
}

// LoRA down-projection of permuted rows on the CUDA cores, one CTA per routed
// slot: out[row] = bf16(s * src_row . A[e]^T) over K, for the few rows of a
// serving batch (the tensor-core projection is built for 128-row tiles).  The
// source row is the token's row of `src` (by_token) or the slot's permuted
// row; with `copy_dst` the source row is also copied to the slot's permuted
// row (the x scatter of the serving forward).  fp32 products and sums.
template <int R>
__global__ void __launch_bounds__(256) lora_rows_kernel(const uint16_t* __restrict__ src, int by_token,
                                                        const int32_t* __restrict__ topk_ids,
                                                        const int32_t* __restrict__ row_of_slot, int N, int k,
                                                        int K, const uint16_t* __restrict__ A, int r, float s,
                                                        uint16_t* __restrict__ copy_dst,
                                                        uint16_t* __restrict__ out) {
  __shared__ float red[8][R];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int vec = K / 8;
  for (int f = blockIdx.x; f < N; f += gridDim.x) {
    const int e = __ldg(topk_ids + f), row = __ldg(row_of_slot + f);
    const uint4* sp = reinterpret_cast<const uint4*>(src + (size_t)(by_token ? f / k : row) * K);
    const uint4* ap = reinterpret_cast<const uint4*>(A + (size_t)e * r * K);
    float acc[R];
#pragma unroll
    for (int j = 0; j < R; ++j) acc[j] = 0.0f;
    for (int pc = threadIdx.x; pc < vec; pc += blockDim.x) {
      const uint4 q = __ldg(sp + pc);
      if (copy_dst != nullptr) reinterpret_cast<uint4*>(copy_dst + (size_t)row * K)[pc] = q;
      const uint32_t* qw = reinterpret_cast<const uint32_t*>(&q);
      float xv[8];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        xv[2 * c] = bf16lo_to_f32(qw[c]);
        xv[2 * c + 1] = bf16hi_to_f32(qw[c]);
      }
#pragma unroll
      for (int j = 0; j < R; ++j)
        if (j < r) {
          const uint4 a = __ldg(ap + (size_t)j * vec + pc);
          const uint32_t* aw = reinterpret_cast<const uint32_t*>(&a);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            acc[j] = fmaf(xv[2 * c], bf16lo_to_f32(aw[c]), acc[j]);
            acc[j] = fmaf(xv[2 * c + 1], bf16hi_to_f32(aw[c]), acc[j]);
          }
        }
    }
#pragma unroll
    for (int j = 0; j < R; ++j) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int j = 0; j < R; ++j) red[warp][j] = acc[j];
    }
    __syncthreads();
    for (int j = threadIdx.x; j < r; j += blockDim.x) {  // r may exceed a one-warp block
      float sum = 0.0f;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) sum += red[w][j];
      const __nv_bfloat16 h = __float2bfloat16_rn(s * sum);
      out[(size_t)row * r + j] = *reinterpret_cast<const uint16_t*>(&h);
    }
    __syncthreads();
  }
}

__device__ __forceinline__ uint4 scale_bf16x8(uint4 q, float w) {
  uint32_t* p = reinterpret_cast<uint32_t*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = pack_bf16x2(w * bf16lo_to_f32(p[i]), w * bf16hi_to_f32(p[i]));
  return q;
}

// One warp per permuted row (padding rows are zero-filled).  A row is moved
// in batches of up to 8 16-byte pieces per lane (4 KB per warp), every load
// of a batch issued before its stores; the next row's slot index is fetched
// one row ahead.
constexpr int kPiecesPerBatch = 8;
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ src,
                                                          const int32_t* __restrict__ slot_of_row,
                                                          const int32_t* __restrict__ tiles,
                                                          const float* __restrict__ scale_w, int H, int k,
                                                          uint16_t* __restrict__ dst) {
  const int rows_used = tiles[1];
  const int vec = H / 8;  // 16-byte pieces per row
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), nw = gridDim.x * (blockDim.x >> 5);
  int slot = (gw < rows_used) ? __ldg(slot_of_row + gw) : -1;
  for (int row = gw; row < rows_used; row += nw) {
    const int next = (row + nw < rows_used) ? __ldg(slot_of_row + row + nw) : -1;
    uint4* d = reinterpret_cast<uint4*>(dst + (size_t)row * H);
    if (slot < 0) {
      for (int i = lane; i < vec; i += 32) d[i] = make_uint4(0, 0, 0, 0);
    } else {
      const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)(slot / k) * H);
      const float w = scale_w ? __ldg(scale_w + slot) : 1.0f;
      for (int b0 = 0; b0 < vec; b0 += 32 * kPiecesPerBatch) {
        uint4 q[kPiecesPerBatch];
#pragma unroll
        for (int i = 0; i < kPiecesPerBatch; ++i) {
          const int pc = b0 + 32 * i + lane;
          if (pc < vec) q[i] = __ldg(s + pc);
        }
#pragma unroll
        for (int i = 0; i < kPiecesPerBatch; ++i) {
          const int pc = b0 + 32 * i + lane;
          if (pc < vec) d[pc] = scale_w ? scale_bf16x8(q[i], w) : q[i];
        }
      }
    }
    slot = next;
  }
}

// One warp per token: the k permuted rows are summed in slot order (weighted
// by the routing weights for y, unweighted for dx) in fp32 per 16-byte piece;
// the rows of a piece are loaded in groups of 8, all in flight together.
constexpr int kRowsPerBatch = 8;
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ src_perm,
                                                      const int32_t* __restrict__ row_of_slot,
                                                      const float* __restrict__ topk_w, int T, int k, int H,
                                                      int split, uint16_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), nw = gridDim.x * (blockDim.x >> 5);
  // a task is one of `split` equal column ranges of a token (split > 1 for small batches)
  const int per = H / 8 / split;
  for (int task = gw; task < T * split; task += nw) {
    const int t = task / split;
    const int pc0 = (task % split) * per;
    const int vec = pc0 + per;
    // lane j < k holds slot j's permuted row and weight
    const int my_row = (lane < k) ? __ldg(row_of_slot + (size_t)t * k + lane) : 0;
    const float my_w = (lane < k) ? (topk_w ? __ldg(topk_w + (size_t)t * k + lane) : 1.0f) : 0.0f;
    if (k <= kRowsPerBatch) {  // common case: the k row pointers and weights stay in registers
      const uint4* rp[kRowsPerBatch];
      float rw[kRowsPerBatch];
#pragma unroll
      for (int j = 0; j < kRowsPerBatch; ++j) {
        rp[j] = reinterpret_cast<const uint4*>(src_perm + (size_t)__shfl_sync(0xffffffffu, my_row, j) * H);
        rw[j] = __shfl_sync(0xffffffffu, my_w, j);
      }
      for (int pc = pc0 + lane; pc < vec; pc += 32) {
        uint4 q[kRowsPerBatch];
#pragma unroll
        for (int j = 0; j < kRowsPerBatch; ++j)
          if (j < k) q[j] = __ldg(rp[j] + pc);
        float acc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
#pragma unroll
        for (int j = 0; j < kRowsPerBatch; ++j)
          if (j < k) {
            const uint32_t* p = reinterpret_cast<const uint32_t*>(&q[j]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              acc[2 * c] += rw[j] * bf16lo_to_f32(p[c]);
              acc[2 * c + 1] += rw[j] * bf16hi_to_f32(p[c]);
            }
          }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        reinterpret_cast<uint4*>(out + (size_t)t * H)[pc] = o;
      }
      continue;
    }
    // k > 8: the row indices and weights come by shuffles inside the loop, so every lane runs
    // every iteration (the loop bound is warp-uniform) and only the loads and stores are guarded.
    for (int pb = pc0; pb < vec; pb += 32) {
      const int pc = pb + lane;
      const bool live = pc < vec;
      float acc[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
      for (int j0 = 0; j0 < k; j0 += kRowsPerBatch) {
        uint4 q[kRowsPerBatch];
#pragma unroll
        for (int j = 0; j < kRowsPerBatch; ++j) {
          const int r = __shfl_sync(0xffffffffu, my_row, (j0 + j) & 31);
          q[j] = (live && j0 + j < k) ? __ldg(reinterpret_cast<const uint4*>(src_perm + (size_t)r * H) + pc)
                                      : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int j = 0; j < kRowsPerBatch; ++j) {
          const float w = __shfl_sync(0xffffffffu, my_w, (j0 + j) & 31);
          if (j0 + j < k) {
            const uint32_t* p = reinterpret_cast<const uint32_t*>(&q[j]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              acc[2 * c] += w * bf16lo_to_f32(p[c]);
              acc[2 * c + 1] += w * bf16hi_to_f32(p[c]);
            }
          }
        }
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      if (live) reinterpret_cast<uint4*>(out + (size_t)t * H)[pc] = o;
    }
  }
}

// Router backward, one warp per token.  dw_j = <dY[t], y_perm[row(t,j)]> in
// fp32 (lanes across H in 16-byte pieces, the k rows of a batch loaded
// together, then a butterfly sum), followed by the backward of the softmax
// over the k selected logits: d_logit[ids_j] = w_j (dw_j - sum_i w_i dw_i);
// every other logit of the row gets 0.
constexpr int kRbwdSlots = 4;
__global__ void __launch_bounds__(256, 4) router_bwd_kernel(const uint16_t* __restrict__ dY,
                                                         const uint16_t* __restrict__ y_perm,
                                                         const int32_t* __restrict__ row_of_slot,
                                                         const int32_t* __restrict__ topk_ids,
                                                         const float* __restrict__ topk_w, int T, int k, int H,
                                                         int E, float* __restrict__ d_logits,
                                                         float* __restrict__ dw_out) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), nw = gridDim.x * (blockDim.x >> 5);
  const int vec = H / 8;
  for (int t = gw; t < T; t += nw) {
    const int my_row = (lane < k) ? __ldg(row_of_slot + (size_t)t * k + lane) : 0;
    const float my_w = (lane < k) ? __ldg(topk_w + (size_t)t * k + lane) : 0.0f;
    const int my_id = (lane < k) ? __ldg(topk_ids + (size_t)t * k + lane) : 0;
    const uint4* dyp = reinterpret_cast<const uint4*>(dY + (size_t)t * H);
    float my_dw = 0.0f;
    for (int j0 = 0; j0 < k; j0 += kRbwdSlots) {
      const uint4* rp[kRbwdSlots];
#pragma unroll
      for (int j = 0; j < kRbwdSlots; ++j)
        rp[j] = reinterpret_cast<const uint4*>(y_perm +
                                               (size_t)__shfl_sync(0xffffffffu, my_row, (j0 + j) & 31) * H);
      float acc[kRbwdSlots];
#pragma unroll
      for (int j = 0; j < kRbwdSlots; ++j) acc[j] = 0.0f;
      for (int pc = lane; pc < vec; pc += 32) {
        const uint4 d = __ldg(dyp + pc);
        uint4 q[kRbwdSlots];
#pragma unroll
        for (int j = 0; j < kRbwdSlots; ++j)
          if (j0 + j < k) q[j] = __ldg(rp[j] + pc);
        const uint32_t* dp = reinterpret_cast<const uint32_t*>(&d);
        float dv[8];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          dv[2 * c] = bf16lo_to_f32(dp[c]);
          dv[2 * c + 1] = bf16hi_to_f32(dp[c]);
        }
#pragma unroll
        for (int j = 0; j < kRbwdSlots; ++j)
          if (j0 + j < k) {
            const uint32_t* p = reinterpret_cast<const uint32_t*>(&q[j]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              acc[j] = fmaf(dv[2 * c], bf16lo_to_f32(p[c]), acc[j]);
              acc[j] = fmaf(dv[2 * c + 1], bf16hi_to_f32(p[c]), acc[j]);
            }
          }
      }
#pragma unroll
      for (int j = 0; j < kRbwdSlots; ++j) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
        if (lane == j0 + j) my_dw = acc[j];
      }
    }
    // sum_i w_i dw_i over the selected slots (lanes >= k contribute 0)
    float mean = my_w * my_dw;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mean += __shfl_xor_sync(0xffffffffu, mean, o);
    const float g = my_w * (my_dw - mean);
    float* row = d_logits + (size_t)t * E;
    if ((E & 3) == 0) {
      for (int e = lane; e < E / 4; e += 32) reinterpret_cast<float4*>(row)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      for (int e = lane; e < E; e += 32) row[e] = 0.0f;
    }
    __syncwarp();  // the zeros are ordered before the selected entries
    if (lane < k) {
      row[my_id] = g;
      if (dw_out != nullptr) dw_out[(size_t)t * k + lane] = my_dw;
    }
  }
}

__global__ void __launch_bounds__(256) nf4_dequant_kernel(const uint8_t* __restrict__ packed,
                                                          const float* __restrict__ absmax, int64_t nblocks,
                                                          uint16_t* __restrict__ out) {
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblocks;
       b += (int64_t)gridDim.x * blockDim.x) {
    const uint4* p = reinterpret_cast<const uint4*>(packed + b * 32);
    const uint4 q0 = __ldg(p), q1 = __ldg(p + 1);
    const uint32_t codes[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    uint32_t v[32];
    nf4_decode_block(codes, __ldg(absmax + b), v);
    uint4* o = reinterpret_cast<uint4*>(out + b * 64);
#pragma unroll
    for (int c = 0; c < 8; ++c) o[c] = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
  }
}

// NF4 quantisation.  The code of x = w / absmax (an IEEE float32 division)
// is the level nearest to x in float32 distance |x - level|, an exact tie
// going to the lower code; a block whose absmax is not positive gets the code
// of the level 0 (7).  The levels ascend, so with c the number of levels
// below x (a 4-step search of the level table) the nearest level is c-1 or c:
// every other level is at least one level gap (> 0.07) further from x, far
// more than float32 rounding of numbers below 2 can close, so comparing the
// two distances takes the same decision as comparing all 16.  A NaN x ends
// at c = 0 and gets code 0, as the full comparison gives.
__device__ __forceinline__ uint32_t nf4_nearest_code(float x, const float* lv) {
  int c = (lv[7] < x) ? 8 : 0;
  c += (lv[c + 3] < x) ? 4 : 0;
  c += (lv[c + 1] < x) ? 2 : 0;
  c += (lv[c] < x) ? 1 : 0;
  const int lo = c > 0 ? c - 1 : 0;
  const float d_lo = fabsf(__fsub_rn(x, lv[lo]));
  const float d_hi = fabsf(__fsub_rn(x, lv[c]));
  return (uint32_t)(d_lo <= d_hi ? lo : c);
}

__device__ __forceinline__ float rcp_approx(float a) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(a));
  return r;
}

__device__ __forceinline__ float ld_shared_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

// The fast decision.  x' = w * rcp(a) is within 2^-21 of the float32
// quotient x = fl(w / a) (|x| <= 1; the reciprocal is within 1 ulp, the
// product within half an ulp).  The level nearest to x changes only at the
// midpoints between adjacent levels (the float32 distance comparison agrees
// with "x above the midpoint" except within a few ulps of it).  Buckets of
// width 1/128 over [-1, 1] each hold the midpoint nearest to them, its
// float32 bits with the low 4 bits replaced by the code just below it (an
// error of at most 15 ulps, under 2^-20): code = that code + (x' above the
// stored midpoint).  Midpoints are more than 0.07 apart, so no other midpoint
// lies between x' and the stored one.  Whenever x' is within 2^-18 of the
// stored midpoint the IEEE division decides instead; further away, x is on
// the same side of the true midpoint as x' by more than 2^-20, far beyond
// the rounding of the distances, so both decisions agree.  Blocks whose a is
// outside [2^-125, 2^125], where the reciprocal may not be a normal number,
// always divide.  Each lane reads its own copy of the table (bank = lane),
// so the lookups never conflict.
constexpr int kQBuckets = 257;
constexpr float kQMargin = 3.814697265625e-06f;  // 2^-18
constexpr float kQMagic = 12583040.0f;           // 1.5 * 2^23 + 128: bits = 0x4B400000 + 128 + round(128 x)

__device__ __forceinline__ void nf4_quantize_piece(uint4 v, bool ok, int64_t p, int lane, const float* lv,
                                                   uint32_t tbl_lane, uint32_t* __restrict__ packed4,
                                                   float* __restrict__ absmax) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
  // absmax: |w| bf16 bit patterns order like unsigned integers (a NaN ranks above every number)
  uint32_t m2 = __vmaxu2(u[0] & 0x7fff7fffu, u[1] & 0x7fff7fffu);
  m2 = __vmaxu2(m2, __vmaxu2(u[2] & 0x7fff7fffu, u[3] & 0x7fff7fffu));
  uint32_t m = max(m2 & 0xffffu, m2 >> 16) << 16;
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 4));
  const float amax = __uint_as_float(m);
  float w[8];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    w[2 * c] = __uint_as_float(mul_lo_u32(u[c], 65536u));  // low half: an integer multiply, off the ALU pipe
    w[2 * c + 1] = bf16hi_to_f32(u[c]);
  }
  uint32_t out = 0x77777777u;
  if (amax > 0.0f) {
    bool exact = !(amax >= 2.350988701644575e-38f && amax <= 4.253529586511730793e+37f);  // 2^-125, 2^125
    if (!exact) {
      const float ra = rcp_approx(amax);
      uint32_t near = 0;  // number of x' within the margin of their stored midpoint
      out = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {  // element 2b in the high nibble of byte b
        const float x = __fmul_rn(w[i], ra);
        const float t = __fmaf_rn(x, 128.0f, kQMagic);
        const float mid = ld_shared_f32(mad_lo_u32(__float_as_uint(t), 128u, tbl_lane));
        const float d = __fsub_rn(mid, x);
        const uint32_t code = mad_hi_u32(__float_as_uint(d), 2u, __float_as_uint(mid) & 15u);
        near = mad_hi_u32(__float_as_uint(__fsub_rn(fabsf(d), kQMargin)), 2u, near);  // sign bit: |d| < margin
        out = mad_lo_u32(code, 1u << (8 * (i >> 1) + ((i & 1) ? 0 : 4)), out);
      }
      exact = near != 0;
    }
    if (exact) {  // rare: some x' near a midpoint, or an extreme block scale
      out = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        out |= nf4_nearest_code(__fdiv_rn(w[i], amax), lv) << (8 * (i >> 1) + ((i & 1) ? 0 : 4));
    }
  }
  if (ok) {
    packed4[p] = out;
    if ((lane & 7) == 0) absmax[p >> 3] = amax;
  }
}

// A warp covers 4 blocks (32 pieces) per quad and loads two quads before
// quantising either.
__global__ void __launch_bounds__(256) nf4_quantize_kernel(const uint4* __restrict__ w8, int64_t nblocks,
                                                           uint32_t* __restrict__ packed4,
                                                           float* __restrict__ absmax) {
  __shared__ float lv[16];
  __shared__ float tbl[kQBuckets * 32];  // [bucket][lane]
  if (threadIdx.x < 16) lv[threadIdx.x] = nf4_level(threadIdx.x);
  for (int e = threadIdx.x; e < kQBuckets; e += blockDim.x) {
    const float center = (float)(e - 128) * 0.0078125f;
    int best = 0;
    float bm = 0.5f * (nf4_level(0) + nf4_level(1)), bd = fabsf(bm - center);
    for (int c = 1; c < 15; ++c) {
      const float mc = 0.5f * (nf4_level(c) + nf4_level(c + 1));
      if (fabsf(mc - center) < bd) {
        bd = fabsf(mc - center);
        bm = mc;
        best = c;
      }
    }
    const float v = __uint_as_float((__float_as_uint(bm) & ~15u) | (uint32_t)best);
    for (int l = 0; l < 32; ++l) tbl[e * 32 + l] = v;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  // shared address of this lane's copy of bucket b is tbl + 128 b + 4 lane = bits(t) * 128 + tbl_lane
  const uint32_t tbl_lane = (uint32_t)__cvta_generic_to_shared(tbl) + 4u * lane - 0x4B400000u * 128u;
  const int64_t n8 = nblocks * 8;
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  // the next iteration's two pieces are loaded before this iteration's are quantised
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  int64_t q = gw * 2;
  uint4 a = (q * 32 + lane < n8) ? __ldg(w8 + q * 32 + lane) : z;
  uint4 b = (q * 32 + 32 + lane < n8) ? __ldg(w8 + q * 32 + 32 + lane) : z;
  for (; q * 32 < n8; q += nw * 2) {
    const int64_t p0 = q * 32 + lane, p1 = p0 + 32;
    const int64_t n0 = p0 + nw * 64, n1 = n0 + 32;
    const uint4 an = (n0 < n8) ? __ldg(w8 + n0) : z;
    const uint4 bn = (n1 < n8) ? __ldg(w8 + n1) : z;
    nf4_quantize_piece(a, p0 < n8, p0, lane, lv, tbl_lane, packed4, absmax);
    nf4_quantize_piece(b, p1 < n8, p1, lane, lv, tbl_lane, packed4, absmax);
    a = an;
    b = bn;
  }
}

// Waits on an mbarrier that nothing ever arrives on: the bounded wait must
// give up, record E4B_ERR_DEVICE_TIMEOUT and let the CTA finish.
__global__ void watchdog_kernel(DeviceError* err, long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ CtaControl ctl;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  mbar_wait(&bar, 0, &ctl, err, timeout_ns, /*site=*/1);
  __syncthreads();
}

// ---------------------------------------------------------------- launchers

cudaError_t launch_route(const float* logits, const uint16_t* x, int T, int E, int H, int k, int32_t* topk_ids,
                         float* topk_w, int32_t* counts, int32_t* offsets, int32_t* row_of_slot,
                         int32_t* slot_of_row, int32_t* tiles, int64_t mt_cap, uint16_t* x_perm,
                         int64_t rows_cap, int32_t* scratch, int num_sms, cudaStream_t stream) {
  const int nblk = (T + kRouteTokensPerBlock - 1) / kRouteTokensPerBlock;
  int32_t* block_counts = scratch;
  int32_t* block_base = scratch + (size_t)nblk * E;
  const size_t smem = (size_t)E * sizeof(int);
  const int epl = (E + 31) / 32;
  {
  LaunchScope scope("route_topk", stream);
  if (epl <= 1)
    route_topk_kernel<1><<<nblk, 1024, smem, stream>>>(logits, T, E, k, topk_ids, topk_w, block_counts);
  else if (epl <= 2)
    route_topk_kernel<2><<<nblk, 1024, smem, stream>>>(logits, T, E, k, topk_ids, topk_w, block_counts);
  else if (epl <= 4)
    route_topk_kernel<4><<<nblk, 1024, smem, stream>>>(logits, T, E, k, topk_ids, topk_w, block_counts);
  else if (epl <= 8)
    route_topk_kernel<8><<<nblk, 1024, smem, stream>>>(logits, T, E, k, topk_ids, topk_w, block_counts);
  else if (epl <= 16)
    route_topk_kernel<16><<<nblk, 1024, smem, stream>>>(logits, T, E, k, topk_ids, topk_w, block_counts);
  else
    route_topk_kernel<32><<<nblk, 1024, smem, stream>>>(logits, T, E, k, topk_ids, topk_w, block_counts);
  }
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  {
    LaunchScope scope("route_scan", stream);
    route_scan_kernel<<<1, 1024, 0, stream>>>(block_counts, nblk, E, block_base, counts, offsets, slot_of_row,
                                              tiles, mt_cap);
  }
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  {
    LaunchScope scope("route_rank", stream);
    route_rank_kernel<<<nblk, 32, smem, stream>>>(topk_ids, T * k, E, kRouteTokensPerBlock * k, block_base,
                                                  row_of_slot, slot_of_row);
  }
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  if (x_perm == nullptr) return cudaSuccess;  // routing tables only
  return launch_gather_rows(x, slot_of_row, tiles, nullptr, H, k, rows_cap, x_perm, num_sms, stream);
}

cudaError_t launch_route_serve(const float* logits, int T, int E, int H, int k, int32_t* topk_ids, float* topk_w,
                               int32_t* counts, int32_t* offsets, int32_t* row_of_slot, int32_t* slot_of_row,
                               int32_t* tiles, int64_t mt_cap, int64_t rows_cap, int32_t* scratch, int num_sms,
                               cudaStream_t stream, int32_t* zero, int64_t n_zero) {
  if (T > kRouteTokensPerBlock) {
    cudaError_t err = launch_route(logits, nullptr, T, E, H, k, topk_ids, topk_w, counts, offsets, row_of_slot,
                                   slot_of_row, tiles, mt_cap, nullptr, rows_cap, scratch, num_sms, stream);
    if (err != cudaSuccess || zero == nullptr || n_zero == 0) return err;
    return cudaMemsetAsync(zero, 0, (size_t)n_zero * sizeof(int32_t), stream);
  }
  const int64_t st_off = stiles_offset(mt_cap, E);
  const int epl = (E + 31) / 32;
  LaunchScope scope("route_small", stream);
#define E4B_ROUTE_SMALL(P)                                                                                   \
  route_small_kernel<P><<<1, 1024, 0, stream>>>(logits, T, E, k, topk_ids, topk_w, counts, offsets, row_of_slot, \
                                                slot_of_row, tiles, st_off, zero, n_zero)
  if (epl <= 1)
    E4B_ROUTE_SMALL(1);
  else if (epl <= 2)
    E4B_ROUTE_SMALL(2);
  else if (epl <= 4)
    E4B_ROUTE_SMALL(4);
  else if (epl <= 8)
    E4B_ROUTE_SMALL(8);
  else if (epl <= 16)
    E4B_ROUTE_SMALL(16);
  else
    E4B_ROUTE_SMALL(32);
#undef E4B_ROUTE_SMALL
  return cudaGetLastError();
}

cudaError_t launch_lora_rows(const uint16_t* src, bool by_token, const int32_t* topk_ids, const int32_t* row_of_slot,
                             int N, int k, int K, const uint16_t* A, int r, float s, uint16_t* copy_dst,
                             uint16_t* out, int num_sms, cudaStream_t stream) {
  const int pieces = K / 8;
  const int threads = pieces >= 256 ? 256 : ((pieces + 31) / 32) * 32;
  const int grid = N < num_sms * 8 ? N : num_sms * 8;
  LaunchScope scope(copy_dst ? "scatter_lora_rows" : "lora_rows", stream);
  const int bt = by_token ? 1 : 0;
  if (r <= 16)
    lora_rows_kernel<16><<<grid, threads, 0, stream>>>(src, bt, topk_ids, row_of_slot, N, k, K, A, r, s, copy_dst, out);
  else if (r <= 32)
    lora_rows_kernel<32><<<grid, threads, 0, stream>>>(src, bt, topk_ids, row_of_slot, N, k, K, A, r, s, copy_dst, out);
  else
    lora_rows_kernel<64><<<grid, threads, 0, stream>>>(src, bt, topk_ids, row_of_slot, N, k, K, A, r, s, copy_dst, out);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const uint16_t* src, const int32_t* slot_of_row, const int32_t* tiles,
                               const float* scale_w, int H, int k, int64_t rows_cap, uint16_t* dst, int num_sms,
                               cudaStream_t stream) {
  const int64_t blocks = (rows_cap + 7) / 8;  // 8 warps of 256 threads, a warp per row
  const int64_t grid = blocks < (int64_t)num_sms * 8 ? blocks : (int64_t)num_sms * 8;
  LaunchScope scope(scale_w ? "gather_dyw" : "gather_x", stream);
  gather_rows_kernel<<<(int)grid, 256, 0, stream>>>(src, slot_of_row, tiles, scale_w, H, k, dst);
  return cudaGetLastError();
}

cudaError_t launch_combine(const uint16_t* src_perm, const int32_t* row_of_slot, const float* topk_w, int T, int k,
                           int H, uint16_t* out, int num_sms, cudaStream_t stream) {
  // a warp per token, or per 1/split of a token's columns when the batch has fewer tokens than 4 warps
  // per SM (split divides the H/8 16-byte pieces and leaves at least 32 per task)
  int split = 1;
  while (T * split < num_sms * 4 && (H / 8) % (2 * split) == 0 && H / 8 / (2 * split) >= 32) split *= 2;
  const int blocks = (T * split + 7) / 8;  // 8 warps of 256 threads
  const int grid = blocks < num_sms * 8 ? blocks : num_sms * 8;
  LaunchScope scope(topk_w ? "combine_y" : "combine_dx", stream);
  combine_kernel<<<grid, 256, 0, stream>>>(src_perm, row_of_slot, topk_w, T, k, H, split, out);
  return cudaGetLastError();
}

cudaError_t launch_router_bwd(const uint16_t* dY, const uint16_t* y_perm, const int32_t* row_of_slot,
                              const int32_t* topk_ids, const float* topk_w, int T, int k, int H, int E,
                              float* d_logits, float* dw, int num_sms, cudaStream_t stream) {
  const int blocks = (T + 7) / 8;  // 8 warps of 256 threads, a warp per token
  const int grid = blocks < num_sms * 8 ? blocks : num_sms * 8;
  LaunchScope scope("router_bwd", stream);
  router_bwd_kernel<<<grid, 256, 0, stream>>>(dY, y_perm, row_of_slot, topk_ids, topk_w, T, k, H, E, d_logits, dw);
  return cudaGetLastError();
}

cudaError_t launch_nf4_dequant(const uint8_t* packed, const float* absmax, int64_t n, uint16_t* out, int num_sms,
                               cudaStream_t stream) {
  const int64_t nblocks = n / 64;
  int64_t grid = (nblocks + 255) / 256;
  if (grid > (int64_t)num_sms * 16) grid = (int64_t)num_sms * 16;
  if (grid < 1) grid = 1;
  LaunchScope scope("nf4_dequant", stream);
  nf4_dequant_kernel<<<(int)grid, 256, 0, stream>>>(packed, absmax, nblocks, out);
  return cudaGetLastError();
}

cudaError_t launch_nf4_quantize(const uint16_t* w, int64_t n, uint8_t* packed, float* absmax, int num_sms,
                                cudaStream_t stream) {
  const int64_t nblocks = n / 64;
  int64_t grid = (nblocks + 63) / 64;  // 8 warps of 256 threads, 8 blocks per warp iteration
  if (grid > (int64_t)num_sms * 6) grid = (int64_t)num_sms * 6;  // 33 KB of tables: 6 CTAs per SM
  if (grid < 1) grid = 1;
  LaunchScope scope("nf4_quantize", stream);
  nf4_quantize_kernel<<<(int)grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(w), nblocks,
                                                     reinterpret_cast<uint32_t*>(packed), absmax);
  return cudaGetLastError();
}

cudaError_t launch_watchdog(DeviceError* err, long long timeout_ns, cudaStream_t stream) {
  LaunchScope scope("watchdog", stream);
  watchdog_kernel<<<1, 32, 0, stream>>>(err, timeout_ns);
  return cudaGetLastError();
}

}  // namespace e4b
