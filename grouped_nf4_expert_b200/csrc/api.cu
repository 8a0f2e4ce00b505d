// C-ABI entry points (include/e4b.h): host-side validation, buffer sizes,
// workspace layout, tensor-map encoding and the launch sequence of each call.
// No entry point allocates device memory; only e4b_check_device_error
// synchronises.
#include <cudaTypedefs.h>
#include <math.h>
#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <vector>
#include <string.h>

#include "e4b_device.cuh"
#include "e4b_internal.h"

namespace e4b {

namespace {

constexpr int kMaxDevices = 64;
std::atomic<int> g_num_sms[kMaxDevices] = {};  // per device, filled on first use (any host thread)
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

cudaError_t device_sms(int* out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  int n = g_num_sms[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    err = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    g_num_sms[dev].store(n, std::memory_order_relaxed);
  }
  *out = n;
  return cudaSuccess;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int r_padded(int r) { return r <= 16 ? 16 : (r <= 32 ? 32 : 64); }

e4b_status check_dims(const e4b_moe_dims* d, int32_t T) {
  if (d == nullptr || T < 0) return E4B_ERR_INVALID_ARG;
  if (d->E < 1 || d->E > E4B_MAX_EXPERTS) return E4B_ERR_UNSUPPORTED;
  if (d->H <= 0 || d->H % 64 || d->I <= 0 || d->I % 64) return E4B_ERR_UNSUPPORTED;
  if (d->top_k < 1 || d->top_k > d->E || d->top_k > E4B_MAX_TOP_K) return E4B_ERR_UNSUPPORTED;
  if (d->r < 8 || d->r > E4B_MAX_RANK || d->r % 8) return E4B_ERR_UNSUPPORTED;
  if (d->blocksize != 64) return E4B_ERR_UNSUPPORTED;
  if (d->act != E4B_ACT_SILU_GLU) return E4B_ERR_UNSUPPORTED;
  if (!isfinite(d->alpha)) return E4B_ERR_INVALID_ARG;
  // 32-bit row and element indices inside the kernels
  const int64_t N = (int64_t)T * d->top_k;
  const int64_t rc = rows_cap(N, d->E);
  if (rc * (int64_t)(2 * d->I > d->H ? 2 * d->I : d->H) >= ((int64_t)1 << 40) || rc >= ((int64_t)1 << 30))
    return E4B_ERR_UNSUPPORTED;
  return E4B_OK;
}

size_t workspace_bytes(const e4b_moe_dims* d, int32_t T) {
  const int64_t nblk = ((int64_t)T + kRouteTokensPerBlock - 1) / kRouteTokensPerBlock;
  size_t ints = (size_t)2 * nblk * d->E;  // routing: per-block histograms and scatter bases
  const int64_t N = (int64_t)T * d->top_k;
  if (use_streaming_forward(N, d->E)) {  // the one-launch serving forward's counters and shares (after routing)
    const int64_t st_cap = stiles_cap(N, d->E);
    const size_t serve = ((size_t)serve_counters(d->E, st_cap, T, d->H) + 63) / 64 * 64 +
                         (size_t)serve_part_floats(st_cap, d->I, d->r);
    if (serve > ints) ints = serve;
  }
  return sizeof(DeviceError) + ((ints * sizeof(int32_t) + 255) / 256) * 256;
}

e4b_status check_ws(const e4b_moe_dims* d, int32_t T, const void* ws, size_t ws_bytes) {
  if (!aligned16(ws)) return E4B_ERR_INVALID_ARG;
  if (ws_bytes < workspace_bytes(d, T)) return E4B_ERR_WORKSPACE_TOO_SMALL;
  return E4B_OK;
}

e4b_status check_routing(const e4b_routing* r) {
  if (r == nullptr) return E4B_ERR_INVALID_ARG;
  if (!aligned16(r->topk_ids) || !aligned16(r->topk_w) || !aligned16(r->counts) || !aligned16(r->offsets) ||
      !aligned16(r->row_of_slot) || !aligned16(r->slot_of_row) || !aligned16(r->tiles))
    return E4B_ERR_INVALID_ARG;
  return E4B_OK;
}

e4b_status check_base(const e4b_nf4_experts* b) {
  if (b == nullptr || !aligned16(b->gate_up_nf4) || !aligned16(b->gate_up_absmax) || !aligned16(b->down_nf4) ||
      !aligned16(b->down_absmax))
    return E4B_ERR_INVALID_ARG;
  return E4B_OK;
}

e4b_status check_lora(const e4b_lora* l) {
  if (l == nullptr || !aligned16(l->A_gu) || !aligned16(l->B_gu) || !aligned16(l->A_d) || !aligned16(l->B_d))
    return E4B_ERR_INVALID_ARG;
  return E4B_OK;
}

e4b_status check_fwd(const e4b_fwd_buffers* f) {
  if (f == nullptr || !aligned16(f->x_perm) || !aligned16(f->p_gu) || !aligned16(f->gu) || !aligned16(f->act) ||
      !aligned16(f->p_d) || !aligned16(f->y_perm))
    return E4B_ERR_INVALID_ARG;
  return E4B_OK;
}

e4b_status check_bwd(const e4b_bwd_buffers* b) {
  if (b == nullptr || !aligned16(b->dyw) || !aligned16(b->q_d) || !aligned16(b->dgu) || !aligned16(b->q_gu) ||
      !aligned16(b->dx_perm))
    return E4B_ERR_INVALID_ARG;
  return E4B_OK;
}

#define E4B_TRY(expr)                     \
  do {                                    \
    const e4b_status _s = (expr);         \
    if (_s != E4B_OK) return _s;          \
  } while (0)

#define E4B_CUDA(expr)                      \
  do {                                      \
    if ((expr) != cudaSuccess) {            \
      (void)cudaGetLastError();             \
      return E4B_ERR_CUDA;                  \
    }                                       \
  } while (0)

}  // namespace

cudaError_t encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                              const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                              CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, []() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (g_encode == nullptr) return cudaErrorNotSupported;
  cuuint64_t d[5];
  cuuint64_t s[4];
  cuuint32_t b[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) s[i] = strides_bytes[i];
  }
  const CUresult r = g_encode(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), d, s, b, es,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// ---- launch counting and optional per-kernel event timing
namespace {
struct ProfRecord {
  const char* name;
  cudaEvent_t start, stop;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRecord> g_prof_records;
std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_prof_pool;
std::atomic<int64_t> g_launches{0};
}  // namespace

LaunchScope::LaunchScope(const char* name, cudaStream_t stream) : name_(name), stream_(stream), slot_(-1) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (!g_prof_on) return;
  // A launch being captured into a CUDA graph is counted but not timed: its
  // events would only be recorded when the graph replays.
  cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream_, &capture) != cudaSuccess) {
    (void)cudaGetLastError();
    return;
  }
  if (capture != cudaStreamCaptureStatusNone) return;
  std::pair<cudaEvent_t, cudaEvent_t> ev;
  if (!g_prof_pool.empty()) {
    ev = g_prof_pool.back();
    g_prof_pool.pop_back();
  } else if (cudaEventCreate(&ev.first) != cudaSuccess || cudaEventCreate(&ev.second) != cudaSuccess) {
    (void)cudaGetLastError();
    return;
  }
  if (cudaEventRecord(ev.first, stream_) != cudaSuccess) {
    (void)cudaGetLastError();
    g_prof_pool.push_back(ev);
    return;
  }
  slot_ = (int)g_prof_records.size();
  g_prof_records.push_back({name_, ev.first, ev.second});
}

LaunchScope::~LaunchScope() {
  if (slot_ < 0) return;
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (slot_ < (int)g_prof_records.size() && cudaEventRecord(g_prof_records[slot_].stop, stream_) != cudaSuccess)
    (void)cudaGetLastError();
}

}  // namespace e4b

using namespace e4b;

extern "C" {

const char* e4b_status_string(e4b_status s) {
  switch (s) {
    case E4B_OK: return "E4B_OK";
    case E4B_ERR_INVALID_ARG: return "E4B_ERR_INVALID_ARG: null or misaligned pointer, or inconsistent sizes";
    case E4B_ERR_UNSUPPORTED: return "E4B_ERR_UNSUPPORTED: shape, rank, block size or epilogue not supported";
    case E4B_ERR_WORKSPACE_TOO_SMALL: return "E4B_ERR_WORKSPACE_TOO_SMALL: workspace below e4b_get_sizes()";
    case E4B_ERR_CUDA: return "E4B_ERR_CUDA: a CUDA call or kernel launch failed";
    case E4B_ERR_DEVICE_TIMEOUT: return "E4B_ERR_DEVICE_TIMEOUT: a device-side wait ran out";
  }
  return "E4B_ERR_UNKNOWN";
}

const char* e4b_version(void) { return "e4b-b200 0.1.0 (sm_100a)"; }

void e4b_nf4_levels(float out[16]) {
  if (out != nullptr)
    for (int c = 0; c < 16; ++c) out[c] = nf4_level(c);
}

e4b_status e4b_get_sizes(const e4b_moe_dims* dims, int32_t T, e4b_sizes* out) {
  E4B_TRY(check_dims(dims, T));
  if (out == nullptr) return E4B_ERR_INVALID_ARG;
  const int64_t N = (int64_t)T * dims->top_k;
  out->slots = N;
  out->rows_cap = rows_cap(N, dims->E);
  out->tiles_cap = tiles_cap(N, dims->E);
  out->workspace_bytes = workspace_bytes(dims, T);
  return E4B_OK;
}

e4b_status e4b_workspace_init(void* ws, size_t ws_bytes, e4b_stream_t stream) {
  if (!aligned16(ws) || ws_bytes < sizeof(DeviceError)) return E4B_ERR_INVALID_ARG;
  E4B_CUDA(cudaMemsetAsync(ws, 0, sizeof(DeviceError), (cudaStream_t)stream));
  return E4B_OK;
}

e4b_status e4b_check_device_error(const void* ws, e4b_stream_t stream) {
  if (!aligned16(ws)) return E4B_ERR_INVALID_ARG;
  DeviceError host;
  E4B_CUDA(cudaMemcpyAsync(&host, ws, sizeof(DeviceError), cudaMemcpyDeviceToHost, (cudaStream_t)stream));
  E4B_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
  if (host.code == E4B_ERR_DEVICE_TIMEOUT) return E4B_ERR_DEVICE_TIMEOUT;
  if (host.code != 0) return E4B_ERR_CUDA;
  return E4B_OK;
}

e4b_status e4b_route_permute(const e4b_moe_dims* dims, int32_t T, const float* logits, const e4b_bf16* x,
                             const e4b_routing* routing, e4b_bf16* x_perm, void* ws, size_t ws_bytes,
                             e4b_stream_t stream) {
  E4B_TRY(check_dims(dims, T));
  if (T == 0) return E4B_OK;  // nothing is read or written: T-sized pointers may be NULL
  E4B_TRY(check_ws(dims, T, ws, ws_bytes));
  E4B_TRY(check_routing(routing));
  if (!aligned16(logits)) return E4B_ERR_INVALID_ARG;
  if (x_perm != nullptr && (!aligned16(x) || !aligned16(x_perm))) return E4B_ERR_INVALID_ARG;
  int sms = 0;
  E4B_CUDA(device_sms(&sms));
  const int64_t N = (int64_t)T * dims->top_k;
  int32_t* scratch = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + sizeof(DeviceError));
  E4B_CUDA(launch_route(logits, x, T, dims->E, dims->H, dims->top_k, routing->topk_ids, routing->topk_w,
                        routing->counts, routing->offsets, routing->row_of_slot, routing->slot_of_row, routing->tiles,
                        mtiles_cap(N, dims->E), x_perm, rows_cap(N, dims->E), scratch, sms,
                        (cudaStream_t)stream));
  return E4B_OK;
}

e4b_status e4b_grouped_nf4_lora_fwd(const e4b_moe_dims* dims, int32_t T, const e4b_routing* routing,
                                    const e4b_nf4_experts* base, const e4b_lora* lora, const e4b_bf16* x,
                                    const e4b_fwd_buffers* fwd, e4b_bf16* y, void* ws, size_t ws_bytes,
                                    e4b_stream_t stream) {
  E4B_TRY(check_dims(dims, T));
  if (T == 0) return E4B_OK;  // nothing is read or written: T-sized pointers may be NULL
  E4B_TRY(check_ws(dims, T, ws, ws_bytes));
  E4B_TRY(check_routing(routing));
  E4B_TRY(check_base(base));
  E4B_TRY(check_lora(lora));
  E4B_TRY(check_fwd(fwd));
  if (!aligned16(y)) return E4B_ERR_INVALID_ARG;
  if (x != nullptr && !aligned16(x)) return E4B_ERR_INVALID_ARG;
  int sms = 0;
  E4B_CUDA(device_sms(&sms));
  const cudaStream_t st = (cudaStream_t)stream;
  const int E = dims->E, H = dims->H, I = dims->I, r = dims->r, k = dims->top_k;
  const int64_t N = (int64_t)T * k;
  const float s = dims->alpha / (float)r;
  DeviceError* err = static_cast<DeviceError*>(ws);

  LoraProjHost lp{};
  lp.E = E;
  lp.r = r;
  lp.r_pad = r_padded(r);
  lp.scale = s;
  lp.tiles = routing->tiles;
  lp.rows_cap = rows_cap(N, E);
  lp.mt_cap = mtiles_cap(N, E);
  lp.err = err;
  lp.timeout_ns = kDefaultTimeoutNs;

  Nf4GemmHost g{};
  g.E = E;
  g.H = H;
  g.I = I;
  g.r = r;
  g.r_pad = r_padded(r);
  g.tiles = routing->tiles;
  g.rows_cap = lp.rows_cap;
  g.mt_cap = lp.mt_cap;
  g.err = err;
  g.timeout_ns = kDefaultTimeoutNs;

  // p_gu = s * x_perm A_gu^T; with x given, x_perm is gathered in the same pass
  lp.act_in = fwd->x_perm;
  lp.K = H;
  lp.w = lora->A_gu;
  lp.w_mn_major = false;
  lp.out = fwd->p_gu;
  if (x != nullptr) {
    lp.gather_src = reinterpret_cast<const uint16_t*>(x);
    lp.slot_of_row = routing->slot_of_row;
    lp.gather_w = nullptr;
    lp.k = k;
    E4B_CUDA(launch_gather_proj(lp, sms, st));
    lp.gather_src = nullptr;
  } else {
    E4B_CUDA(launch_lora_proj(lp, sms, st));
  }
  // gu = W_gu x + p_gu B_gu^T ; act = silu(gate) * up
  g.mode = kFwdGateUp;
  g.nf4 = base->gate_up_nf4;
  g.absmax = base->gate_up_absmax;
  g.stored_rows = 2 * I;
  g.stored_cols = H;
  g.act_in = fwd->x_perm;
  g.K = H;
  g.n_dim = 2 * I;
  g.lora_a_rows = fwd->p_gu;
  g.lora_w = lora->B_gu;
  g.out0 = fwd->gu;
  g.out1 = fwd->act;
  g.aux = nullptr;
  const bool streaming = use_streaming_forward(N, E);  // decode-sized batch: weight-streaming tiles
  E4B_CUDA(streaming ? launch_nf4_stream(g, sms, st) : launch_nf4_gemm(g, sms, st));
  // p_d = s * act A_d^T
  lp.act_in = fwd->act;
  lp.K = I;
  lp.w = lora->A_d;
  lp.out = fwd->p_d;
  E4B_CUDA(launch_lora_proj(lp, sms, st));
  // y_perm = W_d act + p_d B_d^T
  g.mode = kFwdDown;
  g.nf4 = base->down_nf4;
  g.absmax = base->down_absmax;
  g.stored_rows = H;
  g.stored_cols = I;
  g.act_in = fwd->act;
  g.K = I;
  g.n_dim = H;
  g.lora_a_rows = fwd->p_d;
  g.lora_w = lora->B_d;
  g.out0 = fwd->y_perm;
  g.out1 = nullptr;
  E4B_CUDA(streaming ? launch_nf4_stream(g, sms, st) : launch_nf4_gemm(g, sms, st));
  // y[t] = sum_j w[t,j] y_perm[row(t,j)]
  E4B_CUDA(launch_combine(fwd->y_perm, routing->row_of_slot, routing->topk_w, T, k, H, y, sms, st));
  return E4B_OK;
}

e4b_status e4b_moe_serve_fwd(const e4b_moe_dims* dims, int32_t T, const float* logits, const e4b_bf16* x,
                             const e4b_routing* routing, const e4b_nf4_experts* base, const e4b_lora* lora,
                             const e4b_fwd_buffers* fwd, e4b_bf16* y, void* ws, size_t ws_bytes,
                             e4b_stream_t stream) {
  E4B_TRY(check_dims(dims, T));
  if (T == 0) return E4B_OK;  // nothing is read or written: T-sized pointers may be NULL
  E4B_TRY(check_ws(dims, T, ws, ws_bytes));
  E4B_TRY(check_routing(routing));
  E4B_TRY(check_base(base));
  E4B_TRY(check_lora(lora));
  if (fwd == nullptr || !aligned16(fwd->x_perm) || !aligned16(fwd->p_gu) || !aligned16(fwd->act) ||
      !aligned16(fwd->p_d) || !aligned16(fwd->y_perm) || (fwd->gu != nullptr && !aligned16(fwd->gu)))
    return E4B_ERR_INVALID_ARG;
  if (!aligned16(logits) || !aligned16(x) || !aligned16(y)) return E4B_ERR_INVALID_ARG;
  const int64_t N = (int64_t)T * dims->top_k;
  if (!use_streaming_forward(N, dims->E)) {
    // a prefill-sized batch: the training forward (it writes gu, so gu is required)
    if (fwd->gu == nullptr) return E4B_ERR_INVALID_ARG;
    E4B_TRY(e4b_route_permute(dims, T, logits, x, routing, nullptr, ws, ws_bytes, stream));
    return e4b_grouped_nf4_lora_fwd(dims, T, routing, base, lora, x, fwd, y, ws, ws_bytes, stream);
  }
  int sms = 0;
  E4B_CUDA(device_sms(&sms));
  const cudaStream_t st = (cudaStream_t)stream;
  const int E = dims->E, H = dims->H, I = dims->I, r = dims->r, k = dims->top_k;
  const float s = dims->alpha / (float)r;
  int32_t* scratch = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + sizeof(DeviceError));
  const int64_t st_cap = stiles_cap(N, E);
  // routing (one CTA for up to 64 tokens), which also zeroes the counters of the launch after it
  E4B_CUDA(launch_route_serve(logits, T, E, H, k, routing->topk_ids, routing->topk_w, routing->counts,
                              routing->offsets, routing->row_of_slot, routing->slot_of_row, routing->tiles,
                              mtiles_cap(N, E), rows_cap(N, E), scratch, sms, st, scratch,
                              serve_counters(E, st_cap, T, H)));
  // everything else in one launch: x scatter + p_gu, gate_up + SiLU gate, p_d, down, weighted combine
  ServeHost h{};
  h.T = T;
  h.k = k;
  h.E = E;
  h.H = H;
  h.I = I;
  h.r = r;
  h.r_pad = r_padded(r);
  h.s = s;
  h.gate_up_nf4 = base->gate_up_nf4;
  h.gate_up_absmax = base->gate_up_absmax;
  h.down_nf4 = base->down_nf4;
  h.down_absmax = base->down_absmax;
  h.A_gu = lora->A_gu;
  h.B_gu = lora->B_gu;
  h.A_d = lora->A_d;
  h.B_d = lora->B_d;
  h.x = reinterpret_cast<const uint16_t*>(x);
  h.x_perm = fwd->x_perm;
  h.p_gu = fwd->p_gu;
  h.gu = fwd->gu;
  h.act = fwd->act;
  h.p_d = fwd->p_d;
  h.y_perm = fwd->y_perm;
  h.y = reinterpret_cast<uint16_t*>(y);
  h.topk_ids = routing->topk_ids;
  h.topk_w = routing->topk_w;
  h.row_of_slot = routing->row_of_slot;
  h.slot_of_row = routing->slot_of_row;
  h.counts = routing->counts;
  h.tiles = routing->tiles;
  h.counters = scratch;
  h.pd_part = reinterpret_cast<float*>(scratch + (serve_counters(E, st_cap, T, H) + 63) / 64 * 64);
  h.rows_cap = rows_cap(N, E);
  h.mt_cap = mtiles_cap(N, E);
  h.st_cap = st_cap;
  h.err = static_cast<DeviceError*>(ws);
  h.timeout_ns = kDefaultTimeoutNs;
  E4B_CUDA(launch_nf4_serve(h, sms, st));
  return E4B_OK;
}

e4b_status e4b_grouped_nf4_lora_dgrad(const e4b_moe_dims* dims, int32_t T, const e4b_routing* routing,
                                      const e4b_nf4_experts* base, const e4b_lora* lora,
                                      const e4b_fwd_buffers* fwd, const e4b_bf16* dY, const e4b_bwd_buffers* bwd,
                                      e4b_bf16* dx, void* ws, size_t ws_bytes, e4b_stream_t stream) {
  E4B_TRY(check_dims(dims, T));
  if (T == 0) return E4B_OK;  // nothing is read or written: T-sized pointers may be NULL
  E4B_TRY(check_ws(dims, T, ws, ws_bytes));
  E4B_TRY(check_routing(routing));
  E4B_TRY(check_base(base));
  E4B_TRY(check_lora(lora));
  E4B_TRY(check_fwd(fwd));
  E4B_TRY(check_bwd(bwd));
  if (!aligned16(dY) || !aligned16(dx)) return E4B_ERR_INVALID_ARG;
  int sms = 0;
  E4B_CUDA(device_sms(&sms));
  const cudaStream_t st = (cudaStream_t)stream;
  const int E = dims->E, H = dims->H, I = dims->I, r = dims->r, k = dims->top_k;
  const int64_t N = (int64_t)T * k;
  const float s = dims->alpha / (float)r;
  DeviceError* err = static_cast<DeviceError*>(ws);

  LoraProjHost lp{};
  lp.E = E;
  lp.r = r;
  lp.r_pad = r_padded(r);
  lp.scale = s;
  lp.tiles = routing->tiles;
  lp.rows_cap = rows_cap(N, E);
  lp.mt_cap = mtiles_cap(N, E);
  lp.err = err;
  lp.timeout_ns = kDefaultTimeoutNs;
  Nf4GemmHost g{};
  g.E = E;
  g.H = H;
  g.I = I;
  g.r = r;
  g.r_pad = r_padded(r);
  g.tiles = routing->tiles;
  g.rows_cap = lp.rows_cap;
  g.mt_cap = lp.mt_cap;
  g.err = err;
  g.timeout_ns = kDefaultTimeoutNs;

  // dyw[row] = w(slot) * dY[token] and q_d = s * dyw B_d, in one pass over the gathered rows
  lp.act_in = bwd->dyw;
  lp.K = H;
  lp.w = lora->B_d;
  lp.w_mn_major = true;
  lp.out = bwd->q_d;
  lp.gather_src = reinterpret_cast<const uint16_t*>(dY);
  lp.slot_of_row = routing->slot_of_row;
  lp.gather_w = routing->topk_w;
  lp.k = k;
  E4B_CUDA(launch_gather_proj(lp, sms, st));
  // dact = dyw W_d + q_d A_d ; dgu = SwiGLU backward(dact, gu)
  g.mode = kDgradDown;
  g.nf4 = base->down_nf4;
  g.absmax = base->down_absmax;
  g.stored_rows = H;
  g.stored_cols = I;
  g.act_in = bwd->dyw;
  g.K = H;
  g.n_dim = I;
  g.lora_a_rows = bwd->q_d;
  g.lora_w = lora->A_d;
  g.out0 = bwd->dgu;
  g.out1 = nullptr;
  g.aux = fwd->gu;
  E4B_CUDA(launch_nf4_gemm(g, sms, st));
  // q_gu = s * dgu B_gu
  lp.act_in = bwd->dgu;
  lp.K = 2 * I;
  lp.w = lora->B_gu;
  lp.out = bwd->q_gu;
  E4B_CUDA(launch_lora_proj(lp, sms, st));
  // dx_perm = dgu W_gu + q_gu A_gu
  g.mode = kDgradGateUp;
  g.nf4 = base->gate_up_nf4;
  g.absmax = base->gate_up_absmax;
  g.stored_rows = 2 * I;
  g.stored_cols = H;
  g.act_in = bwd->dgu;
  g.K = 2 * I;
  g.n_dim = H;
  g.lora_a_rows = bwd->q_gu;
  g.lora_w = lora->A_gu;
  g.out0 = bwd->dx_perm;
  g.aux = nullptr;
  E4B_CUDA(launch_nf4_gemm(g, sms, st));
  // dx[t] = sum_j dx_perm[row(t,j)]
  E4B_CUDA(launch_combine(bwd->dx_perm, routing->row_of_slot, nullptr, T, k, H, dx, sms, st));
  return E4B_OK;
}

e4b_status e4b_lora_wgrad(const e4b_moe_dims* dims, int32_t T, const e4b_routing* routing,
                          const e4b_fwd_buffers* fwd, const e4b_bwd_buffers* bwd, e4b_bf16* dA_gu, e4b_bf16* dB_gu,
                          e4b_bf16* dA_d, e4b_bf16* dB_d, void* ws, size_t ws_bytes, e4b_stream_t stream) {
  E4B_TRY(check_dims(dims, T));
  E4B_TRY(check_ws(dims, T, ws, ws_bytes));
  E4B_TRY(check_routing(routing));
  E4B_TRY(check_fwd(fwd));
  E4B_TRY(check_bwd(bwd));
  if (!aligned16(dA_gu) || !aligned16(dB_gu) || !aligned16(dA_d) || !aligned16(dB_d)) return E4B_ERR_INVALID_ARG;
  int sms = 0;
  E4B_CUDA(device_sms(&sms));
  const int E = dims->E, H = dims->H, I = dims->I, r = dims->r;
  const int64_t N = (int64_t)T * dims->top_k;
  if (T == 0) {
    // No tokens: every gradient is exactly zero.
    const cudaStream_t st = (cudaStream_t)stream;
    E4B_CUDA(cudaMemsetAsync(dB_gu, 0, (size_t)E * 2 * I * r * 2, st));
    E4B_CUDA(cudaMemsetAsync(dA_gu, 0, (size_t)E * r * H * 2, st));
    E4B_CUDA(cudaMemsetAsync(dB_d, 0, (size_t)E * H * r * 2, st));
    E4B_CUDA(cudaMemsetAsync(dA_d, 0, (size_t)E * r * I * 2, st));
    return E4B_OK;
  }
  WgradHost w{};
  w.act[0] = bwd->dgu;  // dB_gu = dgu^T p_gu
  w.low[0] = fwd->p_gu;
  w.out[0] = dB_gu;
  w.F[0] = 2 * I;
  w.transposed[0] = false;
  w.act[1] = fwd->x_perm;  // dA_gu = (x^T q_gu)^T
  w.low[1] = bwd->q_gu;
  w.out[1] = dA_gu;
  w.F[1] = H;
  w.transposed[1] = true;
  w.act[2] = bwd->dyw;  // dB_d = dyw^T p_d
  w.low[2] = fwd->p_d;
  w.out[2] = dB_d;
  w.F[2] = H;
  w.transposed[2] = false;
  w.act[3] = fwd->act;  // dA_d = (act^T q_d)^T
  w.low[3] = bwd->q_d;
  w.out[3] = dA_d;
  w.F[3] = I;
  w.transposed[3] = true;
  w.E = E;
  w.r = r;
  w.r_pad = r_padded(r);
  w.counts = routing->counts;
  w.offsets = routing->offsets;
  w.tiles = routing->tiles;
  w.rows_cap = rows_cap(N, E);
  w.mt_cap = mtiles_cap(N, E);
  w.err = static_cast<DeviceError*>(ws);
  w.timeout_ns = kDefaultTimeoutNs;
  E4B_CUDA(launch_wgrad(w, sms, (cudaStream_t)stream));
  return E4B_OK;
}

e4b_status e4b_router_backward(const e4b_moe_dims* dims, int32_t T, const e4b_routing* routing,
                               const e4b_bf16* y_perm, const e4b_bf16* dY, float* d_logits, float* dw,
                               e4b_stream_t stream) {
  E4B_TRY(check_dims(dims, T));
  if (T == 0) return E4B_OK;  // nothing is read or written: T-sized pointers may be NULL
  E4B_TRY(check_routing(routing));
  if (!aligned16(y_perm) || !aligned16(dY) || !aligned16(d_logits)) return E4B_ERR_INVALID_ARG;
  if (dw != nullptr && !aligned16(dw)) return E4B_ERR_INVALID_ARG;
  int sms = 0;
  E4B_CUDA(device_sms(&sms));
  E4B_CUDA(launch_router_bwd(reinterpret_cast<const uint16_t*>(dY), reinterpret_cast<const uint16_t*>(y_perm),
                             routing->row_of_slot, routing->topk_ids, routing->topk_w, T, dims->top_k, dims->H,
                             dims->E, d_logits, dw, sms, (cudaStream_t)stream));
  return E4B_OK;
}

e4b_status e4b_nf4_dequant(const uint8_t* packed, const float* absmax, int64_t n, e4b_bf16* out,
                           e4b_stream_t stream) {
  if (n < 0 || n % 64) return E4B_ERR_INVALID_ARG;
  if (n == 0) return E4B_OK;
  if (!aligned16(packed) || absmax == nullptr || (reinterpret_cast<uintptr_t>(absmax) & 3u) || !aligned16(out))
    return E4B_ERR_INVALID_ARG;
  int sms = 0;
  E4B_CUDA(device_sms(&sms));
  E4B_CUDA(launch_nf4_dequant(packed, absmax, n, out, sms, (cudaStream_t)stream));
  return E4B_OK;
}

e4b_status e4b_nf4_quantize(const e4b_bf16* w, int64_t n, uint8_t* packed, float* absmax, e4b_stream_t stream) {
  if (n < 0 || n % 64) return E4B_ERR_INVALID_ARG;
  if (n == 0) return E4B_OK;
  if (!aligned16(w) || !aligned16(packed) || absmax == nullptr || (reinterpret_cast<uintptr_t>(absmax) & 3u))
    return E4B_ERR_INVALID_ARG;
  int sms = 0;
  E4B_CUDA(device_sms(&sms));
  E4B_CUDA(launch_nf4_quantize(reinterpret_cast<const uint16_t*>(w), n, packed, absmax, sms, (cudaStream_t)stream));
  return E4B_OK;
}

e4b_status e4b_profiler_enable(int32_t on) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  g_prof_on = on != 0;
  return E4B_OK;
}

e4b_status e4b_profiler_read(e4b_kernel_time* out, int32_t capacity, int32_t* count) {
  if (count == nullptr || capacity < 0 || (capacity > 0 && out == nullptr)) return E4B_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_prof_mu);
  std::map<std::string, std::pair<int64_t, double>> acc;
  std::vector<std::string> order;
  e4b_status st = E4B_OK;
  for (const ProfRecord& r : g_prof_records) {
    float ms = 0.0f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) {
      (void)cudaGetLastError();
      st = E4B_ERR_CUDA;
    }
    auto it = acc.find(r.name);
    if (it == acc.end()) {
      order.push_back(r.name);
      acc[r.name] = {1, (double)ms};
    } else {
      it->second.first += 1;
      it->second.second += ms;
    }
    g_prof_pool.push_back({r.start, r.stop});
  }
  g_prof_records.clear();
  int n = 0;
  for (const std::string& name : order) {
    if (n < capacity) {
      memset(out[n].name, 0, sizeof(out[n].name));
      strncpy(out[n].name, name.c_str(), sizeof(out[n].name) - 1);
      out[n].launches = acc[name].first;
      out[n].total_ms = acc[name].second;
    }
    ++n;
  }
  *count = n;
  return st;
}

int64_t e4b_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

e4b_status e4b_debug_watchdog(void* ws, size_t ws_bytes, int64_t timeout_ns, e4b_stream_t stream) {
  if (!aligned16(ws) || ws_bytes < sizeof(DeviceError) || timeout_ns <= 0 || timeout_ns > 10000000000LL)
    return E4B_ERR_INVALID_ARG;
  E4B_CUDA(launch_watchdog(static_cast<DeviceError*>(ws), (long long)timeout_ns, (cudaStream_t)stream));
  return E4B_OK;
}

}  // extern "C"
