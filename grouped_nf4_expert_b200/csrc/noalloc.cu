// Routing entry point for callers that cannot allocate device memory.
//
// e4b_route_permute needs a caller-provided workspace for its per-CTA
// histograms and scatter bases.  Some callers have no way to provide one:
// code running while a CUDA graph is being captured in global mode (where
// cudaMalloc is not permitted), plugins of an inference engine that may only
// use memory the engine planned up front, or a runtime with a fixed device
// memory budget where an allocation in the middle of a step may fail.  This
// variant keeps that scratch in a fixed-size array in the library's own
// device memory instead, and allocates nothing.
#include <mutex>

#include "e4b_device.cuh"
#include "e4b_internal.h"

namespace e4b {
namespace {

// 4 MiB of int32: per-CTA expert histograms and scatter bases,
// 2 * ceil(T / kRouteTokensPerBlock) * E entries.  Every GPU that loads the
// library holds this array until the process exits.
constexpr int64_t kNoallocScratchInts = int64_t(1) << 20;
static __device__ __align__(256) int32_t g_route_scratch[kNoallocScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int32_t* g_scratch[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};

// Device address of the scratch array and the SM count of the current
// device.  The first call on a device looks both up (with that device
// current); later calls reuse them.  In host code `g_route_scratch` names a
// host-side stand-in, so only the looked-up address may be given to kernels.
cudaError_t setup_current_device(int32_t** scratch, int* sms) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch[dev] == nullptr) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_route_scratch);
    if (err != cudaSuccess) return err;
    int n = 0;
    err = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    g_sms[dev] = n;
    g_scratch[dev] = static_cast<int32_t*>(p);
  }
  *scratch = g_scratch[dev];
  *sms = g_sms[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace e4b

extern "C" e4b_status e4b_route_permute_noalloc(const e4b_moe_dims* dims, int32_t T, const float* logits,
                                                const e4b_bf16* x, const e4b_routing* routing, e4b_bf16* x_perm,
                                                e4b_stream_t stream) {
  using namespace e4b;
  e4b_sizes sz;
  const e4b_status st = e4b_get_sizes(dims, T, &sz);  // validates dims and T
  if (st != E4B_OK) return st;
  if (T == 0) return E4B_OK;  // nothing is read or written: T-sized pointers may be NULL
  if (routing == nullptr || !aligned16(routing->topk_ids) || !aligned16(routing->topk_w) ||
      !aligned16(routing->counts) || !aligned16(routing->offsets) || !aligned16(routing->row_of_slot) ||
      !aligned16(routing->slot_of_row) || !aligned16(routing->tiles) || !aligned16(logits) ||
      (x_perm != nullptr && (!aligned16(x) || !aligned16(x_perm))))
    return E4B_ERR_INVALID_ARG;
  const int64_t nblk = ((int64_t)T + kRouteTokensPerBlock - 1) / kRouteTokensPerBlock;
  if (2 * nblk * (int64_t)dims->E > kNoallocScratchInts) return E4B_ERR_UNSUPPORTED;
  int32_t* scratch = nullptr;
  int sms = 0;
  if (setup_current_device(&scratch, &sms) != cudaSuccess) {
    (void)cudaGetLastError();
    return E4B_ERR_CUDA;
  }
  // The histograms and bases are fully written by the routing kernels before
  // they are read, so nothing left in the array by an earlier call needs
  // clearing.
  const int64_t N = (int64_t)T * dims->top_k;
  if (launch_route(logits, x, T, dims->E, dims->H, dims->top_k, routing->topk_ids, routing->topk_w,
                   routing->counts, routing->offsets, routing->row_of_slot, routing->slot_of_row, routing->tiles,
                   mtiles_cap(N, dims->E), x_perm, rows_cap(N, dims->E), scratch, sms,
                   (cudaStream_t)stream) != cudaSuccess) {
    (void)cudaGetLastError();
    return E4B_ERR_CUDA;
  }
  return E4B_OK;
}
