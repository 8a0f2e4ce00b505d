// Serving forward for decode-sized batches in one persistent launch.
//
// After routing, the whole block -- the x scatter with its LoRA projection,
// the gate_up weight-streaming GEMM with the SiLU-gated epilogue, the LoRA
// down projection, the down weight-streaming GEMM and the router-weighted
// combine -- runs in ONE grid of persistent CTAs (one per SM).  The work is a
// list of units taken in this order:
//
//   prep:  every CTA first gathers a few routed slots' token rows into the
//          permuted buffer and projects them, p_gu = s x A_gu[e]^T, on the
//          CUDA cores (warps that are idle until their first unit arrives);
//   A:     (slot tile, 64-row gate/up tile) of the gate_up stack: weights are
//          the UMMA M operand (NF4 decoded into tensor memory), up to 32 slots
//          of one expert the N operand; epilogue act = silu(g) * u;
//          each A unit also forms its 64 features' share of the LoRA down
//          projection, act A_d[e]^T over those features, on the CUDA cores,
//          and the unit that completes a slot tile sums the shares in unit
//          order into p_d = s act A_d[e]^T (deterministic);
//   B:     (slot tile, 128-row tile) of the down stack, as A, epilogue y_perm;
//          once all k slots of a token have their rows of a 128-column piece
//          of y_perm, the warp that completed the last of them forms that
//          piece of y[t] = sum_j w[t,j] y_perm[row(t,j)] (fp32, j ascending).
//
// Each unit waits only for work earlier in the list: an A unit for its
// expert's prep, a B unit for its slot tile's p_d (its last A unit).  The waits are device-wide counters and flags written with
// release and read with acquire, polled with a bounded wait (a timeout records
// E4B_ERR_DEVICE_TIMEOUT and the CTA stops), and only the activation loader
// waits: by then every earlier unit of its own CTA has been handed to the
// other roles, which finish it without waiting on anything else.  The
// counters live in the caller's workspace and are zeroed by the routing
// launch that precedes this one.
//
// Pages: "How do I QLoRA-train the fused experts of a MoE", sections "The
// abstraction that fails" (per-expert delta before the activation, act(gate)
// * up) and "Why it happens" (scaling * (x @ A.T) @ B.T); experts4bit-qlora
// package METADATA, section "The package family" (one launch over the packed
// 4-bit expert stacks, codes decoded in registers, fp32 sums) and its
// decode/serving use.
#include "e4b_device.cuh"
#include "e4b_internal.h"

namespace e4b {

namespace {
constexpr uint32_t kFull = 0xffffffffu;
}  // namespace

namespace nf4v {
constexpr int BM = 128;          // weight rows per tile (UMMA M)
constexpr int BN = 32;           // routed slots per tile (UMMA N)
constexpr int BK = 64;
constexpr int RAW_CHUNKS = 4;    // k-chunks per NF4 code stage (128 code bytes per weight row)
constexpr int kTeams = 3;        // decode teams of 4 warps
constexpr int RAW_STAGES = 6;    // slot r always goes to team r % 3
constexpr int X_STAGES = 4;
constexpr int CODE_BYTES = BM * RAW_CHUNKS * BK / 2;   // 16384
constexpr int AMAX_BYTES = BM * RAW_CHUNKS * 4;        // 2048
constexpr int RAW_SLOT = CODE_BYTES + AMAX_BYTES;      // 18432
constexpr int X_BYTES = BN * BK * 2;                   // 4096 per chunk
constexpr int XS_BYTES = RAW_CHUNKS * X_BYTES;         // 16384 per stage
constexpr int LA_BYTES = BM * E4B_MAX_RANK * 2;
constexpr int LB_BYTES = BN * E4B_MAX_RANK * 2;
constexpr int EPI_BYTES = 64 * BN * 4;                 // up values handed to the gate lanes
constexpr int kHand = 4;                               // hand-off ring: epilogue -> publisher
constexpr int kQ = 16;                                 // claimed-unit queue: producer -> the other roles
constexpr int kQConsumers = 19;                        // warps 1-3 and 4-19 read every queue entry
constexpr int ACTS_BYTES = kHand * 64 * BN * 2;        // act tiles (bf16) of the A units in the ring
constexpr int RAW_OFF = 0;
constexpr int X_OFF = RAW_STAGES * RAW_SLOT;
constexpr int LA_OFF = X_OFF + X_STAGES * XS_BYTES;
constexpr int LB_OFF = LA_OFF + LA_BYTES;
constexpr int EPI_OFF = LB_OFF + LB_BYTES;
constexpr int ACTS_OFF = EPI_OFF + EPI_BYTES;
constexpr int BAR_OFF = ACTS_OFF + ACTS_BYTES;
constexpr int SMEM_BYTES = BAR_OFF + 1024 + 1024;
constexpr int kPrepWarp0 = 4;                          // warps 4..19 (teams, epilogue) run the prep first
constexpr int kPrepWarps = 16;
constexpr int kPubWarp = 3;                            // publishes finished units to the other CTAs
constexpr int kEpiWarp0 = 4 + 4 * kTeams;
constexpr int kThreads = 32 * (kEpiWarp0 + 4);         // 640
constexpr int kAccCols = BN;
constexpr int kACols = BK / 2;
constexpr int kAOff = 128;
constexpr int kTeamCols = RAW_CHUNKS * kACols;
constexpr int kTmemCols = 512;
constexpr int kRawFullCount = 1 + 32;
static_assert(X_OFF % 1024 == 0 && LA_OFF % 1024 == 0 && LB_OFF % 1024 == 0, "swizzle atom alignment");
static_assert(SMEM_BYTES > 232448 / 2 && SMEM_BYTES <= 232448, "one CTA per SM, within the budget");
static_assert(RAW_STAGES % kTeams == 0, "each code slot belongs to one team");
static_assert(kAOff + kTeams * kTeamCols <= kTmemCols && 2 * kAccCols <= kAOff, "TMEM budget");
static_assert(kThreads / 32 - kPrepWarp0 == kPrepWarps, "prep group: warps 4..19");
static_assert(kQConsumers == kThreads / 32 - 1, "every warp but the producer reads the unit queue");
}  // namespace nf4v

struct ServeParams {
  const float* gu_absmax;      // [E, 2I, H/64]
  const float* d_absmax;       // [E, H, I/64]
  const uint16_t* x;           // [T, H]
  const uint16_t* A_gu;        // [E, r, H]
  const uint16_t* A_d;         // [E, r, I]
  uint16_t* x_perm;            // [rows_cap, H]
  uint16_t* p_gu;              // [rows_cap, r]
  uint16_t* gu;                // [rows_cap, 2I] or nullptr
  uint16_t* act;               // [rows_cap, I]
  uint16_t* p_d;               // [rows_cap, r]
  uint16_t* y_perm;            // [rows_cap, H]
  uint16_t* y;                 // [T, H]
  const int32_t* topk_ids;     // [T*k]
  const float* topk_w;         // [T*k]
  const int32_t* row_of_slot;  // [T*k]
  const int32_t* slot_of_row;  // [rows_cap]
  const int32_t* counts;       // [E]
  const int32_t* tiles;
  int64_t st_offset;
  int32_t* cnt_prep;           // [E] slots prepped per expert
  int32_t* cnt_a;              // [slot tiles] A-unit epilogue warps done
  int32_t* pd_ready;           // [slot tiles] p_d written
  float* pd_part;              // [slot tiles][I/64][32][r] each A unit's share of act A_d^T
  int32_t* cnt_comb;           // [T * nB_mt] slots of a token whose y_perm piece is written
  int32_t* claim;              // next unit of the list to hand out
  DeviceError* err;
  long long timeout_ns;
  int T, k, E, H, I, r, r_pad;
  float s;
  int nA_mt, nB_mt;            // I / 64 gate/up tiles; ceil(H / 128) down tiles
};

// Unit kinds, in list order.
enum : int { kUnitA = 0, kUnitB = 1 };

struct ServeUnit {
  int kind, st, mt;
  int e, row0, nslots;
  int kchunks;     // k-chunks of 64 over the reduction
  int nq;          // code stages of RAW_CHUNKS k-chunks
  int rA, rB;      // stored weight rows of the tile (two 64-row halves)
  int stored_rows;
};

__device__ __forceinline__ ServeUnit serve_unit(const ServeParams& p, const int32_t* stiles, int n_st, int u) {
  ServeUnit w;
  const int nA = n_st * p.nA_mt;
  if (u < nA) {
    w.kind = kUnitA;
    w.st = u / p.nA_mt;
    w.mt = u - w.st * p.nA_mt;
    w.kchunks = p.H / nf4v::BK;
    w.rA = w.mt * 64;
    w.rB = p.I + w.mt * 64;
    w.stored_rows = 2 * p.I;
  } else {
    w.kind = kUnitB;
    const int v = u - nA;
    w.st = v / p.nB_mt;
    w.mt = v - w.st * p.nB_mt;
    w.kchunks = p.I / nf4v::BK;
    w.rA = w.mt * 128;
    w.rB = w.mt * 128 + 64;
    w.stored_rows = p.H;
  }
  w.nq = (w.kchunks + nf4v::RAW_CHUNKS - 1) / nf4v::RAW_CHUNKS;
  w.e = stiles[3 * w.st];
  w.row0 = stiles[3 * w.st + 1];
  w.nslots = stiles[3 * w.st + 2];
  return w;
}

__device__ __forceinline__ int ld_acquire_gpu(const int32_t* a) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add_gpu(int32_t* a, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(a), "r"(v) : "memory");
}
__device__ __forceinline__ int atom_acq_rel_add_gpu(int32_t* a, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(a), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void st_release_gpu(int32_t* a, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(a), "r"(v) : "memory");
}
// Orders this thread's generic-proxy global accesses with its later async-proxy (TMA) accesses.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Bounded wait until *flag >= want (acquire).  Gives up on the CTA's abort
// flag or after timeout_ns, recording E4B_ERR_DEVICE_TIMEOUT with `site`.
__device__ __forceinline__ bool wait_counter(const int32_t* flag, int want, CtaControl* ctl, DeviceError* err,
                                             long long timeout_ns, int site) {
  if (ld_acquire_gpu(flag) >= want) return true;
  const long long c0 = clock64(), limit = wait_limit_cycles(timeout_ns);
  while (true) {
    __nanosleep(200);
    if (ld_acquire_gpu(flag) >= want) return true;
    if (ctl->abort) return false;
    if (clock64() - c0 > limit) {
      ctl->abort = 1;
      record_error(err, E4B_ERR_DEVICE_TIMEOUT, site);
      return false;
    }
  }
}

__global__ void __launch_bounds__(nf4v::kThreads, 1)
    nf4_serve_kernel(const __grid_constant__ CUtensorMap map_gu_raw, const __grid_constant__ CUtensorMap map_d_raw,
                     const __grid_constant__ CUtensorMap map_x,
                     const __grid_constant__ CUtensorMap map_act, const __grid_constant__ CUtensorMap map_lw_gu,
                     const __grid_constant__ CUtensorMap map_lw_d, const __grid_constant__ CUtensorMap map_lp_gu,
                     const __grid_constant__ CUtensorMap map_lp_d, const ServeParams p) {
  using namespace nf4v;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = align1024(smem_dyn);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* raw_full = bars;                         // [RAW_STAGES]
  uint64_t* raw_empty = raw_full + RAW_STAGES;       // [RAW_STAGES]
  uint64_t* a_ready = raw_empty + RAW_STAGES;        // [kTeams]
  uint64_t* a_empty = a_ready + kTeams;              // [kTeams]
  uint64_t* x_full = a_empty + kTeams;               // [X_STAGES]
  uint64_t* x_empty = x_full + X_STAGES;             // [X_STAGES]
  uint64_t* drain = x_empty + X_STAGES;
  uint64_t* lfull = drain + 1;
  uint64_t* lempty = lfull + 1;
  uint64_t* accfull = lfull + 2;                     // [2]
  uint64_t* accempty = lfull + 4;                    // [2]
  uint64_t* epi_full = lfull + 6;
  uint64_t* epi_empty = lfull + 7;
  uint64_t* hand_full = lfull + 8;                   // [kHand] a unit's outputs stored (four epilogue warps)
  uint64_t* hand_empty = hand_full + kHand;          // [kHand] the publisher is done with that unit
  uint64_t* q_full = hand_empty + kHand;             // [kQ] a claimed unit published by the producer
  uint64_t* q_empty = q_full + kQ;                   // [kQ] every other role has read it
  int* uq = reinterpret_cast<int*>(q_empty + kQ);    // [kQ] claimed unit ids (-1: no more)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_empty + kQ + kQ / 2);
  CtaControl* ctl = reinterpret_cast<CtaControl*>(q_empty + kQ + kQ / 2 + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < RAW_STAGES; ++s) {
      mbar_init(&raw_full[s], kRawFullCount);
      mbar_init(&raw_empty[s], 4);
    }
    for (int m = 0; m < kTeams; ++m) {
      mbar_init(&a_ready[m], 4);
      mbar_init(&a_empty[m], 1);
    }
    for (int s = 0; s < X_STAGES; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], 1);
    }
    mbar_init(drain, 1);
    mbar_init(lfull, 1);
    mbar_init(lempty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 4);
    }
    mbar_init(epi_full, 2);
    mbar_init(epi_empty, 2);
    for (int b = 0; b < kHand; ++b) {
      mbar_init(&hand_full[b], 4);
      mbar_init(&hand_empty[b], 1);
    }
    for (int q = 0; q < kQ; ++q) {
      mbar_init(&q_full[q], 1);
      mbar_init(&q_empty[q], kQConsumers);
    }
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int32_t* stiles = p.tiles + p.st_offset;
  const int n_st = p.tiles[3];
  const int n_units = n_st * (p.nA_mt + p.nB_mt);
  const int N = p.T * p.k;
  // The units are handed out in list order from a device-wide counter: the producer warp claims one
  // when it is about to load it and publishes the id to the CTA's other roles through a queue, so
  // every CTA works until the list runs out and a unit is only ever claimed by a running CTA.  Whole
  // warp: the id of this CTA's i-th unit, or -1 once the list is exhausted (or a wait gave up).
  auto next_unit = [&](uint32_t i, int site) -> int {
    const uint32_t qs = i % kQ, qph = (i / kQ) & 1;
    if (!__all_sync(kFull, mbar_wait_lazy(&q_full[qs], qph, ctl, p.err, p.timeout_ns, site, 64))) return -1;
    const int u = uq[qs];
    __syncwarp();
    if (lane == 0) mbar_arrive(&q_empty[qs]);
    return u;
  };

  if (warp == 0) {
    // ------------------------------------------------ weights: NF4 codes + absmax
    if (lane == 0) {
      tma_prefetch_desc(&map_gu_raw);
      tma_prefetch_desc(&map_d_raw);
    }
    uint32_t j = 0, issued = 0, last_par = 0;
    bool ok = true;
    for (uint32_t ui = 0; ok; ++ui) {
      // claim the next unit of the list and publish it to the other roles
      const uint32_t qs = ui % kQ, qph = (ui / kQ) & 1;
      ok = __all_sync(kFull, mbar_wait_lazy(&q_empty[qs], qph ^ 1, ctl, p.err, p.timeout_ns, 415, 64));
      int u = -1;
      if (lane == 0) {
        if (ok) {
          u = atomicAdd(p.claim, 1);
          if (u >= n_units) u = -1;
        }
        uq[qs] = u;
        mbar_arrive(&q_full[qs]);
      }
      u = __shfl_sync(kFull, u, 0);
      if (u < 0) break;
      const ServeUnit w = serve_unit(p, stiles, n_st, u);
      const CUtensorMap* map = (w.kind == kUnitA) ? &map_gu_raw : &map_d_raw;
      const float* absmax = (w.kind == kUnitA) ? p.gu_absmax : p.d_absmax;
      const int blocks_per_row = ((w.kind == kUnitA) ? p.H : p.I) / 64;
      const bool amax16 = (w.kchunks % RAW_CHUNKS) == 0 && (reinterpret_cast<uintptr_t>(absmax) & 15u) == 0;
      for (int q = 0; q < w.nq; ++q, ++j) {
        const uint32_t r = j % RAW_STAGES, ph = (j / RAW_STAGES) & 1;
        ok = __all_sync(kFull, mbar_wait_lazy(&raw_empty[r], ph ^ 1, ctl, p.err, p.timeout_ns, 410, 128));
        if (!ok) break;
        uint8_t* slot = smem + RAW_OFF + r * RAW_SLOT;
        if (lane == 0) {
          mbar_arrive_expect_tx(&raw_full[r], CODE_BYTES);
          tma_load_3d(slot, map, &raw_full[r], q * (RAW_CHUNKS * BK / 2), w.rA, w.e);
          tma_load_3d(slot + CODE_BYTES / 2, map, &raw_full[r], q * (RAW_CHUNKS * BK / 2), w.rB, w.e);
        }
        float* amax = reinterpret_cast<float*>(slot + CODE_BYTES);
        const int nb = min(RAW_CHUNKS, w.kchunks - q * RAW_CHUNKS);
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const int t = lane + 32 * qq;
          const int srow = (t < 64) ? w.rA + t : w.rB + (t - 64);
          if (srow < w.stored_rows) {
            const float* src = absmax + ((size_t)w.e * w.stored_rows + srow) * blocks_per_row + q * RAW_CHUNKS;
            if (amax16) {
              cp_async_16(amax + t * RAW_CHUNKS, src);
            } else {
              for (int c = 0; c < nb; ++c) cp_async_4(amax + t * RAW_CHUNKS + c, src + c);
            }
          }
        }
        cp_async_arrive_noinc(&raw_full[r]);
        issued |= 1u << r;
        last_par = (last_par & ~(1u << r)) | (ph << r);
      }
    }
    if (!ok && lane == 0) {
      for (int i = 0; i < RAW_STAGES; ++i)
        if (issued & (1u << i)) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&raw_full[i], (last_par >> i) & 1u) &&
                 (long long)(globaltimer_ns() - t0) < p.timeout_ns) {
          }
        }
    }
  } else if (warp == 2) {
    // ------------------------------------------------ activation rows + LoRA operands, after the unit's inputs exist
    if (lane == 0) {
      tma_prefetch_desc(&map_x);
      tma_prefetch_desc(&map_act);
      tma_prefetch_desc(&map_lw_gu);
      tma_prefetch_desc(&map_lw_d);
      tma_prefetch_desc(&map_lp_gu);
      tma_prefetch_desc(&map_lp_d);
      uint32_t j = 0, ti = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (;; ++ti) {
        const uint32_t qs = ti % kQ, qph = (ti / kQ) & 1;
        if (!(ok = mbar_wait_lazy(&q_full[qs], qph, ctl, p.err, p.timeout_ns, 420, 64))) break;
        const int u = uq[qs];
        mbar_arrive(&q_empty[qs]);
        if (u < 0) break;
        const ServeUnit w = serve_unit(p, stiles, n_st, u);
        // inputs of this unit: written by other CTAs with release, read here with acquire
        if (w.kind == kUnitA)
          ok = wait_counter(p.cnt_prep + w.e, kPrepWarps * p.counts[w.e], ctl, p.err, p.timeout_ns, 421);
        else
          ok = wait_counter(p.pd_ready + w.st, 1, ctl, p.err, p.timeout_ns, 423);
        if (!ok) break;
        fence_proxy_async_global();  // the TMA reads below see those generic-proxy writes
        if (!(ok = mbar_wait_lazy(lempty, (ti & 1) ^ 1, ctl, p.err, p.timeout_ns, 424, 128))) break;
        mbar_arrive_expect_tx(lfull, (uint32_t)((BM + BN) * 2 * p.r_pad));
        uint8_t* la = smem + LA_OFF;
        const CUtensorMap* lw = (w.kind == kUnitA) ? &map_lw_gu : &map_lw_d;
        tma_load_3d(la, lw, lfull, 0, w.rA, w.e);
        tma_load_3d(la + 128 * p.r_pad, lw, lfull, 0, w.rB, w.e);
        tma_load_2d(smem + LB_OFF, (w.kind == kUnitA) ? &map_lp_gu : &map_lp_d, lfull, 0, w.row0);
        const CUtensorMap* xm = (w.kind == kUnitA) ? &map_x : &map_act;
        for (int q = 0; q < w.nq; ++q, ++j) {
          const uint32_t s = j % X_STAGES, ph = (j / X_STAGES) & 1;
          if (!(ok = mbar_wait_lazy(&x_empty[s], ph ^ 1, ctl, p.err, p.timeout_ns, 425, 128))) break;
          const int nb = min(RAW_CHUNKS, w.kchunks - q * RAW_CHUNKS);
          mbar_arrive_expect_tx(&x_full[s], (uint32_t)(nb * X_BYTES));
          for (int c = 0; c < nb; ++c)
            tma_load_2d(smem + X_OFF + s * XS_BYTES + c * X_BYTES, xm, &x_full[s], (q * RAW_CHUNKS + c) * BK,
                        w.row0);
          issued |= 1u << s;
          last_par = (last_par & ~(1u << s)) | (ph << s);
        }
      }
      if (!ok) {
        for (int i = 0; i < X_STAGES; ++i)
          if (issued & (1u << i)) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&x_full[i], (last_par >> i) & 1u) &&
                   (long long)(globaltimer_ns() - t0) < p.timeout_ns) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ UMMA issuer (whole warp, one elected lane issues)
    const uint32_t idesc = make_idesc_bf16(BM, BN, false, false);
    const uint32_t lswz = swz_for_row_bytes(2 * p.r_pad);
    const uint32_t la_u = smem_u32(smem + LA_OFF), lb_u = smem_u32(smem + LB_OFF);
    const uint64_t xdesc0 = make_sdesc(smem_u32(smem + X_OFF), 16, 1024, kSw128);
    uint32_t ti = 0, rq = 0, xs = 0, xph = 0;
    bool ok = true;
    for (;; ++ti) {
      const int u = next_unit(ti, 434);
      if (u < 0) break;
      const ServeUnit w = serve_unit(p, stiles, n_st, u);
      const uint32_t b = ti & 1, use = ti >> 1;
      const uint32_t d = tmem + b * kAccCols;
      if (!(ok = __all_sync(kFull, mbar_wait(&accempty[b], (use & 1) ^ 1, ctl, p.err, p.timeout_ns, 430)))) break;
      if (!(ok = __all_sync(kFull, mbar_wait(lfull, ti & 1, ctl, p.err, p.timeout_ns, 431)))) break;
      tc_fence_after();
      if (elect_one_sync()) {
        for (int kk = 0; kk < p.r_pad / 16; ++kk)
          umma_bf16(d, make_sdesc(la_u + 32 * kk, 16, 16 * p.r_pad, lswz),
                    make_sdesc(lb_u + 32 * kk, 16, 16 * p.r_pad, lswz), idesc, kk > 0 ? 1u : 0u);
        umma_commit(lempty);
      }
      __syncwarp();
      for (int q = 0; q < w.nq; ++q, ++rq) {
        const uint32_t team = rq % kTeams, aph = (rq / kTeams) & 1;
        ok = __all_sync(kFull, mbar_wait(&a_ready[team], aph, ctl, p.err, p.timeout_ns, 432));
        if (ok) ok = __all_sync(kFull, mbar_wait(&x_full[xs], xph, ctl, p.err, p.timeout_ns, 433));
        if (!ok) break;
        tc_fence_after();
        if (elect_one_sync()) {
          const int nb = min(RAW_CHUNKS, w.kchunks - q * RAW_CHUNKS);
          const uint32_t a_col = tmem + kAOff + team * kTeamCols;
          const uint64_t xdesc = xdesc0 + (uint64_t)((xs * XS_BYTES) >> 4);
          for (int c = 0; c < nb; ++c)
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)  // K16 step: 8 TMEM columns of A, +32 bytes of x
              umma_bf16_ta(d, a_col + c * kACols + 8 * kk, xdesc + (uint64_t)(c * (X_BYTES >> 4) + 2 * kk), idesc,
                           1u);
          umma_commit(&a_empty[team]);
          umma_commit(&x_empty[xs]);
        }
        __syncwarp();
        if (++xs == X_STAGES) {
          xs = 0;
          xph ^= 1;
        }
      }
      if (!ok) break;
      if (elect_one_sync()) umma_commit(&accfull[b]);
      __syncwarp();
    }
    if (elect_one_sync()) umma_commit(drain);
    __syncwarp();
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(drain, 0) && (long long)(globaltimer_ns() - t0) < p.timeout_ns) {
    }
  } else if (warp >= kPrepWarp0) {
    {
      // ------------------------------------------------ prep (warps 4..19): x scatter + p_gu of a few slots
      // (the first gate_up units wait for it, so all of these warps share it before their own roles)
      const int pw = warp - kPrepWarp0;  // 0..15
      const int vec = p.H / 8;           // 16-byte pieces of a row
      for (int f = blockIdx.x; f < N; f += gridDim.x) {
        const int e = __ldg(p.topk_ids + f), row = __ldg(p.row_of_slot + f), t = f / p.k;
        const uint4* xs = reinterpret_cast<const uint4*>(p.x + (size_t)t * p.H);
        // Each lane keeps kPrepBatch 16-byte pieces of a row in flight at once: a loop that waited for
        // each piece in turn made this phase ~8 us long, and the first gate_up units wait for it.
        constexpr int kPrepBatch = 4;
        if (pw == 0) {
          uint4* dst = reinterpret_cast<uint4*>(p.x_perm + (size_t)row * p.H);
          for (int c0 = lane; c0 < vec; c0 += 32 * kPrepBatch) {
            uint4 xq[kPrepBatch];
#pragma unroll
            for (int i = 0; i < kPrepBatch; ++i)
              if (c0 + 32 * i < vec) xq[i] = __ldg(xs + c0 + 32 * i);
#pragma unroll
            for (int i = 0; i < kPrepBatch; ++i)
              if (c0 + 32 * i < vec) dst[c0 + 32 * i] = xq[i];
          }
        }
        for (int jr = pw; jr < p.r; jr += kPrepWarps) {
          const uint4* ap = reinterpret_cast<const uint4*>(p.A_gu + ((size_t)e * p.r + jr) * p.H);
          float acc = 0.0f;
          for (int c0 = lane; c0 < vec; c0 += 32 * kPrepBatch) {
            uint4 xq[kPrepBatch], aq[kPrepBatch];
#pragma unroll
            for (int i = 0; i < kPrepBatch; ++i) {
              const bool in = c0 + 32 * i < vec;
              xq[i] = in ? __ldg(xs + c0 + 32 * i) : make_uint4(0u, 0u, 0u, 0u);
              aq[i] = in ? __ldg(ap + c0 + 32 * i) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int q = 0; q < kPrepBatch; ++q) {
              const uint32_t* xw = reinterpret_cast<const uint32_t*>(&xq[q]);
              const uint32_t* aw = reinterpret_cast<const uint32_t*>(&aq[q]);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                acc = fmaf(bf16lo_to_f32(xw[i]), bf16lo_to_f32(aw[i]), acc);
                acc = fmaf(bf16hi_to_f32(xw[i]), bf16hi_to_f32(aw[i]), acc);
              }
            }
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
          if (lane == 0) {
            const __nv_bfloat16 h = __float2bfloat16_rn(p.s * acc);
            p.p_gu[(size_t)row * p.r + jr] = *reinterpret_cast<const uint16_t*>(&h);
          }
        }
        // this warp's stores of the slot (its lanes ordered by __syncwarp, the proxy fence for the TMA
        // readers) are released with its count: an A unit of expert e starts once every prep warp has
        // counted each of e's slots
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) red_release_add_gpu(p.cnt_prep + e, 1);
      }
    }
    if (warp < kEpiWarp0) {
      // ------------------------------------------------ decode teams: NF4 -> TMEM
      const uint32_t team = (uint32_t)(warp - 4) >> 2;
      const int t = (threadIdx.x - 128) & 127;
      const Nf4Shift ks = nf4_shift_consts();
      const uint32_t a_base = tmem + kAOff + team * kTeamCols + ((uint32_t)(warp & 3) * 32u << 16);
      uint32_t rq = 0, tuse = 0;
      bool ok = true;
      for (uint32_t ui = 0; ok; ++ui) {
        const int u = next_unit(ui, 444);
        if (u < 0) break;
        const ServeUnit w = serve_unit(p, stiles, n_st, u);
        const bool valid = ((t < 64) ? w.rA + t : w.rB + (t - 64)) < w.stored_rows;
        for (int q = 0; q < w.nq; ++q, ++rq) {
          if (rq % kTeams != team) continue;
          const uint32_t r = rq % RAW_STAGES, rph = (rq / RAW_STAGES) & 1;
          const uint32_t aph = tuse++ & 1;
          ok = __all_sync(kFull, mbar_wait(&raw_full[r], rph, ctl, p.err, p.timeout_ns, 440));
          if (!ok) break;
          const uint8_t* slot = smem + RAW_OFF + r * RAW_SLOT;
          const uint8_t* crow = slot + t * 128;  // 128B-swizzled row t: 16-byte piece c at c ^ (t % 8)
          const int nb = min(RAW_CHUNKS, w.kchunks - q * RAW_CHUNKS);
          const float* amax = reinterpret_cast<const float*>(slot + CODE_BYTES) + t * RAW_CHUNKS;
          for (int c = 0; c < nb; ++c) {
            const uint4 q0 = *reinterpret_cast<const uint4*>(crow + (((2 * c) ^ (t & 7)) << 4));
            const uint4 q1 = *reinterpret_cast<const uint4*>(crow + (((2 * c + 1) ^ (t & 7)) << 4));
            const float a = amax[c];
            if (c == nb - 1) {
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) mbar_arrive(&raw_empty[r]);
            }
            const uint32_t codes[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
            const Nf4Planes pl = nf4_block_planes(valid ? a : 0.0f);
            uint32_t v[32];
#pragma unroll
            for (int i = 0; i < 8; ++i) nf4_decode_word(codes[i], pl, ks, &v[4 * i]);
            if (c == 0) {
              ok = __all_sync(kFull, mbar_wait(&a_empty[team], aph ^ 1, ctl, p.err, p.timeout_ns, 441));
              if (!ok) break;
              tc_fence_after();
            }
            tmem_st32(a_base + c * kACols, v);
          }
          if (!ok) break;
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_ready[team]);
        }
      }
    } else {
      // ------------------------------------------------ epilogue: lane = weight row, 32 slot columns
      // Only TMEM loads and stores here: every wait on other CTAs' work and every device-scope fence or
      // atomic is left to the publisher warp, through a two-slot hand-off ring.
      const int qrt = warp & 3;
      const int wrow = qrt * 32 + lane;
      float* epi = reinterpret_cast<float*>(smem + EPI_OFF);
      uint32_t ti = 0, ai = 0;  // units; A units (the gate/up hand-off alternates with them)
      bool ok = true;
      for (; ok; ++ti) {
        const int u = next_unit(ti, 455);
        if (u < 0) break;
        const ServeUnit w = serve_unit(p, stiles, n_st, u);
        const size_t row0 = (size_t)w.row0;
        const uint32_t b = ti & 1, use = ti >> 1;
        ok = __all_sync(kFull, mbar_wait_lazy(&accfull[b], use & 1, ctl, p.err, p.timeout_ns, 450, 256));
        if (!ok) break;
        tc_fence_after();
        float v[32];
        {
          float v0[16], v1[16];
          const uint32_t tl = tmem + b * kAccCols + ((uint32_t)(qrt * 32) << 16);
          tmem_ld16(tl, v0);
          tmem_ld16(tl + 16, v1);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            v[i] = v0[i];
            v[16 + i] = v1[i];
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accempty[b]);  // the accumulator is in registers now
        // hand-off slot of this unit: free once the publisher finished the unit kHand back
        const uint32_t hb = ti % kHand, huse = ti / kHand;
        if (w.kind == kUnitA) {
          const int il = wrow & 63;  // the lane's feature within the unit's 64
          const int i = w.mt * 64 + il;
          const int I2 = 2 * p.I;
          const uint32_t aph = ai & 1;
          if (qrt >= 2) {
            ok = __all_sync(kFull, mbar_wait(epi_empty, aph ^ 1, ctl, p.err, p.timeout_ns, 451));
            if (!ok) break;
#pragma unroll
            for (int sl = 0; sl < 32; ++sl) epi[sl * 64 + il] = v[sl];
            __syncwarp();
            if (lane == 0) mbar_arrive(epi_full);
            if (p.gu != nullptr) {
#pragma unroll
              for (int sl = 0; sl < 32; ++sl)
                if (sl < w.nslots) {
                  const __nv_bfloat16 h = __float2bfloat16_rn(v[sl]);
                  p.gu[(row0 + sl) * I2 + p.I + i] = *reinterpret_cast<const uint16_t*>(&h);
                }
            }
            ok = __all_sync(kFull, mbar_wait(&hand_empty[hb], (huse & 1) ^ 1, ctl, p.err, p.timeout_ns, 453));
            if (!ok) break;
          } else {
            ok = __all_sync(kFull, mbar_wait(epi_full, aph, ctl, p.err, p.timeout_ns, 452));
            if (!ok) break;
            uint16_t a[32];
#pragma unroll
            for (int sl = 0; sl < 32; ++sl) {
              const float g = v[sl], uu = epi[sl * 64 + il];
              const __nv_bfloat16 ha = __float2bfloat16_rn(silu_f(g) * uu);
              a[sl] = *reinterpret_cast<const uint16_t*>(&ha);  // the stored act, as the down projection reads it
              if (sl < w.nslots) {
                const __nv_bfloat16 hg = __float2bfloat16_rn(g);
                if (p.gu != nullptr) p.gu[(row0 + sl) * I2 + i] = *reinterpret_cast<const uint16_t*>(&hg);
                p.act[(row0 + sl) * p.I + i] = a[sl];
              }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(epi_empty);
            // the act tile for the publisher's share of the LoRA down projection
            ok = __all_sync(kFull, mbar_wait(&hand_empty[hb], (huse & 1) ^ 1, ctl, p.err, p.timeout_ns, 453));
            if (!ok) break;
            uint16_t* acts = reinterpret_cast<uint16_t*>(smem + ACTS_OFF) + hb * (64 * BN);
#pragma unroll
            for (int sl = 0; sl < 32; ++sl) acts[sl * 64 + il] = a[sl];
          }
          ++ai;
        } else {
          const int f = w.mt * 128 + wrow;
          if (f < p.H) {
#pragma unroll
            for (int sl = 0; sl < 32; ++sl)
              if (sl < w.nslots) {
                const __nv_bfloat16 h = __float2bfloat16_rn(v[sl]);
                p.y_perm[(row0 + sl) * p.H + f] = *reinterpret_cast<const uint16_t*>(&h);
              }
          }
          ok = __all_sync(kFull, mbar_wait(&hand_empty[hb], (huse & 1) ^ 1, ctl, p.err, p.timeout_ns, 453));
          if (!ok) break;
        }
        // the unit's global stores (and act tile) go to the publisher: the arrival is a CTA-scope release,
        // and the publisher's device-scope release after it covers these stores
        fence_proxy_async_global();  // the act rows are read by TMA in other CTAs
        __syncwarp();
        if (lane == 0) mbar_arrive(&hand_full[hb]);
      }
    }
  } else if (warp == kPubWarp) {
    // ------------------------------------------------ publisher: counts finished units for the other CTAs,
    // forms p_d once a slot tile's gate_up units are all done, and y once a token's slots are all done
    uint32_t ti = 0;
    bool ok = true;
    for (; ok; ++ti) {
      const int u = next_unit(ti, 465);
      if (u < 0) break;
      const ServeUnit w = serve_unit(p, stiles, n_st, u);
      const size_t row0 = (size_t)w.row0;
      const uint32_t hb = ti % kHand, huse = ti / kHand;
      ok = __all_sync(kFull, mbar_wait_lazy(&hand_full[hb], huse & 1, ctl, p.err, p.timeout_ns, 460, 128));
      if (!ok) break;
      if (w.kind == kUnitA) {
        // this unit's share of p_d: part[sl][j] = sum_i act[sl][i] A_d[e][j][i] over its 64 features (i ascending)
        const uint16_t* acts = reinterpret_cast<const uint16_t*>(smem + ACTS_OFF) + hb * (64 * BN);
        float* part = p.pd_part + ((size_t)w.st * p.nA_mt + w.mt) * BN * p.r;
        for (int o = lane; o < w.nslots * p.r; o += 32) {
          const int sl = o / p.r, jr = o - sl * p.r;
          const uint4* ap = reinterpret_cast<const uint4*>(p.A_d + ((size_t)w.e * p.r + jr) * p.I + w.mt * 64);
          uint4 aq[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) aq[c] = __ldg(ap + c);
          const uint4* ar = reinterpret_cast<const uint4*>(acts + sl * 64);
          float sum = 0.0f;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 xq = ar[c];
            const uint32_t* aw = reinterpret_cast<const uint32_t*>(&aq[c]);
            const uint32_t* xw = reinterpret_cast<const uint32_t*>(&xq);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              sum = fmaf(bf16lo_to_f32(xw[h]), bf16lo_to_f32(aw[h]), sum);
              sum = fmaf(bf16hi_to_f32(xw[h]), bf16hi_to_f32(aw[h]), sum);
            }
          }
          part[o] = sum;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&hand_empty[hb]);
        // Publish this unit (the act rows the epilogue stored and this warp's shares; the acq_rel add
        // releases both, the warp's lanes ordered by __syncwarp).  The unit that completes the slot tile
        // sums the shares in unit order into p_d and releases the tile to its down units.
        int old = 0;
        if (lane == 0) old = atom_acq_rel_add_gpu(p.cnt_a + w.st, 1);
        old = __shfl_sync(kFull, old, 0);
        if (old == p.nA_mt - 1) {
          const float* parts = p.pd_part + (size_t)w.st * p.nA_mt * BN * p.r;
          for (int o = lane; o < w.nslots * p.r; o += 32) {
            float sum = 0.0f;
            for (int m = 0; m < p.nA_mt; ++m) sum += __ldcg(parts + (size_t)m * BN * p.r + o);
            const int sl = o / p.r, jr = o - sl * p.r;
            const __nv_bfloat16 h = __float2bfloat16_rn(p.s * sum);
            p.p_d[(row0 + sl) * p.r + jr] = *reinterpret_cast<const uint16_t*>(&h);
          }
          fence_proxy_async_global();  // p_d is read by TMA in other CTAs
          __syncwarp();
          if (lane == 0) st_release_gpu(p.pd_ready + w.st, 1);
        }
      } else {
        __syncwarp();
        if (lane == 0) mbar_arrive(&hand_empty[hb]);
        // count this unit's 128 columns for each slot's token (acq_rel: releases the epilogue's y_perm rows,
        // acquires the other slots'); the count that completes a token's k slots forms its 128 columns of
        // y = sum_j w[t,j] y_perm[row(t,j)] (fp32, j ascending, one rounding)
        bool done = false;
        int tok = 0;
        if (lane < w.nslots) {
          tok = __ldg(p.slot_of_row + row0 + lane) / p.k;
          done = atom_acq_rel_add_gpu(p.cnt_comb + (size_t)tok * p.nB_mt + w.mt, 1) == p.k - 1;
        }
        uint32_t pending = __ballot_sync(kFull, done);  // also orders the other lanes' reads after the acquires
        const int col = w.mt * 128 + 4 * lane;  // this lane's 4 columns (H is a multiple of 64)
        while (pending) {
          const int src = __ffs(pending) - 1;
          pending &= pending - 1;
          const int t = __shfl_sync(kFull, tok, src);
          int my_row = 0;
          float my_w = 0.0f;
          if (lane < p.k) {
            my_row = __ldg(p.row_of_slot + (size_t)t * p.k + lane);
            my_w = __ldg(p.topk_w + (size_t)t * p.k + lane);
          }
          uint2 yv[E4B_MAX_TOP_K];
#pragma unroll
          for (int jj = 0; jj < E4B_MAX_TOP_K; ++jj) {
            const int rr = __shfl_sync(kFull, my_row, jj);
            yv[jj] = (jj < p.k && col < p.H)
                         ? __ldcg(reinterpret_cast<const uint2*>(p.y_perm + (size_t)rr * p.H + col))
                         : make_uint2(0u, 0u);
          }
          float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int jj = 0; jj < E4B_MAX_TOP_K; ++jj) {
            const float wj = __shfl_sync(kFull, my_w, jj);
            if (jj < p.k) {
              acc[0] = fmaf(wj, bf16lo_to_f32(yv[jj].x), acc[0]);
              acc[1] = fmaf(wj, bf16hi_to_f32(yv[jj].x), acc[1]);
              acc[2] = fmaf(wj, bf16lo_to_f32(yv[jj].y), acc[2]);
              acc[3] = fmaf(wj, bf16hi_to_f32(yv[jj].y), acc[3]);
            }
          }
          if (col < p.H)
            *reinterpret_cast<uint2*>(p.y + (size_t)t * p.H + col) =
                make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]));
        }
      }
    }
  }

  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

cudaError_t launch_nf4_serve(const ServeHost& h, int num_sms, cudaStream_t stream) {
  using namespace nf4v;
  CUtensorMap mgu, md, mx, mact, mlwgu, mlwd, mlpgu, mlpd;
  cudaError_t err;
  const CUtensorMapSwizzle rswz = swizzle_for_bytes(2 * h.r_pad);
  if ((err = map_u8_3d(&mgu, h.gate_up_nf4, h.H / 2, 2 * (uint64_t)h.I, h.E, RAW_CHUNKS * BK / 2, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess)
    return err;
  if ((err = map_u8_3d(&md, h.down_nf4, h.I / 2, h.H, h.E, RAW_CHUNKS * BK / 2, 64, CU_TENSOR_MAP_SWIZZLE_128B)) !=
      cudaSuccess)
    return err;
  if ((err = map_bf16_2d(&mx, h.x_perm, h.H, h.rows_cap, BK, BN, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess)
    return err;
  if ((err = map_bf16_2d(&mact, h.act, h.I, h.rows_cap, BK, BN, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess)
    return err;
  if ((err = map_bf16_3d(&mlwgu, h.B_gu, h.r, 2 * (uint64_t)h.I, h.E, h.r_pad, 64, rswz)) != cudaSuccess) return err;
  if ((err = map_bf16_3d(&mlwd, h.B_d, h.r, h.H, h.E, h.r_pad, 64, rswz)) != cudaSuccess) return err;
  if ((err = map_bf16_2d(&mlpgu, h.p_gu, h.r, h.rows_cap, h.r_pad, BN, rswz)) != cudaSuccess) return err;
  if ((err = map_bf16_2d(&mlpd, h.p_d, h.r, h.rows_cap, h.r_pad, BN, rswz)) != cudaSuccess) return err;
  ServeParams p;
  p.gu_absmax = h.gate_up_absmax;
  p.d_absmax = h.down_absmax;
  p.x = h.x;
  p.A_gu = h.A_gu;
  p.A_d = h.A_d;
  p.x_perm = h.x_perm;
  p.p_gu = h.p_gu;
  p.gu = h.gu;
  p.act = h.act;
  p.p_d = h.p_d;
  p.y_perm = h.y_perm;
  p.y = h.y;
  p.topk_ids = h.topk_ids;
  p.topk_w = h.topk_w;
  p.row_of_slot = h.row_of_slot;
  p.slot_of_row = h.slot_of_row;
  p.counts = h.counts;
  p.tiles = h.tiles;
  p.st_offset = stiles_offset(h.mt_cap, h.E);
  p.cnt_prep = h.counters;
  p.cnt_a = h.counters + serve_cnt_a_offset(h.E);
  p.pd_ready = h.counters + serve_pd_offset(h.E, h.st_cap);
  p.cnt_comb = h.counters + serve_comb_offset(h.E, h.st_cap);
  p.pd_part = h.pd_part;
  p.claim = h.counters + serve_claim_offset(h.E, h.st_cap, h.T, h.H);
  p.err = h.err;
  p.timeout_ns = h.timeout_ns;
  p.T = h.T;
  p.k = h.k;
  p.E = h.E;
  p.H = h.H;
  p.I = h.I;
  p.r = h.r;
  p.r_pad = h.r_pad;
  p.s = h.s;
  p.nA_mt = h.I / 64;
  p.nB_mt = (h.H + 127) / 128;
  // every unit waits only for units listed before it, which running CTAs hold: one CTA per SM
  const int64_t units_max = h.st_cap * (int64_t)(p.nA_mt + p.nB_mt);
  int64_t grid = units_max < num_sms ? units_max : num_sms;
  const int64_t nslots = (int64_t)h.T * h.k;
  if (grid < nslots && grid < num_sms) grid = nslots < num_sms ? nslots : num_sms;
  if (grid < 1) grid = 1;
  const int smem = SMEM_BYTES;
  LaunchScope scope("nf4_serve", stream);
  if ((err = cudaFuncSetAttribute(nf4_serve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
      cudaSuccess)
    return err;
  nf4_serve_kernel<<<(int)grid, kThreads, smem, stream>>>(mgu, md, mx, mact, mlwgu, mlwd, mlpgu, mlpd, p);
  return cudaGetLastError();
}

}  // namespace e4b
