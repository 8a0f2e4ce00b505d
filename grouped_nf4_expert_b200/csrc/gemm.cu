// Grouped GEMMs on the 5th-generation tensor cores (tcgen05, TMEM
// accumulators, TMA-fed shared memory) for the NF4 expert block:
//
//  * nf4_gemm_kernel: persistent CTA pairs, one 256x256 output tile per work
//    unit (cta_group::2 UMMAs) of a grouped GEMM whose B operand is a frozen
//    NF4 expert matrix, dequantised into shared memory by four decode groups
//    (bit-exact bf16 weights), with the LoRA term as an extra K = r MMA into
//    the same TMEM accumulator.  Four modes: forward gate_up (SiLU-gated
//    epilogue), forward down, down dgrad (transposed base, SwiGLU backward
//    epilogue), gate_up dgrad.
//  * lora_proj_kernel: s * (rows x LoRA factor) -> [rows, r], the low-rank
//    projections p = s x A^T and q = s dy B.
//  * gather_proj_kernel: the row gather of x (or w * dY) into the permuted
//    buffer fused with its LoRA projection.
//  * wgrad_kernel: variable-K grouped GEMM for the LoRA weight gradients
//    (K = the rows of one expert).
//
// Pages: "How do I QLoRA-train the fused experts of a MoE", section "The
// abstraction that fails" (pre-activation per-expert delta over the fused
// stacks), section "Why it happens" (scaling * (x @ A.T) @ B.T; the backward
// decodes the 4-bit base again), section "Which project solves it" (grouped
// forward and a dgrad kernel); package METADATA "The package family" (4-bit
// codes decoded in registers, fp32 sums).
#include <math.h>

#include "e4b_device.cuh"
#include "e4b_internal.h"

namespace e4b {

namespace {

constexpr uint32_t kFull = 0xffffffffu;

// 16 bf16 (32 bytes) from registers to global memory: one full-sector store
// when the destination is 32-byte aligned, else two 16-byte stores.
__device__ __forceinline__ void store_row16(uint16_t* dst, const uint32_t (&w)[8], bool v8) {
  if (v8) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(w[0]), "r"(w[1]),
                 "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
  } else {
    uint4* d = reinterpret_cast<uint4*>(dst);
    d[0] = make_uint4(w[0], w[1], w[2], w[3]);
    d[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

}  // namespace

// =============================================================================
// NF4 grouped GEMM on CTA pairs (2-SM UMMA)
// =============================================================================
// Work unit: up to 256 rows of one expert (a 256-row m-unit) x 256 output
// columns, computed by a cluster of two CTAs with cta_group::2 UMMAs
// (M = 256, N = 256).  CTA rank c holds rows [128c, 128c+128) of the
// activation tile and decodes weight rows (output columns) [128c, 128c+128)
// of the tile; its TMEM receives its 128 rows x 256 columns.  Each CTA loads
// only its own tiles (no multicast loads).
// Roles per CTA: warp 0 = NF4 codes into a ring of their own (one TMA per
// k-chunk, filled far ahead), warp 1 = TMEM owner (both CTAs) and UMMA issuer
// (even CTA only), warp 2 = relay, warp 3 = activation tiles and LoRA
// operands, warps 4-19 = four decode groups taking the k-chunks round robin,
// warps 20-23 = epilogue.  Operands are staged in two rings: activation slots
// (six; a unit's LoRA operands take two of them ahead of its k-chunks, so the
// LoRA step needs no buffers of its own) and decoded-tile slots (one per decode
// group).  The activation tile is the operand that arrives last (a TMA load of
// ~1000+ cycles), so its ring is the deeper one; decoders decode into registers
// from the code ring (block scales: their own loads, a chunk ahead) and only
// wait for their own slot to be free to store.
// Each CTA's relay (warp 2) waits for its own operands of an MMA step (xfull,
// bdone) and signals the even CTA's full[], the one barrier the UMMA issuer
// tests per step: the even CTA's relay with an arrive that also arms 4
// transaction bytes, the odd CTA's with a 4-byte st.async whose mbarrier
// complete_tx carries the cluster-scope release (a release-arrive would stall
// the signalling warp for about a microsecond).  The issuer's instruction
// stream is one dependent chain per k-chunk sharing its scheduler with four
// decode warps, so it is kept short.  The issuer's commits arrive on both
// CTAs' aempty / bempty / accfull barriers.
namespace nf4g {
constexpr int BM = 128;   // activation rows per CTA (256 per pair)
constexpr int BN = 128;   // weight rows decoded per CTA (256 output columns per pair)
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;                 // activation tile, K-major SW128
constexpr int B_BYTES = BN * BK * 2;                 // dequantised weight tile
constexpr int kGroups = 4;          // decode groups; group g decodes the k-chunks j with j % 4 == g
constexpr int kGroupWarps = 4;      // warps per decode group (one per 32 weight rows)
// Activation ring: SA slots.  A unit takes two activation uses for its LoRA operands (its p or q
// rows, 128 x r_pad, and its LoRA weight rows, 128 x r_pad), then one per k-chunk.
constexpr int SA = 6;
// Decoded-tile ring: one slot per decode group (group g's chunks always use slot g).
constexpr int SB = kGroups;
constexpr int RAW_STAGES = 2 * kGroups;  // code slot r always belongs to group r % 4 (no phase aliasing)
constexpr int RAW_BYTES = BN * BK / 2;               // NF4 codes as loaded
constexpr int RAW_SLOT = RAW_BYTES;
constexpr int B_OFF = SA * A_BYTES;
constexpr int RAW_OFF = B_OFF + SB * B_BYTES;
static_assert(BM * E4B_MAX_RANK * 2 <= A_BYTES && BN * E4B_MAX_RANK * 2 <= A_BYTES, "LoRA operands fit a slot");
// Epilogue staging: per epilogue warp, two steps x up to three 32-row x 16-column output tiles.
constexpr int kEpiTileBytes = 32 * 16 * 2;
constexpr int kEpiStepBytes = 3 * kEpiTileBytes;
constexpr int kEpiWarpBytes = 2 * kEpiStepBytes;
static_assert(kEpiWarpBytes >= 3 * 2 * kEpiTileBytes, "three 2-tile buffers for the plain epilogue");
constexpr int kDgAhead = 3;  // down dgrad epilogue: gate/up copies in flight, 2 KB per step per warp
static_assert(kEpiWarpBytes >= kDgAhead * 4 * 512, "down dgrad gate/up ring");
constexpr int EPI_OFF = RAW_OFF + RAW_STAGES * RAW_SLOT;
constexpr int BAR_OFF = EPI_OFF + 4 * kEpiWarpBytes;
constexpr int BAR_BYTES = 1024;
constexpr int SMEM_BYTES = BAR_OFF + BAR_BYTES + 1024;
constexpr int kEpiWarp0 = 4 + kGroups * kGroupWarps;
constexpr int kThreads = 32 * (kEpiWarp0 + 4);
constexpr int kTmemCols = 512;      // 2 accumulator buffers x 256 columns
static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0 && B_OFF % 1024 == 0, "swizzle atom alignment");
static_assert(RAW_STAGES % kGroups == 0, "code slots are owned by one decode group each");
// Every barrier is waited on phase by phase by the roles that use it: the activation loader,
// relays and issuer go through all activation uses and MMA steps in order, and a decode group
// owns its decoded-tile slot and code slots, so no parity wait can alias.
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
}  // namespace nf4g

struct Nf4GemmParams {
  const float* absmax;
  const int32_t* tiles;
  uint16_t* out0;
  uint16_t* out1;
  const uint16_t* aux;
  DeviceError* err;
  long long timeout_ns;
  int K, n_dim, I, r_pad;
  int stored_rows, stored_cols;
  int n_nt;
  int v8;             // (down dgrad) dgu and its row pitch are 32-byte aligned: 32-byte stores
  int64_t mu_offset;  // start of the m-unit list in `tiles`
};

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(nf4g::kThreads, 1)
    nf4_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_raw,
                    const __grid_constant__ CUtensorMap map_la, const __grid_constant__ CUtensorMap map_lb,
                    const __grid_constant__ CUtensorMap map_o0, const __grid_constant__ CUtensorMap map_o1,
                    const Nf4GemmParams p) {
  using namespace nf4g;
  constexpr bool kMN = (MODE == kDgradDown || MODE == kDgradGateUp);  // B operand N-contiguous
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = align1024(smem_dyn);
  uint8_t* aring = smem;          // [SA] activation tiles / LoRA operands
  uint8_t* bring = smem + B_OFF;  // [SB] decoded weight tiles
  uint8_t* rawbuf = smem + RAW_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* raw_full = bars;                   // [RAW_STAGES] codes landed
  uint64_t* raw_empty = raw_full + RAW_STAGES; // [RAW_STAGES] codes read into registers (group's 4 warps)
  uint64_t* xfull = raw_empty + RAW_STAGES;    // [SA] activation use landed
  uint64_t* aempty = xfull + SA;               // [SA] activation slot consumed by the UMMAs
  uint64_t* full = aempty + SA;                // [SA] (even CTA) both CTAs' operands of an MMA step in place
  uint64_t* bdone = full + SA;                 // [SB] this CTA's decoded tile written (group's 4 warps)
  uint64_t* bempty = bdone + SB;               // [SB] decoded-tile slot consumed by the UMMAs
  uint64_t* accfull = bempty + SB;             // [2] accumulator buffer complete
  uint64_t* accempty = accfull + 2;            // [2] (even CTA) accumulator buffer drained in both CTAs
  uint64_t* drain = accfull + 4;               // (even CTA) all issued UMMAs finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfull + 5);
  CtaControl* ctl = reinterpret_cast<CtaControl*>(accfull + 6);
  uint32_t* sig = reinterpret_cast<uint32_t*>(accfull + 7);  // target word of the st.async signals

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  if (threadIdx.x == 0) {
    for (int r = 0; r < RAW_STAGES; ++r) {
      mbar_init(&raw_full[r], 1);
      mbar_init(&raw_empty[r], kGroupWarps);
    }
    for (int s = 0; s < SA; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&aempty[s], 1);
      mbar_init(&full[s], 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(&bdone[s], kGroupWarps);
      mbar_init(&bempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 8);
    }
    mbar_init(drain, 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_2sm(tmem_slot, kTmemCols);
    tmem_relinquish_2sm();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int32_t* units = p.tiles + p.mu_offset;
  const int n_units = p.tiles[2] * p.n_nt;
  const int kchunks = p.K / BK;
  const int blocks_per_row = p.stored_cols / 64;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  // First of the 128 consecutive stored rows of this CTA's weight tile (K-major modes).
  auto kmajor_row0 = [&](int nt) -> int {
    if (MODE == kFwdGateUp) return (rank ? p.I : 0) + nt * 128;  // even CTA: gate rows, odd CTA: up rows
    return nt * 256 + rank * 128;
  };
  // Decoded tile row t of this CTA is valid (exists in the stored matrix / output).
  auto row_valid = [&](int nt, int t) -> bool {
    if (!kMN) {
      if (MODE == kFwdGateUp) return nt * 128 + t < p.I;
      return nt * 256 + rank * 128 + t < p.stored_rows;
    }
    return nt * 4 + rank * 2 + (t >> 6) < blocks_per_row;
  };

  if (warp == 0) {
    // ------------------------------------------------ NF4 codes into the code ring (one lane)
    // One TMA per k-chunk: the 128 weight rows x 64 codes of this CTA (K-major: 128 consecutive stored rows;
    // N-contiguous: 64 stored rows x 128 codes).  The block scales are read by the decoders themselves, a
    // chunk ahead: gathered here they made this role slower than the k-chunk rate.
    if (lane == 0) {
      tma_prefetch_desc(&map_raw);
      uint32_t j = 0, issued = 0, last_par = 0;  // issued/last_par: per code slot
      bool ok = true;
      int e_next = (pair < n_units) ? units[3 * (pair / p.n_nt)] : 0;
      for (int u = pair; u < n_units && ok; u += n_pairs) {
        const int nt = u % p.n_nt;
        const int e = e_next;
        if (u + n_pairs < n_units) e_next = units[3 * ((u + n_pairs) / p.n_nt)];
        const int rA = kMN ? 0 : kmajor_row0(nt);
        for (int kc = 0; kc < kchunks; ++kc, ++j) {
          const uint32_t r = j % RAW_STAGES, ph = (j / RAW_STAGES) & 1;
          if (!(ok = mbar_wait_lazy(&raw_empty[r], ph ^ 1, ctl, p.err, p.timeout_ns, 11, 64))) break;
          uint8_t* slot = rawbuf + r * RAW_SLOT;
          mbar_arrive_expect_tx(&raw_full[r], (uint32_t)RAW_BYTES);
          if (!kMN)
            tma_load_3d(slot, &map_raw, &raw_full[r], kc * (BK / 2), rA, e);
          else
            tma_load_3d(slot, &map_raw, &raw_full[r], (nt * 256 + rank * 128) / 2, kc * BK, e);
          issued |= 1u << r;
          last_par = (last_par & ~(1u << r)) | (ph << r);
        }
      }
      if (!ok) {
        // Let copies already issued land before the CTA's shared memory goes away.
        for (int i = 0; i < RAW_STAGES; ++i)
          if (issued & (1u << i)) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&raw_full[i], (last_par >> i) & 1u) &&
                   (long long)(globaltimer_ns() - t0) < p.timeout_ns) {
            }
          }
      }
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------ activation tiles + LoRA operands (one lane)
    // Activation uses in order: per unit two for its LoRA operands (p or q rows into slot a, LoRA weight
    // rows into slot a + 1, both copies completing on xfull[a]; xfull[a + 1] gets a plain arrival), then
    // one per k-chunk.
    if (lane == 0) {
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_la);
      tma_prefetch_desc(&map_lb);
      uint32_t s = 0, ph = 0, issued = 0, last_par = 0;  // issued/last_par: per activation slot
      auto issued_next = [&]() {
        issued |= 1u << s;
        last_par = (last_par & ~(1u << s)) | (ph << s);
        if (++s == SA) {
          s = 0;
          ph ^= 1;
        }
      };
      bool ok = true;
      for (int u = pair; u < n_units && ok; u += n_pairs) {
        const int nt = u % p.n_nt;
        const int e = units[3 * (u / p.n_nt)], row0 = units[3 * (u / p.n_nt) + 1] + (int)rank * 128;
        const int rA = kMN ? 0 : kmajor_row0(nt);
        const uint32_t s1 = (s + 1 == SA) ? 0 : s + 1, ph1 = (s + 1 == SA) ? ph ^ 1 : ph;
        if (!(ok = mbar_wait(&aempty[s], ph ^ 1, ctl, p.err, p.timeout_ns, 10))) break;
        if (!(ok = mbar_wait(&aempty[s1], ph1 ^ 1, ctl, p.err, p.timeout_ns, 10))) break;
        {
          uint8_t* la = aring + s * A_BYTES;
          uint8_t* lb = aring + s1 * A_BYTES;
          mbar_arrive_expect_tx(&xfull[s], (uint32_t)(512 * p.r_pad));
          tma_load_2d(la, &map_la, &xfull[s], 0, row0);
          if (!kMN) {
            tma_load_3d(lb, &map_lb, &xfull[s], 0, rA, e);
            tma_load_3d(lb + 128 * p.r_pad, &map_lb, &xfull[s], 0, rA + 64, e);
          } else {
            const int c0 = nt * 256 + rank * 128;
            tma_load_3d(lb, &map_lb, &xfull[s], c0, 0, e);
            tma_load_3d(lb + 128 * p.r_pad, &map_lb, &xfull[s], c0 + 64, 0, e);
          }
          mbar_arrive(&xfull[s1]);
          issued_next();
          issued_next();
        }
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!(ok = mbar_wait(&aempty[s], ph ^ 1, ctl, p.err, p.timeout_ns, 12))) break;
          mbar_arrive_expect_tx(&xfull[s], (uint32_t)A_BYTES);
          tma_load_2d(aring + s * A_BYTES, &map_a, &xfull[s], kc * BK, row0);
          issued_next();
        }
      }
      if (!ok) {
        for (int i = 0; i < SA; ++i)
          if (issued & (1u << i)) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&xfull[i], (last_par >> i) & 1u) &&
                   (long long)(globaltimer_ns() - t0) < p.timeout_ns) {
            }
          }
      }
    }
  } else if (warp == 1 && rank == 0) {
    // ------------------------------------------------ UMMA issuer (even CTA, one elected lane)
    // A 256x256x16 pair UMMA keeps the tensor pipe busy for about as long as
    // the issuing thread is blocked handing in the next one, so any gap between
    // the last UMMA of a k-chunk and the first of the next leaves the pipe
    // idle.  The readiness of the next k-chunk is therefore tested (without
    // blocking) while the current chunk's UMMAs are being handed in; only if it
    // is not ready yet does the thread fall back to a bounded wait.
    if (elect_one_sync()) {
      const uint32_t idesc = make_idesc_bf16(256, 256, false, kMN);
      const uint32_t lswz = swz_for_row_bytes(2 * p.r_pad);
      const uint32_t a_u = smem_u32(aring), b_u = smem_u32(bring);
      const uint32_t bstep = kMN ? 128u : 2u;  // K16 step of B in the descriptor address field
      // Descriptors of slot 0 of each ring; slot s adds s * slot bytes to the address field (bits 0-13,
      // address / 16: shared memory stays below 256 KB, so the sum cannot carry out of it).
      const uint64_t adesc0 = make_sdesc(a_u, 16, 1024, kSw128);
      const uint64_t bdesc0 = kMN ? make_sdesc(b_u, 8192, 1024, kSw128) : make_sdesc(b_u, 16, 1024, kSw128);
      uint32_t ti = 0;            // unit counter
      uint32_t sa = 0, sb = 0;    // activation slot, decoded-tile slot
      uint32_t fs = 0, fph = 0;   // MMA step: full[] slot and parity
      bool ok = true;
      auto next_a = [&]() { sa = (sa + 1 == SA) ? 0 : sa + 1; };
      auto next_f = [&]() {
        if (++fs == SA) {
          fs = 0;
          fph ^= 1;
        }
      };
      // Both CTAs' operands of the MMA step are in place (one barrier, signalled by the two relays).
      auto wait_step = [&]() -> bool { return mbar_wait_cluster(&full[fs], fph, ctl, p.err, p.timeout_ns, 23); };
      for (int u = pair; u < n_units && ok; u += n_pairs, ++ti) {
        const uint32_t b = ti & 1, use = ti >> 1;
        const uint32_t d = tmem + b * 256;
        if (!(ok = mbar_wait_cluster(&accempty[b], (use & 1) ^ 1, ctl, p.err, p.timeout_ns, 20))) break;
        tc_fence_after();
        // LoRA step first: acc = (s*p) . B_lora^T over K = r (overwrites the accumulator), from the unit's
        // two activation uses (p or q rows, then the LoRA weight rows).
        if (!(ok = wait_step())) break;
        tc_fence_after();
        {
          const uint32_t sa1 = (sa + 1 == SA) ? 0 : sa + 1;
          const uint32_t la_u = a_u + sa * A_BYTES, lb_u = a_u + sa1 * A_BYTES;
          for (int ks = 0; ks < p.r_pad / 16; ++ks) {
            const uint64_t bd = kMN ? make_sdesc(lb_u + 2048 * ks, 128 * p.r_pad, 1024, kSw128)
                                    : make_sdesc(lb_u + 32 * ks, 16, 16 * p.r_pad, lswz);
            umma_bf16_2sm(d, make_sdesc(la_u + 32 * ks, 16, 16 * p.r_pad, lswz), bd, idesc, ks > 0 ? 1u : 0u);
          }
          umma_commit_2sm(&aempty[sa], 0x3);
          umma_commit_2sm(&aempty[sa1], 0x3);
          next_a();
          next_a();
          next_f();
        }
        if (!(ok = wait_step())) break;
        tc_fence_after();
        for (int kc = 0; kc < kchunks; ++kc) {
          const uint64_t adesc = adesc0 + (uint64_t)(sa * (A_BYTES >> 4));
          const uint64_t bdesc = bdesc0 + (uint64_t)(sb * (B_BYTES >> 4));
          const uint32_t fs1 = (fs + 1 == SA) ? 0 : fs + 1, fph1 = (fs + 1 == SA) ? fph ^ 1 : fph;
          const bool more = kc + 1 < kchunks;
#pragma unroll
          for (int kk = 0; kk < BK / 16 - 1; ++kk)  // K16 step: +32 bytes of A; +32 (K-major) / +2048 bytes of B
            umma_bf16_2sm(d, adesc + 2 * kk, bdesc + bstep * kk, idesc, 1u);
          // Peek at the next k-chunk while the UMMAs above execute.
          const bool next_ready = more && mbar_test_wait_cluster(&full[fs1], fph1);
          umma_bf16_2sm(d, adesc + 2 * (BK / 16 - 1), bdesc + bstep * (BK / 16 - 1), idesc, 1u);
          umma_commit_2sm(&aempty[sa], 0x3);
          umma_commit_2sm(&bempty[sb], 0x3);
          next_a();
          sb = (sb + 1 == SB) ? 0 : sb + 1;
          fs = fs1;
          fph = fph1;
          if (more) {
            if (!next_ready && !(ok = wait_step())) break;
            tc_fence_after();
          }
        }
        if (!ok) break;
        umma_commit_2sm(&accfull[b], 0x3);
      }
      umma_commit_2sm(drain, 0x1);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0) && (long long)(globaltimer_ns() - t0) < p.timeout_ns) {
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------ relays: this CTA's operands of each MMA step (a
    // unit's LoRA operands, or a k-chunk's activation and decoded tiles) are in place -> the even CTA's
    // full[].  The odd CTA signals with one 4-byte st.async; the even CTA's relay arrives locally and
    // arms the 4 bytes (which may land first: the transaction count goes negative until then).  Off the
    // issuer's scheduler partition, so that the issuer tests one barrier per MMA step.
    const uint32_t full_even = mapa_shared(smem_u32(full), 0);
    const uint32_t sig_even = mapa_shared(smem_u32(sig), 0);
    uint32_t sa = 0, pha = 0, jb = 0, fs = 0;
    bool ok = true;
    auto wait_a = [&]() -> bool {
      const bool r = __all_sync(kFull, mbar_wait(&xfull[sa], pha, ctl, p.err, p.timeout_ns, 52));
      if (++sa == SA) {
        sa = 0;
        pha ^= 1;
      }
      return r;
    };
    auto signal = [&]() {
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive_expect_tx(&full[fs], 4);
        else
          st_async_signal(sig_even, full_even + 8 * fs, 1u);
      }
      fs = (fs + 1 == SA) ? 0 : fs + 1;
    };
    for (int u = pair; u < n_units && ok; u += n_pairs) {
      if (!(ok = wait_a()) || !(ok = wait_a())) break;  // the unit's two LoRA operand uses
      signal();
      for (int kc = 0; kc < kchunks; ++kc, ++jb) {
        ok = __all_sync(kFull, mbar_wait(&bdone[jb % SB], (jb / SB) & 1, ctl, p.err, p.timeout_ns, 51));
        if (!ok || !(ok = wait_a())) break;
        signal();
      }
    }
  } else if (warp >= 4 && warp < kEpiWarp0) {
    // ------------------------------------------------ NF4 decode, groups take the k-chunks round robin
    // Group g decodes the pair's k-chunks jj with jj % 4 == g (chunk jj: unit jj / kchunks of the pair,
    // k-chunk jj % kchunks) from code slot jj % RAW_STAGES into registers, then waits for its decoded-tile
    // slot g to be free and stores the tile.  Each thread loads the block scale of its row for its
    // group's next chunk while decoding the current one.
    const uint32_t grp = (warp - 4) >> 2;
    const int t = (threadIdx.x - 128) & 127;  // the weight row (K-major) / code column pair this thread decodes
    const Nf4Shift ks = nf4_shift_consts();
    const int raw_off = kMN ? (t & 63) * 64 + (t >> 6) * 32 : t * 32;
    // Row `drow` of the decoded 128B-swizzled tile: 16-byte chunk c at c ^ (drow % 8).
    const int drow = kMN ? (t & 63) : t;
    const uint32_t drow_off = (kMN ? (t >> 6) * 8192 : 0) + (drow >> 3) * 1024 + (drow & 7) * 128;
    const uint32_t b_u = smem_u32(bring) + grp * B_BYTES;
    // A cursor over this group's chunks, kept one chunk ahead of the decode: its k-chunk kc, unit u,
    // the unit's n-tile nt and expert e.  The block scale of this thread's row for the
    // cursor's chunk is loaded a group iteration before it is used, with no division and no dependent
    // load on the way (the expert of the unit after the cursor's is loaded a unit ahead): a stall there
    // would hold up the decode that follows it in this warp's instruction stream.
    const uint32_t n_chunks = (uint32_t)((n_units - pair + n_pairs - 1) / n_pairs) * (uint32_t)kchunks;
    auto unit_expert = [&](int u) -> int { return u < n_units ? units[3 * (u / p.n_nt)] : 0; };
    int c_kc = (int)grp, c_u = pair;
    while (c_kc >= kchunks) {
      c_kc -= kchunks;
      c_u += n_pairs;
    }
    int c_nt = c_u % p.n_nt, c_e = unit_expert(c_u), e_after = unit_expert(c_u + n_pairs);
    auto advance = [&]() {
      c_kc += kGroups;
      while (c_kc >= kchunks) {
        c_kc -= kchunks;
        c_u += n_pairs;
        c_nt = c_u % p.n_nt;
        c_e = e_after;
        e_after = unit_expert(c_u + n_pairs);
      }
    };
    // Block scale of this thread's row for the cursor's chunk (0 for rows past the end of the matrix:
    // all-zero decode).
    auto block_scale = [&]() -> float {
      if (c_u >= n_units || !row_valid(c_nt, t)) return 0.0f;
      size_t idx;
      if (!kMN)
        idx = ((size_t)c_e * p.stored_rows + kmajor_row0(c_nt) + t) * blocks_per_row + c_kc;
      else
        idx = ((size_t)c_e * p.stored_rows + c_kc * BK + (t & 63)) * blocks_per_row + c_nt * 4 + rank * 2 + (t >> 6);
      return __ldg(p.absmax + idx);
    };
    float amax_next = block_scale();
    bool ok = true;
    for (uint32_t jj = grp; jj < n_chunks && ok; jj += kGroups) {
      const float amax = amax_next;
      advance();  // the cursor moves to this group's next chunk
      const uint32_t r = jj % RAW_STAGES, rph = (jj / RAW_STAGES) & 1;
      ok = __all_sync(kFull, mbar_wait(&raw_full[r], rph, ctl, p.err, p.timeout_ns, 30));
      if (!ok) break;
      const uint8_t* slot = rawbuf + r * RAW_SLOT;
      const uint4 q0 = *reinterpret_cast<const uint4*>(slot + raw_off);
      const uint4 q1 = *reinterpret_cast<const uint4*>(slot + raw_off + 16);
      const uint32_t codes[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
      // The codes are in registers: hand the code slot back before decoding, so the producer refills it
      // a whole decode earlier (the proxy fence orders these generic reads before the next TMA write).
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&raw_empty[r]);
      amax_next = block_scale();
      const Nf4Planes pl = nf4_block_planes(amax);
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < 8; ++c) nf4_decode_word(codes[c], pl, ks, &v[4 * c]);
      // slot grp's previous use (this group's chunk jj - 4) consumed by its UMMAs
      ok = __all_sync(kFull, mbar_wait(&bempty[grp], ((jj / kGroups) & 1) ^ 1, ctl, p.err, p.timeout_ns, 31));
      if (!ok) break;
      const uint32_t dbase = b_u + drow_off;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        st_shared_v4(dbase + ((c ^ (drow & 7)) << 4), v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
      // The proxy fence orders the tile stores before the UMMA reads them.
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bdone[grp]);
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------ epilogue
    // Output tiles of a 16-column step (32 rows x 16 columns, 1 KB each) are
    // staged in this warp's shared memory and written by TMA bulk stores:
    // per-row global stores (32 rows per warp instruction) congest the L1
    // path that the UMMAs read their operands through (measured: the k-chunks
    // running beside an epilogue took twice as long).  The down dgrad keeps
    // direct stores (see there).
    const int qrt = warp & 3;  // TMEM lane quarter of this warp
    const uint32_t accempty_even = mapa_shared(smem_u32(accempty), 0);
    const uint32_t ebuf = smem_u32(smem + EPI_OFF + qrt * kEpiWarpBytes);
    if (lane == 0) {
      tma_prefetch_desc(&map_o0);
      tma_prefetch_desc(&map_o1);
    }
    uint32_t ti = 0, step = 0;
    bool ok = true;
    // Staging buffer of this step, free once the stores of the step two back have read it.
    auto step_buffer = [&]() -> uint32_t {
      if (lane == 0) bulk_wait_read<1>();
      __syncwarp();
      return ebuf + (step & 1) * kEpiStepBytes;
    };
    auto stage = [&](uint32_t buf, int tile, const uint32_t (&w)[8]) {
      const uint32_t a = buf + tile * kEpiTileBytes + lane * 32;
      st_shared_v4(a, w[0], w[1], w[2], w[3]);
      st_shared_v4(a + 16, w[4], w[5], w[6], w[7]);
    };
    auto publish = [&]() {  // the staged tiles are visible to the TMA (async proxy)
      fence_proxy_async_smem();
      __syncwarp();
    };
    for (int u = pair; u < n_units && ok; u += n_pairs, ++ti) {
      const int mu = u / p.n_nt, nt = u % p.n_nt;
      const int nrows = units[3 * mu + 2];
      const bool store = (int)rank * 128 < nrows;
      const int wrow0 = units[3 * mu + 1] + (int)rank * 128 + qrt * 32;  // this warp's first row
      const size_t row = (size_t)wrow0 + lane;
      const uint32_t b = ti & 1, use = ti >> 1;
      ok = __all_sync(kFull, mbar_wait(&accfull[b], use & 1, ctl, p.err, p.timeout_ns, 40));
      if (!ok) break;
      tc_fence_after();
      const uint32_t tl = tmem + b * 256 + ((uint32_t)(qrt * 32) << 16);
      if (MODE == kFwdGateUp) {
        // columns [0,128): gate, [128,256): up, of gate/up columns nt*128 ..
        const int c0 = nt * 128;
#pragma unroll 1
        for (int jj = 0; jj < 128; jj += 16) {
          if (c0 + jj >= p.I) break;
          float g[16], up[16];
          tmem_ld16(tl + jj, g);
          tmem_ld16(tl + 128 + jj, up);
          if (!store) continue;
          uint32_t gw[8], uw[8], aw[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            gw[i] = pack_bf16x2(g[2 * i], g[2 * i + 1]);
            uw[i] = pack_bf16x2(up[2 * i], up[2 * i + 1]);
            aw[i] = pack_bf16x2(silu_f(g[2 * i]) * up[2 * i], silu_f(g[2 * i + 1]) * up[2 * i + 1]);
          }
          const uint32_t buf = step_buffer();
          stage(buf, 0, gw);
          stage(buf, 1, uw);
          stage(buf, 2, aw);
          publish();
          if (lane == 0) {
            tma_store_2d(&map_o0, buf, c0 + jj, wrow0);
            tma_store_2d(&map_o0, buf + kEpiTileBytes, p.I + c0 + jj, wrow0);
            tma_store_2d(&map_o1, buf + 2 * kEpiTileBytes, c0 + jj, wrow0);
            bulk_commit();
          }
          ++step;
        }
      } else if (MODE == kDgradDown) {
        // SwiGLU backward.  The forward gate/up values of a row are copied
        // with cp.async into a per-warp ring in the (here unused) staging
        // area, kDgAhead steps ahead of their use, so that the step loop waits
        // for none of them: one step ahead left this epilogue longer than the
        // unit's UMMAs.  Ring slot layout [step % kDgAhead][piece][lane] x 16
        // bytes: a warp's reads of one piece are 512 contiguous bytes.
        const int I2 = 2 * p.I, c0 = nt * 256;
        const int ncol = min(256, p.I - c0);  // a multiple of 64
        const uint16_t* grow = p.aux + row * I2 + c0;
        if (store) {
          // The unit's gate/up values of this row (2 x ncol bf16, from HBM: the
          // buffer is larger than L2) are pulled into L2 up front.
          for (int off = 0; off < ncol; off += 64) {
            asm volatile("prefetch.global.L2 [%0];" ::"l"(grow + off));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(grow + p.I + off));
          }
        }
        uint8_t* ring = smem + EPI_OFF + qrt * kEpiWarpBytes + lane * 16;
        // copies of 16-column step js (gate: pieces 0-1, up: pieces 2-3); past the row's end nothing is read
        auto issue = [&](int js) {
          const int col = js * 16;
          const uint32_t n = (store && col < ncol) ? 16u : 0u;
          const uint16_t* g = n ? grow + col : grow;
          uint8_t* dst = ring + (js % kDgAhead) * 4 * 512;
          cp_async_16_zfill(dst, g, n);
          cp_async_16_zfill(dst + 512, g + 8, n);
          cp_async_16_zfill(dst + 1024, n ? g + p.I : grow, n);
          cp_async_16_zfill(dst + 1536, n ? g + p.I + 8 : grow, n);
          cp_async_commit();
        };
#pragma unroll
        for (int js = 0; js < kDgAhead - 1; ++js) issue(js);
#pragma unroll 1
        for (int jj = 0; jj < ncol; jj += 16) {
          issue(jj / 16 + kDgAhead - 1);
          cp_async_wait_group<kDgAhead - 1>();  // this thread's copies of step jj/16 have landed
          float da[16];
          tmem_ld16(tl + jj, da);
          if (store) {
            const uint8_t* src = ring + ((jj / 16) % kDgAhead) * 4 * 512;
            const uint4 g0 = *reinterpret_cast<const uint4*>(src);
            const uint4 g1 = *reinterpret_cast<const uint4*>(src + 512);
            const uint4 u0 = *reinterpret_cast<const uint4*>(src + 1024);
            const uint4 u1 = *reinterpret_cast<const uint4*>(src + 1536);
            const uint32_t gw[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            const uint32_t uw[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            uint32_t dgw[8], duw[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float dg[2], du[2];
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                const float gg = hh ? bf16hi_to_f32(gw[i]) : bf16lo_to_f32(gw[i]);
                const float uu = hh ? bf16hi_to_f32(uw[i]) : bf16lo_to_f32(uw[i]);
                const float dd = da[2 * i + hh];
                const float sg = sigmoid_f(gg);
                dg[hh] = dd * uu * sg * (1.0f + gg * (1.0f - sg));
                du[hh] = dd * gg * sg;
              }
              dgw[i] = pack_bf16x2(dg[0], dg[1]);
              duw[i] = pack_bf16x2(du[0], du[1]);
            }
            // Direct full-sector stores here: this epilogue is as long as the
            // unit's UMMAs, and the staging hand-off would lengthen it.
            store_row16(p.out0 + row * I2 + c0 + jj, dgw, p.v8);
            store_row16(p.out0 + row * I2 + p.I + c0 + jj, duw, p.v8);
          }
        }
      } else {
        // 32-column steps (n_dim is a multiple of 64): two 16-column tiles per step from a ring of
        // three 2 KB buffers, so that a unit's accumulator is drained in 8 steps, each with one
        // TMEM wait and one proxy fence (in the down projection's short units the epilogue would
        // otherwise hold the accumulator past the next unit's start).
        const int c0 = nt * 256;
#pragma unroll 1
        for (int jj = 0; jj < 256; jj += 32) {
          if (c0 + jj >= p.n_dim) break;
          float v[32];
          tmem_ld32(tl + jj, v);
          if (!store) continue;
          uint32_t w0[8], w1[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            w0[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
            w1[i] = pack_bf16x2(v[16 + 2 * i], v[16 + 2 * i + 1]);
          }
          if (lane == 0) bulk_wait_read<2>();
          __syncwarp();
          const uint32_t buf = ebuf + (step % 3) * (2 * kEpiTileBytes);
          stage(buf, 0, w0);
          stage(buf, 1, w1);
          publish();
          if (lane == 0) {
            tma_store_2d(&map_o0, buf, c0 + jj, wrow0);
            tma_store_2d(&map_o0, buf + kEpiTileBytes, c0 + jj + 16, wrow0);
            bulk_commit();
          }
          ++step;
        }
      }
      // The issuer needs only this warp's TMEM reads to be complete (tcgen05.ld
      // waited, then the tcgen05 fence), not its global stores: the odd CTA's
      // arrival is relaxed, since a release would first wait for the stores.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(&accempty[b]);
        else
          mbar_arrive_cluster_relaxed(accempty_even + 8 * b);
      }
    }
    // Every bulk store of this warp has written global memory (and stopped
    // reading its staging buffer), and every cp.async has landed, before the CTA goes away.
    if (lane == 0) bulk_wait<0>();
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncwarp();
  }

  __syncwarp();  // reconverge each warp (its lane 0 ran a role loop) before the cluster barrier
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_2sm(tmem, kTmemCols);
  }
}

// =============================================================================
// LoRA projection: out[rows, r] = bf16(scale * act[rows, K] . W_e)
// =============================================================================
namespace lproj {
constexpr int BM = 128, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BK * E4B_MAX_RANK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 24 KB
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 1024;
constexpr int kThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kAccCols = 64;    // one accumulator: 128 rows x r_pad <= 64 fp32 columns
constexpr int kTmemCols = 2 * kAccCols;  // two: a unit's MMAs overlap the previous unit's epilogue
static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
}  // namespace lproj

struct LoraProjParams {
  const int32_t* tiles;
  uint16_t* out;
  DeviceError* err;
  long long timeout_ns;
  float scale;
  int K, r, r_pad;
};

template <bool W_MN>
__global__ void __launch_bounds__(lproj::kThreads)
    lora_proj_kernel(const __grid_constant__ CUtensorMap map_act, const __grid_constant__ CUtensorMap map_w,
                     const LoraProjParams p) {
  using namespace lproj;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = align1024(smem_dyn);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* accfull = bars + 2 * STAGES;  // [2]
  uint64_t* accempty = accfull + 2;       // [2]
  uint64_t* drain = accfull + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfull + 5);
  CtaControl* ctl = reinterpret_cast<CtaControl*>(accfull + 6);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 4);
    }
    mbar_init(drain, 1);
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
  const int n_units = p.tiles[0];
  const int kchunks = p.K / BK;
  const uint32_t b_bytes = BK * p.r_pad * 2;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&map_act);
      tma_prefetch_desc(&map_w);
      int s = 0;
      uint32_t ph = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const int e = p.tiles[kTileHeader + 2 * u], row0 = p.tiles[kTileHeader + 2 * u + 1];
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!(ok = mbar_wait(&empty[s], ph ^ 1, ctl, p.err, p.timeout_ns, 110))) break;
          uint8_t* st = smem + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], A_BYTES + b_bytes);
          tma_load_2d(st, &map_act, &full[s], kc * BK, row0);
          if (W_MN)
            tma_load_3d(st + A_BYTES, &map_w, &full[s], 0, kc * BK, e);
          else
            tma_load_3d(st + A_BYTES, &map_w, &full[s], kc * BK, 0, e);
          issued |= 1u << s;
          last_par = (last_par & ~(1u << s)) | (ph << s);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok) {
        for (int i = 0; i < STAGES; ++i)
          if (issued & (1u << i)) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&full[i], (last_par >> i) & 1u) &&
                   (long long)(globaltimer_ns() - t0) < p.timeout_ns) {
            }
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc_bf16(BM, p.r_pad, false, W_MN);
      const uint32_t wswz = swz_for_row_bytes(2 * p.r_pad);
      int s = 0;
      uint32_t ph = 0, ti = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++ti) {
        const uint32_t b = ti & 1, use = ti >> 1;
        if (!(ok = mbar_wait(&accempty[b], (use & 1) ^ 1, ctl, p.err, p.timeout_ns, 120))) break;
        tc_fence_after();
        const uint32_t acc = tmem + b * kAccCols;
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!(ok = mbar_wait(&full[s], ph, ctl, p.err, p.timeout_ns, 121))) break;
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * STAGE_BYTES), b0 = a0 + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = make_sdesc(a0 + 32 * kk, 16, 1024, kSw128);
            const uint64_t bd = W_MN ? make_sdesc(b0 + 32 * p.r_pad * kk, b_bytes, 16 * p.r_pad, wswz)
                                     : make_sdesc(b0 + 32 * kk, 16, 1024, kSw128);
            umma_bf16(acc, ad, bd, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&accfull[b]);
      }
      umma_commit(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0) && (long long)(globaltimer_ns() - t0) < p.timeout_ns) {
      }
    }
  } else {
    const int q = ((warp & 3) << 5) | lane;  // TMEM lane of this thread
    uint32_t ti = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++ti) {
      const uint32_t b = ti & 1, use = ti >> 1;
      const uint32_t tl = tmem + b * kAccCols + ((uint32_t)(32 * (warp & 3)) << 16);
      const size_t row = (size_t)p.tiles[kTileHeader + 2 * u + 1] + q;
      ok = mbar_wait(&accfull[b], use & 1, ctl, p.err, p.timeout_ns, 130);
      ok = __all_sync(kFull, ok);
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int j = 0; j < p.r_pad; j += 16) {
        float v[16];
        tmem_ld16(tl + j, v);
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(p.scale * v[2 * i], p.scale * v[2 * i + 1]);
        uint4* d = reinterpret_cast<uint4*>(p.out + row * p.r + j);
        if (j < p.r) d[0] = make_uint4(w[0], w[1], w[2], w[3]);
        if (j + 8 < p.r) d[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[b]);
    }
  }
  __syncwarp();  // reconverge each warp (its lane 0 ran a role loop) before the CTA barrier
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// =============================================================================
// Row gather fused with the LoRA projection:
//   dst[row] = bf16(w(slot) * src[token of row])  (zero for padding rows)
//   out[row] = bf16(scale * dst[row] . W_e)       over K, r outputs
// The gathered 128-row x 64-column tile is copied into shared memory (in the
// UMMA's 128B-swizzled K-major layout) by four loader warps with cp.async
// (8 lanes per 128-byte row piece, coalesced; zero-filled for padding rows),
// as many k-chunks ahead as there are free slots; for a weighted gather four
// more warps scale the landed tile in place.  The tensor core reads the tile
// as the A operand of the projection and a TMA bulk store writes the same tile
// to dst, so the permuted rows are read from HBM by no later projection.
// =============================================================================
namespace gproj {
constexpr int BM = 128, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BK * E4B_MAX_RANK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 24 KB
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 1024;
// warps 0-3 row loaders (32 tile rows each), 4-7 scalers (weighted gather only), 8 W loader,
// 9 UMMA issuer + TMEM owner, 10 tile storer, 11-14 epilogue
constexpr int kLoadWarps = 4, kScaleWarp0 = 4, kScaleWarps = 4;
constexpr int kWLoadWarp = 8, kIssueWarp = 9, kStoreWarp = 10, kEpiWarp0 = 11;
constexpr int kThreads = 15 * 32;
constexpr int kAccCols = 64;
constexpr int kTmemCols = 2 * kAccCols;
static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
}  // namespace gproj

struct GatherProjParams {
  const uint16_t* src;        // [T, K] token rows
  const int32_t* slot_of_row;
  const float* scale_w;       // [T*k] per-slot factor, or nullptr
  const int32_t* tiles;
  uint16_t* out;              // [rows_cap, r]
  DeviceError* err;
  long long timeout_ns;
  float scale;
  int K, r, r_pad, k;
};

template <bool W_MN>
__global__ void __launch_bounds__(gproj::kThreads, 2)  // two CTAs per SM: <= 64 registers
    gather_proj_kernel(const __grid_constant__ CUtensorMap map_dst, const __grid_constant__ CUtensorMap map_w,
                       const GatherProjParams p) {
  using namespace gproj;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = align1024(smem_dyn);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* full = bars;                 // [STAGES] tile complete (+ the W bytes)
  uint64_t* empty = bars + STAGES;       // [STAGES] the UMMAs read the slot
  uint64_t* stored = bars + 2 * STAGES;  // [STAGES] the bulk store read the tile
  uint64_t* landed = bars + 3 * STAGES;  // [STAGES] (weighted gather) the row copies landed
  uint64_t* accfull = bars + 4 * STAGES;  // [2]
  uint64_t* accempty = accfull + 2;       // [2]
  uint64_t* drain = accfull + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfull + 5);
  CtaControl* ctl = reinterpret_cast<CtaControl*>(accfull + 6);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    const bool scaled = p.scale_w != nullptr;
    for (int i = 0; i < STAGES; ++i) {
      // each loader thread's cp.async arrival (.noinc) counts once; the W loader's expect_tx once
      mbar_init(&full[i], (scaled ? kScaleWarps : kLoadWarps * 32) + 1);
      mbar_init(&empty[i], 1);
      mbar_init(&stored[i], 1);
      mbar_init(&landed[i], kLoadWarps * 32);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 4);
    }
    mbar_init(drain, 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == kIssueWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_units = p.tiles[0];
  const int rows_used = p.tiles[1];
  const int kchunks = p.K / BK;
  const uint32_t b_bytes = BK * p.r_pad * 2;

  if (warp < kLoadWarps) {
    // ------------------------------------------------ row loaders: warp w copies rows 32w..32w+31; per
    // instruction i lane l copies 16-byte piece l%8 of row 32w + 4i + l/8 (cp.async, no registers held)
    const int c = lane & 7;
    uint64_t* done = (p.scale_w != nullptr) ? landed : full;
    uint32_t s = 0, ph = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const int row0 = p.tiles[kTileHeader + 2 * u + 1];
      const uint16_t* src[8];
      uint32_t nbytes[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int row = row0 + 32 * warp + 4 * i + (lane >> 3);
        const int slot = (row < rows_used) ? __ldg(p.slot_of_row + row) : -1;
        src[i] = p.src + ((slot >= 0) ? (size_t)(slot / p.k) * p.K : 0) + 8 * c;
        nbytes[i] = (slot >= 0) ? 16u : 0u;  // padding rows: zero fill, nothing read
      }
      for (int kc = 0; kc < kchunks; ++kc) {
        // warp-uniform waits: every lane leaves the loop together on a timeout
        if (!(ok = __all_sync(kFull, mbar_wait(&empty[s], ph ^ 1, ctl, p.err, p.timeout_ns, 60)))) break;
        if (!(ok = __all_sync(kFull, mbar_wait(&stored[s], ph ^ 1, ctl, p.err, p.timeout_ns, 61)))) break;
        uint8_t* tile = smem + s * STAGE_BYTES;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int q = 32 * warp + 4 * i + (lane >> 3);  // tile row
          cp_async_16_zfill(tile + (q >> 3) * 1024 + (q & 7) * 128 + ((c ^ (q & 7)) << 4), src[i] + kc * BK,
                            nbytes[i]);
        }
        cp_async_arrive_noinc(&done[s]);
        if (++s == STAGES) {
          s = 0;
          ph ^= 1;
        }
      }
    }
    // every copy of this thread has landed before the CTA's shared memory can go away (a timeout
    // elsewhere may end the loops with copies still in flight)
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp < kScaleWarp0 + kScaleWarps) {
    // ------------------------------------------------ scalers (weighted gather): row *= w(slot) in place
    if (p.scale_w != nullptr) {
      const int sw = warp - kScaleWarp0, c = lane & 7;
      uint32_t s = 0, ph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const int row0 = p.tiles[kTileHeader + 2 * u + 1];
        float w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int row = row0 + 32 * sw + 4 * i + (lane >> 3);
          const int slot = (row < rows_used) ? __ldg(p.slot_of_row + row) : -1;
          w[i] = (slot >= 0) ? __ldg(p.scale_w + slot) : 0.0f;
        }
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!(ok = __all_sync(kFull, mbar_wait(&landed[s], ph, ctl, p.err, p.timeout_ns, 67)))) break;
          uint8_t* tile = smem + s * STAGE_BYTES;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int q = 32 * sw + 4 * i + (lane >> 3);
            uint4* pc = reinterpret_cast<uint4*>(tile + (q >> 3) * 1024 + (q & 7) * 128 + ((c ^ (q & 7)) << 4));
            uint4 x = *pc;
            uint32_t* xw = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              xw[e] = pack_bf16x2(w[i] * bf16lo_to_f32(xw[e]), w[i] * bf16hi_to_f32(xw[e]));
            *pc = x;
          }
          fence_proxy_async_smem();  // visible to the tensor core and the bulk store
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[s]);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
      }
    }
  } else if (warp == kWLoadWarp) {
    // ------------------------------------------------ LoRA factor chunks (TMA, one lane)
    if (lane == 0) {
      tma_prefetch_desc(&map_w);
      uint32_t s = 0, ph = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const int e = p.tiles[kTileHeader + 2 * u];
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!(ok = mbar_wait(&empty[s], ph ^ 1, ctl, p.err, p.timeout_ns, 62))) break;
          uint8_t* st = smem + s * STAGE_BYTES + A_BYTES;
          mbar_arrive_expect_tx(&full[s], b_bytes);
          if (W_MN)
            tma_load_3d(st, &map_w, &full[s], 0, kc * BK, e);
          else
            tma_load_3d(st, &map_w, &full[s], kc * BK, 0, e);
          issued |= 1u << s;
          last_par = (last_par & ~(1u << s)) | (ph << s);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok) {  // let issued copies land before shared memory goes away
        for (int i = 0; i < STAGES; ++i)
          if (issued & (1u << i)) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&full[i], (last_par >> i) & 1u) &&
                   (long long)(globaltimer_ns() - t0) < p.timeout_ns) {
            }
          }
      }
    }
  } else if (warp == kIssueWarp) {
    // ------------------------------------------------ UMMA issuer (one lane)
    if (lane == 0) {
      const uint32_t idesc = make_idesc_bf16(BM, p.r_pad, false, W_MN);
      const uint32_t wswz = swz_for_row_bytes(2 * p.r_pad);
      uint32_t s = 0, ph = 0, ti = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++ti) {
        const uint32_t b = ti & 1, use = ti >> 1;
        if (!(ok = mbar_wait(&accempty[b], (use & 1) ^ 1, ctl, p.err, p.timeout_ns, 63))) break;
        tc_fence_after();
        const uint32_t acc = tmem + b * kAccCols;
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!(ok = mbar_wait(&full[s], ph, ctl, p.err, p.timeout_ns, 64))) break;
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * STAGE_BYTES), b0 = a0 + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = make_sdesc(a0 + 32 * kk, 16, 1024, kSw128);
            const uint64_t bd = W_MN ? make_sdesc(b0 + 32 * p.r_pad * kk, b_bytes, 16 * p.r_pad, wswz)
                                     : make_sdesc(b0 + 32 * kk, 16, 1024, kSw128);
            umma_bf16(acc, ad, bd, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&accfull[b]);
      }
      umma_commit(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0) && (long long)(globaltimer_ns() - t0) < p.timeout_ns) {
      }
    }
  } else if (warp == kStoreWarp) {
    // ------------------------------------------------ gathered tiles -> dst (TMA bulk stores, one lane)
    // A slot is handed back once its store's shared-memory reads are done: for
    // the plain gather that is checked when the next chunk's store has been
    // issued (two stores in flight), for the weighted gather (whose slots also
    // pass through the scalers) right after each store.  A slot held until the
    // store two chunks later was issued kept the row loads ~2 chunks deep: both
    // gathers ran 15-25% longer (measured).
    constexpr int kStoreLag = 1;
    const bool wait_each = p.scale_w != nullptr;
    if (lane == 0) {
      tma_prefetch_desc(&map_dst);
      uint32_t s = 0, ph = 0, pend[kStoreLag];
      int n_pend = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const int row0 = p.tiles[kTileHeader + 2 * u + 1];
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!(ok = mbar_wait(&full[s], ph, ctl, p.err, p.timeout_ns, 65))) break;
          fence_proxy_async_smem();
          tma_store_2d(&map_dst, smem_u32(smem + s * STAGE_BYTES), kc * BK, row0);
          bulk_commit();
          if (wait_each) {
            bulk_wait_read<0>();
            mbar_arrive(&stored[s]);
          } else if (n_pend == kStoreLag) {
            bulk_wait_read<kStoreLag>();  // the oldest pending store has read its slot
            mbar_arrive(&stored[pend[0]]);
#pragma unroll
            for (int i = 0; i + 1 < kStoreLag; ++i) pend[i] = pend[i + 1];
            --n_pend;
          }
          if (!wait_each) pend[n_pend++] = s;
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      bulk_wait<0>();  // reads and writes of every store done
      for (int i = 0; i < n_pend; ++i) mbar_arrive(&stored[pend[i]]);
    }
  } else {
    // ------------------------------------------------ epilogue: TMEM -> bf16(scale * acc) rows
    const int q = ((warp & 3) << 5) | lane;  // TMEM lane of this thread
    uint32_t ti = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++ti) {
      const uint32_t b = ti & 1, use = ti >> 1;
      const uint32_t tl = tmem + b * kAccCols + ((uint32_t)(32 * (warp & 3)) << 16);
      const size_t row = (size_t)p.tiles[kTileHeader + 2 * u + 1] + q;
      ok = mbar_wait(&accfull[b], use & 1, ctl, p.err, p.timeout_ns, 66);
      ok = __all_sync(kFull, ok);
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int j = 0; j < p.r_pad; j += 16) {
        float v[16];
        tmem_ld16(tl + j, v);
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(p.scale * v[2 * i], p.scale * v[2 * i + 1]);
        uint4* d = reinterpret_cast<uint4*>(p.out + row * p.r + j);
        if (j < p.r) d[0] = make_uint4(w[0], w[1], w[2], w[3]);
        if (j + 8 < p.r) d[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[b]);
    }
  }
  __syncwarp();
  __syncthreads();
  if (warp == kIssueWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// =============================================================================
// LoRA weight gradients: out_g[e] = act_g[rows of e]^T . low_g[rows of e]
// =============================================================================
namespace wg {
constexpr int BM = 128, BK = 64, STAGES = 4;
constexpr int A_BYTES = BK * BM * 2;            // 64 rows x 128 features, MN-major SW128
constexpr int B_BYTES = BK * E4B_MAX_RANK * 2;  // 64 rows x r_pad, MN-major
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 1024;
constexpr int kThreads = 192;
constexpr int kAccCols = 64;             // one accumulator: 128 features x r_pad <= 64 fp32 columns
constexpr int kTmemCols = 2 * kAccCols;  // two: a unit's MMAs overlap the previous unit's epilogue
static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
}  // namespace wg

struct WgradParams {
  uint16_t* out[4];
  int F[4];
  int n_ft[4];
  int transposed_mask;
  int units_per_expert;
  int E, r, r_pad;
  int64_t mt_cap;
  const int32_t* counts;
  const int32_t* offsets;
  const int32_t* tiles;
  DeviceError* err;
  long long timeout_ns;
};

struct WgradUnit {
  int g, ft, e, nk;
};

__device__ __forceinline__ WgradUnit wgrad_unit(const WgradParams& p, int u) {
  WgradUnit w;
  const int erank = u / p.units_per_expert;
  int rem = u - erank * p.units_per_expert;
  w.g = 0;
#pragma unroll
  for (int i = 0; i < 3; ++i)
    if (w.g == i && rem >= p.n_ft[i]) {
      rem -= p.n_ft[i];
      w.g = i + 1;
    }
  w.ft = rem;
  w.e = p.tiles[kTileHeader + 2 * p.mt_cap + erank];
  w.nk = ((p.counts[w.e] + 127) / 128) * 2;  // 64-row K chunks over the padded group
  return w;
}

__global__ void __launch_bounds__(wg::kThreads)
    wgrad_kernel(const __grid_constant__ CUtensorMap act0, const __grid_constant__ CUtensorMap act1,
                 const __grid_constant__ CUtensorMap act2, const __grid_constant__ CUtensorMap act3,
                 const __grid_constant__ CUtensorMap low0, const __grid_constant__ CUtensorMap low1,
                 const __grid_constant__ CUtensorMap low2, const __grid_constant__ CUtensorMap low3,
                 const WgradParams p) {
  using namespace wg;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = align1024(smem_dyn);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* accfull = bars + 2 * STAGES;  // [2]
  uint64_t* accempty = accfull + 2;       // [2]
  uint64_t* drain = accfull + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfull + 5);
  CtaControl* ctl = reinterpret_cast<CtaControl*>(accfull + 6);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 4);
    }
    mbar_init(drain, 1);
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
  const int n_units = p.E * p.units_per_expert;
  const uint32_t b_bytes = BK * p.r_pad * 2;

  if (warp == 0) {
    if (lane == 0) {
      const CUtensorMap* amaps[4] = {&act0, &act1, &act2, &act3};
      const CUtensorMap* lmaps[4] = {&low0, &low1, &low2, &low3};
      int s = 0;
      uint32_t ph = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const WgradUnit w = wgrad_unit(p, u);
        const int row0 = p.offsets[w.e];
        for (int kc = 0; kc < w.nk; ++kc) {
          if (!(ok = mbar_wait(&empty[s], ph ^ 1, ctl, p.err, p.timeout_ns, 210))) break;
          uint8_t* st = smem + s * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], A_BYTES + b_bytes);
          tma_load_2d(st, amaps[w.g], &full[s], w.ft * BM, row0 + kc * BK);
          tma_load_2d(st + A_BYTES / 2, amaps[w.g], &full[s], w.ft * BM + 64, row0 + kc * BK);
          tma_load_2d(st + A_BYTES, lmaps[w.g], &full[s], 0, row0 + kc * BK);
          issued |= 1u << s;
          last_par = (last_par & ~(1u << s)) | (ph << s);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok) {
        for (int i = 0; i < STAGES; ++i)
          if (issued & (1u << i)) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&full[i], (last_par >> i) & 1u) &&
                   (long long)(globaltimer_ns() - t0) < p.timeout_ns) {
            }
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc_bf16(BM, p.r_pad, true, true);
      const uint32_t lswz = swz_for_row_bytes(2 * p.r_pad);
      int s = 0;
      uint32_t ph = 0, ti = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++ti) {
        const WgradUnit w = wgrad_unit(p, u);
        const uint32_t b = ti & 1, use = ti >> 1;
        if (!(ok = mbar_wait(&accempty[b], (use & 1) ^ 1, ctl, p.err, p.timeout_ns, 220))) break;
        tc_fence_after();
        const uint32_t acc = tmem + b * kAccCols;
        for (int kc = 0; kc < w.nk; ++kc) {
          if (!(ok = mbar_wait(&full[s], ph, ctl, p.err, p.timeout_ns, 221))) break;
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * STAGE_BYTES), b0 = a0 + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = make_sdesc(a0 + 2048 * kk, A_BYTES / 2, 1024, kSw128);
            const uint64_t bd = make_sdesc(b0 + 32 * p.r_pad * kk, b_bytes, 16 * p.r_pad, lswz);
            umma_bf16(acc, ad, bd, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&accfull[b]);
      }
      umma_commit(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0) && (long long)(globaltimer_ns() - t0) < p.timeout_ns) {
      }
    }
  } else {
    const int q = ((warp & 3) << 5) | lane;
    uint32_t ti = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++ti) {
      const WgradUnit w = wgrad_unit(p, u);
      const uint32_t b = ti & 1, use = ti >> 1;
      const uint32_t tl = tmem + b * kAccCols + ((uint32_t)(32 * (warp & 3)) << 16);
      ok = mbar_wait(&accfull[b], use & 1, ctl, p.err, p.timeout_ns, 230);
      ok = __all_sync(kFull, ok);
      if (!ok) break;
      tc_fence_after();
      const int F = p.F[w.g];
      const int m = w.ft * BM + q;
      const bool tr = (p.transposed_mask >> w.g) & 1;
      uint16_t* out = p.out[w.g];
#pragma unroll 1
      for (int j = 0; j < p.r_pad; j += 16) {
        float v[16];
        if (w.nk > 0) {
          tmem_ld16(tl + j, v);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = 0.0f;
        }
        if (m < F) {
          if (!tr) {
            uint32_t pw[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) pw[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
            uint4* d = reinterpret_cast<uint4*>(out + ((size_t)w.e * F + m) * p.r + j);
            if (j < p.r) d[0] = make_uint4(pw[0], pw[1], pw[2], pw[3]);
            if (j + 8 < p.r) d[1] = make_uint4(pw[4], pw[5], pw[6], pw[7]);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (j + i < p.r) {
                const __nv_bfloat16 b = __float2bfloat16_rn(v[i]);
                out[((size_t)w.e * p.r + j + i) * F + m] = *reinterpret_cast<const uint16_t*>(&b);
              }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[b]);
    }
  }
  __syncwarp();  // reconverge each warp (its lane 0 ran a role loop) before the CTA barrier
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// =============================================================================
// Host-side launchers
// =============================================================================
CUtensorMapSwizzle swizzle_for_bytes(int row_bytes) {
  return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// 2-D bf16 matrix [rows, cols] row-major.
cudaError_t map_bf16_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                        uint32_t box_rows, CUtensorMapSwizzle swz) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t strides[1] = {cols * 2};
  const uint32_t box[2] = {box_cols, box_rows};
  return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, swz);
}

// 3-D bf16 stack [E, rows, cols].
cudaError_t map_bf16_3d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t E,
                        uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  const uint64_t dims[3] = {cols, rows, E};
  const uint64_t strides[2] = {cols * 2, cols * rows * 2};
  const uint32_t box[3] = {box_cols, box_rows, 1};
  return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, swz);
}

// 3-D byte stack [E, rows, bytes].
cudaError_t map_u8_3d(CUtensorMap* m, const void* base, uint64_t bytes, uint64_t rows, uint64_t E,
                      uint32_t box_bytes, uint32_t box_rows, CUtensorMapSwizzle swz) {
  const uint64_t dims[3] = {bytes, rows, E};
  const uint64_t strides[2] = {bytes, bytes * rows};
  const uint32_t box[3] = {box_bytes, box_rows, 1};
  return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box, swz);
}

namespace {
template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}
}  // namespace

cudaError_t launch_nf4_gemm(const Nf4GemmHost& h, int num_sms, cudaStream_t stream) {
  const bool mn = (h.mode == kDgradDown || h.mode == kDgradGateUp);
  CUtensorMap ma, mraw, mla, mlb, mo0, mo1;
  cudaError_t err;
  if ((err = map_bf16_2d(&ma, h.act_in, h.K, h.rows_cap, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess)
    return err;
  // Epilogue outputs, written as 32-row x 16-column tiles: out0 [rows, n_dim] (gate_up forward: [rows, 2I]
  // with n_dim = 2I; down dgrad: dgu [rows, 2I] with n_dim = I), out1 [rows, I] (gate_up forward: act).
  const int64_t out0_cols = (h.mode == kDgradDown) ? 2 * (int64_t)h.I : h.n_dim;
  if ((err = map_bf16_2d(&mo0, h.out0, out0_cols, h.rows_cap, 16, 32, CU_TENSOR_MAP_SWIZZLE_NONE)) != cudaSuccess)
    return err;
  if (h.out1 != nullptr)
    err = map_bf16_2d(&mo1, h.out1, h.I, h.rows_cap, 16, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
  else
    mo1 = mo0;
  if (err != cudaSuccess) return err;
  if (!mn)
    err = map_u8_3d(&mraw, h.nf4, h.stored_cols / 2, h.stored_rows, h.E, 32, 128);
  else
    err = map_u8_3d(&mraw, h.nf4, h.stored_cols / 2, h.stored_rows, h.E, 64, 64);
  if (err != cudaSuccess) return err;
  const CUtensorMapSwizzle rswz = swizzle_for_bytes(2 * h.r_pad);
  if ((err = map_bf16_2d(&mla, h.lora_a_rows, h.r, h.rows_cap, h.r_pad, 128, rswz)) != cudaSuccess) return err;
  if (!mn)  // B_lora [E, stored_rows, r], K-major rows
    err = map_bf16_3d(&mlb, h.lora_w, h.r, h.stored_rows, h.E, h.r_pad, 64, rswz);
  else  // A_lora [E, r, stored_cols], rows are the K = r dimension
    err = map_bf16_3d(&mlb, h.lora_w, h.stored_cols, h.r, h.E, 64, h.r_pad, CU_TENSOR_MAP_SWIZZLE_128B);
  if (err != cudaSuccess) return err;

  Nf4GemmParams p;
  p.absmax = h.absmax;
  p.tiles = h.tiles;
  p.out0 = h.out0;
  p.out1 = h.out1;
  p.aux = h.aux;
  p.err = h.err;
  p.timeout_ns = h.timeout_ns;
  p.K = h.K;
  p.n_dim = h.n_dim;
  p.I = h.I;
  p.r_pad = h.r_pad;
  p.stored_rows = h.stored_rows;
  p.stored_cols = h.stored_cols;
  p.n_nt = (h.mode == kFwdGateUp) ? (h.I + 127) / 128 : (h.n_dim + 255) / 256;
  p.v8 = ((reinterpret_cast<uintptr_t>(h.out0) & 31u) == 0 && (h.I * 4) % 32 == 0) ? 1 : 0;
  p.mu_offset = munits_offset(h.mt_cap, h.E);
  const int64_t units_max = h.mt_cap * p.n_nt;
  const int64_t pairs = units_max < num_sms / 2 ? units_max : num_sms / 2;
  const int grid = 2 * (int)(pairs > 0 ? pairs : 1);
  const int smem = nf4g::SMEM_BYTES;
  static const char* kNames[4] = {"nf4_gemm_fwd_gate_up", "nf4_gemm_fwd_down", "nf4_gemm_dgrad_down",
                                  "nf4_gemm_dgrad_gate_up"};
  LaunchScope scope(kNames[h.mode & 3], stream);
  switch (h.mode) {
    case kFwdGateUp:
      if ((err = set_smem(nf4_gemm_kernel<kFwdGateUp>, smem)) != cudaSuccess) return err;
      nf4_gemm_kernel<kFwdGateUp><<<grid, nf4g::kThreads, smem, stream>>>(ma, mraw, mla, mlb, mo0, mo1, p);
      break;
    case kFwdDown:
      if ((err = set_smem(nf4_gemm_kernel<kFwdDown>, smem)) != cudaSuccess) return err;
      nf4_gemm_kernel<kFwdDown><<<grid, nf4g::kThreads, smem, stream>>>(ma, mraw, mla, mlb, mo0, mo1, p);
      break;
    case kDgradDown:
      if ((err = set_smem(nf4_gemm_kernel<kDgradDown>, smem)) != cudaSuccess) return err;
      nf4_gemm_kernel<kDgradDown><<<grid, nf4g::kThreads, smem, stream>>>(ma, mraw, mla, mlb, mo0, mo1, p);
      break;
    default:
      if ((err = set_smem(nf4_gemm_kernel<kDgradGateUp>, smem)) != cudaSuccess) return err;
      nf4_gemm_kernel<kDgradGateUp><<<grid, nf4g::kThreads, smem, stream>>>(ma, mraw, mla, mlb, mo0, mo1, p);
      break;
  }
  return cudaGetLastError();
}

cudaError_t launch_lora_proj(const LoraProjHost& h, int num_sms, cudaStream_t stream) {
  CUtensorMap mact, mw;
  cudaError_t err;
  if ((err = map_bf16_2d(&mact, h.act_in, h.K, h.rows_cap, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess)
    return err;
  if (h.w_mn_major)  // B [E, K, r]: K rows of r values
    err = map_bf16_3d(&mw, h.w, h.r, h.K, h.E, h.r_pad, 64, swizzle_for_bytes(2 * h.r_pad));
  else  // A [E, r, K]: r rows of K values
    err = map_bf16_3d(&mw, h.w, h.K, h.r, h.E, 64, h.r_pad, CU_TENSOR_MAP_SWIZZLE_128B);
  if (err != cudaSuccess) return err;
  LoraProjParams p;
  p.tiles = h.tiles;
  p.out = h.out;
  p.err = h.err;
  p.timeout_ns = h.timeout_ns;
  p.scale = h.scale;
  p.K = h.K;
  p.r = h.r;
  p.r_pad = h.r_pad;
  const int64_t cap = (int64_t)num_sms * 2;
  const int grid = (int)(h.mt_cap < cap ? h.mt_cap : cap);
  const int smem = lproj::SMEM_BYTES;
  LaunchScope scope("lora_proj", stream);
  if (h.w_mn_major) {
    if ((err = set_smem(lora_proj_kernel<true>, smem)) != cudaSuccess) return err;
    lora_proj_kernel<true><<<grid, lproj::kThreads, smem, stream>>>(mact, mw, p);
  } else {
    if ((err = set_smem(lora_proj_kernel<false>, smem)) != cudaSuccess) return err;
    lora_proj_kernel<false><<<grid, lproj::kThreads, smem, stream>>>(mact, mw, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_gather_proj(const LoraProjHost& h, int num_sms, cudaStream_t stream) {
  CUtensorMap mdst, mw;
  cudaError_t err;
  if ((err = map_bf16_2d(&mdst, h.act_in, h.K, h.rows_cap, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess)
    return err;
  if (h.w_mn_major)
    err = map_bf16_3d(&mw, h.w, h.r, h.K, h.E, h.r_pad, 64, swizzle_for_bytes(2 * h.r_pad));
  else
    err = map_bf16_3d(&mw, h.w, h.K, h.r, h.E, 64, h.r_pad, CU_TENSOR_MAP_SWIZZLE_128B);
  if (err != cudaSuccess) return err;
  GatherProjParams p;
  p.src = h.gather_src;
  p.slot_of_row = h.slot_of_row;
  p.scale_w = h.gather_w;
  p.tiles = h.tiles;
  p.out = h.out;
  p.err = h.err;
  p.timeout_ns = h.timeout_ns;
  p.scale = h.scale;
  p.K = h.K;
  p.r = h.r;
  p.r_pad = h.r_pad;
  p.k = h.k;
  const int64_t cap = (int64_t)num_sms * 2;
  const int grid = (int)(h.mt_cap < cap ? h.mt_cap : cap);
  const int smem = gproj::SMEM_BYTES;
  LaunchScope scope(h.gather_w ? "gather_proj_dyw" : "gather_proj_x", stream);
  if (h.w_mn_major) {
    if ((err = set_smem(gather_proj_kernel<true>, smem)) != cudaSuccess) return err;
    gather_proj_kernel<true><<<grid, gproj::kThreads, smem, stream>>>(mdst, mw, p);
  } else {
    if ((err = set_smem(gather_proj_kernel<false>, smem)) != cudaSuccess) return err;
    gather_proj_kernel<false><<<grid, gproj::kThreads, smem, stream>>>(mdst, mw, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_wgrad(const WgradHost& h, int num_sms, cudaStream_t stream) {
  CUtensorMap ma[4], ml[4];
  cudaError_t err;
  WgradParams p;
  p.units_per_expert = 0;
  p.transposed_mask = 0;
  for (int g = 0; g < 4; ++g) {
    if ((err = map_bf16_2d(&ma[g], h.act[g], h.F[g], h.rows_cap, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B)) !=
        cudaSuccess)
      return err;
    if ((err = map_bf16_2d(&ml[g], h.low[g], h.r, h.rows_cap, h.r_pad, 64, swizzle_for_bytes(2 * h.r_pad))) !=
        cudaSuccess)
      return err;
    p.out[g] = h.out[g];
    p.F[g] = h.F[g];
    p.n_ft[g] = (h.F[g] + 127) / 128;
    p.units_per_expert += p.n_ft[g];
    if (h.transposed[g]) p.transposed_mask |= 1 << g;
  }
  p.E = h.E;
  p.r = h.r;
  p.r_pad = h.r_pad;
  p.mt_cap = h.mt_cap;
  p.counts = h.counts;
  p.offsets = h.offsets;
  p.tiles = h.tiles;
  p.err = h.err;
  p.timeout_ns = h.timeout_ns;
  const int64_t units = (int64_t)h.E * p.units_per_expert;
  const int64_t cap = (int64_t)num_sms * 2;
  const int grid = (int)(units < cap ? units : cap);
  const int smem = wg::SMEM_BYTES;
  if ((err = set_smem(wgrad_kernel, smem)) != cudaSuccess) return err;
  LaunchScope scope("lora_wgrad", stream);
  wgrad_kernel<<<grid, wg::kThreads, smem, stream>>>(ma[0], ma[1], ma[2], ma[3], ml[0], ml[1], ml[2], ml[3], p);
  return cudaGetLastError();
}

}  // namespace e4b
