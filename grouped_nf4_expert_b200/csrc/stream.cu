// Weight-streaming grouped NF4 forward for decode-sized batches.
//
// When a batch routes only a few slots to each expert, the block's cost is
// reading every touched expert's NF4 weights once.  Here the weights are the
// UMMA M operand (128 weight rows per tile, decoded into shared memory) and
// up to 32 routed slots of one expert are the N operand, so each weight byte is
// fetched and decoded once per 32 slots.  Deep rings of NF4 code tiles and of
// activation-row tiles keep enough memory traffic in flight; a shorter ring
// holds the decoded tiles the UMMAs consume.  Same exact decode routine, same outputs as the training
// tiles (gu / act for gate_up, y_perm for down), with the LoRA term as K = r
// UMMAs into the same accumulator.
//
// Pages: "How do I QLoRA-train the fused experts of a MoE", section "The
// abstraction that fails" (per-expert delta before the activation) and
// section "Why it happens" (the LoRA term); package METADATA "The package
// family" (4-bit decode, fp32 accumulation) and its decode/serving use.
#include "e4b_device.cuh"
#include "e4b_internal.h"

namespace e4b {

namespace {
constexpr uint32_t kFull = 0xffffffffu;
}  // namespace

namespace nf4s {
constexpr int BM = 128;          // weight rows per tile (UMMA M)
constexpr int BN = 32;           // routed slots per tile (UMMA N)
constexpr int BK = 64;
constexpr int RAW_STAGES = 16;   // NF4 codes + absmax (the HBM stream)
constexpr int AB_STAGES = 4;     // decoded weights
constexpr int X_STAGES = 12;     // activation rows (prefetched like the codes)
constexpr int RAW_BYTES = BM * BK / 2;                 // 4096
constexpr int AMAX_BYTES = BM * 4;                     // 512
constexpr int RAW_SLOT = RAW_BYTES + AMAX_BYTES;       // 4608 (128-byte multiple)
constexpr int A_BYTES = BM * BK * 2;                   // 16384, K-major SW128
constexpr int X_BYTES = BN * BK * 2;                   // 4096, K-major SW128

constexpr int LA_BYTES = BM * E4B_MAX_RANK * 2;        // LoRA B rows of the tile (UMMA A of the K=r step)
constexpr int LB_BYTES = BN * E4B_MAX_RANK * 2;        // p rows of the slots (UMMA B of the K=r step)
constexpr int EPI_BYTES = 64 * BN * 4;                 // up values handed to the gate lanes
constexpr int RAW_OFF = 0;
constexpr int AB_OFF = RAW_STAGES * RAW_SLOT;          // 73728, 1024-aligned
constexpr int X_OFF = AB_OFF + AB_STAGES * A_BYTES;
constexpr int LA_OFF = X_OFF + X_STAGES * X_BYTES;
constexpr int LB_OFF = LA_OFF + LA_BYTES;
constexpr int EPI_OFF = LB_OFF + LB_BYTES;
constexpr int BAR_OFF = EPI_OFF + EPI_BYTES;
constexpr int SMEM_BYTES = BAR_OFF + 1024 + 1024;
constexpr int kDecodeGroups = 4;  // groups of 4 warps; group g decodes the k-chunks j with j % 4 == g
constexpr int kEpiWarp0 = 4 + 4 * kDecodeGroups;
// warp 0 codes, warp 1 UMMA, warp 2 activations + LoRA, 4.. decode, last 4 epilogue
constexpr int kThreads = 32 * (kEpiWarp0 + 4);
constexpr int kTmemCols = 64;   // 2 accumulator buffers x 32 columns
constexpr int kRawFullCount = 1 + 32;
static_assert(AB_OFF % 1024 == 0 && X_OFF % 1024 == 0 && LA_OFF % 1024 == 0 && LB_OFF % 1024 == 0,
              "swizzle atom alignment");
static_assert(RAW_STAGES % kDecodeGroups == 0 && AB_STAGES % kDecodeGroups == 0,
              "each ring slot must belong to one decode group");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
}  // namespace nf4s

struct Nf4StreamParams {
  const float* absmax;
  const int32_t* tiles;
  uint16_t* out0;        // gu [rows, 2I] or y_perm [rows, H]
  uint16_t* out1;        // act [rows, I] or nullptr
  DeviceError* err;
  long long timeout_ns;
  int K, n_dim, I, r_pad;
  int stored_rows, stored_cols;
  int n_mt;              // weight tiles per slot tile
  int64_t st_offset;     // slot-tile list in `tiles`
};

template <int MODE>
__global__ void __launch_bounds__(nf4s::kThreads, 1)
    nf4_stream_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_raw,
                      const __grid_constant__ CUtensorMap map_lw, const __grid_constant__ CUtensorMap map_lp,
                      const Nf4StreamParams p) {
  using namespace nf4s;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = align1024(smem_dyn);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* raw_full = bars;                         // [RAW_STAGES] codes + absmax landed
  uint64_t* raw_empty = raw_full + RAW_STAGES;       // [RAW_STAGES] codes decoded
  uint64_t* a_full = raw_empty + RAW_STAGES;         // [AB_STAGES] decoded tile written
  uint64_t* ab_empty = a_full + AB_STAGES;           // [AB_STAGES] decoded tile consumed by the UMMAs
  uint64_t* x_full = ab_empty + AB_STAGES;           // [X_STAGES] activation rows landed
  uint64_t* x_empty = x_full + X_STAGES;             // [X_STAGES] activation rows consumed
  uint64_t* lfull = x_empty + X_STAGES;              // LoRA operands landed
  uint64_t* lempty = lfull + 1;                      // LoRA operands consumed
  uint64_t* accfull = lfull + 2;                     // [2]
  uint64_t* accempty = lfull + 4;                    // [2]
  uint64_t* epi_full = lfull + 6;                    // up values in EPI
  uint64_t* epi_empty = lfull + 7;                   // up values consumed
  uint64_t* drain = lfull + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lfull + 9);
  CtaControl* ctl = reinterpret_cast<CtaControl*>(lfull + 10);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < RAW_STAGES; ++s) {
      mbar_init(&raw_full[s], kRawFullCount);
      mbar_init(&raw_empty[s], 4);
    }
    for (int s = 0; s < AB_STAGES; ++s) {
      mbar_init(&a_full[s], 4);
      mbar_init(&ab_empty[s], 1);
    }
    for (int s = 0; s < X_STAGES; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], 1);
    }
    mbar_init(lfull, 1);
    mbar_init(lempty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 4);
    }
    mbar_init(epi_full, 2);
    mbar_init(epi_empty, 2);
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

  const int32_t* stiles = p.tiles + p.st_offset;
  const int n_units = p.tiles[3] * p.n_mt;
  const int kchunks = p.K / BK;
  const int blocks_per_row = p.stored_cols / 64;

  // Stored weight rows of tile mt: two 64-row halves.
  auto rows_of = [&](int mt, int& rA, int& rB) {
    if (MODE == kFwdGateUp) {
      rA = mt * 64;
      rB = p.I + mt * 64;
    } else {
      rA = mt * 128;
      rB = mt * 128 + 64;
    }
  };

  if (warp == 0) {
    // ------------------------------------------------ NF4 codes + absmax (whole warp), far ahead
    if (lane == 0) tma_prefetch_desc(&map_raw);
    uint32_t j = 0, issued = 0, last_par = 0;
    bool ok = true;
    int e_next = (blockIdx.x < n_units) ? stiles[3 * (blockIdx.x / p.n_mt)] : 0;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const int mt = u % p.n_mt;
      const int e = e_next;
      if (u + (int)gridDim.x < n_units) e_next = stiles[3 * ((u + gridDim.x) / p.n_mt)];
      int rA, rB;
      rows_of(mt, rA, rB);
      for (int kc = 0; kc < kchunks; ++kc, ++j) {
        const uint32_t r = j % RAW_STAGES, ph = (j / RAW_STAGES) & 1;
        ok = __all_sync(kFull, mbar_wait(&raw_empty[r], ph ^ 1, ctl, p.err, p.timeout_ns, 310));
        if (!ok) break;
        uint8_t* slot = smem + RAW_OFF + r * RAW_SLOT;
        if (lane == 0) {
          mbar_arrive_expect_tx(&raw_full[r], RAW_BYTES);
          tma_load_3d(slot, &map_raw, &raw_full[r], kc * (BK / 2), rA, e);
          tma_load_3d(slot + RAW_BYTES / 2, &map_raw, &raw_full[r], kc * (BK / 2), rB, e);
        }
        float* amax = reinterpret_cast<float*>(slot + RAW_BYTES);
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const int t = lane + 32 * qq;
          const int srow = (t < 64) ? rA + t : rB + (t - 64);
          if (srow < p.stored_rows)
            cp_async_4(amax + t, p.absmax + ((size_t)e * p.stored_rows + srow) * blocks_per_row + kc);
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
    // ------------------------------------------------ activation rows + LoRA operands
    if (lane == 0) {
      tma_prefetch_desc(&map_x);
      tma_prefetch_desc(&map_lw);
      tma_prefetch_desc(&map_lp);
      uint32_t j = 0, ti = 0, issued = 0, last_par = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++ti) {
        const int st = u / p.n_mt, mt = u % p.n_mt;
        const int e = stiles[3 * st], row0 = stiles[3 * st + 1];
        int rA, rB;
        rows_of(mt, rA, rB);
        if (!(ok = mbar_wait(lempty, (ti & 1) ^ 1, ctl, p.err, p.timeout_ns, 320))) break;
        mbar_arrive_expect_tx(lfull, (uint32_t)((BM + BN) * 2 * p.r_pad));
        uint8_t* la = smem + LA_OFF;
        tma_load_3d(la, &map_lw, lfull, 0, rA, e);
        tma_load_3d(la + 128 * p.r_pad, &map_lw, lfull, 0, rB, e);
        tma_load_2d(smem + LB_OFF, &map_lp, lfull, 0, row0);
        for (int kc = 0; kc < kchunks; ++kc, ++j) {
          const uint32_t s = j % X_STAGES, ph = (j / X_STAGES) & 1;
          if (!(ok = mbar_wait(&x_empty[s], ph ^ 1, ctl, p.err, p.timeout_ns, 321))) break;
          mbar_arrive_expect_tx(&x_full[s], X_BYTES);
          tma_load_2d(smem + X_OFF + s * X_BYTES, &map_x, &x_full[s], kc * BK, row0);
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
    const uint32_t ab_u = smem_u32(smem + AB_OFF), x_u = smem_u32(smem + X_OFF);
    uint32_t j = 0, ti = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++ti) {
      const uint32_t b = ti & 1, use = ti >> 1;
      const uint32_t d = tmem + b * BN;
      if (!(ok = __all_sync(kFull, mbar_wait(&accempty[b], (use & 1) ^ 1, ctl, p.err, p.timeout_ns, 330)))) break;
      if (!(ok = __all_sync(kFull, mbar_wait(lfull, ti & 1, ctl, p.err, p.timeout_ns, 331)))) break;
      tc_fence_after();
      if (elect_one_sync()) {
        for (int ks = 0; ks < p.r_pad / 16; ++ks)
          umma_bf16(d, make_sdesc(la_u + 32 * ks, 16, 16 * p.r_pad, lswz),
                    make_sdesc(lb_u + 32 * ks, 16, 16 * p.r_pad, lswz), idesc, ks > 0 ? 1u : 0u);
        umma_commit(lempty);
      }
      __syncwarp();
      for (int kc = 0; kc < kchunks; ++kc, ++j) {
        const uint32_t s = j % AB_STAGES, ph = (j / AB_STAGES) & 1;
        const uint32_t xs = j % X_STAGES, xph = (j / X_STAGES) & 1;
        if (!(ok = __all_sync(kFull, mbar_wait(&a_full[s], ph, ctl, p.err, p.timeout_ns, 332)))) break;
        if (!(ok = __all_sync(kFull, mbar_wait(&x_full[xs], xph, ctl, p.err, p.timeout_ns, 333)))) break;
        tc_fence_after();
        const uint64_t adesc = make_sdesc(ab_u + s * A_BYTES, 16, 1024, kSw128);
        const uint64_t xdesc = make_sdesc(x_u + xs * X_BYTES, 16, 1024, kSw128);
        if (elect_one_sync()) {
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)  // +32 bytes along K = +2 in the address field
            umma_bf16(d, adesc + 2 * kk, xdesc + 2 * kk, idesc, 1u);
          umma_commit(&ab_empty[s]);
          umma_commit(&x_empty[xs]);
        }
        __syncwarp();
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
  } else if (warp >= 4 && warp < kEpiWarp0) {
    // ------------------------------------------------ NF4 decode, groups take k-chunks round robin
    const uint32_t grp = (uint32_t)(warp - 4) >> 2;
    const int t = (threadIdx.x - 128) & 127;  // weight row of the tile
    uint32_t j = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const int mt = u % p.n_mt;
      int rA, rB;
      rows_of(mt, rA, rB);
      const bool valid = ((t < 64) ? rA + t : rB + (t - 64)) < p.stored_rows;
      for (int kc = 0; kc < kchunks; ++kc, ++j) {
        if (j % kDecodeGroups != grp) continue;
        const uint32_t r = j % RAW_STAGES, rph = (j / RAW_STAGES) & 1;
        const uint32_t s = j % AB_STAGES, sph = (j / AB_STAGES) & 1;
        ok = __all_sync(kFull, mbar_wait(&raw_full[r], rph, ctl, p.err, p.timeout_ns, 340));
        if (ok) ok = __all_sync(kFull, mbar_wait(&ab_empty[s], sph ^ 1, ctl, p.err, p.timeout_ns, 341));
        if (!ok) break;
        const uint8_t* slot = smem + RAW_OFF + r * RAW_SLOT;
        uint8_t* arow = smem + AB_OFF + s * A_BYTES + (t >> 3) * 1024 + (t & 7) * 128;
        if (valid) {
          const uint4 q0 = *reinterpret_cast<const uint4*>(slot + t * 32);
          const uint4 q1 = *reinterpret_cast<const uint4*>(slot + t * 32 + 16);
          const uint32_t codes[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
          const Nf4Planes pl = nf4_block_planes(reinterpret_cast<const float*>(slot + RAW_BYTES)[t]);
#pragma unroll
          for (int c = 0; c < 8; ++c) {  // 16-byte chunk c of the 128-byte row, 128B-swizzled
            uint32_t w4[4];
            nf4_decode_word(codes[c], pl, w4);
            *reinterpret_cast<uint4*>(arow + ((c ^ (t & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(arow + (c << 4)) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&raw_empty[r]);
          mbar_arrive(&a_full[s]);
        }
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------ epilogue: lane = weight row, 32 slot columns
    const int qrt = warp & 3;
    const int wrow = qrt * 32 + lane;
    float* epi = reinterpret_cast<float*>(smem + EPI_OFF);
    uint32_t ti = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++ti) {
      const int st = u / p.n_mt, mt = u % p.n_mt;
      const size_t row0 = (size_t)stiles[3 * st + 1];
      const uint32_t b = ti & 1, use = ti >> 1;
      ok = __all_sync(kFull, mbar_wait(&accfull[b], use & 1, ctl, p.err, p.timeout_ns, 350));
      if (!ok) break;
      tc_fence_after();
      float v[32];
      {
        float v0[16], v1[16];
        const uint32_t tl = tmem + b * BN + ((uint32_t)(qrt * 32) << 16);
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
      if (MODE == kFwdGateUp) {
        const int i = mt * 64 + (wrow & 63);  // gate/up feature of this lane
        const int I2 = 2 * p.I;
        if (qrt >= 2) {
          // up rows: store u, hand it to the gate lanes
          ok = __all_sync(kFull, mbar_wait(epi_empty, (ti & 1) ^ 1, ctl, p.err, p.timeout_ns, 351));
          if (!ok) break;
#pragma unroll
          for (int sl = 0; sl < 32; ++sl) epi[sl * 64 + (wrow - 64)] = v[sl];
          __syncwarp();
          if (lane == 0) mbar_arrive(epi_full);
#pragma unroll
          for (int sl = 0; sl < 32; ++sl) {
            const __nv_bfloat16 h = __float2bfloat16_rn(v[sl]);
            p.out0[(row0 + sl) * I2 + p.I + i] = *reinterpret_cast<const uint16_t*>(&h);
          }
        } else {
          ok = __all_sync(kFull, mbar_wait(epi_full, ti & 1, ctl, p.err, p.timeout_ns, 352));
          if (!ok) break;
#pragma unroll
          for (int sl = 0; sl < 32; ++sl) {
            const float g = v[sl], uu = epi[sl * 64 + wrow];
            const __nv_bfloat16 hg = __float2bfloat16_rn(g);
            const __nv_bfloat16 ha = __float2bfloat16_rn(silu_f(g) * uu);
            p.out0[(row0 + sl) * I2 + i] = *reinterpret_cast<const uint16_t*>(&hg);
            p.out1[(row0 + sl) * p.I + i] = *reinterpret_cast<const uint16_t*>(&ha);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(epi_empty);
        }
      } else {
        const int f = mt * 128 + wrow;
        if (f < p.n_dim) {
#pragma unroll
          for (int sl = 0; sl < 32; ++sl) {
            const __nv_bfloat16 h = __float2bfloat16_rn(v[sl]);
            p.out0[(row0 + sl) * p.n_dim + f] = *reinterpret_cast<const uint16_t*>(&h);
          }
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

cudaError_t launch_nf4_stream(const Nf4GemmHost& h, int num_sms, cudaStream_t stream) {
  using namespace nf4s;
  if (h.mode != kFwdGateUp && h.mode != kFwdDown) return cudaErrorInvalidValue;
  CUtensorMap mx, mraw, mlw, mlp;
  cudaError_t err;
  const CUtensorMapSwizzle rswz = swizzle_for_bytes(2 * h.r_pad);
  if ((err = map_bf16_2d(&mx, h.act_in, h.K, h.rows_cap, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess)
    return err;
  if ((err = map_u8_3d(&mraw, h.nf4, h.stored_cols / 2, h.stored_rows, h.E, 32, 64)) != cudaSuccess) return err;
  if ((err = map_bf16_3d(&mlw, h.lora_w, h.r, h.stored_rows, h.E, h.r_pad, 64, rswz)) != cudaSuccess) return err;
  if ((err = map_bf16_2d(&mlp, h.lora_a_rows, h.r, h.rows_cap, h.r_pad, BN, rswz)) != cudaSuccess) return err;
  Nf4StreamParams p;
  p.absmax = h.absmax;
  p.tiles = h.tiles;
  p.out0 = h.out0;
  p.out1 = h.out1;
  p.err = h.err;
  p.timeout_ns = h.timeout_ns;
  p.K = h.K;
  p.n_dim = h.n_dim;
  p.I = h.I;
  p.r_pad = h.r_pad;
  p.stored_rows = h.stored_rows;
  p.stored_cols = h.stored_cols;
  p.n_mt = (h.mode == kFwdGateUp) ? h.I / 64 : (h.n_dim + 127) / 128;
  p.st_offset = stiles_offset(h.mt_cap, h.E);
  const int64_t units_max = 4 * h.mt_cap * p.n_mt;
  const int grid = (int)(units_max < num_sms ? units_max : num_sms);
  const int smem = SMEM_BYTES;
  static const char* kNames[2] = {"nf4_stream_fwd_gate_up", "nf4_stream_fwd_down"};
  LaunchScope scope(kNames[h.mode & 1], stream);
  if (h.mode == kFwdGateUp) {
    if ((err = cudaFuncSetAttribute(nf4_stream_kernel<kFwdGateUp>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    smem)) != cudaSuccess)
      return err;
    nf4_stream_kernel<kFwdGateUp><<<grid, kThreads, smem, stream>>>(mx, mraw, mlw, mlp, p);
  } else {
    if ((err = cudaFuncSetAttribute(nf4_stream_kernel<kFwdDown>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    smem)) != cudaSuccess)
      return err;
    nf4_stream_kernel<kFwdDown><<<grid, kThreads, smem, stream>>>(mx, mraw, mlw, mlp, p);
  }
  return cudaGetLastError();
}

}  // namespace e4b
