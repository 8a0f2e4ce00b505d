// Weight-streaming grouped NF4 forward for decode-sized batches.
//
// When a batch routes only a few slots to each expert, the block's cost is
// reading every touched expert's NF4 weights once.  Here the weights are the
// UMMA M operand (128 weight rows per tile) and up to 32 routed slots of one
// expert are the N operand, so each weight byte is fetched and decoded once
// per 32 slots.  Decoded tiles go straight to tensor memory, which the UMMA
// reads as its A operand.  A code stage holds 4 k-chunks, so
// every weight row contributes one whole 128-byte line (and one 16-byte run
// of block scales) per stage; rings of code stages and of activation-row tiles
// keep enough memory traffic in flight.
//
// Three teams of four decode warps take the code stages round robin, so that
// while one team waits on its barriers the other two decode; a team writes
// the decoded rows of its stage's four k-chunks straight into its own A
// buffer in tensor memory, and one warp issues every stage's UMMAs in order
// with those tiles as the A operand read from tensor memory.  Outputs match the training tiles (gu /
// act for gate_up, y_perm for down; the serving call skips gu), with the LoRA
// term as K = r UMMAs into the same accumulator.
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
constexpr int RAW_CHUNKS = 4;    // k-chunks per code stage: 128 contiguous code bytes per weight row
constexpr int kTeams = 3;        // decode teams of 4 warps (one per TMEM lane quadrant)
constexpr int RAW_STAGES = 6;    // NF4 codes + absmax (the HBM stream); slot r always goes to team r % 3
constexpr int X_STAGES = 4;      // activation rows of a code stage's 4 chunks (prefetched like the codes)
constexpr int CODE_BYTES = BM * RAW_CHUNKS * BK / 2;   // 16384, 128B-swizzled rows of 128 bytes
constexpr int AMAX_BYTES = BM * RAW_CHUNKS * 4;        // 2048, 4 block scales per row
constexpr int RAW_SLOT = CODE_BYTES + AMAX_BYTES;      // 18432 (1024-byte multiple)
constexpr int X_BYTES = BN * BK * 2;                   // 4096 per chunk, K-major SW128
constexpr int XS_BYTES = RAW_CHUNKS * X_BYTES;         // 16384 per stage

constexpr int LA_BYTES = BM * E4B_MAX_RANK * 2;        // LoRA B rows of the tile (UMMA A of the K=r step)
constexpr int LB_BYTES = BN * E4B_MAX_RANK * 2;        // p rows of the slots (UMMA B of the K=r step)
constexpr int EPI_BYTES = 64 * BN * 4;                 // up values handed to the gate lanes
constexpr int RAW_OFF = 0;
constexpr int X_OFF = RAW_STAGES * RAW_SLOT;           // 147456, 1024-aligned
constexpr int LA_OFF = X_OFF + X_STAGES * XS_BYTES;
constexpr int LB_OFF = LA_OFF + LA_BYTES;
constexpr int EPI_OFF = LB_OFF + LB_BYTES;
constexpr int BAR_OFF = EPI_OFF + EPI_BYTES;
constexpr int SMEM_BYTES = BAR_OFF + 1024 + 1024;
constexpr int kEpiWarp0 = 4 + 4 * kTeams;
// warp 0 codes, warp 1 UMMA, warp 2 activations + LoRA, 4.. decode, last 4 epilogue
constexpr int kThreads = 32 * (kEpiWarp0 + 4);
// TMEM columns: 2 accumulator buffers x 32 slot columns at 0, then one A
// buffer per team (4 chunks x 32 columns = 4 x 64 bf16 per lane) from 128.
constexpr int kAccCols = BN;
constexpr int kACols = BK / 2;
constexpr int kAOff = 128;
constexpr int kTeamCols = RAW_CHUNKS * kACols;         // 128
constexpr int kTmemCols = 512;
constexpr int kRawFullCount = 1 + 32;
static_assert(X_OFF % 1024 == 0 && LA_OFF % 1024 == 0 && LB_OFF % 1024 == 0, "swizzle atom alignment");
static_assert(kTmemCols == 512, "one CTA per SM owns all of TMEM");
static_assert(SMEM_BYTES > 232448 / 2, "shared memory keeps one CTA per SM (TMEM is not shared)");
static_assert(RAW_STAGES % kTeams == 0, "each code slot belongs to one team (no phase aliasing)");
static_assert(kAOff + kTeams * kTeamCols <= kTmemCols && 2 * kAccCols <= kAOff, "TMEM budget");
static_assert(RAW_SLOT % 1024 == 0, "code tiles are 128B-swizzled");
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
  uint64_t* raw_empty = raw_full + RAW_STAGES;       // [RAW_STAGES] codes read into registers (team's 4 warps)
  uint64_t* a_ready = raw_empty + RAW_STAGES;        // [kTeams] team's decoded stage written (4 warps)
  uint64_t* a_empty = a_ready + kTeams;              // [kTeams] team's A buffer consumed by the UMMAs
  uint64_t* x_full = a_empty + kTeams;               // [X_STAGES] activation rows landed
  uint64_t* x_empty = x_full + X_STAGES;             // [X_STAGES] activation rows consumed
  uint64_t* drain = x_empty + X_STAGES;              // every UMMA completed
  uint64_t* lfull = drain + 1;                       // LoRA operands landed
  uint64_t* lempty = lfull + 1;                      // LoRA operands consumed
  uint64_t* accfull = lfull + 2;                     // [2] accumulator final
  uint64_t* accempty = lfull + 4;                    // [2] epilogue read the accumulators
  uint64_t* epi_full = lfull + 6;                    // up values in EPI
  uint64_t* epi_empty = lfull + 7;                   // up values consumed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lfull + 8);
  CtaControl* ctl = reinterpret_cast<CtaControl*>(lfull + 9);

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
  const int nq = (kchunks + RAW_CHUNKS - 1) / RAW_CHUNKS;  // code stages per unit; the last may be partial
  // Block scales of a full stage are one aligned 16-byte run per row when
  // rows hold a multiple of 4 blocks.
  const bool amax16 = (kchunks % RAW_CHUNKS) == 0 && (reinterpret_cast<uintptr_t>(p.absmax) & 15u) == 0;

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
      for (int q = 0; q < nq; ++q, ++j) {
        const uint32_t r = j % RAW_STAGES, ph = (j / RAW_STAGES) & 1;
        ok = __all_sync(kFull, mbar_wait_lazy(&raw_empty[r], ph ^ 1, ctl, p.err, p.timeout_ns, 310, 128));
        if (!ok) break;
        uint8_t* slot = smem + RAW_OFF + r * RAW_SLOT;
        if (lane == 0) {
          // Codes past the end of a row (a partial last stage) are zero-filled.
          mbar_arrive_expect_tx(&raw_full[r], CODE_BYTES);
          tma_load_3d(slot, &map_raw, &raw_full[r], q * (RAW_CHUNKS * BK / 2), rA, e);
          tma_load_3d(slot + CODE_BYTES / 2, &map_raw, &raw_full[r], q * (RAW_CHUNKS * BK / 2), rB, e);
        }
        float* amax = reinterpret_cast<float*>(slot + CODE_BYTES);
        const int nb = min(RAW_CHUNKS, kchunks - q * RAW_CHUNKS);
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const int t = lane + 32 * qq;
          const int srow = (t < 64) ? rA + t : rB + (t - 64);
          if (srow < p.stored_rows) {
            const float* src = p.absmax + ((size_t)e * p.stored_rows + srow) * blocks_per_row + q * RAW_CHUNKS;
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
        if (!(ok = mbar_wait_lazy(lempty, (ti & 1) ^ 1, ctl, p.err, p.timeout_ns, 320, 128))) break;
        mbar_arrive_expect_tx(lfull, (uint32_t)((BM + BN) * 2 * p.r_pad));
        uint8_t* la = smem + LA_OFF;
        tma_load_3d(la, &map_lw, lfull, 0, rA, e);
        tma_load_3d(la + 128 * p.r_pad, &map_lw, lfull, 0, rB, e);
        tma_load_2d(smem + LB_OFF, &map_lp, lfull, 0, row0);
        for (int q = 0; q < nq; ++q, ++j) {
          const uint32_t s = j % X_STAGES, ph = (j / X_STAGES) & 1;
          if (!(ok = mbar_wait_lazy(&x_empty[s], ph ^ 1, ctl, p.err, p.timeout_ns, 321, 128))) break;
          const int nb = min(RAW_CHUNKS, kchunks - q * RAW_CHUNKS);
          mbar_arrive_expect_tx(&x_full[s], (uint32_t)(nb * X_BYTES));
          for (int c = 0; c < nb; ++c)
            tma_load_2d(smem + X_OFF + s * XS_BYTES + c * X_BYTES, &map_x, &x_full[s], (q * RAW_CHUNKS + c) * BK,
                        row0);
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
    uint32_t ti = 0, rq = 0, xs = 0, xph = 0;  // units, code stages, activation ring slot and parity
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++ti) {
      const uint32_t b = ti & 1, use = ti >> 1;
      const uint32_t d = tmem + b * kAccCols;
      if (!(ok = __all_sync(kFull, mbar_wait(&accempty[b], (use & 1) ^ 1, ctl, p.err, p.timeout_ns, 330)))) break;
      if (!(ok = __all_sync(kFull, mbar_wait(lfull, ti & 1, ctl, p.err, p.timeout_ns, 331)))) break;
      tc_fence_after();
      if (elect_one_sync()) {
        for (int k = 0; k < p.r_pad / 16; ++k)
          umma_bf16(d, make_sdesc(la_u + 32 * k, 16, 16 * p.r_pad, lswz),
                    make_sdesc(lb_u + 32 * k, 16, 16 * p.r_pad, lswz), idesc, k > 0 ? 1u : 0u);
        umma_commit(lempty);
      }
      __syncwarp();
      for (int q = 0; q < nq; ++q, ++rq) {
        const uint32_t team = rq % kTeams, aph = (rq / kTeams) & 1;
        ok = __all_sync(kFull, mbar_wait(&a_ready[team], aph, ctl, p.err, p.timeout_ns, 332));
        if (ok) ok = __all_sync(kFull, mbar_wait(&x_full[xs], xph, ctl, p.err, p.timeout_ns, 333));
        if (!ok) break;
        tc_fence_after();
        if (elect_one_sync()) {
          const int nb = min(RAW_CHUNKS, kchunks - q * RAW_CHUNKS);
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
  } else if (warp >= 4 && warp < kEpiWarp0) {
    // ------------------------------------------------ NF4 decode into TMEM, teams take code stages round robin
    // Team m decodes every code stage rq with rq % 3 == m; thread t owns
    // weight row t, which is TMEM lane t, and writes the stage's decoded
    // rows (4 k-chunks x 64 bf16) straight into the team's A buffer there.
    const uint32_t team = (uint32_t)(warp - 4) >> 2;
    const int t = (threadIdx.x - 128) & 127;
    const Nf4Shift ks = nf4_shift_consts();
    const uint32_t a_base = tmem + kAOff + team * kTeamCols + ((uint32_t)(warp & 3) * 32u << 16);
    uint32_t rq = 0, tuse = 0;  // code stages seen, stages this team decoded
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const int mt = u % p.n_mt;
      int rA, rB;
      rows_of(mt, rA, rB);
      const bool valid = ((t < 64) ? rA + t : rB + (t - 64)) < p.stored_rows;
      for (int q = 0; q < nq; ++q, ++rq) {
        if (rq % kTeams != team) continue;
        const uint32_t r = rq % RAW_STAGES, rph = (rq / RAW_STAGES) & 1;
        const uint32_t aph = tuse++ & 1;
        const int nb = min(RAW_CHUNKS, kchunks - q * RAW_CHUNKS);  // a partial last stage has fewer chunks
        ok = __all_sync(kFull, mbar_wait(&raw_full[r], rph, ctl, p.err, p.timeout_ns, 340));
        if (!ok) break;
        const uint8_t* slot = smem + RAW_OFF + r * RAW_SLOT;
        const uint8_t* crow = slot + t * 128;  // 128B-swizzled: 16-byte piece c sits at c ^ (t % 8)
        const float* amax = reinterpret_cast<const float*>(slot + CODE_BYTES) + t * RAW_CHUNKS;
        for (int c = 0; c < nb; ++c) {
          const uint4 q0 = *reinterpret_cast<const uint4*>(crow + (((2 * c) ^ (t & 7)) << 4));
          const uint4 q1 = *reinterpret_cast<const uint4*>(crow + (((2 * c + 1) ^ (t & 7)) << 4));
          const float a = amax[c];
          if (c == nb - 1) {
            // The stage's codes are in registers.  A proxy fence orders these
            // generic reads before the next TMA write into the slot.
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&raw_empty[r]);
          }
          const uint32_t codes[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
          // Rows past the end of the matrix get a zero scale, so every entry
          // of their table (and every decoded weight) is zero whatever the codes.
          const Nf4Planes pl = nf4_block_planes(valid ? a : 0.0f);
          uint32_t v[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) nf4_decode_word(codes[i], pl, ks, &v[4 * i]);
          if (c == 0) {
            // The UMMAs of this team's previous stage have finished reading the buffer.
            ok = __all_sync(kFull, mbar_wait(&a_empty[team], aph ^ 1, ctl, p.err, p.timeout_ns, 341));
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
      ok = __all_sync(kFull, mbar_wait_lazy(&accfull[b], use & 1, ctl, p.err, p.timeout_ns, 350, 256));
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
          if (p.out0 != nullptr) {  // gu is kept for a backward; a serving forward passes none
#pragma unroll
            for (int sl = 0; sl < 32; ++sl) {
              const __nv_bfloat16 h = __float2bfloat16_rn(v[sl]);
              p.out0[(row0 + sl) * I2 + p.I + i] = *reinterpret_cast<const uint16_t*>(&h);
            }
          }
        } else {
          ok = __all_sync(kFull, mbar_wait(epi_full, ti & 1, ctl, p.err, p.timeout_ns, 352));
          if (!ok) break;
#pragma unroll
          for (int sl = 0; sl < 32; ++sl) {
            const float g = v[sl], uu = epi[sl * 64 + wrow];
            const __nv_bfloat16 hg = __float2bfloat16_rn(g);
            const __nv_bfloat16 ha = __float2bfloat16_rn(silu_f(g) * uu);
            if (p.out0 != nullptr) p.out0[(row0 + sl) * I2 + i] = *reinterpret_cast<const uint16_t*>(&hg);
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
  if ((err = map_u8_3d(&mraw, h.nf4, h.stored_cols / 2, h.stored_rows, h.E, RAW_CHUNKS * BK / 2, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess)
    return err;
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
