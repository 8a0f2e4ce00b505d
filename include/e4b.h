/*
 * e4b.h -- C ABI of the grouped NF4 expert block with per-expert LoRA,
 * hand-written for NVIDIA B200 (sm_100a).
 *
 * The block is the routed-expert MoE layer over a frozen, NF4-quantised,
 * fused expert stack; each expert carries a trainable low-rank delta that is
 * added to its pre-activation (inside the activation, not after it):
 *
 *     y[t] = sum_j w[t,j] * yd(t, e = ids[t,j])
 *     gu   = W_gu[e] x + s * B_gu[e] (A_gu[e] x)         s = alpha / r
 *     act  = silu(gu[:I]) * gu[I:]
 *     yd   = W_d[e] act + s * B_d[e] (A_d[e] act)
 *
 * Sources (page title, section):
 *   "How do I QLoRA-train the fused experts of a MoE (per-expert LoRA on
 *   4-bit experts)?", section "The abstraction that fails, and what replaces
 *   it": the fused 3-D stacks (gate_up_proj [E,2I,H], down_proj [E,H,I]);
 *   each routed expert computes act(W_e x + B[e] A[e] x), the delta inside
 *   the activation; the base is frozen and B starts at zero.
 *   Same page, section "Why it happens": the LoRA term is
 *   scaling * (x @ A[e].T) @ B[e].T with stacked per-expert A and B; the
 *   backward decodes the 4-bit base again, so no bf16 copy of a weight is
 *   ever kept.
 *   Same page, sections "Which project solves it" and "Limitations": a
 *   grouped forward, an input-gradient (dgrad) kernel, the stock epilogue
 *   act(gate) * up, and loud refusal instead of a silent fallback.
 *   experts4bit-qlora package METADATA, section "The package family": a
 *   single kernel launch covers all the packed 4-bit experts, decoding in
 *   registers and summing in fp32.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major
 *     (C order), 16-byte aligned.  The library never allocates, never frees
 *     and never synchronises (e4b_check_device_error excepted); all work is
 *     enqueued on `stream` in order.
 *   - bfloat16 tensors are passed as e4b_bf16 (their 16-bit patterns).
 *   - Arguments are validated on the host before anything is launched; a
 *     failed check returns a status and launches nothing.  With T == 0 the
 *     calls return E4B_OK without reading or writing anything (pointers to
 *     T-sized arrays may then be NULL); e4b_lora_wgrad still writes its
 *     all-zero gradients.
 *   - A launch failure returns E4B_ERR_CUDA.  Device-side waits are bounded:
 *     a wait that runs out records E4B_ERR_DEVICE_TIMEOUT in the workspace,
 *     the kernel ends cleanly, and e4b_check_device_error reports it.
 *   - Permuted buffers ("rows") hold the routed slots grouped by expert;
 *     every expert's group starts at a multiple of E4B_ROW_ALIGN rows and its
 *     padding rows are zero.  Their row capacity is e4b_sizes.rows_cap.
 */
#ifndef E4B_H
#define E4B_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *e4b_stream_t; /* a cudaStream_t; NULL is the legacy default stream */
typedef uint16_t e4b_bf16;                 /* bfloat16 bit pattern */

typedef enum {
  E4B_OK = 0,
  E4B_ERR_INVALID_ARG = 1,          /* null/misaligned pointer, negative size, inconsistent dims */
  E4B_ERR_UNSUPPORTED = 2,          /* a shape, rank, block size or epilogue the library refuses */
  E4B_ERR_WORKSPACE_TOO_SMALL = 3,  /* ws_bytes < e4b_sizes.workspace_bytes */
  E4B_ERR_CUDA = 4,                 /* a CUDA runtime/driver call or a launch failed */
  E4B_ERR_DEVICE_TIMEOUT = 5        /* a device-side wait ran out (see e4b_check_device_error) */
} e4b_status;

enum { E4B_ACT_SILU_GLU = 0 };   /* the only epilogue: silu(gate) * up */
enum { E4B_ROW_ALIGN = 128 };    /* every expert's group of rows starts at a multiple of this */
enum { E4B_MAX_EXPERTS = 1024, E4B_MAX_TOP_K = 32, E4B_MAX_RANK = 64 };

/* Problem dimensions.  Requirements (else E4B_ERR_UNSUPPORTED):
 * 1 <= E <= 1024; H, I positive multiples of 64; 1 <= top_k <= min(E, 32);
 * r a multiple of 8 in [8, 64]; blocksize == 64; act == E4B_ACT_SILU_GLU;
 * alpha finite.  The LoRA scaling is s = alpha / r. */
typedef struct {
  int32_t E, H, I, top_k, r;
  float alpha;
  int32_t blocksize;
  int32_t act;
} e4b_moe_dims;

/* The frozen base, NF4 with one float32 absmax per 64 consecutive elements
 * of a row.  Element 2m of a row is the HIGH nibble of byte m, element 2m+1
 * the LOW nibble.  gate_up rows [0, I) are the gate projection, rows [I, 2I)
 * the up projection.  A weight dequantises to
 * bf16_rn(float32(NF4[code]) * float32(absmax)). */
typedef struct {
  const uint8_t *gate_up_nf4;   /* [E, 2I, H/2]  */
  const float   *gate_up_absmax;/* [E, 2I, H/64] */
  const uint8_t *down_nf4;      /* [E, H, I/2]   */
  const float   *down_absmax;   /* [E, H, I/64]  */
} e4b_nf4_experts;

/* Per-expert LoRA factors (bf16). */
typedef struct {
  const e4b_bf16 *A_gu;  /* [E, r, H]  */
  const e4b_bf16 *B_gu;  /* [E, 2I, r] */
  const e4b_bf16 *A_d;   /* [E, r, I]  */
  const e4b_bf16 *B_d;   /* [E, H, r]  */
} e4b_lora;

/* Routing results, written by e4b_route_permute, read by the other calls. */
typedef struct {
  int32_t *topk_ids;     /* [T, top_k]  experts of each token, descending logit */
  float   *topk_w;       /* [T, top_k]  softmax over the selected logits */
  int32_t *counts;       /* [E]         slots routed to each expert */
  int32_t *offsets;      /* [E + 1]     first row of each expert's group; offsets[E] = rows used */
  int32_t *row_of_slot;  /* [T*top_k]   row of flat slot t*top_k + j */
  int32_t *slot_of_row;  /* [rows_cap]  flat slot held by each used row, -1 for padding rows */
  int32_t *tiles;        /* [tiles_cap] device work list (opaque) */
} e4b_routing;

/* Forward activations, all [rows_cap, .] bf16.  Written by the forward and
 * kept for the backward (the base weights are never stored dequantised). */
typedef struct {
  e4b_bf16 *x_perm;  /* [rows_cap, H]  token rows grouped by expert (e4b_route_permute) */
  e4b_bf16 *p_gu;    /* [rows_cap, r]  s * (x A_gu^T) */
  e4b_bf16 *gu;      /* [rows_cap, 2I] pre-activation, gate | up */
  e4b_bf16 *act;     /* [rows_cap, I]  silu(gate) * up */
  e4b_bf16 *p_d;     /* [rows_cap, r]  s * (act A_d^T) */
  e4b_bf16 *y_perm;  /* [rows_cap, H]  expert output of each slot (unweighted) */
} e4b_fwd_buffers;

/* Backward intermediates, all [rows_cap, .] bf16. */
typedef struct {
  e4b_bf16 *dyw;     /* [rows_cap, H]  w * dY of each slot */
  e4b_bf16 *q_d;     /* [rows_cap, r]  s * (dyw B_d) */
  e4b_bf16 *dgu;     /* [rows_cap, 2I] gradient of the pre-activation */
  e4b_bf16 *q_gu;    /* [rows_cap, r]  s * (dgu B_gu) */
  e4b_bf16 *dx_perm; /* [rows_cap, H]  input gradient of each slot */
} e4b_bwd_buffers;

typedef struct {
  int64_t slots;           /* N = T * top_k */
  int64_t rows_cap;        /* rows of every permuted buffer: N + E*(E4B_ROW_ALIGN-1), rounded up */
  int64_t tiles_cap;       /* int32 entries of e4b_routing.tiles */
  size_t  workspace_bytes; /* bytes of the `ws` argument every call needs */
} e4b_sizes;

/* Human-readable name of a status.  Never NULL. */
const char *e4b_status_string(e4b_status s);

/* Library version string. */
const char *e4b_version(void);

/* The 16 NF4 levels the library decodes with (float32, ascending): the
 * NormalFloat-4 code book of the QLoRA paper (Dettmers et al., 2023), which
 * the pages name as the default base format without printing it. */
void e4b_nf4_levels(float out[16]);

/* Buffer sizes for `dims` and T tokens.  Host only; no CUDA call. */
e4b_status e4b_get_sizes(const e4b_moe_dims *dims, int32_t T, e4b_sizes *out);

/* Clears the workspace's device error word (enqueued on `stream`).  Call
 * once after allocating a workspace; the word is sticky afterwards. */
e4b_status e4b_workspace_init(void *ws, size_t ws_bytes, e4b_stream_t stream);

/* Synchronises `stream`, then returns E4B_ERR_DEVICE_TIMEOUT if any kernel
 * recorded a timed-out wait in `ws`, E4B_ERR_CUDA on a CUDA error, else
 * E4B_OK.  The only entry point that blocks the host. */
e4b_status e4b_check_device_error(const void *ws, e4b_stream_t stream);

/* Routing and grouping: per token the top_k largest logits (ties to the lower
 * expert id, NaN lowest), the softmax over them, the stable grouping of the
 * T*top_k slots by expert (ascending flat slot within an expert), the device
 * work list, and x_perm[row] = x[token of row] (zero for padding rows).
 * logits: float32 [T, E]; x: bf16 [T, H]; x_perm: [rows_cap, H].  With
 * x_perm NULL only the routing tables are written (x is not read and may be
 * NULL): the permutation is then left to e4b_grouped_nf4_lora_fwd, which
 * gathers the rows in the same pass as its first LoRA projection.
 * Deterministic: identical inputs give identical bits.
 * Pages: same page, section "Which project solves it" (grouped execution);
 * the router's logits are inputs (router frozen, section "The abstraction
 * that fails"). */
e4b_status e4b_route_permute(const e4b_moe_dims *dims, int32_t T, const float *logits,
                             const e4b_bf16 *x, const e4b_routing *routing, e4b_bf16 *x_perm,
                             void *ws, size_t ws_bytes, e4b_stream_t stream);

/* Routing and grouping exactly as e4b_route_permute, for callers that
 * cannot allocate device memory and so cannot supply a workspace: code
 * running while a CUDA graph is captured in global mode (cudaMalloc is not
 * permitted there), engine plugins limited to memory the engine planned up
 * front, or runtimes with a fixed device-memory budget.  The pages have no
 * counterpart; this is an addition of this library.
 * Scratch lives in a fixed 4 MiB array in the library's own device memory
 * (held on every GPU that loads the library until the process exits); calls
 * whose 2 * ceil(T / 64) * E int32 scratch entries exceed 1,048,576 are
 * refused with E4B_ERR_UNSUPPORTED.  Allocates nothing (no cudaMalloc,
 * cudaFree or allocating library call).  The first call on a device looks
 * up the array's device address (a one-time set-up per device, made with
 * that device current); make that first call before any stream capture.
 * All calls share the one array: calls whose work overlaps on the GPU (other
 * streams, other host threads) race on it and must be serialised by the
 * caller.  Nothing in the array needs to start at zero.  As with
 * e4b_route_permute, x_perm NULL writes the routing tables only (x unread),
 * and T == 0 returns E4B_OK with nothing launched. */
e4b_status e4b_route_permute_noalloc(const e4b_moe_dims *dims, int32_t T, const float *logits,
                                     const e4b_bf16 *x, const e4b_routing *routing, e4b_bf16 *x_perm,
                                     e4b_stream_t stream);

/* Forward: p_gu, gu/act (SiLU-gated epilogue), p_d, y_perm, then the
 * router-weighted un-permute y[t] = sum_j w[t,j] * y_perm[row(t,j)] (fp32
 * sum in j order, rounded once to bf16).  y: bf16 [T, H].  With x (bf16
 * [T, H]) given, the call writes fwd->x_perm itself (x_perm[row] = x[token of
 * row], zero for padding rows, as e4b_route_permute would) in the same pass
 * as p_gu, so the permuted rows are not read back from memory; with x NULL,
 * fwd->x_perm must hold what e4b_route_permute wrote.
 * Pages: section "The abstraction that fails" (pre-activation delta) and
 * section "Why it happens" (the LoRA term); METADATA "The package family". */
e4b_status e4b_grouped_nf4_lora_fwd(const e4b_moe_dims *dims, int32_t T,
                                    const e4b_routing *routing, const e4b_nf4_experts *base,
                                    const e4b_lora *lora, const e4b_bf16 *x, const e4b_fwd_buffers *fwd,
                                    e4b_bf16 *y, void *ws, size_t ws_bytes, e4b_stream_t stream);

/* Serving forward: routing and the forward in one call, for inference
 * (decode-sized batches above all): y = the block's output for x (bf16
 * [T, H]) and logits (float32 [T, E]), the same arithmetic as
 * e4b_route_permute + e4b_grouped_nf4_lora_fwd.  Batches with at most
 * 16 * E routed slots take the serving pipeline: the routing tables in one
 * launch (T <= 64) or three, then ONE persistent launch for everything else
 * -- the x scatter with the LoRA projection s * x A_gu^T, the weight-
 * streaming gate_up GEMM with the SiLU-gated epilogue, the projection
 * s * act A_d^T, the weight-streaming down GEMM and the router-weighted
 * combine, its work units ordered so that each waits (device-side, bounded:
 * a wait that runs out records E4B_ERR_DEVICE_TIMEOUT in the workspace) only
 * for units before it.  Nothing is kept for a backward: fwd->gu may be NULL
 * (then not written), padding rows of the permuted buffers are left
 * unspecified and the m-tile lists in routing->tiles are not built, so the
 * routing and buffers of a serving call must not be passed to
 * e4b_grouped_nf4_lora_dgrad or e4b_lora_wgrad.  The launch keeps its
 * counters and partial sums in ws (e4b_get_sizes accounts for them), so two
 * serving calls that share a workspace must not overlap on the GPU.
 * Larger batches run e4b_route_permute + e4b_grouped_nf4_lora_fwd (fwd->gu
 * is then required).  Argument checks, ownership and errors as for those two
 * calls; the call allocates nothing and never synchronises, so it can be
 * captured into a CUDA graph.
 * Pages: section "Which project solves it" (grouped forward), section
 * "Limitations" (the fast forward for inference) and METADATA "The package
 * family" (a single launch covers all packed experts). */
e4b_status e4b_moe_serve_fwd(const e4b_moe_dims *dims, int32_t T, const float *logits, const e4b_bf16 *x,
                             const e4b_routing *routing, const e4b_nf4_experts *base, const e4b_lora *lora,
                             const e4b_fwd_buffers *fwd, e4b_bf16 *y, void *ws, size_t ws_bytes,
                             e4b_stream_t stream);

/* Input gradient for upstream dY (bf16 [T, H]): dyw = w * dY per slot,
 * q_d, the down-projection dgrad through the transposed re-dequantised base
 * plus LoRA with the SwiGLU backward fused in (dgu), q_gu, the gate_up dgrad
 * (dx_perm), and dx[t] = sum_j dx_perm[row(t,j)] (bf16 [T, H]).
 * Pages: section "Which project solves it" (dgrad kernel) and section "Why it
 * happens" (re-dequantisation in backward). */
e4b_status e4b_grouped_nf4_lora_dgrad(const e4b_moe_dims *dims, int32_t T,
                                      const e4b_routing *routing, const e4b_nf4_experts *base,
                                      const e4b_lora *lora, const e4b_fwd_buffers *fwd,
                                      const e4b_bf16 *dY, const e4b_bwd_buffers *bwd, e4b_bf16 *dx,
                                      void *ws, size_t ws_bytes, e4b_stream_t stream);

/* LoRA weight gradients, fp32 accumulation, bf16 out, for every expert
 * (an expert with no tokens gets exact zeros):
 *   dB_gu[e] = dgu_e^T p_gu_e  [2I, r]     dA_gu[e] = q_gu_e^T x_e   [r, H]
 *   dB_d[e]  = dyw_e^T p_d_e   [H, r]      dA_d[e]  = q_d_e^T act_e  [r, I]
 * (p and q already carry the scaling s).  The frozen base gets no gradient.
 * Pages: section "The abstraction that fails" (trainable A[e]/B[e], frozen
 * base). */
e4b_status e4b_lora_wgrad(const e4b_moe_dims *dims, int32_t T, const e4b_routing *routing,
                          const e4b_fwd_buffers *fwd, const e4b_bwd_buffers *bwd,
                          e4b_bf16 *dA_gu, e4b_bf16 *dB_gu, e4b_bf16 *dA_d, e4b_bf16 *dB_d,
                          void *ws, size_t ws_bytes, e4b_stream_t stream);

/* Router-logit gradient, for a trained router (the router is frozen by
 * default and its logits are inputs; this is the extra step that training it
 * needs).  The top-k selection is piecewise constant, so the logits get a
 * gradient through the routing weights only:
 *   dw[t,j]  = <dY[t], y_perm[row(t,j)]>   (fp32 sum of bf16 products)
 *   d_logits[t, ids[t,j]] = w[t,j] * (dw[t,j] - sum_i w[t,i] dw[t,i])
 * and every other entry of d_logits is 0 (the whole [T, E] array is written).
 * routing: what e4b_route_permute wrote for these T tokens (ids, weights,
 * row_of_slot are read); y_perm: the unweighted expert outputs the forward
 * wrote (e4b_fwd_buffers.y_perm); dY: bf16 [T, H], the upstream gradient the
 * dgrad also takes.  d_logits: float32 [T, E]; dw: float32 [T, top_k] or NULL
 * (not written).  All device pointers, 16-byte aligned, owned by the caller;
 * invalid arguments -> E4B_ERR_INVALID_ARG / E4B_ERR_UNSUPPORTED with no
 * launch; T == 0 launches nothing.  Needs no workspace.  Deterministic.
 * Pages: "How do I QLoRA-train the fused experts of a MoE", section "The
 * abstraction that fails, and what replaces it" (TRAIN_ROUTER trains the
 * router `mlp.gate.weight`; the weights are the softmax over the selected
 * logits). */
e4b_status e4b_router_backward(const e4b_moe_dims *dims, int32_t T, const e4b_routing *routing,
                               const e4b_bf16 *y_perm, const e4b_bf16 *dY, float *d_logits, float *dw,
                               e4b_stream_t stream);

/* Dequantises n NF4 elements (n a multiple of 64): packed uint8 [n/2],
 * absmax float32 [n/64] -> bf16 [n], with the same device routine the
 * grouped GEMMs decode with.  For bit-exact testing of the decode.  Device
 * pointers owned by the caller (packed and out 16-byte aligned, absmax 4-byte
 * aligned); invalid sizes or alignment -> E4B_ERR_INVALID_ARG, no launch.
 * Pages: experts4bit-qlora package METADATA, section "The package family"
 * (the 4-bit codes decoded in registers); the element layout is the one
 * e4b_nf4_experts states. */
e4b_status e4b_nf4_dequant(const uint8_t *packed, const float *absmax, int64_t n, e4b_bf16 *out,
                           e4b_stream_t stream);

/* Quantises n bf16 weights (n a multiple of 64; blocks of 64 consecutive
 * elements, i.e. along the rows of a row-major [..., K] stack with K % 64 ==
 * 0) to NF4: packed uint8 [n/2] (element 2m in the high nibble of byte m),
 * absmax float32 [n/64].  Per block absmax = max |w|; each code is the level
 * nearest to w / absmax, computed as an IEEE float32 division and float32
 * distances |w/absmax - level| with an exact tie going to the lower code; a
 * block whose absmax is 0 gets code 7 (the level 0) throughout.  This is the
 * step that turns a bf16 fused expert stack into the frozen NF4 base the
 * grouped GEMMs read (and that e4b_nf4_dequant inverts up to rounding).
 * w and packed 16-byte aligned, absmax 4-byte aligned; device pointers owned
 * by the caller; invalid sizes or alignment -> E4B_ERR_INVALID_ARG with no
 * launch.  Non-finite weights give what the same float32 rules give (a NaN
 * makes the block's absmax NaN and its codes 7).
 * Pages: "How do I QLoRA-train the fused experts of a MoE", section "The
 * abstraction that fails, and what replaces it" (the packed NF4 base chosen
 * with quant_type= on the loader) and section "Smallest correct example"
 * (the loader quantising the fused stacks to 4 bit). */
e4b_status e4b_nf4_quantize(const e4b_bf16 *w, int64_t n, uint8_t *packed, float *absmax, e4b_stream_t stream);

/* Watchdog self-test: launches one CTA that waits on an mbarrier nothing
 * arrives on, with a limit of `timeout_ns` nanoseconds, so that the bounded
 * wait runs out and records E4B_ERR_DEVICE_TIMEOUT in `ws`.  No GPU fault. */
e4b_status e4b_debug_watchdog(void *ws, size_t ws_bytes, int64_t timeout_ns, e4b_stream_t stream);

/* ---- Measurement -------------------------------------------------------
 * Optional per-kernel timing.  While enabled, every kernel the library
 * launches is bracketed by two CUDA events recorded on that launch's stream;
 * e4b_profiler_read waits for the recorded events, returns per-kernel launch
 * counts and summed device times, and clears the record.  Off by default; it
 * creates CUDA events (host handles), never device buffers.  Launches made
 * while their stream is being captured into a CUDA graph are not timed. */
typedef struct {
  char name[48];      /* kernel (and mode) name */
  int64_t launches;   /* launches recorded */
  double total_ms;    /* summed event-to-event device time */
} e4b_kernel_time;

e4b_status e4b_profiler_enable(int32_t on);
e4b_status e4b_profiler_read(e4b_kernel_time *out, int32_t capacity, int32_t *count);

/* Number of kernels this library has launched in this process so far. */
int64_t e4b_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* E4B_H */
