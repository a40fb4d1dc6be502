/*
 * scion.h -- C ABI of libscion: the forward pass of one mixture-of-experts block
 * whose expert banks are ternary ({-1, 0, +1} codes with one fp16 scale per 128
 * weights), plus a rank-r low-rank correction added to the block output.
 * All compute runs in hand-written CUDA kernels for sm_100a (NVIDIA B200).
 *
 * Sources (page titles and sections):
 *  [P1] "Scion: ternary MoE quantization with trained corrections", The idea:
 *       ternary expert banks at 2.125 bpw; rank-512 correction branches on the
 *       MoE block output; router deltas.
 *  [P3] "Scion-35B-A3B" model card: Model Overview (256 experts, top-8 plus a
 *       shared expert), Weight Representation (codes in {-1,0,+1} plus one fp16
 *       group scale per 128 weights = 2.125 bpw; routers stay F32).
 *  [P4] "Scion-FlashNext-176B-A6B" model card: Model Overview (512 experts,
 *       top-10 routed + 1 shared), Highlights and Weight Representation (PTQ1_0:
 *       base-3 trits plus an fp16 scale, 28 bytes per 128 weights = 1.75 bpw).
 *  [P1 Serving notes] the expert matmul computes k experts per token.
 *
 * Conventions for every entry point:
 *  - Returns an int status (scion_status); never throws, never aborts.
 *  - "device" pointers are CUDA global memory of the current device; "host"
 *    pointers are CPU memory.  The caller owns every buffer it passes.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy stream).
 *    Device work is enqueued asynchronously; no entry point synchronises the
 *    stream except scion_layer_create (which validates codes once).
 *  - Asynchronous CUDA faults surface as SCION_ECUDA on a later call.
 */
#ifndef SCION_H
#define SCION_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SCION_OK = 0,
  SCION_EINVAL = -1,   /* bad argument: null pointer, size out of range, bad descriptor */
  SCION_ENOMEM = -2,   /* device or host allocation failed */
  SCION_ECUDA = -3,    /* a CUDA runtime call or kernel launch failed */
  SCION_EFORMAT = -4,  /* a packed block holds an invalid code (PQ2_0 field 3, PTQ1_0 byte > 242 / tail > 26) */
  SCION_ETIMEOUT = -5  /* a bounded device-side wait gave up */
} scion_status;

/* Container formats.  Bit orders are this library's container specification
 * (the pages give only the sizes):
 *  SCION_PQ2_0  (34 B / 128 weights, [P3] Weight Representation): byte i < 32
 *     holds weights 4i..4i+3, weight 4i+j in bits 2j..2j+1; field 0 -> -1,
 *     1 -> 0, 2 -> +1, 3 invalid; bytes 32..33 = fp16 scale, little-endian.
 *  SCION_PTQ1_0 (28 B / 128 weights, [P4] Weight Representation): byte q < 25 =
 *     sum_{j<5} t_{5q+j} 3^j; byte 25 = t125 + 3 t126 + 9 t127; trit t -> code
 *     t - 1; bytes 26..27 = fp16 scale, little-endian.
 * A weight is code * scale. */
typedef enum { SCION_PQ2_0 = 0, SCION_PTQ1_0 = 1 } scion_fmt;

/* Bytes per 128-weight block: 34 (PQ2_0), 28 (PTQ1_0), 0 for an unknown format. */
size_t scion_block_bytes(int fmt);

/* Human-readable name of a status code (static storage). */
const char* scion_status_str(int status);

/* ------------------------------------------------------------------ packing
 * Host packers.  codes: n_groups*128 int8 values in {-1,0,+1}; scales:
 * n_groups fp16 bit patterns; out: n_groups*scion_block_bytes(fmt) bytes.  All
 * host memory, caller-owned.  EINVAL on a null pointer, n_groups < 0 or a code
 * outside {-1,0,+1} (out is then unspecified). */
int scion_pack_pq2(const int8_t* codes, const uint16_t* scales, int64_t n_groups, uint8_t* out);
int scion_pack_ptq1(const int8_t* codes, const uint16_t* scales, int64_t n_groups, uint8_t* out);

/* Host unpacker, the inverse of the packers.  Invalid fields decode to code 0
 * and the call returns SCION_EFORMAT after decoding everything. */
int scion_unpack(int fmt, const uint8_t* in, int64_t n_groups, int8_t* codes, uint16_t* scales);

/* Device packer: same contract as the host packers, all three pointers device
 * memory, enqueued on `stream`.  A code outside {-1,0,+1} is packed as 0 and
 * counted; if `bad_count` (device int64, may be NULL) is given, the number of
 * such codes is ADDED to it. */
int scion_pack_device(int fmt, const int8_t* codes, const uint16_t* scales, int64_t n_groups, uint8_t* out,
                      int64_t* bad_count, void* stream);

/* Device unpacker: inverse of scion_pack_device.  Invalid fields decode to 0;
 * if `bad_count` (device int64, may be NULL) is given the number of invalid
 * fields is ADDED to it. */
int scion_unpack_device(int fmt, const uint8_t* in, int64_t n_groups, int8_t* codes, uint16_t* scales,
                        int64_t* bad_count, void* stream);

/* Test support for the failure path of the device-side waits: one kernel waits on a barrier
 * phase that nothing completes, with a limit of limit_us (1 .. 10^6) microseconds; a second warp
 * waits on another such phase with ten times the limit.  The first must give up on its clock
 * and write SCION_ETIMEOUT, the second must leave on the abort flag the first raised.  result
 * (host int[3]) receives {the status word, first wait's return, second wait's return} (expected
 * {SCION_ETIMEOUT, 0, 0}); *elapsed_ms the time until both gave up.  No fault, no hang: the
 * kernel ends after about limit_us plus the wait's suspend time (1 ms).  Synchronises `stream`.
 * EINVAL on a bad argument, ENOMEM, ECUDA. */
int scion_selftest_bounded_wait(int limit_us, int* result, double* elapsed_ms, void* stream);

/* Float -> ternary quantizers ("Scion: ternary MoE quantization with trained corrections",
 * Findings: the deployable Lloyd quantizer against one-shot absmean; "Scion-35B-A3B" model
 * card, Highlights: ternary Lloyd g128).  w: device fp32, n_groups groups of 128 consecutive
 * weights (a row-major [rows][K] matrix with K % 128 == 0 is rows * K / 128 groups along K),
 * 16-byte aligned, finite, |w| <= 65504.  Writes codes (device int8 [n_groups][128], 4-byte
 * aligned) in {-1, 0, +1} and scale_f16 (device binary16 bits [n_groups]) such that
 * w ~ code * scale; feed them to scion_pack_device for the PQ2_0 / PTQ1_0 containers.
 *   SCION_QUANT_ABSMEAN: s = mean |w| of the group; code = sign(w) where 2|w| >= s, else 0.
 *   SCION_QUANT_LLOYD:   Lloyd's algorithm for the levels {-s, 0, +s} from the absmean start:
 *     s = mean |w| over the nonzero codes, then every code re-chosen by the rule above, until
 *     no code changes or `iters` (0..1000) rounds ran; s = mean |w| over the final nonzero codes.
 * Sums and decisions in fp64; the scale is rounded to the nearest binary16.  Enqueued on
 * `stream`.  EINVAL on a bad method, count, iteration limit, null or misaligned pointer. */
enum { SCION_QUANT_ABSMEAN = 0, SCION_QUANT_LLOYD = 1 };
int scion_quantize_device(int method, const float* w, int64_t n_groups, int iters, int8_t* codes, uint16_t* scale_f16,
                          void* stream);

/* -------------------------------------------------------------------- layer
 * One MoE block.  d = hidden size, E = experts, k = top-k, F = expert ffn,
 * Fs = shared-expert ffn (0 = no shared expert), r = correction rank (0 = none).
 * d and F must be multiples of 128; 1 <= k <= E <= 4096; Fs % 128 == 0;
 * r % 16 == 0.
 *
 * Expert banks (device, packed blocks in `fmt`, groups of 128 along each row's
 * reduction axis; [P3]/[P4] Weight Representation):
 *   gate_exps, up_exps : [E][F][d/128] blocks     (rows = ffn units, K = d)
 *   down_exps          : [E][d][F/128] blocks     (rows = hidden units, K = F)
 * Router ([P1] The idea; [P3] Weight Representation): w_router and
 * w_router_delta are [E][d], fp32 when router_fp32 = 1, else bf16; the logit of
 * expert e is x.w_router[e] + x.w_router_delta[e].
 * Shared expert ([P3]/[P4] Model Overview), bf16: sh_gate, sh_up [Fs][d];
 * sh_down [d][Fs]; sh_gate_vec [d] or NULL (if given, the shared output is
 * multiplied by sigmoid(x . sh_gate_vec)).
 * Correction ([P1] The idea: rank-r branch on the MoE block output), bf16:
 * corr_a [r][d], corr_b [d][r]; it adds corr_b (corr_a x) to the output, where x
 * is the block input (the branch runs beside the block on the residual stream,
 * scale 1).
 * Gates: norm_topk = 1 -> softmax over the k selected logits; 0 -> the selected
 * entries of a softmax over all E logits. */
typedef struct {
  int d, n_experts, top_k, ffn, shared_ffn, rank;
  int fmt;         /* scion_fmt */
  int router_fp32; /* 1: router and delta fp32; 0: bf16 */
  int norm_topk;   /* 1 (default reading) or 0 */
  const void* w_router;
  const void* w_router_delta;
  const void* gate_exps;
  const void* up_exps;
  const void* down_exps;
  const void* sh_gate;
  const void* sh_up;
  const void* sh_down;
  const void* sh_gate_vec;
  const void* corr_a;
  const void* corr_b;
  /* 0: corr_a / corr_b are bf16 [rank][d] and [d][rank].  1: ternary correction factors
   * ("Scion-35B-A3B" model card, Weight Representation: the corrections ship as 2-bit codes
   * plus one fp16 scale per 128, the q1_0_g128 container) as PQ2_0 blocks, corr_a [rank][d/128] and corr_b [d][rank/128] (groups of 128 along each
   * factor's reduction axis; rank a multiple of 128; 2-byte aligned).  Decode reads both
   * factors' blocks in place (they must outlive the handle); the tensor-core path (batches
   * above 64 tokens) uses exact fp16 copies (code * scale). */
  int corr_packed;
  /* Expert parallelism: this handle holds experts [expert_lo, expert_lo + n_local_experts) of the
   * n_experts the router scores (n_local_experts = 0: all of them, expert_lo must be 0).  The
   * banks then hold n_local_experts experts ([n_local][F][d/128] and [n_local][d][F/128] blocks);
   * routing still picks the top-k of all n_experts logits, and only the entries whose expert is
   * local are grouped and computed (the grouping outputs of scion_moe_forward_debug are indexed
   * by local expert).  With SCION_OPT_PARTS the handle computes the routed and / or the dense part
   * (shared expert + correction) of the block; summing the routed parts of the ranks that hold all
   * experts and one dense part gives the block output. */
  int expert_lo;
  int n_local_experts;
} scion_layer_desc;

typedef struct scion_layer scion_layer;

/* Builds a layer handle for batches of up to max_tokens tokens.
 * Copies the expert banks into the device layout used by the kernels (same
 * bytes per 128 weights, regrouped into 16-byte-aligned tiles), converts
 * sh_down and corr_b to an fp16 copy, and allocates the workspace.  After it
 * returns, the caller may free gate_exps / up_exps / down_exps / sh_down /
 * corr_b (not corr_b's blocks when corr_packed); w_router, w_router_delta, sh_gate,
 * sh_up, sh_gate_vec and corr_a are read in place and must outlive the handle.  Synchronises `stream` once to
 * validate every code: SCION_EFORMAT if a block holds an invalid code (no
 * handle is returned), EINVAL on a bad descriptor, ENOMEM, ECUDA.  Descriptor
 * limits: d and ffn multiples of 128 with d <= 4096, shared_ffn a multiple of 128,
 * rank a multiple of 16 (of 128 with corr_packed), 1 <= top_k <= min(E, 32), E <= 4096.
 * With corr_packed, a correction-A scale whose 256-fold overflows fp16 on a PQ2_0 layer with
 * max_tokens > 64 counts as an invalid code (its fp16 copy is stored in the experts' column
 * order, scaled by the same powers of 4 as their inputs). */
int scion_layer_create(const scion_layer_desc* desc, int max_tokens, void* stream, scion_layer** out);

/* Frees the handle and everything it allocated (synchronises the device). */
void scion_layer_destroy(scion_layer* layer);

/* Bytes of device memory owned by the handle (banks, fp16 copies, workspace). */
size_t scion_layer_device_bytes(const scion_layer* layer);

/* The block forward ([P1] The idea; [P3]/[P4] Model Overview):
 *   out[t] = sum_{j<k} g_{t,j} E_{e(t,j)}(x_t) + S(x_t) + B (A x_t)
 * with E_e(x) = W_d,e (silu(W_g,e x) * (W_u,e x)), S the shared expert and
 * g, e(t, .) the gates and ids of the top-k router logits.
 * x: device bf16 [T][d]; out: device fp32 [T][d], OVERWRITTEN (no residual add); both
 * 16-byte aligned.
 * 0 <= T <= max_tokens (T = 0 is a no-op).  Batches of at most 64 tokens stream the
 * weights through warp-level MMA kernels; larger batches (layers created with
 * max_tokens > 64) run as tcgen05 grouped GEMMs.  Calls on one handle must not
 * overlap on the GPU (they share its workspace): issue them on one stream.  Batches of
 * 16..64 tokens fork the dense down projection onto a stream owned by the handle and
 * join it back (events) before the call's work on `stream` ends; stream capture into
 * a CUDA graph records the fork and the join.
 * Activation range: any finite bf16 x.  The expert GEMMs and the stored hidden values run in
 * fp16; every token whose largest |x| lies outside [2^-3, 2^6) is scaled by a power of two
 * 2^s (s = 2 - floor(log2 max|x|), clamped to [-40, 40]) on its way into them and scaled back
 * exactly where its results enter out, so tokens with outlier channels (tested up to 3e4),
 * tokens of tiny magnitude (tested near 1e-6) and large ones keep the block tolerance; max|x|
 * inside [2^-38, 2^42] is fully normalised.  The output itself is fp32: a block output beyond
 * the fp32 range overflows.
 * EINVAL on a null or misaligned pointer or T out of range; ECUDA if a launch fails. */
int scion_moe_forward(const void* x, int T, const scion_layer* layer, float* out, void* stream);

/* The block added to the residual stream ("Scion: ternary MoE quantization with trained
 * corrections", The idea: the block output and its correction are added to the residual
 * stream):  out[t] = resid[t] + block(x_t), with block(x_t) the output of scion_moe_forward.
 * resid: device fp32 [T][d], 16-byte aligned; it may be the same buffer as out (in-place
 * accumulation), otherwise it is only read.  The residual enters where out is first written
 * (the first kernel of the call), so the cost is one read of resid.
 * EINVAL on a null or misaligned pointer or T out of range; ECUDA if a launch fails. */
int scion_moe_forward_residual(const void* x, int T, const scion_layer* layer, const float* resid, float* out,
                               void* stream);

/* Tuning options of a layer (scion_layer_set_option).
 *  SCION_OPT_STREAM_MIN_TOKENS (default 16): batches of at least this many tokens (and at
 *    most 64) run the expert GEMMs on persistent kernels (128 expert rows per work item);
 *    smaller batches split K over the warps of one CTA per 16 rows, which spreads the few
 *    active experts over more SMs.
 *  SCION_OPT_DECODE_TC (default 0): 0 runs those persistent kernels as mma.sync kernels fed by a
 *    bulk-copy ring; 1 as tcgen05 kernels (codes expanded into tensor memory at one instruction
 *    per two weights, tiles of up to 16 tokens of one expert, one accumulator per 128-column
 *    group folded into registers with the group scales; the down projection adds its
 *    gate-weighted rows into out).  Layers of up to 512 experts.
 *  SCION_OPT_DETERMINISTIC (default 1): batches above 64 tokens are bit-reproducible: the down
 *    projection writes one fp16 row per routed entry and a combine kernel sums each token's rows
 *    in slot order.  0: the down projection adds its rows into out with fp32 reductions (no row
 *    buffer, order of the additions not fixed).
 *    All settings give the same result up to fp32 summation order.
 * EINVAL for an unknown option or an out-of-range value. */
enum { SCION_OPT_STREAM_MIN_TOKENS = 1, SCION_OPT_DECODE_TC = 2, SCION_OPT_DETERMINISTIC = 3, SCION_OPT_PARTS = 4 };
/* SCION_OPT_PARTS (default SCION_PART_ROUTED | SCION_PART_DENSE): which part of the block a forward
 * computes: the routed experts (the handle's local ones), the dense part (shared expert and
 * correction), or both.  out is overwritten with the selected part (plus resid). */
enum { SCION_PART_ROUTED = 1, SCION_PART_DENSE = 2 };
int scion_layer_set_option(scion_layer* layer, int option, int value);

/* Waits for `stream`, then returns the layer's device status word and clears it:
 * SCION_ETIMEOUT if a tensor-core kernel of an earlier forward gave up a bounded wait
 * (its outputs are then invalid), SCION_ECUDA on an asynchronous CUDA fault, else OK. */
int scion_layer_check(const scion_layer* layer, void* stream);

/* Same forward with x and out in HOST memory (pinned for asynchronous copies):
 * enqueues the host-to-device copy of x, the forward and the device-to-host copy
 * of out on `stream`.  The caller synchronises the stream before reading out. */
int scion_moe_forward_host(const void* x_host, int T, const scion_layer* layer, float* out_host, void* stream);

/* Intermediate results of a forward, for tests and debugging.  Every pointer is
 * device memory and may be NULL (not written). */
typedef struct {
  float* logits;    /* [T][E] router logits (fp32) */
  int32_t* ids;     /* [T][k] selected experts, descending logit, ties -> lower id */
  float* gates;     /* [T][k] gate weights */
  int32_t* counts;  /* [E] tokens routed to each expert */
  int32_t* offsets; /* [E+1] exclusive scan of counts */
  int32_t* perm;    /* [T*k] entries t*k+j, grouped by expert, token order within an expert */
  uint16_t* h;      /* fp16 [T*k][F] expert SwiGLU hidden, row p for perm[p], times 2^(2s) */
  uint16_t* hz;     /* fp16 [T][Fs + r] shared SwiGLU hidden then correction z = A x, times 2^p */
} scion_debug_out;
/* (s is the token's range exponent of scion_moe_forward, 0 for max|x| in [2^-3, 2^6); p = s on a
 * layer without a shared expert, 2s on a layer without a correction, and with both s for s > 0,
 * else 2s.) */

/* scion_moe_forward, then copies the intermediates requested in `dbg`. */
int scion_moe_forward_debug(const void* x, int T, const scion_layer* layer, float* out, const scion_debug_out* dbg,
                            void* stream);

/* The routing of a batch alone ([P3]/[P4] Model Overview: top-k of the router logits; [P1]
 * Serving notes: tokens grouped per expert for the expert matmul).  Runs the block forward on x
 * (bf16 [T][d], device, 16-byte aligned) with the output going to the handle's own staging
 * buffer, then copies ids [T][k] (int32), gates [T][k] (fp32), offsets [E+1] (int32) and perm
 * [T*k] (int32) -- the same values and orders as the fields of scion_debug_out -- into the
 * given device buffers; any of the four may be NULL (not written).  Calls on one handle must
 * not overlap (the staging buffer is shared with scion_moe_forward_host).  EINVAL on a null x,
 * a misaligned x or T out of range; ECUDA if a launch or copy fails. */
int scion_debug_route(const void* x, int T, const scion_layer* layer, int32_t* ids, float* gates, int32_t* offsets,
                      int32_t* perm, void* stream);

/* ------------------------------------------ correction branch on the attention output
 * The second correction branch of the method ("Scion: ternary MoE quantization with trained
 * corrections", The idea: rank-512 branches on the attention output and on the MoE block output;
 * Findings: the attention-output branch ships as a standard low-rank adapter on the attention
 * output projection; "Scion-35B-A3B" model card, Weight Representation: the corrections ship as
 * 2-bit codes plus one fp16 scale per 128).  The branch takes the input v of the attention
 * output projection (the attention heads' concatenated output, d_in wide) and adds its low-rank
 * product to the projection's output (d_out wide), scale 1:
 *   out[t] = base[t] + B (A v_t)
 * The attention itself and its output projection are the caller's; base is typically that
 * projection's output, or the residual stream with it already added.
 *   packed = 0: corr_a bf16 [rank][d_in], corr_b bf16 [d_out][rank], 16-byte aligned, read in place
 *              (they must outlive the handle; a fp16 copy of B is made);
 *   packed = 1: PQ2_0 blocks, corr_a [rank][d_in/128], corr_b [d_out][rank/128] (groups of 128
 *              along each factor's reduction axis), 2-byte aligned; rank a multiple of 128.
 * Limits: d_in a multiple of 128 and <= 4096, d_out a multiple of 128, rank a multiple of 16 and
 * <= 4096.  EINVAL on a bad descriptor, EFORMAT on an invalid code (packed), ENOMEM, ECUDA.
 * Batches of up to 64 tokens run split-K weight-streaming kernels, larger ones (handles created
 * with max_tokens > 64) tcgen05 GEMMs. */
typedef struct {
  int d_in, d_out, rank;
  int packed;
  const void* corr_a;
  const void* corr_b;
} scion_corr_desc;
typedef struct scion_corr scion_corr;
int scion_corr_create(const scion_corr_desc* desc, int max_tokens, void* stream, scion_corr** out);
void scion_corr_destroy(scion_corr* corr);
size_t scion_corr_device_bytes(const scion_corr* corr);
/* v: device bf16 [T][d_in]; base: device fp32 [T][d_out] or NULL (zero), may equal out; out:
 * device fp32 [T][d_out], written; all 16-byte aligned.  0 <= T <= max_tokens.  Activations get
 * the same per-token power-of-two range scaling as scion_moe_forward.  Calls on one handle must
 * not overlap on the GPU.  EINVAL on a null or misaligned pointer or T out of range; ECUDA. */
int scion_corr_forward(const void* v, int T, const scion_corr* corr, const float* base, float* out, void* stream);
/* Waits for `stream`, then returns and clears the handle's device status word (SCION_ETIMEOUT if
 * a bounded wait of the tensor-core path gave up), like scion_layer_check. */
int scion_corr_check(const scion_corr* corr, void* stream);

/* ------------------------------------------------------------ measurement
 * Kernel-level timing for benchmarks.  Between scion_profile_begin and
 * scion_profile_end, every kernel a forward launches is bracketed by a pair of CUDA
 * events recorded on the stream it is launched on, tagged with its stage:           */
enum {
  SCION_STAGE_ROUTER_F32 = 0,  /* fp32 router logits (FFMA) */
  SCION_STAGE_XPROJ = 1,       /* bf16 router + delta, shared gate/up + SwiGLU, correction A */
  SCION_STAGE_ROUTE = 2,       /* top-k, gates, histogram / scan / stable scatter */
  SCION_STAGE_GATEUP = 3,      /* ternary expert gate/up + SwiGLU */
  SCION_STAGE_DOWN_ROUTED = 4, /* ternary expert down + gate-weighted scatter-add */
  SCION_STAGE_DOWN_DENSE = 5,  /* shared down + correction B */
  SCION_STAGE_X16 = 6,         /* x -> fp16 in container column order (tensor-core path) */
  SCION_STAGE_COMBINE = 7,     /* gate-weighted sum of the k expert rows per token (tensor-core path) */
  SCION_N_STAGES = 8
};
/* Creates a pool for `max_launches` launches and starts recording (EINVAL if already
 * recording or max_launches < 1).  Launches past the pool are not recorded.  Not
 * thread-safe: one recording per process at a time. */
int scion_profile_begin(int max_launches);
/* Waits for the recorded events, stops recording, and writes per stage the summed
 * device time in milliseconds and the number of recorded launches (arrays of
 * n_stages entries, host memory).  Frees the pool. */
int scion_profile_end(int n_stages, double* ms_total, int64_t* launches);
/* Number of kernels the forward entry points have launched since the library loaded. */
int64_t scion_kernel_launches(void);

/* ------------------------------------------------------- no-allocation entry
 * Router logits for callers that cannot allocate device memory (their memory belongs
 * to another allocator, or they run where allocation is not allowed).  The pages
 * describe no counterpart of this entry point; it is a deployment aid.
 *   logits[t][e] = x_t . w_router[e] + x_t . w_router_delta[e]      (fp32)
 * x: device bf16 [T][d]; w_router, w_router_delta: device bf16 [E][d], all three 16-byte
 * aligned (they are read with 16-byte loads); logits: device fp32 [T][E], 4-byte aligned,
 * written.  A null or misaligned pointer returns SCION_EINVAL and launches nothing.  Limits: T <= 64, E <= 512, d <= 4096 and d % 128 == 0; larger
 * sizes return SCION_EINVAL and launch nothing.  The split-K scratch lives in a static
 * device array inside the library (1 MiB + 128 B on every GPU that loads it, held until
 * the process exits); the call allocates nothing.  The first call on a device looks the
 * array's address up (cudaGetSymbolAddress) with that device current -- make that first
 * call before any stream capture.  All calls share the array, so calls that could
 * overlap on the GPU (different streams, or devices sharing a context) race: issue them
 * in order on one stream.  Each call clears the array's counters before its kernel. */
int scion_router_logits_static(const void* x, int T, const void* w_router, const void* w_router_delta, int n_experts,
                               int d, float* logits, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SCION_H */
