/*
 * fmoe.h -- C ABI of libfmoe.so: the routed Mixture-of-Experts FFN block at
 * decode time, as hand-written CUDA kernels for sm_100a (B200).
 *
 * The block follows the Flash-MoE pages:
 *   - "What is Flash-MoE" (a2a-mcp.org), MoE section: per layer a router picks
 *     4 of 512 routed experts and one shared expert always runs;
 *   - same page, section 2: group-wise affine codes, dequantised as
 *     code * scale + bias (4-bit production, 2-bit experimental);
 *   - same page, section 3 (hand-tuned Metal shaders): two-pass RMSNorm, fused
 *     SwiGLU, and one combine pass of weighted experts + residual + sigmoid-gated
 *     shared expert;
 *   - "Flash-MoE" wiki summary (jeongsk), per-layer pipeline: routing projection,
 *     softmax, top-K.
 *
 * Conventions for every call:
 *   - Pointers are DEVICE pointers owned by the caller unless stated; the
 *     library never allocates or frees memory.
 *   - Calls are stream-ordered and asynchronous: they validate their arguments
 *     on the host, enqueue kernels on `stream` and return.  Errors in the
 *     arguments are reported before anything is enqueued.  A failed launch
 *     returns FMOE_ERR_CUDA.  Asynchronous device faults surface at the
 *     caller's next synchronisation.
 *   - No call aborts, throws or exits; fmoe_last_error() returns a message for
 *     the last non-OK status of the calling host thread.
 *   - Layouts are row-major.  bf16 values are passed as uint16_t bit patterns.
 *
 * Packed matrix [out][in] with b-bit codes (b = 2 or 4; 8 as a further format) and
 * group size G (64; 128 as a further format, for hidden and inter >= 1024), after
 * "Running MoE models on Apple Silicon with flash-moe" (gillilab), which lists INT2/3/4/8
 * and groups of 64 or 128:
 *   qw    uint32[out][in*b/32]  code of column c at word c/(32/b), bits
 *                               [b*(c%(32/b)), +b) counted from the LSB;
 *   scale bf16[out][in/G], bias bf16[out][in/G]: group g of row r covers
 *                               columns [G*g, G*g + G-1];
 *   weight (r, c) = code(r, c) * scale[r][c/G] + bias[r][c/G].
 * Only the per-token kernels take 8-bit codes and groups of 128; the grouped, fused and
 * two-kernel paths run 2/4-bit codes in groups of 64 and leave other formats to them.
 * Expert record: gate [I][H] | up [I][H] | down [H][I], each {qw, scale, bias},
 * every sub-array 16-byte aligned; at I = 1024, H = 4096 a record is
 * 7,077,888 bytes at 4-bit (the pages' "6.75 MB per expert") and 3,932,160
 * bytes at 2-bit (their "~3.9 MB").  A bank is `num_experts` records at a
 * fixed stride.
 */
#ifndef FMOE_H
#define FMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* fmoe_stream_t;

typedef enum {
  FMOE_OK = 0,
  FMOE_ERR_INVALID_ARG = 1,   /* NULL pointer, bad shape or count */
  FMOE_ERR_ALIGNMENT = 2,     /* a pointer, offset or stride is not 16-byte aligned */
  FMOE_ERR_UNSUPPORTED = 3,   /* a shape or width these kernels do not handle */
  FMOE_ERR_WORKSPACE = 4,     /* workspace missing or smaller than the size query returns */
  FMOE_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed */
  FMOE_ERR_DEVICE_TIMEOUT = 6, /* a kernel's bounded wait ran out (reported by fmoe_workspace_check) */
  FMOE_ERR_DEVICE_BOUNDS = 7   /* a device-side bounds check failed (debug build only; fmoe_workspace_check) */
} fmoe_status;

/* A bank of expert records in device memory.
 * bits: 2, 4 or 8.  group_size: 64 or 128 (128 needs hidden and inter >= 1024).
 * hidden (H), inter (I): model width and expert intermediate width.
 * reserved: set to 0 (it spells out the padding before `base`, so that the layout is
 * the same under every compiler).
 * base: record 0 (16-byte aligned); stride: bytes between records (multiple of 16).
 * off[9]: byte offsets inside a record of gate.qw, gate.scale, gate.bias,
 *         up.qw, up.scale, up.bias, down.qw, down.scale, down.bias (multiples of 16). */
typedef struct {
  int32_t bits;
  int32_t group_size;
  int32_t hidden;
  int32_t inter;
  int32_t num_experts;
  int32_t reserved;
  const void* base;
  int64_t stride;
  int64_t off[9];
} fmoe_bank;

/* One MoE layer.
 * routed: E = routed.num_experts experts.  shared: the always-on expert (record 0 used).
 * w_router: bf16 [E][H].  router_bias: fp32 [E] added to the logits, or NULL.
 * w_shared_gate: bf16 [H]; the shared expert's output is scaled by sigmoid(w_shared_gate . x).
 * gamma: fp32 [H] RMSNorm weight; NULL skips the normalisation (x = h).
 * eps: RMSNorm epsilon (1e-6 for the Qwen3.5-397B-A17B shapes).  top_k: K, 1 <= K <= min(E, 32). */
typedef struct {
  fmoe_bank routed;
  fmoe_bank shared;
  const uint16_t* w_router;
  const float* router_bias;
  const uint16_t* w_shared_gate;
  const float* gamma;
  float eps;
  int32_t top_k;
} fmoe_layer;

/* Canonical record layout for (bits, group_size, hidden, inter): writes the
 * record size and the nine sub-array offsets.  Host-only helper. */
fmoe_status fmoe_bank_layout(int bits, int group_size, int hidden, int inter, int64_t* record_bytes, int64_t off[9]);

/* Two-pass RMSNorm ("What is Flash-MoE", section 3: sum of squares, then apply):
 *   y[t][i] = h[t][i] / sqrt(mean_i h[t][i]^2 + eps) * gamma[i].
 * h, y: fp32 [T][H] (y may equal h).  gamma: fp32 [H] or NULL for unit weights.
 * T >= 0 (T = 0 enqueues nothing), H >= 1. */
fmoe_status fmoe_rmsnorm(const float* h, const float* gamma, float eps, int T, int H, float* y, fmoe_stream_t stream);

/* Router GEMV + softmax + top-K ("Flash-MoE" wiki summary, per-layer pipeline:
 * routing projection, then softmax and top-K; the pages run the selection on
 * the CPU, here it stays on the GPU):
 *   l[t][e] = sum_i w_router[e][i] x[t][i] (+ logit_bias[e]);  p = softmax_e(l);
 *   idx[t][0..K-1] = the K largest p in descending order, ties to the lower index;
 *   w[t][k] = p[idx[t][k]] / sum_k' p[idx[t][k']].
 * x: fp32 [T][H] (already normalised).  w_router: bf16 [E][H].  logit_bias: fp32 [E] or NULL.
 * idx: int32 [T][K]; w: fp32 [T][K]; probs: fp32 [T][E] or NULL.
 * ws: device workspace of fmoe_router_topk_workspace_size(T, E) bytes, 256-byte
 * aligned, zeroed once before first use (fmoe_workspace_init); every call
 * leaves it ready for the next.  Requirements: H % 128 == 0, 1 <= K <= min(E, 32), E <= 4096. */
fmoe_status fmoe_router_topk(const float* x, const uint16_t* w_router, const float* logit_bias, int T, int H, int E,
                             int K, int32_t* idx, float* w, float* probs, void* ws, size_t ws_bytes,
                             fmoe_stream_t stream);
size_t fmoe_router_topk_workspace_size(int T, int E);

/* One expert's FFN for one token ("What is Flash-MoE", sections 2-3: dequant
 * matvec, fused SwiGLU):
 *   g = Wg x, u = Wu x, a = silu(g) * u with silu(z) = z / (1 + exp(-z)), y = Wd a.
 * bank: the expert bank; expert: record index in [0, num_experts).
 * x: fp32 [H]; y: fp32 [H].  ws: fmoe_expert_ffn_workspace_size(bank) bytes,
 * 256-byte aligned, zeroed once (fmoe_workspace_init).
 * Requirements: bits 2, 4 or 8, group 64 or 128 (see fmoe_bank), H and I each 64 times a power of two,
 * 128 <= H, I <= 8192. */
fmoe_status fmoe_expert_ffn(const fmoe_bank* bank, int expert, const float* x, float* y, void* ws, size_t ws_bytes,
                            fmoe_stream_t stream);
size_t fmoe_expert_ffn_workspace_size(const fmoe_bank* bank);

/* The whole block for T tokens (the MoE section and sections 2-3 of "What is
 * Flash-MoE"; pipeline of the jeongsk wiki summary):
 *   x = RMSNorm(h) (skipped when gamma is NULL); routing as fmoe_router_topk;
 *   sigma = sigmoid(w_shared_gate . x);
 *   out[t] = h[t] + sum_k w[t][k] FFN_{idx[t][k]}(x[t]) + sigma[t] FFN_shared(x[t]).
 * h, out: fp32 [T][H]; out may equal h (in-place residual), no other overlap.
 * topk_idx (int32 [T][K]) and topk_w (fp32 [T][K]) receive the routing, or NULL.
 * ws: fmoe_moe_layer_workspace_size(layer, T) bytes, 256-byte aligned, zeroed
 * once before first use (fmoe_workspace_init); calls on one workspace must be
 * ordered on one stream.  The size for T serves every call of at most T tokens.
 * T >= 8 tokens run expert-grouped (each active expert's rows read once for
 * its token group) when the workspace holds the grouped layout of T tokens
 * (one of fmoe_moe_layer_workspace_size(layer, T') bytes, T' >= T, does),
 * hidden and inter are >= 512 and FMOE_GROUPED is not "0";
 * otherwise token by token, for which the T = 1 size suffices (a smaller
 * workspace gives FMOE_ERR_WORKSPACE).  Requirements: those of fmoe_expert_ffn for both
 * banks (same bits, hidden, inter), 1 <= K <= min(E, 32), E <= 4096,
 * hidden <= 8192, and K + 1 expert slots of the down kernel within its shared
 * memory (K <= 9 at inter 1024, 4-bit; FMOE_ERR_UNSUPPORTED otherwise).
 * T = 0 enqueues nothing. */
fmoe_status fmoe_moe_layer(const fmoe_layer* layer, const float* h, int T, float* out, int32_t* topk_idx,
                           float* topk_w, void* ws, size_t ws_bytes, fmoe_stream_t stream);
size_t fmoe_moe_layer_workspace_size(const fmoe_layer* layer, int T);

/* Bytes of the library's static scratch used by fmoe_moe_layer_static. */
#define FMOE_STATIC_SCRATCH_BYTES 524288

/* fmoe_moe_layer without a workspace argument: the pages have no counterpart
 * (their engine owns all its buffers); this is an interface convenience.
 * Computes what fmoe_moe_layer computes, but its scratch is a fixed device array
 * inside libfmoe.so of FMOE_STATIC_SCRATCH_BYTES (512 KiB) per device, so the call
 * allocates nothing.  Batches of T >= 8 tokens take the expert-grouped kernels only
 * when their grouped layout fits the scratch (small layers); otherwise, e.g. for the
 * Qwen3.5-397B-A17B shapes, they run token by token, which reads every selected
 * expert's rows once per token.  It serves callers that
 * cannot hand over a workspace: a plain-C or FFI host that keeps no device
 * allocator, or an engine whose memory planner has reserved the whole device.
 * Arguments as fmoe_moe_layer, plus:
 *   dev_err: device int (caller-owned, 4-byte aligned) that the kernels set
 *            non-zero when a bounded wait gives up or an expert index lies
 *            outside the bank; it must start at zero and is never cleared by
 *            the library.  NULL: such failures are recorded only inside the
 *            static scratch, where no call reports them.
 * The scratch needs no set-up: it is zero when the library's module loads on
 * a device, and the first kernel of every token clears the counters the later
 * ones use.  A call after which dev_err is non-zero has invalid outputs; the
 * scratch itself needs no reset, since the next call clears its counters again.  Its address is
 * looked up (cudaGetSymbolAddress) on the first call on each device; make that
 * first call outside any CUDA stream capture.
 * One scratch per device is shared by every caller of this function: two calls
 * on the same device whose kernels may overlap (different streams without an
 * ordering between them, or different host threads) race on it and give wrong
 * results.  Order all calls on a device on one stream.
 * A layer whose per-token scratch (fmoe_moe_layer_workspace_size(layer, 1))
 * exceeds FMOE_STATIC_SCRATCH_BYTES is rejected with FMOE_ERR_WORKSPACE before
 * anything is enqueued.  Every shape the other requirements admit needs at
 * most 435,968 bytes (the Qwen3.5-397B-A17B layer 214,016), so today that
 * check only guards against shapes later versions may admit. */
fmoe_status fmoe_moe_layer_static(const fmoe_layer* layer, const float* h, int T, float* out, int32_t* topk_idx,
                                  float* topk_w, int* dev_err, fmoe_stream_t stream);

/* The block with the routing given by the caller instead of selected from the logits
 * (for a routing recorded earlier or made elsewhere; the pages' engine selects on the
 * CPU and hands the choice to the GPU, "Flash-MoE" wiki summary, per-layer pipeline):
 *   out[t] = h[t] + sum_k topk_w[t][k] FFN_{topk_idx[t][k]}(x[t]) + sigma[t] FFN_shared(x[t]),
 * with x = RMSNorm(h) and sigma = sigmoid(w_shared_gate . x) as in fmoe_moe_layer; the
 * weights are used as given (not renormalised).
 * topk_idx: device int32 [T][K]; topk_w: device fp32 [T][K] (4-byte aligned).  Other
 * arguments and requirements as fmoe_moe_layer (token by token; the T = 1 workspace
 * size suffices).  An index outside [0, num_experts) is not checked on the host: the
 * kernels replace it by expert 0 and record it, and fmoe_workspace_check then returns
 * FMOE_ERR_INVALID_ARG. */
fmoe_status fmoe_moe_layer_routed(const fmoe_layer* layer, const float* h, int T, const int32_t* topk_idx,
                                  const float* topk_w, float* out, void* ws, size_t ws_bytes, fmoe_stream_t stream);

/* Stream-ordered, bounded wait: work enqueued on `stream` after this call starts once
 * *flag == value (a device word, or mapped host memory, set by another stream, the host
 * or a peer), or once limit_ns (1 ns .. 60 s) have passed; in that case the workspace's
 * error word records it and fmoe_workspace_check returns FMOE_ERR_DEVICE_TIMEOUT.  The
 * kernels of this library bound every wait the same way.  ws: any workspace of this
 * library, initialised by fmoe_workspace_init (its control words are used; every size
 * query of this library returns at least their size).  flag: 4-byte aligned. */
fmoe_status fmoe_wait_flag(const uint32_t* flag, uint32_t value, int64_t limit_ns, void* ws, fmoe_stream_t stream);

/* A stack of L layers applied in order, each block's output feeding the next
 * (the 60-layer decode loop of the jeongsk wiki summary, without the attention
 * layers): h_0 = h, h_{l+1} = block_l(h_l), out = h_L.  out may equal h.
 * ws: max over l of fmoe_moe_layer_workspace_size(&layers[l], T) bytes. */
fmoe_status fmoe_moe_stack(const fmoe_layer* layers, int L, const float* h, int T, float* out, void* ws,
                           size_t ws_bytes, fmoe_stream_t stream);

/* Tracing hook for per-kernel timing: the next fmoe_moe_layer call made by
 * this host thread records the caller's CUDA events (cudaEvent_t handles) on
 * its stream: events[0] before the router kernel, events[1] after it,
 * events[2] after the gate/up kernel, events[3] after the down/combine kernel
 * (first token only when T > 1).  On the expert-grouped path (T >= 8) the
 * events bracket the whole batch: [0] before the router, [1] after the
 * selection and sort, [2] after the grouped gate/up kernel, [3] after the
 * combine.  n must be 4; events = NULL cancels. */
fmoe_status fmoe_trace_next_layer(void* const* events, int n);

/* Zeroes the workspace's control words (enqueued on `stream`).  Call once after
 * allocating a workspace, before its first use. */
fmoe_status fmoe_workspace_init(void* ws, size_t ws_bytes, fmoe_stream_t stream);

/* Synchronises `stream`, then reads and clears the workspace's device error
 * word: FMOE_OK, or FMOE_ERR_DEVICE_TIMEOUT if a kernel gave up a bounded wait. */
fmoe_status fmoe_workspace_check(void* ws, fmoe_stream_t stream);

/* Message for the last non-OK status returned to this host thread ("" if none). */
const char* fmoe_last_error(void);

/* Static name of a status code. */
const char* fmoe_status_string(fmoe_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
int fmoe_version(void);

/* 1 if this library is the debug build, whose kernels check their indices, row ranges
 * and copies against their buffers and report a failure as FMOE_ERR_DEVICE_BOUNDS
 * (libfmoe_debug.so, built beside libfmoe.so); 0 otherwise. */
int fmoe_debug_bounds(void);

#ifdef __cplusplus
}
#endif

#endif /* FMOE_H */
