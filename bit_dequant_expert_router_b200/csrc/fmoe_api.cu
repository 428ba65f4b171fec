// fmoe_api.cu -- the C ABI of libfmoe.so: argument validation, workspace
// layout and kernel dispatch.  Every entry point validates on the host before
// enqueuing anything and reports through fmoe_status (never aborts).
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "fmoe.h"
#include "fmoe_cache.h"
#include "fmoe_gdn.h"
#include "fmoe_internal.h"

namespace fmoe {

cudaError_t launch_xq(const float* x, int H, int bits, uint8_t* limbs, float2* cs, cudaStream_t s);

namespace {

thread_local char g_msg[512] = "";
thread_local cudaEvent_t g_trace[4] = {nullptr, nullptr, nullptr, nullptr};
thread_local bool g_trace_on = false;

fmoe_status fail(fmoe_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

fmoe_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FMOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr size_t kAlign = 256;
size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
bool pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

// Workspace regions (byte offsets), in this order.
struct WsLayout {
  size_t ctrl, xq_limbs, xq_cs, logits, route_idx, route_w, act, act_limbs, act_cs, grp_cnt, xlog, xact, xh, total;
};

// Workspace: control words, digits of x (3 bytes per element + one float2 per
// chunk of at most 32 elements), router logits [T][E+1], the routing [T][K]
// and weights [T][K+1], the activations of the K+1 expert slots with their
// digits, per-group completion counters, and the single-kernel path's
// epoch-tagged exchange words (8 bytes each, two copies): logits [E+1],
// activations [(K+1) I] and a stacked layer's output [H].
WsLayout layout(int H, int E, int K, int I, int T) {
  WsLayout L;
  const size_t ne = (size_t)K + 1;
  L.ctrl = 0;
  L.xq_limbs = up(sizeof(WsControl));
  L.xq_cs = L.xq_limbs + up((size_t)T * 3 * H);
  L.logits = L.xq_cs + up((size_t)T * (H / 32) * 8);
  L.route_idx = L.logits + up((size_t)T * (E + 1) * 4);
  L.route_w = L.route_idx + up((size_t)T * ne * 4);
  L.act = L.route_w + up((size_t)T * ne * 4);
  L.act_limbs = L.act + up(ne * I * 4);
  L.act_cs = L.act_limbs + up(ne * 3 * I);
  L.grp_cnt = L.act_cs + up(ne * (I / 32) * 8);
  L.xlog = L.grp_cnt + up(ne * (I / 64 > 0 ? I / 64 : 1) * 4);
  L.xact = L.xlog + up(2 * (size_t)(E + 1) * 8);
  L.xh = L.xact + up(2 * ne * I * 8);
  L.total = L.xh + up(2 * (size_t)H * 8);
  return L;
}

// Workspace of the expert-grouped path for T tokens: regions in this order,
// placed after the whole per-token layout (whose counters must stay zero
// between calls); the control block is the per-token one at offset 0.
struct GLayout {
  size_t ctrl, logits, xq_limbs, xq_cs, route_idx, route_w, n_active, act_expert, act_off, pair_tok, pair_pos, work,
      act, act_limbs, act_cs, y, x, rt_part, total;
};

GLayout glayout(int H, int E, int K, int I, int T) {
  GLayout L;
  const size_t np = (size_t)T * K, nr = np + T;
  L.ctrl = 0;
  L.logits = layout(H, E, K, I, 1).total;
  L.xq_limbs = L.logits + up((size_t)T * (E + 1) * 4);
  L.xq_cs = L.xq_limbs + up((size_t)T * 3 * H);
  L.route_idx = L.xq_cs + up((size_t)T * (H / 32) * 8);
  L.route_w = L.route_idx + up(np * 4);
  L.n_active = L.route_w + up((size_t)T * (K + 1) * 4);
  L.act_expert = L.n_active + up(8);
  L.act_off = L.act_expert + up(np * 4);
  L.pair_tok = L.act_off + up((np + 1) * 4);
  L.pair_pos = L.pair_tok + up(np * 4);
  L.work = L.pair_pos + up(np * 4);
  L.act = L.work + up(nr * sizeof(UnitDesc));
  L.act_limbs = L.act + up(nr * I * 4);
  L.act_cs = L.act_limbs + up(nr * 3 * I);
  L.y = L.act_cs + up(nr * (I / 32) * 8);
  L.x = L.y + up(nr * H * 4);
  L.rt_part = L.x + up((size_t)T * H * 4);
  L.total = L.rt_part + up((size_t)grouped_router_split(H, E, T) * (E + 1) * T * 4);
  return L;
}

constexpr int kGroupedMinT = 8;  // batches at least this large take the expert-grouped path

fmoe_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return fail(FMOE_ERR_WORKSPACE, "workspace is NULL");
  if (((uintptr_t)ws & (kAlign - 1)) != 0) return fail(FMOE_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  if (ws_bytes < need) return fail(FMOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  return FMOE_OK;
}

fmoe_status check_bank(const fmoe_bank* b, const char* name) {
  if (!b) return fail(FMOE_ERR_INVALID_ARG, "%s bank is NULL", name);
  if (!b->base) return fail(FMOE_ERR_INVALID_ARG, "%s bank base is NULL", name);
  if (b->bits != 2 && b->bits != 4 && b->bits != 8)
    return fail(FMOE_ERR_UNSUPPORTED, "%s bank: bits %d (2, 4 or 8)", name, b->bits);
  if (b->group_size != kGroup && b->group_size != 2 * kGroup)
    return fail(FMOE_ERR_UNSUPPORTED, "%s bank: group_size %d (64 or 128)", name, b->group_size);
  if (b->group_size == 2 * kGroup && (b->hidden < 1024 || b->inter < 1024))
    return fail(FMOE_ERR_UNSUPPORTED, "%s bank: groups of 128 need hidden and inter of at least 1024", name);
  if (b->num_experts < 1) return fail(FMOE_ERR_INVALID_ARG, "%s bank: num_experts %d", name, b->num_experts);
  const int H = b->hidden, I = b->inter;
  if (H < 128 || I < 128 || H % 128 || I % 128)
    return fail(FMOE_ERR_UNSUPPORTED, "%s bank: hidden %d and inter %d must be positive multiples of 128", name, H, I);
  if (!pow2(H / 64) || H > 8192 || !pow2(I / 64) || I > 8192)
    return fail(FMOE_ERR_UNSUPPORTED, "%s bank: hidden %d and inter %d must be 64 times a power of two, at most 8192",
                name, H, I);
  if (!expert_shapes_supported(b->bits, H, I, 1))
    return fail(FMOE_ERR_UNSUPPORTED, "%s bank: shapes exceed the kernels' shared memory", name);
  if (!aligned16(b->base) || (b->stride & 15)) return fail(FMOE_ERR_ALIGNMENT, "%s bank: base/stride not 16-byte aligned", name);
  if (b->num_experts > 1 && b->stride <= 0) return fail(FMOE_ERR_INVALID_ARG, "%s bank: stride %lld", name, (long long)b->stride);
  for (int i = 0; i < 9; ++i)
    if (b->off[i] < 0 || (b->off[i] & 15)) return fail(FMOE_ERR_ALIGNMENT, "%s bank: off[%d] not 16-byte aligned", name, i);
  return FMOE_OK;
}

BankRef ref(const fmoe_bank& b) {
  BankRef r;
  r.base = static_cast<const uint8_t*>(b.base);
  r.stride = b.stride;
  for (int i = 0; i < 9; ++i) r.off[i] = b.off[i];
  r.num_experts = b.num_experts;
  return r;
}

cudaStream_t cs(fmoe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// Records a trace event; under stream capture it becomes an event-record node
// of the graph (an external event), so the replay timestamps it.
cudaError_t trace_record(cudaEvent_t ev, cudaStream_t s) {
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &st);
  if (e != cudaSuccess) return e;
  return cudaEventRecordWithFlags(ev, s, st == cudaStreamCaptureStatusActive ? cudaEventRecordExternal
                                                                              : cudaEventRecordDefault);
}

}  // namespace

int num_sms() {
  static std::atomic<int> cache[64] = {};  // per device; calls may come from several host threads
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// L2 prefetch of the routed experts' down matrices from the gate/up kernel: 1 as soon as
// the routing is known, 2 once a CTA's last chunk of gate/up rows has landed (so that it
// does not share DRAM with the gate/up stream), 0 not at all (FMOE_PREFETCH; default 0:
// measured fastest, the down kernel requests its rows itself before its dependency wait).
int prefetch_down() {
  static const int mode = [] {  // read once (thread-safe static initialisation)
    const char* v = getenv("FMOE_PREFETCH");
    return (v && v[0] == '1') ? 1 : (v && v[0] == '2') ? 2 : 0;
  }();
  return mode;
}

// Dependent launch between the block's kernels; FMOE_PDL=0 in the environment turns it off.
bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("FMOE_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

}  // namespace fmoe

using namespace fmoe;

extern "C" {

int fmoe_version(void) { return 100; }

int fmoe_debug_bounds(void) {
#ifdef FMOE_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

const char* fmoe_last_error(void) { return g_msg; }

const char* fmoe_status_string(fmoe_status s) {
  switch (s) {
    case FMOE_OK: return "FMOE_OK";
    case FMOE_ERR_INVALID_ARG: return "FMOE_ERR_INVALID_ARG";
    case FMOE_ERR_ALIGNMENT: return "FMOE_ERR_ALIGNMENT";
    case FMOE_ERR_UNSUPPORTED: return "FMOE_ERR_UNSUPPORTED";
    case FMOE_ERR_WORKSPACE: return "FMOE_ERR_WORKSPACE";
    case FMOE_ERR_CUDA: return "FMOE_ERR_CUDA";
    case FMOE_ERR_DEVICE_TIMEOUT: return "FMOE_ERR_DEVICE_TIMEOUT";
    case FMOE_ERR_DEVICE_BOUNDS: return "FMOE_ERR_DEVICE_BOUNDS";
  }
  return "unknown fmoe_status";
}

fmoe_status fmoe_bank_layout(int bits, int group_size, int hidden, int inter, int64_t* record_bytes, int64_t off[9]) {
  if (!record_bytes || !off) return fail(FMOE_ERR_INVALID_ARG, "NULL output");
  if (bits != 2 && bits != 4 && bits != 8) return fail(FMOE_ERR_UNSUPPORTED, "bits %d", bits);
  if (group_size != kGroup && group_size != 2 * kGroup) return fail(FMOE_ERR_UNSUPPORTED, "group_size %d", group_size);
  if (hidden <= 0 || inter <= 0 || hidden % group_size || inter % group_size)
    return fail(FMOE_ERR_INVALID_ARG, "hidden %d / inter %d", hidden, inter);
  const int64_t dims[3][2] = {{inter, hidden}, {inter, hidden}, {hidden, inter}};
  int64_t pos = 0;
  for (int m = 0; m < 3; ++m) {
    const int64_t rows = dims[m][0], cols = dims[m][1];
    const int64_t sizes[3] = {rows * cols * bits / 8, rows * (cols / group_size) * 2, rows * (cols / group_size) * 2};
    for (int k = 0; k < 3; ++k) {
      off[3 * m + k] = pos;
      pos = (pos + sizes[k] + 15) / 16 * 16;
    }
  }
  *record_bytes = pos;
  return FMOE_OK;
}

fmoe_status fmoe_rmsnorm(const float* h, const float* gamma, float eps, int T, int H, float* y, fmoe_stream_t stream) {
  if (T < 0 || H < 1) return fail(FMOE_ERR_INVALID_ARG, "T %d, H %d", T, H);
  if (T == 0) return FMOE_OK;
  if (!h || !y) return fail(FMOE_ERR_INVALID_ARG, "h or y is NULL");
  if (!(eps >= 0.0f)) return fail(FMOE_ERR_INVALID_ARG, "eps %g", (double)eps);
  cudaError_t e = launch_rmsnorm(h, gamma, eps, T, H, y, cs(stream));
  return e == cudaSuccess ? FMOE_OK : cuda_fail(e, "rmsnorm launch");
}

fmoe_status fmoe_gdn_step(float* state, const float* q, const float* k, const float* v, const float* alpha,
                          const float* beta, float* o, int n, int dk, int dv, unsigned flags, fmoe_stream_t stream) {
  if (n < 0 || dv < 1) return fail(FMOE_ERR_INVALID_ARG, "n %d, dv %d", n, dv);
  if (flags & ~FMOE_GDN_STATE_EARLY) return fail(FMOE_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (!gdn_shape_supported(dk)) return fail(FMOE_ERR_UNSUPPORTED, "dk %d (128, 256, 384 or 512)", dk);
  if ((long long)n * dv > 0x7fffffffLL) return fail(FMOE_ERR_UNSUPPORTED, "n * dv = %lld rows", (long long)n * dv);
  if (n == 0) return FMOE_OK;
  if (!state || !q || !k || !v || !alpha || !beta || !o)
    return fail(FMOE_ERR_INVALID_ARG, "state, q, k, v, alpha, beta and o must be non-NULL");
  if (!aligned16(state) || !aligned16(q) || !aligned16(k))
    return fail(FMOE_ERR_ALIGNMENT, "state, q and k must be 16-byte aligned");
  if ((((uintptr_t)v | (uintptr_t)alpha | (uintptr_t)beta | (uintptr_t)o) & 3u) != 0)
    return fail(FMOE_ERR_ALIGNMENT, "v, alpha, beta and o must be 4-byte aligned");
  GdnParams p{};
  p.state = state;
  p.q = q;
  p.k = k;
  p.v = v;
  p.alpha = alpha;
  p.beta = beta;
  p.o = o;
  p.rows = n * dv;
  p.dk = dk;
  p.dv = dv;
  p.early = (flags & FMOE_GDN_STATE_EARLY) ? 1 : 0;
  cudaError_t e = launch_gdn_step(p, pdl_enabled(), cs(stream));
  return e == cudaSuccess ? FMOE_OK : cuda_fail(e, "gdn step launch");
}

// The per-token path: three kernels (router, gate/up, down) unless FMOE_TOKEN_KERNELS=2
// selects the two-kernel path (router, fused expert kernel).
static bool three_kernel_path() {
  const char* v = getenv("FMOE_TOKEN_KERNELS");
  return !(v && v[0] == '2');
}

size_t fmoe_router_topk_workspace_size(int T, int E) {
  if (T < 1) T = 1;
  if (T > 1024) T = 1024;
  return layout(0, E, 32, 0, T).total;
}

fmoe_status fmoe_router_topk(const float* x, const uint16_t* w_router, const float* logit_bias, int T, int H, int E,
                             int K, int32_t* idx, float* w, float* probs, void* ws, size_t ws_bytes,
                             fmoe_stream_t stream) {
  if (T < 0) return fail(FMOE_ERR_INVALID_ARG, "T %d", T);
  if (H < 128 || H % 128 || H > 12288) return fail(FMOE_ERR_UNSUPPORTED, "H %d: a multiple of 128 in [128, 12288]", H);
  if (E < 1 || E > 4096) return fail(FMOE_ERR_UNSUPPORTED, "E %d (1..4096)", E);
  if (K < 1 || K > E || K > 32) return fail(FMOE_ERR_INVALID_ARG, "K %d (1..min(E, 32))", K);
  if (T == 0) return FMOE_OK;
  if (!x || !w_router || !idx || !w) return fail(FMOE_ERR_INVALID_ARG, "x, w_router, idx or w is NULL");
  if (!aligned16(x) || !aligned16(w_router)) return fail(FMOE_ERR_ALIGNMENT, "x and w_router must be 16-byte aligned");
  const int Tc = T > 1024 ? 1024 : T;
  const WsLayout L = layout(0, E, 32, 0, Tc);
  fmoe_status st = check_ws(ws, ws_bytes, L.total);
  if (st != FMOE_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(ws);
  WsControl* ctrl = reinterpret_cast<WsControl*>(base + L.ctrl);
  for (int t0 = 0; t0 < T; t0 += 1024) {
    const int n = T - t0 < 1024 ? T - t0 : 1024;
    RouterParams p{};
    p.h = x + (size_t)t0 * H;
    p.norm = 0;
    p.w_router = w_router;
    p.bias = logit_bias;
    p.w_sgate = nullptr;
    p.T = n;
    p.H = H;
    p.E = E;
    p.logits = reinterpret_cast<float*>(base + L.logits);
    p.err = &ctrl->err;
    cudaError_t e = launch_router(p, 0, false, cs(stream));
    if (e != cudaSuccess) return cuda_fail(e, "router launch");
    TopkParams q{};
    q.logits = p.logits;
    q.T = n;
    q.E = E;
    q.K = K;
    q.idx = idx + (size_t)t0 * K;
    q.w = w + (size_t)t0 * K;
    q.probs = probs ? probs + (size_t)t0 * E : nullptr;
    if ((e = launch_topk(q, cs(stream))) != cudaSuccess) return cuda_fail(e, "top-K launch");
  }
  return FMOE_OK;
}

size_t fmoe_expert_ffn_workspace_size(const fmoe_bank* bank) {
  if (!bank) return 0;
  return layout(bank->hidden, 0, 1, bank->inter, 1).total;
}

fmoe_status fmoe_expert_ffn(const fmoe_bank* bank, int expert, const float* x, float* y, void* ws, size_t ws_bytes,
                            fmoe_stream_t stream) {
  fmoe_status st = check_bank(bank, "expert");
  if (st != FMOE_OK) return st;
  if (expert < 0 || expert >= bank->num_experts)
    return fail(FMOE_ERR_INVALID_ARG, "expert %d outside [0, %d)", expert, bank->num_experts);
  if (!x || !y) return fail(FMOE_ERR_INVALID_ARG, "x or y is NULL");
  if (!aligned16(x)) return fail(FMOE_ERR_ALIGNMENT, "x must be 16-byte aligned");
  const WsLayout L = layout(bank->hidden, 0, 1, bank->inter, 1);
  if ((st = check_ws(ws, ws_bytes, L.total)) != FMOE_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(ws);
  WsControl* ctrl = reinterpret_cast<WsControl*>(base + L.ctrl);
  const int bits = bank->bits;
  if (!three_kernel_path() && bank->group_size == kGroup &&
      token_path_supported(bits, bank->hidden, bank->inter, 1, 0, ref(*bank), ref(*bank))) {
    const bool pdl = pdl_enabled();
    cudaError_t e = launch_tok_xq(x, bank->hidden, bits, base + L.xq_limbs, reinterpret_cast<float2*>(base + L.xq_cs),
                                  &ctrl->tok_count, pdl, cs(stream));
    if (e != cudaSuccess) return cuda_fail(e, "digits launch");
    TokExpertParams p{};
    p.routed = ref(*bank);
    p.shared = ref(*bank);
    p.fixed_expert = expert;
    p.E = bank->num_experts;
    p.K = 1;
    p.has_shared = 0;
    p.H = bank->hidden;
    p.I = bank->inter;
    p.xq_limbs = base + L.xq_limbs;
    p.xq_cs = reinterpret_cast<const float2*>(base + L.xq_cs);
    p.act = reinterpret_cast<float*>(base + L.act);
    p.count = &ctrl->tok_count;
    p.out = y;
    p.err = &ctrl->err;
    if ((e = launch_tok_expert(p, bits, pdl, cs(stream))) != cudaSuccess) return cuda_fail(e, "expert launch");
    return FMOE_OK;
  }
  cudaError_t e = launch_xq(x, bank->hidden, bits, base + L.xq_limbs, reinterpret_cast<float2*>(base + L.xq_cs),
                            cs(stream));
  if (e != cudaSuccess) return cuda_fail(e, "digits launch");
  ExpertParams p{};
  p.routed = ref(*bank);
  p.shared = ref(*bank);
  p.gsh = bank->group_size == 2 * kGroup ? 1 : 0;
  p.route_idx = nullptr;
  p.route_w = nullptr;
  p.E = bank->num_experts;
  p.fixed_expert = expert;
  p.K = 1;
  p.has_shared = 0;
  p.H = bank->hidden;
  p.I = bank->inter;
  p.xq_limbs = reinterpret_cast<const uint32_t*>(base + L.xq_limbs);
  p.xq_cs = reinterpret_cast<const float2*>(base + L.xq_cs);
  p.act = reinterpret_cast<float*>(base + L.act);
  p.act_limbs = base + L.act_limbs;
  p.act_cs = reinterpret_cast<float2*>(base + L.act_cs);
  p.grp_cnt = reinterpret_cast<unsigned int*>(base + L.grp_cnt);
  p.resid = nullptr;
  p.out = y;
  p.err = &ctrl->err;
  const bool pdl = pdl_enabled();
  if ((e = launch_gateup(p, bits, pdl, cs(stream))) != cudaSuccess) return cuda_fail(e, "gate/up launch");
  if ((e = launch_down(p, bits, pdl, cs(stream))) != cudaSuccess) return cuda_fail(e, "down launch");
  return FMOE_OK;
}

static fmoe_status check_layer(const fmoe_layer* layer) {
  if (!layer) return fail(FMOE_ERR_INVALID_ARG, "layer is NULL");
  fmoe_status st = check_bank(&layer->routed, "routed");
  if (st != FMOE_OK) return st;
  if ((st = check_bank(&layer->shared, "shared")) != FMOE_OK) return st;
  const fmoe_bank &r = layer->routed, &s = layer->shared;
  if (r.bits != s.bits || r.hidden != s.hidden || r.inter != s.inter || r.group_size != s.group_size)
    return fail(FMOE_ERR_UNSUPPORTED, "routed and shared banks must share bits, group size, hidden and inter");
  if (!layer->w_router || !layer->w_shared_gate) return fail(FMOE_ERR_INVALID_ARG, "w_router or w_shared_gate is NULL");
  if (!aligned16(layer->w_router) || !aligned16(layer->w_shared_gate))
    return fail(FMOE_ERR_ALIGNMENT, "w_router and w_shared_gate must be 16-byte aligned");
  const int E = r.num_experts, K = layer->top_k;
  if (E > 4096) return fail(FMOE_ERR_UNSUPPORTED, "E %d > 4096", E);
  if (r.hidden > 12288) return fail(FMOE_ERR_UNSUPPORTED, "hidden %d > 12288", r.hidden);
  if (K < 1 || K > E || K > 32) return fail(FMOE_ERR_INVALID_ARG, "top_k %d (1..min(E, 32))", K);
  if (!expert_shapes_supported(r.bits, r.hidden, r.inter, K + 1))
    return fail(FMOE_ERR_UNSUPPORTED, "top_k %d with inter %d at %d bits exceeds the down kernel's shared memory", K,
                r.inter, r.bits);
  if (!(layer->eps >= 0.0f)) return fail(FMOE_ERR_INVALID_ARG, "eps %g", (double)layer->eps);
  return FMOE_OK;
}

size_t fmoe_moe_layer_workspace_size(const fmoe_layer* layer, int T) {
  if (!layer) return 0;
  const int H = layer->routed.hidden, E = layer->routed.num_experts, K = layer->top_k, I = layer->routed.inter;
  size_t need = layout(H, E, K, I, 1).total;
  // The grouped layout is not monotone in T (the router's split of H shrinks as token
  // tiles are added), so take its largest size over every batch of at most T tokens:
  // a workspace sized for T then takes the grouped path for any smaller batch too.
  // Once the split is down to 1 it stays there, and the size only grows with t.
  if (K >= 1 && E >= 1 && H > 0 && I > 0)
    for (int t = kGroupedMinT; t <= T; ++t) {
      const size_t g = glayout(H, E, K, I, t).total;
      need = g > need ? g : need;
      if (t < T && grouped_router_split(H, E, t) == 1) t = T - 1;
    }
  return need;
}

static fmoe_status layer_token_3k(const fmoe_layer* layer, const float* h, float* out, int32_t* idx_out, float* w_out,
                                  uint8_t* base, const WsLayout& L, cudaStream_t s, int* err_word,
                                  const int32_t* given_idx = nullptr, const float* given_w = nullptr,
                                  const CacheParams* cache = nullptr);

// One token through the block: router kernel (RMSNorm, logits, digits of x), then
// the expert kernel (top-K, gate/up + SwiGLU, down + combine + residual).
// err_word: where the kernels report a failed bounded wait; NULL means the workspace's own error word.
static fmoe_status layer_token(const fmoe_layer* layer, const float* h, float* out, int32_t* idx_out, float* w_out,
                               uint8_t* base, const WsLayout& L, cudaStream_t s, int* err_word = nullptr) {
  const fmoe_bank& r = layer->routed;
  if (three_kernel_path() || r.group_size != kGroup ||
      !token_path_supported(r.bits, r.hidden, r.inter, layer->top_k, 1, ref(r), ref(layer->shared)))
    return layer_token_3k(layer, h, out, idx_out, w_out, base, L, s, err_word);
  const int H = r.hidden, E = r.num_experts, K = layer->top_k, I = r.inter, bits = r.bits;
  WsControl* ctrl = reinterpret_cast<WsControl*>(base + L.ctrl);
  TokRouterParams rp{};
  rp.h = h;
  rp.gamma = layer->gamma;
  rp.eps = layer->eps;
  rp.norm = layer->gamma != nullptr;
  rp.w_router = layer->w_router;
  rp.bias = layer->router_bias;
  rp.w_sgate = layer->w_shared_gate;
  rp.H = H;
  rp.E = E;
  rp.row0 = 0;
  rp.xq_limbs = base + L.xq_limbs;
  rp.xq_cs = reinterpret_cast<float2*>(base + L.xq_cs);
  rp.logits = reinterpret_cast<float*>(base + L.logits);
  rp.count = &ctrl->tok_count;
  rp.err = err_word ? err_word : &ctrl->err;
  const bool trace = g_trace_on;
  g_trace_on = false;
  const bool pdl = pdl_enabled() && !trace;
  cudaError_t e;
  if (trace && (e = trace_record(g_trace[0], s)) != cudaSuccess) return cuda_fail(e, "trace event");
  if ((e = launch_tok_router(rp, bits, pdl, s)) != cudaSuccess) return cuda_fail(e, "router launch");
  if (trace && (e = trace_record(g_trace[1], s)) != cudaSuccess) return cuda_fail(e, "trace event");
  TokExpertParams p{};
  p.routed = ref(r);
  p.shared = ref(layer->shared);
  p.logits = rp.logits;
  p.idx_out = idx_out;
  p.w_out = w_out;
  p.E = E;
  p.K = K;
  p.has_shared = 1;
  p.H = H;
  p.I = I;
  p.xq_limbs = base + L.xq_limbs;
  p.xq_cs = reinterpret_cast<const float2*>(base + L.xq_cs);
  p.act = reinterpret_cast<float*>(base + L.act);
  p.count = &ctrl->tok_count;
  p.resid = h;
  p.out = out;
  p.err = rp.err;
  if ((e = launch_tok_expert(p, bits, pdl, s)) != cudaSuccess) return cuda_fail(e, "expert launch");
  if (trace && (e = trace_record(g_trace[2], s)) != cudaSuccess) return cuda_fail(e, "trace event");
  if (trace && (e = trace_record(g_trace[3], s)) != cudaSuccess) return cuda_fail(e, "trace event");
  return FMOE_OK;
}

// given_idx / given_w ([K] each, device): the routing given by the caller instead of the
// top-K of the logits (the router still runs, for x, its digits and the shared gate).
// cache: the routed experts sit behind an expert cache; the router's last CTA selects the
// top-K, one cache lookup maps them to slots, and the expert kernels read the slots with
// that routing (layer->routed then describes the slots).
static fmoe_status layer_token_3k(const fmoe_layer* layer, const float* h, float* out, int32_t* idx_out, float* w_out,
                                  uint8_t* base, const WsLayout& L, cudaStream_t s, int* err_word,
                                  const int32_t* given_idx, const float* given_w, const CacheParams* cache) {
  const fmoe_bank& r = layer->routed;
  const int H = r.hidden, E = cache ? cache->E : r.num_experts, K = layer->top_k, I = r.inter, bits = r.bits;
  WsControl* ctrl = reinterpret_cast<WsControl*>(base + L.ctrl);
  RouterParams rp{};
  rp.h = h;
  rp.gamma = layer->gamma;
  rp.eps = layer->eps;
  rp.norm = layer->gamma != nullptr;
  rp.w_router = layer->w_router;
  rp.bias = layer->router_bias;
  rp.w_sgate = layer->w_shared_gate;
  rp.T = 1;
  rp.H = H;
  rp.E = E;
  rp.xq_limbs = base + L.xq_limbs;
  rp.xq_cs = reinterpret_cast<float2*>(base + L.xq_cs);
  rp.xq_limb_stride = 3LL * H;
  rp.xq_cs_stride = H / 32;
  rp.logits = reinterpret_cast<float*>(base + L.logits);
  rp.top_k = 0;  // the expert kernels select the experts from the logits themselves
  rp.tickets = ctrl->tickets;
  rp.route_ready = &ctrl->route_ready;
  rp.clear = reinterpret_cast<unsigned int*>(base + L.grp_cnt);
  rp.nclear = (K + 1) * (I / 64 > 0 ? I / 64 : 1);
  rp.err = err_word ? err_word : &ctrl->err;
  const bool trace = g_trace_on;
  g_trace_on = false;
  const bool pdl = pdl_enabled() && !trace;
  cudaError_t e;
  if (trace && (e = trace_record(g_trace[0], s)) != cudaSuccess) return cuda_fail(e, "trace event");
  if (cache) {  // the router's last CTA selects; the lookup maps the experts to slots
    rp.top_k = K;
    rp.route_idx = reinterpret_cast<int32_t*>(base + L.route_idx);
    rp.route_w = reinterpret_cast<float*>(base + L.route_w);
    rp.idx_out = idx_out;
    rp.w_out = w_out;
    rp.cache = *cache;
    given_idx = cache_slot_out(*cache);
    given_w = rp.route_w;
  }
  e = launch_router(rp, bits, pdl, s);
  if (e != cudaSuccess) return cuda_fail(e, "router launch");
  if (cache && (e = launch_cache_copy(*cache, pdl, s)) != cudaSuccess) return cuda_fail(e, "cache copy launch");
  if (trace && (e = trace_record(g_trace[1], s)) != cudaSuccess) return cuda_fail(e, "trace event");
  ExpertParams p{};
  p.routed = ref(r);
  p.shared = ref(layer->shared);
  p.gsh = r.group_size == 2 * kGroup ? 1 : 0;
  p.logits = rp.logits;
  p.idx_out = idx_out;
  p.w_out = w_out;
  p.E = E;
  p.fixed_expert = 0;
  p.K = K;
  p.has_shared = 1;
  p.H = H;
  p.I = I;
  p.xq_limbs = reinterpret_cast<const uint32_t*>(base + L.xq_limbs);
  p.xq_cs = reinterpret_cast<const float2*>(base + L.xq_cs);
  p.act = reinterpret_cast<float*>(base + L.act);
  p.act_limbs = base + L.act_limbs;
  p.act_cs = reinterpret_cast<float2*>(base + L.act_cs);
  p.grp_cnt = reinterpret_cast<unsigned int*>(base + L.grp_cnt);
  p.resid = h;
  p.out = out;
  p.prefetch_down = prefetch_down();
  p.err = rp.err;
  p.rt_idx = reinterpret_cast<int32_t*>(base + L.route_idx);
  p.rt_w = reinterpret_cast<float*>(base + L.route_w);
  p.route_ready = &ctrl->route_ready;  // gate/up CTA 0 sets it once rt_idx / rt_w are written
  if (given_idx) {
    p.logits = nullptr;
    p.route_idx = given_idx;
    p.idx_out = nullptr;
    p.w_out = nullptr;
    p.route_ready = nullptr;
  }
  if ((e = launch_gateup(p, bits, pdl, s)) != cudaSuccess) return cuda_fail(e, "gate/up launch");
  if (trace && (e = trace_record(g_trace[2], s)) != cudaSuccess) return cuda_fail(e, "trace event");
  ExpertParams pd = p;  // the down kernel reads the routing the gate/up kernel wrote
  pd.logits = nullptr;
  pd.route_idx = p.rt_idx;
  pd.route_w = p.rt_w;
  if (given_idx) {  // launched below with the caller's routing
    pd.route_idx = given_idx;
    pd.route_w = given_w;
    pd.sigma_logit = rp.logits + E;
    pd.route_ready = nullptr;
  }
  if ((e = launch_down(pd, bits, pdl, s)) != cudaSuccess) return cuda_fail(e, "down launch");
  if (trace && (e = trace_record(g_trace[3], s)) != cudaSuccess) return cuda_fail(e, "trace event");
  return FMOE_OK;
}

// The single-kernel path (k_fused.cu) when FMOE_FUSED=1 is set in the environment.
static bool fused_enabled() {
  const char* v = getenv("FMOE_FUSED");
  return v && v[0] == '1';
}

static bool same_offsets(const fmoe_bank& a, const fmoe_bank& b) {
  for (int i = 0; i < 9; ++i)
    if (a.off[i] != b.off[i]) return false;
  return true;
}

// Runs layers[0..nl) over T tokens as one launch of the single-kernel path, if
// that path takes these shapes; `taken` tells whether it did.
static fmoe_status run_fused(const fmoe_layer* layers, int nl, const float* h, int T, float* out, int32_t* idx_out,
                             float* w_out, uint8_t* base, const WsLayout& L, cudaStream_t s, int* err_word,
                             bool& taken) {
  taken = false;
  if (!fused_enabled() || nl < 1 || nl > kFusedMaxLayers || layers[0].routed.group_size != kGroup) return FMOE_OK;
  const fmoe_bank& r0 = layers[0].routed;
  for (int l = 0; l < nl; ++l) {
    const fmoe_layer& y = layers[l];
    if (y.routed.bits != r0.bits || y.routed.hidden != r0.hidden || y.routed.inter != r0.inter ||
        y.routed.group_size != r0.group_size ||
        y.routed.num_experts != r0.num_experts || y.top_k != layers[0].top_k || !same_offsets(y.routed, r0) ||
        !same_offsets(y.shared, r0))
      return FMOE_OK;
  }
  const int H = r0.hidden, I = r0.inter, E = r0.num_experts, K = layers[0].top_k;
  const FusedPlan pl = plan_fused(r0.bits, H, I, E, K);
  if (!pl.ok) return FMOE_OK;
  WsControl* ctrl = reinterpret_cast<WsControl*>(base + L.ctrl);
  FusedParams p{};
  for (int l = 0; l < nl; ++l) {
    const fmoe_layer& y = layers[l];
    FusedLayer& f = p.layers[l];
    f.routed = static_cast<const uint8_t*>(y.routed.base);
    f.stride = y.routed.stride;
    f.shared = static_cast<const uint8_t*>(y.shared.base);
    f.w_router = y.w_router;
    f.bias = y.router_bias;
    f.w_sgate = y.w_shared_gate;
    f.gamma = y.gamma;
    f.eps = y.eps;
  }
  for (int i = 0; i < 9; ++i) p.off[i] = r0.off[i];
  p.L = nl;
  p.T = T;
  p.H = H;
  p.I = I;
  p.E = E;
  p.K = K;
  p.h = h;
  p.out = out;
  p.idx_out = idx_out;
  p.w_out = w_out;
  p.xlog = reinterpret_cast<unsigned long long*>(base + L.xlog);
  p.xact = reinterpret_cast<unsigned long long*>(base + L.xact);
  p.xh = reinterpret_cast<unsigned long long*>(base + L.xh);
  p.epoch = &ctrl->epoch;
  p.err = err_word ? err_word : &ctrl->err;
  p.nbuf = pl.nbuf;
  p.chb = pl.chb;
  p.cu = pl.cu;
  p.rt_rows = pl.rt_rows;
  p.ru = pl.ru;
  p.rd = pl.rd;
  p.dn_rows_max = pl.dn_rows_max;
  p.dn_slot_bytes = pl.dn_slot_bytes;
  p.dn_off = pl.dn_off;
  p.ring_off = pl.ring_off;
  const bool trace = g_trace_on;
  g_trace_on = false;
  cudaError_t e;
  if (trace && (e = trace_record(g_trace[0], s)) != cudaSuccess) return cuda_fail(e, "trace event");
  if ((e = launch_fused(p, pl, r0.bits, pdl_enabled() && !trace, s)) != cudaSuccess) return cuda_fail(e, "fused launch");
  for (int i = 1; trace && i < 4; ++i)
    if ((e = trace_record(g_trace[i], s)) != cudaSuccess) return cuda_fail(e, "trace event");
  taken = true;
  return FMOE_OK;
}

// The expert-grouped path (k_grouped.cu) for T >= kGroupedMinT tokens, unless
// FMOE_GROUPED=0 is set in the environment, the shapes are outside it, or the
// workspace is too small for it; `taken` tells whether it ran.
static fmoe_status run_grouped(const fmoe_layer* layer, const float* h, int T, float* out, int32_t* idx_out,
                               float* w_out, uint8_t* base, size_t ws_bytes, cudaStream_t s, int* err_word,
                               bool& taken) {
  taken = false;
  const char* v = getenv("FMOE_GROUPED");
  if (T < kGroupedMinT || (v && v[0] == '0')) return FMOE_OK;
  const fmoe_bank& r = layer->routed;
  const int H = r.hidden, E = r.num_experts, K = layer->top_k, I = r.inter, bits = r.bits;
  if (r.group_size != kGroup || !grouped_shapes_supported(bits, H, I, E, K, T) || !same_offsets(r, layer->shared))
    return FMOE_OK;
  const GLayout G = glayout(H, E, K, I, T);
  if (ws_bytes < G.total) return FMOE_OK;
  WsControl* ctrl = reinterpret_cast<WsControl*>(base + G.ctrl);
  int* err = err_word ? err_word : &ctrl->err;
  RouterBatch rb{};
  rb.gamma = layer->gamma;
  rb.eps = layer->eps;
  rb.w_router = layer->w_router;
  rb.w_sgate = layer->w_shared_gate;
  rb.bias = layer->router_bias;
  rb.x = reinterpret_cast<float*>(base + G.x);
  GroupedParams p{};
  p.routed = ref(r);
  p.shared = ref(layer->shared);
  p.T = T;
  p.E = E;
  p.K = K;
  p.H = H;
  p.I = I;
  p.logits = reinterpret_cast<float*>(base + G.logits);
  p.xq_limbs = base + G.xq_limbs;
  p.xq_cs = reinterpret_cast<float2*>(base + G.xq_cs);
  p.route_idx = reinterpret_cast<int32_t*>(base + G.route_idx);
  p.route_w = reinterpret_cast<float*>(base + G.route_w);
  p.idx_out = idx_out;
  p.w_out = w_out;
  p.n_active = reinterpret_cast<int32_t*>(base + G.n_active);
  p.act_expert = reinterpret_cast<int32_t*>(base + G.act_expert);
  p.act_off = reinterpret_cast<int32_t*>(base + G.act_off);
  p.pair_tok = reinterpret_cast<int32_t*>(base + G.pair_tok);
  p.pair_pos = reinterpret_cast<int32_t*>(base + G.pair_pos);
  p.units = reinterpret_cast<UnitDesc*>(base + G.work);
  p.rt_part = reinterpret_cast<float*>(base + G.rt_part);
  p.rt_split = grouped_router_split(H, E, T);
  p.rt_bias = layer->router_bias;
  p.act = reinterpret_cast<float*>(base + G.act);
  p.act_limbs = base + G.act_limbs;
  p.act_cs = reinterpret_cast<float2*>(base + G.act_cs);
  p.y = reinterpret_cast<float*>(base + G.y);
  p.h = h;
  p.out = out;
  p.err = err;
  // with tracing on: events before the router, the gate/up kernel, the activation
  // digits, and after the combine
  const bool trace = g_trace_on;
  g_trace_on = false;
  cudaError_t e;
  if (trace && (e = trace_record(g_trace[0], s)) != cudaSuccess) return cuda_fail(e, "trace event");
  const bool pdl = pdl_enabled() && !trace;
  if ((e = launch_grouped_router(p, rb, bits, pdl, s)) != cudaSuccess)
    return cuda_fail(e, "router launch");
  if ((e = launch_grouped_select(p, pdl, s)) != cudaSuccess) return cuda_fail(e, "select launch");
  if (trace && (e = trace_record(g_trace[1], s)) != cudaSuccess) return cuda_fail(e, "trace event");
  if ((e = launch_grouped_gateup(p, bits, pdl, s)) != cudaSuccess) return cuda_fail(e, "grouped gate/up launch");
  if (trace && (e = trace_record(g_trace[2], s)) != cudaSuccess) return cuda_fail(e, "trace event");
  if ((e = launch_grouped_actq(p, bits, pdl, s)) != cudaSuccess) return cuda_fail(e, "activation digits launch");
  if ((e = launch_grouped_down(p, bits, pdl, s)) != cudaSuccess) return cuda_fail(e, "grouped down launch");
  if ((e = launch_grouped_combine(p, pdl, s)) != cudaSuccess) return cuda_fail(e, "combine launch");
  if (trace && (e = trace_record(g_trace[3], s)) != cudaSuccess) return cuda_fail(e, "trace event");
  taken = true;
  return FMOE_OK;
}

// The block for T tokens of one layer on a checked workspace of ws_bytes.
static fmoe_status moe_layer_impl(const fmoe_layer* layer, const float* h, int T, float* out, int32_t* topk_idx,
                                  float* topk_w, uint8_t* base, size_t ws_bytes, const WsLayout& L, cudaStream_t s,
                                  int* err_word) {
  bool taken = false;
  fmoe_status gst = run_grouped(layer, h, T, out, topk_idx, topk_w, base, ws_bytes, s, err_word, taken);
  if (gst != FMOE_OK || taken) return gst;
  fmoe_status st = run_fused(layer, 1, h, T, out, topk_idx, topk_w, base, L, s, err_word, taken);
  if (st != FMOE_OK || taken) return st;
  const int H = layer->routed.hidden, K = layer->top_k;
  for (int t = 0; t < T; ++t) {
    st = layer_token(layer, h + (size_t)t * H, out + (size_t)t * H, topk_idx ? topk_idx + (size_t)t * K : nullptr,
                     topk_w ? topk_w + (size_t)t * K : nullptr, base, L, s, err_word);
    if (st != FMOE_OK) return st;
  }
  return FMOE_OK;
}

fmoe_status fmoe_moe_layer(const fmoe_layer* layer, const float* h, int T, float* out, int32_t* topk_idx,
                           float* topk_w, void* ws, size_t ws_bytes, fmoe_stream_t stream) {
  fmoe_status st = check_layer(layer);
  if (st != FMOE_OK) return st;
  if (T < 0) return fail(FMOE_ERR_INVALID_ARG, "T %d", T);
  if (T == 0) return FMOE_OK;
  if (!h || !out) return fail(FMOE_ERR_INVALID_ARG, "h or out is NULL");
  if (!aligned16(h) || !aligned16(out)) return fail(FMOE_ERR_ALIGNMENT, "h and out must be 16-byte aligned");
  const int H = layer->routed.hidden, K = layer->top_k;
  const WsLayout L = layout(H, layer->routed.num_experts, K, layer->routed.inter, 1);
  if ((st = check_ws(ws, ws_bytes, L.total)) != FMOE_OK) return st;
  return moe_layer_impl(layer, h, T, out, topk_idx, topk_w, static_cast<uint8_t*>(ws), ws_bytes, L, cs(stream),
                        nullptr);
}

// ---- fmoe_moe_layer_static: the same block with library-owned scratch.
//
// For callers that cannot hand over a workspace: a plain-C or FFI host that
// keeps no device allocator of its own, or an engine whose memory planner has
// already reserved every byte of the device and cannot grow.  The scratch is a
// fixed file-scope device array, so the call allocates nothing.  Static device
// memory starts zeroed when the module loads, which is the state the ticket and
// group counters need; every call returns them to zero.

constexpr size_t kStaticScratchBytes = FMOE_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device, looked up once per device.
static fmoe_status static_scratch(uint8_t** out) {
  static std::mutex mu;
  static uint8_t* cache[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < 64 && cache[dev]) {
    *out = cache[dev];
    return FMOE_OK;
  }
  void* p = nullptr;
  if ((e = cudaGetSymbolAddress(&p, g_static_scratch)) != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
  if (dev >= 0 && dev < 64) cache[dev] = static_cast<uint8_t*>(p);
  *out = static_cast<uint8_t*>(p);
  return FMOE_OK;
}

fmoe_status fmoe_moe_layer_static(const fmoe_layer* layer, const float* h, int T, float* out, int32_t* topk_idx,
                                  float* topk_w, int* dev_err, fmoe_stream_t stream) {
  fmoe_status st = check_layer(layer);
  if (st != FMOE_OK) return st;
  if (T < 0) return fail(FMOE_ERR_INVALID_ARG, "T %d", T);
  if (T == 0) return FMOE_OK;
  if (!h || !out) return fail(FMOE_ERR_INVALID_ARG, "h or out is NULL");
  if (!aligned16(h) || !aligned16(out)) return fail(FMOE_ERR_ALIGNMENT, "h and out must be 16-byte aligned");
  if (dev_err && ((uintptr_t)dev_err & 3u) != 0) return fail(FMOE_ERR_ALIGNMENT, "dev_err must be 4-byte aligned");
  const int H = layer->routed.hidden, K = layer->top_k;
  const WsLayout L = layout(H, layer->routed.num_experts, K, layer->routed.inter, 1);
  if (L.total > kStaticScratchBytes)
    return fail(FMOE_ERR_WORKSPACE,
                "layer needs %zu bytes of scratch, the static scratch holds %zu (use fmoe_moe_layer with a workspace)",
                L.total, kStaticScratchBytes);
  uint8_t* base = nullptr;
  if ((st = static_scratch(&base)) != FMOE_OK) return st;
  return moe_layer_impl(layer, h, T, out, topk_idx, topk_w, base, kStaticScratchBytes, L, cs(stream), dev_err);
}

fmoe_status fmoe_moe_layer_routed(const fmoe_layer* layer, const float* h, int T, const int32_t* topk_idx,
                                  const float* topk_w, float* out, void* ws, size_t ws_bytes, fmoe_stream_t stream) {
  fmoe_status st = check_layer(layer);
  if (st != FMOE_OK) return st;
  if (T < 0) return fail(FMOE_ERR_INVALID_ARG, "T %d", T);
  if (T == 0) return FMOE_OK;
  if (!h || !out || !topk_idx || !topk_w) return fail(FMOE_ERR_INVALID_ARG, "h, out, topk_idx or topk_w is NULL");
  if (!aligned16(h) || !aligned16(out)) return fail(FMOE_ERR_ALIGNMENT, "h and out must be 16-byte aligned");
  if (((uintptr_t)topk_idx & 3u) || ((uintptr_t)topk_w & 3u))
    return fail(FMOE_ERR_ALIGNMENT, "topk_idx and topk_w must be 4-byte aligned");
  const int H = layer->routed.hidden, K = layer->top_k;
  const WsLayout L = layout(H, layer->routed.num_experts, K, layer->routed.inter, 1);
  if ((st = check_ws(ws, ws_bytes, L.total)) != FMOE_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(ws);
  for (int t = 0; t < T; ++t) {
    st = layer_token_3k(layer, h + (size_t)t * H, out + (size_t)t * H, nullptr, nullptr, base, L, cs(stream), nullptr,
                        topk_idx + (size_t)t * K, topk_w + (size_t)t * K);
    if (st != FMOE_OK) return st;
  }
  return FMOE_OK;
}

// ---- expert cache (fmoe_cache.h)

// True if p is pinned host memory that the device reads at the same address.
static bool host_mapped(const void* p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost && a.devicePointer == p;
}

static bool device_memory(const void* p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

static fmoe_status check_cache(const fmoe_expert_cache* c, CacheParams& cp) {
  if (!c) return fail(FMOE_ERR_INVALID_ARG, "cache is NULL");
  if (!c->host_base || !c->slots || !c->state) return fail(FMOE_ERR_INVALID_ARG, "host_base, slots or state is NULL");
  if (c->num_experts < 1 || c->num_experts > (1 << 24) || c->num_slots < 1 || c->num_slots > (1 << 24))
    return fail(FMOE_ERR_INVALID_ARG, "num_experts %d, num_slots %d", c->num_experts, c->num_slots);
  if (c->record_bytes < 16 || (c->record_bytes & 15) || (c->host_stride & 15) || (c->slot_stride & 15) ||
      !aligned16(c->host_base) || !aligned16(c->slots) || !aligned16(c->state))
    return fail(FMOE_ERR_ALIGNMENT, "record_bytes, strides, host_base, slots and state must be multiples of 16");
  if (c->host_stride < c->record_bytes || c->slot_stride < c->record_bytes)
    return fail(FMOE_ERR_INVALID_ARG, "a stride is smaller than record_bytes");
  if (!host_mapped(c->host_base))
    return fail(FMOE_ERR_INVALID_ARG, "host_base is not pinned host memory mapped at the same device address");
  if (!device_memory(c->slots) || !device_memory(c->state))
    return fail(FMOE_ERR_INVALID_ARG, "slots and state must be device memory");
  cp.host = static_cast<const uint8_t*>(c->host_base);
  cp.host_stride = c->host_stride;
  cp.slots = static_cast<uint8_t*>(c->slots);
  cp.slot_stride = c->slot_stride;
  cp.rec = c->record_bytes;
  cp.E = c->num_experts;
  cp.C = c->num_slots;
  cp.state = static_cast<uint8_t*>(c->state);
  return FMOE_OK;
}

size_t fmoe_expert_cache_state_size(int num_experts, int num_slots) {
  if (num_experts < 1 || num_slots < 1) return 0;
  return cache_state_bytes(num_experts, num_slots);
}

fmoe_status fmoe_expert_cache_reset(const fmoe_expert_cache* cache, fmoe_stream_t stream) {
  CacheParams cp{};
  fmoe_status st = check_cache(cache, cp);
  if (st != FMOE_OK) return st;
  cudaError_t e = launch_cache_reset(cp, cs(stream));
  return e == cudaSuccess ? FMOE_OK : cuda_fail(e, "cache reset launch");
}

fmoe_status fmoe_expert_cache_fetch(const fmoe_expert_cache* cache, const int32_t* idx, int K, int32_t* slot,
                                    fmoe_stream_t stream) {
  CacheParams cp{};
  fmoe_status st = check_cache(cache, cp);
  if (st != FMOE_OK) return st;
  if (!idx) return fail(FMOE_ERR_INVALID_ARG, "idx is NULL");
  if (K < 1 || K > kCacheMaxK || K > cp.C) return fail(FMOE_ERR_INVALID_ARG, "K %d (1..min(num_slots, 32))", K);
  if (((uintptr_t)idx & 3u) || ((uintptr_t)slot & 3u)) return fail(FMOE_ERR_ALIGNMENT, "idx and slot must be 4-byte aligned");
  CacheHeader* hd = reinterpret_cast<CacheHeader*>(cp.state);
  cudaError_t e = launch_cache_lookup(cp, idx, K, slot, &hd->err, pdl_enabled(), cs(stream));
  return e == cudaSuccess ? FMOE_OK : cuda_fail(e, "cache lookup launch");
}

fmoe_status fmoe_expert_cache_stats(const fmoe_expert_cache* cache, int64_t* hits, int64_t* misses, int64_t* bytes,
                                    fmoe_stream_t stream) {
  CacheParams cp{};
  fmoe_status st = check_cache(cache, cp);
  if (st != FMOE_OK) return st;
  cudaError_t e = cudaStreamSynchronize(cs(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  CacheHeader hd{};
  if ((e = cudaMemcpy(&hd, cp.state, sizeof(hd), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "cudaMemcpy");
  if (hits) *hits = (int64_t)hd.hits;
  if (misses) *misses = (int64_t)hd.misses;
  if (bytes) *bytes = (int64_t)hd.bytes;
  if (hd.err != 0) {
    const int zero = 0;
    if ((e = cudaMemcpy(&reinterpret_cast<CacheHeader*>(cp.state)->err, &zero, sizeof(int), cudaMemcpyHostToDevice)) !=
        cudaSuccess)
      return cuda_fail(e, "cudaMemcpy");
    if (hd.err == kDevBounds) return fail(FMOE_ERR_DEVICE_BOUNDS, "a device-side bounds check failed");
    return fail(FMOE_ERR_INVALID_ARG, "a lookup met an expert index outside the bank");
  }
  return FMOE_OK;
}

fmoe_status fmoe_moe_layer_cached(const fmoe_layer* layer, const fmoe_expert_cache* cache, const float* h, int T,
                                  float* out, int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                                  fmoe_stream_t stream) {
  if (!layer) return fail(FMOE_ERR_INVALID_ARG, "layer is NULL");
  CacheParams cp{};
  fmoe_status st = check_cache(cache, cp);
  if (st != FMOE_OK) return st;
  if (layer->routed.num_experts != cp.E)
    return fail(FMOE_ERR_INVALID_ARG, "layer E %d differs from the cache's %d", layer->routed.num_experts, cp.E);
  // the routed bank as the expert kernels see it: the cache's slots
  fmoe_layer lc = *layer;
  lc.routed.base = cp.slots;
  lc.routed.stride = cp.slot_stride;
  if ((st = check_layer(&lc)) != FMOE_OK) return st;
  const int H = lc.routed.hidden, I = lc.routed.inter, K = lc.top_k, b = lc.routed.bits;
  if (K > cp.C) return fail(FMOE_ERR_INVALID_ARG, "top_k %d > num_slots %d", K, cp.C);
  const int gs = lc.routed.group_size;
  const int64_t qg = (int64_t)I * H * b / 8, sg = (int64_t)I * (H / gs) * 2, sd = (int64_t)H * (I / gs) * 2;
  const int64_t len[9] = {qg, sg, sg, qg, sg, sg, qg, sd, sd};
  for (int i = 0; i < 9; ++i)
    if (lc.routed.off[i] + len[i] > cp.rec)
      return fail(FMOE_ERR_INVALID_ARG, "record_bytes %lld does not cover sub-array %d", (long long)cp.rec, i);
  lc.routed.num_experts = cp.C;
  if (T < 0) return fail(FMOE_ERR_INVALID_ARG, "T %d", T);
  if (T == 0) return FMOE_OK;
  if (!h || !out) return fail(FMOE_ERR_INVALID_ARG, "h or out is NULL");
  if (!aligned16(h) || !aligned16(out)) return fail(FMOE_ERR_ALIGNMENT, "h and out must be 16-byte aligned");
  const WsLayout L = layout(H, cp.E, K, I, 1);
  if ((st = check_ws(ws, ws_bytes, L.total)) != FMOE_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(ws);
  for (int t = 0; t < T; ++t) {
    st = layer_token_3k(&lc, h + (size_t)t * H, out + (size_t)t * H, topk_idx ? topk_idx + (size_t)t * K : nullptr,
                        topk_w ? topk_w + (size_t)t * K : nullptr, base, L, cs(stream), nullptr, nullptr, nullptr,
                        &cp);
    if (st != FMOE_OK) return st;
  }
  return FMOE_OK;
}

fmoe_status fmoe_wait_flag(const uint32_t* flag, uint32_t value, int64_t limit_ns, void* ws, fmoe_stream_t stream) {
  if (!flag) return fail(FMOE_ERR_INVALID_ARG, "flag is NULL");
  if (((uintptr_t)flag & 3u) != 0) return fail(FMOE_ERR_ALIGNMENT, "flag must be 4-byte aligned");
  if (limit_ns <= 0 || limit_ns > 60000000000LL) return fail(FMOE_ERR_INVALID_ARG, "limit_ns %lld (1 ns .. 60 s)",
                                                             (long long)limit_ns);
  if (!ws) return fail(FMOE_ERR_WORKSPACE, "workspace is NULL");
  if (((uintptr_t)ws & (kAlign - 1)) != 0) return fail(FMOE_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  WsControl* ctrl = static_cast<WsControl*>(ws);
  cudaError_t e = launch_wait_flag(flag, value, (unsigned long long)limit_ns, &ctrl->err, cs(stream));
  return e == cudaSuccess ? FMOE_OK : cuda_fail(e, "wait launch");
}

fmoe_status fmoe_moe_stack(const fmoe_layer* layers, int nl, const float* h, int T, float* out, void* ws,
                           size_t ws_bytes, fmoe_stream_t stream) {
  if (!layers || nl < 1) return fail(FMOE_ERR_INVALID_ARG, "layers NULL or count %d", nl);
  for (int l = 0; l < nl; ++l) {
    fmoe_status st = check_layer(&layers[l]);
    if (st != FMOE_OK) return fail(st, "layer %d: %s", l, g_msg);
    if (layers[l].routed.hidden != layers[0].routed.hidden)
      return fail(FMOE_ERR_INVALID_ARG, "layer %d: hidden differs from layer 0", l);
  }
  if (T < 0) return fail(FMOE_ERR_INVALID_ARG, "T %d", T);
  if (T == 0) return FMOE_OK;
  if (!h || !out) return fail(FMOE_ERR_INVALID_ARG, "h or out is NULL");
  if (!aligned16(h) || !aligned16(out)) return fail(FMOE_ERR_ALIGNMENT, "h and out must be 16-byte aligned");
  // one launch per run of up to kFusedMaxLayers layers when the single-kernel path takes them
  size_t need = 0;
  for (int l = 0; l < nl; ++l) {
    const WsLayout Ll = layout(layers[l].routed.hidden, layers[l].routed.num_experts, layers[l].top_k,
                               layers[l].routed.inter, 1);
    need = Ll.total > need ? Ll.total : need;
  }
  fmoe_status st = check_ws(ws, ws_bytes, need);
  if (st != FMOE_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(ws);
  for (int l0 = 0; l0 < nl;) {
    const int n = nl - l0 < kFusedMaxLayers ? nl - l0 : kFusedMaxLayers;
    const WsLayout Ll = layout(layers[l0].routed.hidden, layers[l0].routed.num_experts, layers[l0].top_k,
                               layers[l0].routed.inter, 1);
    bool taken = false;
    st = run_fused(&layers[l0], n, l0 == 0 ? h : out, T, out, nullptr, nullptr, base, Ll, cs(stream), nullptr, taken);
    if (st != FMOE_OK) return st;
    if (taken) {
      l0 += n;
      continue;
    }
    st = fmoe_moe_layer(&layers[l0], l0 == 0 ? h : out, T, out, nullptr, nullptr, ws, ws_bytes, stream);
    if (st != FMOE_OK) return st;
    ++l0;
  }
  return FMOE_OK;
}

fmoe_status fmoe_trace_next_layer(void* const* events, int n) {
  if (!events) {
    g_trace_on = false;
    return FMOE_OK;
  }
  if (n != 4) return fail(FMOE_ERR_INVALID_ARG, "trace needs 4 events, got %d", n);
  for (int i = 0; i < 4; ++i) {
    if (!events[i]) return fail(FMOE_ERR_INVALID_ARG, "trace event %d is NULL", i);
    g_trace[i] = static_cast<cudaEvent_t>(events[i]);
  }
  g_trace_on = true;
  return FMOE_OK;
}

fmoe_status fmoe_workspace_init(void* ws, size_t ws_bytes, fmoe_stream_t stream) {
  if (!ws) return fail(FMOE_ERR_WORKSPACE, "workspace is NULL");
  if (ws_bytes < sizeof(WsControl)) return fail(FMOE_ERR_WORKSPACE, "workspace smaller than its control block");
  cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, cs(stream));
  return e == cudaSuccess ? FMOE_OK : cuda_fail(e, "cudaMemsetAsync");
}

fmoe_status fmoe_workspace_check(void* ws, fmoe_stream_t stream) {
  if (!ws) return fail(FMOE_ERR_WORKSPACE, "workspace is NULL");
  cudaError_t e = cudaStreamSynchronize(cs(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  WsControl* ctrl = static_cast<WsControl*>(ws);
  int err = 0;
  if ((e = cudaMemcpy(&err, &ctrl->err, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "cudaMemcpy");
  if (err == 0) return FMOE_OK;
  const int zero = 0;
  if ((e = cudaMemcpy(&ctrl->err, &zero, sizeof(int), cudaMemcpyHostToDevice)) != cudaSuccess)
    return cuda_fail(e, "cudaMemcpy");
  if (err == kDevBadIndex) return fail(FMOE_ERR_INVALID_ARG, "a kernel met an expert index outside the bank");
  if (err == kDevBounds) return fail(FMOE_ERR_DEVICE_BOUNDS, "a device-side bounds check failed");
  return fail(FMOE_ERR_DEVICE_TIMEOUT, "a kernel gave up a bounded wait (code %d)", err);
}

}  // extern "C"
