// extern "C" entry points of libmoe (declared and documented in include/moe.h):
// argument validation, workspace carving, and the sequence of launches.
// The library is built from this single translation unit.
#include <atomic>
#include <cmath>
#include <mutex>

#include "../../include/moe.h"
#include "internal.h"
// one translation unit: the kernels share the per-device error word
#include "router_permute_combine.cuh"
#include "gemm_launch.cuh"
#include "glm_variant.cuh"

namespace {

using moe::Launch;

std::atomic<unsigned long long> g_wait_limit_ns{1000000000ull};

// stage events (moe_set_stage_events)
constexpr int kStages = 5;
enum { ST_ROUTER = 0, ST_DISPATCH = 1, ST_GATEUP = 2, ST_DOWN = 3, ST_COMBINE = 4 };
std::mutex g_ev_mu;
cudaEvent_t g_ev_start[kStages] = {};
cudaEvent_t g_ev_stop[kStages] = {};

void stage_mark(int stage, bool start, cudaStream_t st) {
  cudaEvent_t ev;
  {
    std::lock_guard<std::mutex> g(g_ev_mu);
    ev = start ? g_ev_start[stage] : g_ev_stop[stage];
  }
  if (ev != nullptr) cudaEventRecord(ev, st);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ptr_ok(const void* p) { return p != nullptr && aligned16(p); }

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

moe_status_t check_cfg(const moe_config_t* c) {
  if (c == nullptr) return MOE_ERR_INVALID_ARG;
  const int D = c->hidden_size, F = c->intermediate_size, E = c->num_local_experts, k = c->num_experts_per_tok;
  if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (c->wfmt != MOE_W_DENSE && c->wfmt != MOE_W_MXFP4 && c->wfmt != MOE_W_MXFP4_A8) return MOE_ERR_INVALID_ARG;
  if (E < 1 || E > 256 || k < 1 || k > 8 || k > E) return MOE_ERR_INVALID_ARG;
  if (D <= 0 || F <= 0 || D > (1 << 20) || F > (1 << 20)) return MOE_ERR_INVALID_ARG;
  const int mult = c->wfmt == MOE_W_DENSE ? 16 : 32;
  if (D % mult != 0 || F % mult != 0) return MOE_ERR_INVALID_ARG;
  if (!std::isfinite(c->swiglu_limit) || !(c->swiglu_limit > 0.0f) || !std::isfinite(c->swiglu_alpha))
    return MOE_ERR_INVALID_ARG;
  if (c->y_f32 != 0 && c->y_f32 != 1) return MOE_ERR_INVALID_ARG;
  if (c->h_split != 0 && c->h_split != 1) return MOE_ERR_INVALID_ARG;
  if (c->wfmt != MOE_W_DENSE && c->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (c->wfmt != MOE_W_DENSE && c->h_split != 0) return MOE_ERR_UNSUPPORTED;
  if (c->wfmt != MOE_W_DENSE) {
    // the scale relayout kernels index a matrix's scales with 32-bit integers
    const int64_t big = D > F ? D : F;
    if (int64_t(E) * big * ((big + 63) / 64) * 2 >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
  }
  return MOE_OK;
}

bool mxfp4_weights(const moe_config_t* c) { return c->wfmt == MOE_W_MXFP4 || c->wfmt == MOE_W_MXFP4_A8; }

// h kept as two bf16 halves (bf16 layers; fp32 layers keep h in fp32 and ignore the flag)
int h_halves(const moe_config_t* c) { return (c->dtype == MOE_BF16 && c->h_split != 0) ? 2 : 1; }

// checked before any launch: the weights-in-M pair kernels have no two-halves form
moe_status_t check_variant(const moe_config_t* c) {
  return (h_halves(c) == 2 && moe::g_gemm_variant.load() == 4) ? MOE_ERR_UNSUPPORTED : MOE_OK;
}

// the layer output is bf16 only for a bf16 layer without y_f32
bool out_bf16(const moe_config_t* c) { return c->dtype == MOE_BF16 && c->y_f32 == 0; }

bool check_T(int64_t T, int k) { return T >= 0 && T * k < (int64_t(1) << 31); }

size_t elem_size(const moe_config_t* c) { return c->dtype == MOE_BF16 ? 2 : 4; }

// Scratch of the expert GEMMs: none for dense weights; for MXFP4 the three scale
// tensors relaid for TMA ([E][ceil(K/64)][N][2] each, 256-byte aligned regions).
struct MxScaleRegions {
  size_t gate, up, down, total;
};
MxScaleRegions mx_regions(const moe_config_t* c) {
  const int D = c->hidden_size, F = c->intermediate_size, E = c->num_local_experts;
  MxScaleRegions r{};
  r.gate = 0;
  r.up = align256(moe::mx_scale_bytes(F, D, E));
  r.down = r.up + align256(moe::mx_scale_bytes(F, D, E));
  r.total = r.down + align256(moe::mx_scale_bytes(D, F, E));
  return r;
}
size_t ffn_ws_bytes(const moe_config_t* c, int64_t) { return c->wfmt == MOE_W_MXFP4 ? mx_regions(c).total : 0; }

struct Layout {
  size_t ids, w, off, ros, sor, pscr, xperm, h, rpart, ys, ffn, total;
  bool dl;                        // the decode layer's regions follow
  size_t dlog, dcnt, dpart, dys;  // its router logits, counters, partial sums, weighted rows
};

// Whether a layer of T tokens can run as the two-kernel decode layer (dense bf16 weights).
bool decode_layer_shape(const moe_config_t* c, int64_t T) {
  return c->wfmt == MOE_W_DENSE &&
         moe::decode_layer_shape(c->dtype == MOE_BF16, T, c->num_experts_per_tok, c->num_local_experts,
                                 c->hidden_size, c->intermediate_size);
}

Layout layout(const moe_config_t* c, int64_t T) {
  const size_t R = size_t(T) * c->num_experts_per_tok, es = elem_size(c);
  Layout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L.ids = take(R * 4);
  L.w = take(R * 4);
  L.off = take(size_t(c->num_local_experts + 1) * 4);
  L.ros = take(R * 4);
  L.sor = take(R * 4);
  L.pscr = take(moe::permute_scratch_words(T, c->num_local_experts) * 4);
  // x_perm is dead once gate/up has run: the weighted fp32 expert outputs reuse its region
  L.xperm = take(R * c->hidden_size * (es > 4 ? es : 4));
  L.ys = L.xperm;
  // the router's K-split partial logits are dead before gate/up writes h: they share it
  const size_t h_bytes = R * c->intermediate_size * es * h_halves(c);
  const size_t rpart_bytes = moe::router_partial_bytes(T, c->num_local_experts);
  L.h = take(h_bytes > rpart_bytes ? h_bytes : rpart_bytes);
  L.rpart = L.h;
  L.ffn = take(ffn_ws_bytes(c, T));
  L.dl = decode_layer_shape(c, T);
  if (L.dl) {
    // the decode layer writes the weighted rows while other CTAs still read x_perm: own region
    L.dlog = take(size_t(T) * c->num_local_experts * 4);
    L.dcnt = take(moe::decode_layer_counter_words(T, c->num_experts_per_tok, c->num_local_experts, c->hidden_size,
                                                  c->intermediate_size) * 4);
    L.dpart = take(moe::decode_layer_part_bytes());
    L.dys = take(R * c->hidden_size * 4);
  }
  L.total = o;
  return L;
}

// Workspace of moe_layer_forward with MOE_W_MXFP4_A8: the maps, then x and x_perm in
// MXFP8 (E4M3 rows and scale rows), h in MXFP8, the weighted fp32 rows, and the
// weights' scale rows padded for 32-bit loads.
struct LayoutA8 {
  size_t ids, w, off, ros, sor, pscr, xq, sfx, xpq, sfa, hq, sfh, ys, sfw_g, sfw_u, sfw_d, rpart, total;
};

LayoutA8 layout_a8(const moe_config_t* c, int64_t T) {
  const size_t R = size_t(T) * c->num_experts_per_tok;
  const size_t D = c->hidden_size, F = c->intermediate_size, E = c->num_local_experts;
  const size_t sd = moe::mx8_sf_bytes_per_row(c->hidden_size), sf = moe::mx8_sf_bytes_per_row(c->intermediate_size);
  LayoutA8 L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L.ids = take(R * 4);
  L.w = take(R * 4);
  L.off = take((E + 1) * 4);
  L.ros = take(R * 4);
  L.sor = take(R * 4);
  L.pscr = take(moe::permute_scratch_words(T, c->num_local_experts) * 4);
  L.xq = take(size_t(T) * D);
  L.sfx = take(size_t(T) * sd);
  L.xpq = take(R * D);
  L.sfa = take(R * sd);
  // the router's K-split partial logits are dead before gate/up writes hq: they share it
  const size_t rpart_bytes = moe::router_partial_bytes(T, c->num_local_experts);
  L.hq = take(R * F > rpart_bytes ? R * F : rpart_bytes);
  L.rpart = L.hq;
  L.sfh = take(R * sf);
  L.ys = take(R * D * 4);
  L.sfw_g = take(E * F * sd);
  L.sfw_u = take(E * F * sd);
  L.sfw_d = take(E * D * sf);
  L.total = o;
  return L;
}

size_t layer_ws_bytes(const moe_config_t* c, int64_t T) {
  return c->wfmt == MOE_W_MXFP4_A8 ? layout_a8(c, T).total : layout(c, T).total;
}

bool get_launch(void* stream, Launch* L) {
  static std::mutex mu;
  static int sms[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  int n = 0;
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev < 64 && sms[dev] > 0) {
      n = sms[dev];
    } else {
      if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
      if (dev < 64) sms[dev] = n;
    }
  }
  L->stream = static_cast<cudaStream_t>(stream);
  L->num_sms = n;
  L->wait_limit_ns = g_wait_limit_ns.load();
  return true;
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

bool weights_ok(const moe_config_t* c, const moe_expert_weights_t* w) {
  if (w == nullptr) return false;
  if (!ptr_ok(w->w_gate) || !ptr_ok(w->w_up) || !ptr_ok(w->w_down)) return false;
  if (!ptr_ok(w->b_gate) || !ptr_ok(w->b_up) || !ptr_ok(w->b_down)) return false;
  if (mxfp4_weights(c) && (!ptr_ok(w->s_gate) || !ptr_ok(w->s_up) || !ptr_ok(w->s_down))) return false;
  return true;
}

moe::ExpertWeights to_internal(const moe_expert_weights_t* w) {
  moe::ExpertWeights x;
  x.w_gate = w->w_gate;
  x.w_up = w->w_up;
  x.w_down = w->w_down;
  x.s_gate = w->s_gate;
  x.s_up = w->s_up;
  x.s_down = w->s_down;
  x.b_gate = w->b_gate;
  x.b_up = w->b_up;
  x.b_down = w->b_down;
  return x;
}

// gate/up then down (into y_perm, or weighted into slot order when slot_of_row != null)
moe_status_t run_experts(const moe_config_t* c, const Launch& L, int64_t T, const void* x_perm,
                         const int32_t* eoff, const moe_expert_weights_t* wts, void* h, void* out,
                         const int32_t* slot_of_row, const float* topk_w, void* ffn_ws,
                         const moe::GateupGather* gather = nullptr) {
  const bool bf16 = c->dtype == MOE_BF16;
  const int D = c->hidden_size, F = c->intermediate_size, E = c->num_local_experts;
  const int64_t R = T * c->num_experts_per_tok;
  moe::ExpertWeights w = to_internal(wts);
  stage_mark(ST_GATEUP, true, L.stream);
  if (c->wfmt == MOE_W_MXFP4) {
    const MxScaleRegions rg = mx_regions(c);
    uint8_t* ws = static_cast<uint8_t*>(ffn_ws);
    if (moe::mx_scale_relayout(L, D, F, E, w, ws + rg.gate, ws + rg.up, ws + rg.down) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (moe::expert_gateup_mxfp4(L, R, D, F, E, x_perm, eoff, w, ws + rg.gate, ws + rg.up, c->swiglu_limit,
                                 c->swiglu_alpha, h) != cudaSuccess)
      return MOE_ERR_CUDA;
    stage_mark(ST_GATEUP, false, L.stream);
    stage_mark(ST_DOWN, true, L.stream);
    const moe_status_t st =
        cuda_status(moe::expert_down_mxfp4(L, R, D, F, E, h, eoff, w, ws + rg.down, slot_of_row, topk_w, out));
    stage_mark(ST_DOWN, false, L.stream);
    return st;
  }
  const int hh = h_halves(c);
  if (moe::expert_gateup(L, bf16, R, D, F, E, x_perm, eoff, w, c->swiglu_limit, c->swiglu_alpha, h, 0.0f, hh,
                         gather) != cudaSuccess)
    return MOE_ERR_CUDA;
  stage_mark(ST_GATEUP, false, L.stream);
  stage_mark(ST_DOWN, true, L.stream);
  const moe_status_t st =
      cuda_status(moe::expert_down(L, bf16, R, D, F, E, h, eoff, w, slot_of_row, topk_w, out, hh));
  stage_mark(ST_DOWN, false, L.stream);
  return st;
}

// ---------------------------------------------------------------------------
// moe_permute_noalloc: the dispatch with its scratch in a fixed device array
// ---------------------------------------------------------------------------
// Histogram and scan scratch of moe_permute_noalloc: 2 * E * ceil(T / 256)
// int32 words at most kNoAllocWords (256 KiB).  One copy per GPU that loads
// the library, kept until the process exits; every call on a device shares it.
constexpr size_t kNoAllocWords = 65536;
static __device__ __align__(256) int32_t g_permute_scratch[kNoAllocWords];

// Host code cannot use g_permute_scratch's name as a device address: the address
// is looked up with cudaGetSymbolAddress in the current CUDA context.  It belongs
// to that context, so lookups are cached per context, keyed by the context's unique
// id (cuCtxGetId, never reused within a process): a context the caller made current
// itself, or the new primary context after a cudaDeviceReset, gets its own lookup.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

int32_t* permute_scratch_address() {
  struct Entry {
    unsigned long long ctx_id;
    int32_t* addr;
  };
  constexpr int kSlots = 64;
  static Entry cache[kSlots] = {};
  static int next = 0;
  static std::mutex mu;
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id);   // false before the runtime made a context current
  std::lock_guard<std::mutex> g(mu);
  if (have_id)
    for (const Entry& e : cache)
      if (e.addr != nullptr && e.ctx_id == id) return e.addr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr) return nullptr;
  if (have_id || current_context_id(&id)) {
    cache[next] = Entry{id, static_cast<int32_t*>(p)};
    next = (next + 1) % kSlots;
  }
  return static_cast<int32_t*>(p);
}

// ---------------------------------------------------------------------------
// the GLM4-MoE-Lite variant
// ---------------------------------------------------------------------------
moe_status_t check_glm(const moe_config_t* c, const moe_glm_params_t* p) {
  moe_status_t s = check_cfg(c);
  if (s != MOE_OK) return s;
  if (p == nullptr || !std::isfinite(p->routed_scaling_factor)) return MOE_ERR_INVALID_ARG;
  const int Fs = p->shared_intermediate_size;
  if (Fs < 0 || Fs > (1 << 20) || Fs % 16 != 0) return MOE_ERR_INVALID_ARG;
  if (c->wfmt != MOE_W_DENSE) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

struct GlmLayout {
  size_t ids, w, off, ros, sor, pscr, xperm, ys, h, rpart, zb, soff, sid, sone, hs, ysh, total;
};

GlmLayout glm_layout(const moe_config_t* c, const moe_glm_params_t* p, int64_t T) {
  const size_t R = size_t(T) * c->num_experts_per_tok, es = elem_size(c);
  const size_t D = c->hidden_size, F = c->intermediate_size, E = c->num_local_experts;
  const size_t Fs = p->shared_intermediate_size;
  GlmLayout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L.ids = take(R * 4);
  L.w = take(R * 4);
  L.off = take((E + 1) * 4);
  L.ros = take(R * 4);
  L.sor = take(R * 4);
  L.pscr = take(moe::permute_scratch_words(T, c->num_local_experts) * 4);
  L.xperm = take(R * D * (es > 4 ? es : 4));   // x_perm, then the weighted fp32 rows
  L.ys = L.xperm;
  const size_t h_bytes = R * F * es * h_halves(c), rpart_bytes = moe::router_partial_bytes(T, c->num_local_experts);
  L.h = take(h_bytes > rpart_bytes ? h_bytes : rpart_bytes);
  L.rpart = L.h;
  // zero biases: [E, F] for gate/up, [E, D] for down, [1, Fs] / [1, D] for the shared expert
  size_t zb = E * (F > D ? F : D);
  if (Fs > zb) zb = Fs;
  L.zb = take(zb * es);
  if (Fs > 0) {
    L.soff = take(2 * 4);
    L.sid = take(size_t(T) * 4);
    L.sone = take(size_t(T) * 4);
    L.hs = take(size_t(T) * Fs * es * h_halves(c));
    L.ysh = take(size_t(T) * D * 4);
  }
  L.total = o;
  return L;
}

// moe_layer_forward with MXFP4 weights and MXFP8 activations (arguments already checked)
moe_status_t layer_forward_a8(const moe_config_t* cfg, const Launch& L, int64_t T, const void* x,
                              const void* w_router, const void* b_router, const moe_expert_weights_t* weights, void* y,
                              int32_t* topk_ids_out, float* topk_w_out, void* ws) {
  const LayoutA8 LY = layout_a8(cfg, T);
  uint8_t* base = static_cast<uint8_t*>(ws);
  int32_t* ids = topk_ids_out ? topk_ids_out : reinterpret_cast<int32_t*>(base + LY.ids);
  float* w = topk_w_out ? topk_w_out : reinterpret_cast<float*>(base + LY.w);
  int32_t* eoff = reinterpret_cast<int32_t*>(base + LY.off);
  int32_t* ros = reinterpret_cast<int32_t*>(base + LY.ros);
  int32_t* sor = reinterpret_cast<int32_t*>(base + LY.sor);
  int32_t* pscr = reinterpret_cast<int32_t*>(base + LY.pscr);
  const int D = cfg->hidden_size, F = cfg->intermediate_size, E = cfg->num_local_experts,
            k = cfg->num_experts_per_tok;
  const int64_t R = T * k;
  const moe::ExpertWeights wt = to_internal(weights);

  stage_mark(ST_ROUTER, true, L.stream);
  if (moe::router_topk(L, true, T, D, E, k, x, w_router, b_router, ids, w,
                       reinterpret_cast<float*>(base + LY.rpart)) != cudaSuccess)
    return MOE_ERR_CUDA;
  stage_mark(ST_ROUTER, false, L.stream);
  stage_mark(ST_DISPATCH, true, L.stream);
  if (moe::permute(L, true, T, D, E, k, ids, nullptr, eoff, ros, sor, nullptr, pscr) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (moe::mx8_quant_rows(L, T, D, x, base + LY.xq, base + LY.sfx) != cudaSuccess) return MOE_ERR_CUDA;
  if (moe::gather_rows(L, base + LY.xq, sor, R, k, T, D, base + LY.xpq) != cudaSuccess) return MOE_ERR_CUDA;
  if (moe::gather_rows(L, base + LY.sfx, sor, R, k, T, moe::mx8_sf_bytes_per_row(D), base + LY.sfa) != cudaSuccess)
    return MOE_ERR_CUDA;
  stage_mark(ST_DISPATCH, false, L.stream);
  stage_mark(ST_GATEUP, true, L.stream);
  if (moe::mx8_weight_scales(L, D, F, E, wt, base + LY.sfw_g, base + LY.sfw_u, base + LY.sfw_d) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (moe::expert_gateup_mx8(L, R, D, F, E, base + LY.xpq, base + LY.sfa, eoff, wt, base + LY.sfw_g,
                             base + LY.sfw_u, cfg->swiglu_limit, cfg->swiglu_alpha, base + LY.hq,
                             base + LY.sfh) != cudaSuccess)
    return MOE_ERR_CUDA;
  stage_mark(ST_GATEUP, false, L.stream);
  stage_mark(ST_DOWN, true, L.stream);
  float* ys = reinterpret_cast<float*>(base + LY.ys);
  if (moe::expert_down_mx8(L, R, D, F, E, base + LY.hq, base + LY.sfh, eoff, wt, base + LY.sfw_d, sor, w, ys) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  stage_mark(ST_DOWN, false, L.stream);
  stage_mark(ST_COMBINE, true, L.stream);
  const moe_status_t s = cuda_status(moe::combine_slots(L, out_bf16(cfg), T, D, k, ys, y));
  stage_mark(ST_COMBINE, false, L.stream);
  return s;
}

}  // namespace

extern "C" {

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: unsupported configuration";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing or too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA call or launch failed";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a bounded device wait gave up";
    case MOE_ERR_DEVICE_BOUNDS: return "MOE_ERR_DEVICE_BOUNDS: out-of-range index read on the device";
  }
  return "unknown moe_status_t";
}

moe_status_t moe_config_check(const moe_config_t* cfg) { return check_cfg(cfg); }

size_t moe_permute_workspace_size(const moe_config_t* cfg, int64_t T) {
  if (check_cfg(cfg) != MOE_OK || !check_T(T, cfg->num_experts_per_tok)) return size_t(-1);
  return moe::permute_scratch_words(T, cfg->num_local_experts) * 4;
}

size_t moe_expert_ffn_workspace_size(const moe_config_t* cfg, int64_t T) {
  if (check_cfg(cfg) != MOE_OK || !check_T(T, cfg->num_experts_per_tok)) return size_t(-1);
  return ffn_ws_bytes(cfg, T);
}

size_t moe_workspace_size(const moe_config_t* cfg, int64_t T) {
  if (check_cfg(cfg) != MOE_OK || !check_T(T, cfg->num_experts_per_tok)) return size_t(-1);
  return layer_ws_bytes(cfg, T);
}

moe_status_t moe_router_topk(const moe_config_t* cfg, int64_t T, const void* x, const void* w_router,
                             const void* b_router, int32_t* topk_ids, float* topk_w, void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (!check_T(T, cfg->num_experts_per_tok)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!ptr_ok(x) || !ptr_ok(w_router) || !ptr_ok(b_router) || !ptr_ok(topk_ids) || !ptr_ok(topk_w))
    return MOE_ERR_INVALID_ARG;
  Launch L;
  if (!get_launch(stream, &L)) return MOE_ERR_CUDA;
  return cuda_status(moe::router_topk(L, cfg->dtype == MOE_BF16, T, cfg->hidden_size, cfg->num_local_experts,
                                      cfg->num_experts_per_tok, x, w_router, b_router, topk_ids, topk_w));
}

moe_status_t moe_permute(const moe_config_t* cfg, int64_t T, const int32_t* topk_ids, const void* x,
                         int32_t* expert_off, int32_t* row_of_slot, int32_t* slot_of_row, void* x_perm, void* ws,
                         size_t ws_bytes, void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (!check_T(T, cfg->num_experts_per_tok)) return MOE_ERR_INVALID_ARG;
  if (!ptr_ok(expert_off)) return MOE_ERR_INVALID_ARG;
  if (T > 0) {
    if (!ptr_ok(topk_ids) || !ptr_ok(row_of_slot) || !ptr_ok(slot_of_row)) return MOE_ERR_INVALID_ARG;
    if ((x == nullptr) != (x_perm == nullptr)) return MOE_ERR_INVALID_ARG;
    if (x != nullptr && (!aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
    const size_t need = moe::permute_scratch_words(T, cfg->num_local_experts) * 4;
    if (ws == nullptr || !aligned16(ws) || ws_bytes < need) return MOE_ERR_WORKSPACE;
  }
  Launch L;
  if (!get_launch(stream, &L)) return MOE_ERR_CUDA;
  return cuda_status(moe::permute(L, cfg->dtype == MOE_BF16, T, cfg->hidden_size, cfg->num_local_experts,
                                  cfg->num_experts_per_tok, topk_ids, x, expert_off, row_of_slot, slot_of_row,
                                  x_perm, static_cast<int32_t*>(ws)));
}

moe_status_t moe_permute_noalloc(const moe_config_t* cfg, int64_t T, const int32_t* topk_ids, const void* x,
                                 int32_t* expert_off, int32_t* row_of_slot, int32_t* slot_of_row, void* x_perm,
                                 void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (!check_T(T, cfg->num_experts_per_tok)) return MOE_ERR_INVALID_ARG;
  if (!ptr_ok(expert_off)) return MOE_ERR_INVALID_ARG;
  if (T > 0) {
    if (!ptr_ok(topk_ids) || !ptr_ok(row_of_slot) || !ptr_ok(slot_of_row)) return MOE_ERR_INVALID_ARG;
    if ((x == nullptr) != (x_perm == nullptr)) return MOE_ERR_INVALID_ARG;
    if (x != nullptr && (!aligned16(x) || !aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
    if (moe::permute_scratch_words(T, cfg->num_local_experts) > kNoAllocWords) return MOE_ERR_UNSUPPORTED;
  }
  int32_t* scratch = permute_scratch_address();
  if (scratch == nullptr) return MOE_ERR_CUDA;
  Launch L;
  if (!get_launch(stream, &L)) return MOE_ERR_CUDA;
  return cuda_status(moe::permute(L, cfg->dtype == MOE_BF16, T, cfg->hidden_size, cfg->num_local_experts,
                                  cfg->num_experts_per_tok, topk_ids, x, expert_off, row_of_slot, slot_of_row,
                                  x_perm, scratch));
}

moe_status_t moe_expert_ffn(const moe_config_t* cfg, int64_t T, const void* x_perm, const int32_t* expert_off,
                            const moe_expert_weights_t* weights, void* h, void* y_perm, void* ws, size_t ws_bytes,
                            void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (!check_T(T, cfg->num_experts_per_tok)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!ptr_ok(x_perm) || !ptr_ok(expert_off) || !ptr_ok(h) || !ptr_ok(y_perm) || !weights_ok(cfg, weights))
    return MOE_ERR_INVALID_ARG;
  if ((s = check_variant(cfg)) != MOE_OK) return s;
  if (cfg->wfmt == MOE_W_MXFP4_A8) return MOE_ERR_UNSUPPORTED;   // its activations never leave MXFP8
  const size_t need = ffn_ws_bytes(cfg, T);
  if (need > 0 && (ws == nullptr || !aligned16(ws) || ws_bytes < need)) return MOE_ERR_WORKSPACE;
  Launch L;
  if (!get_launch(stream, &L)) return MOE_ERR_CUDA;
  return run_experts(cfg, L, T, x_perm, expert_off, weights, h, y_perm, nullptr, nullptr, ws);
}

moe_status_t moe_combine(const moe_config_t* cfg, int64_t T, const void* y_perm, const int32_t* row_of_slot,
                         const float* topk_w, void* y, void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (!check_T(T, cfg->num_experts_per_tok)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!ptr_ok(y_perm) || !ptr_ok(row_of_slot) || !ptr_ok(topk_w) || !ptr_ok(y)) return MOE_ERR_INVALID_ARG;
  Launch L;
  if (!get_launch(stream, &L)) return MOE_ERR_CUDA;
  return cuda_status(moe::combine_gather(L, cfg->dtype == MOE_BF16, cfg->y_f32 != 0, T, cfg->hidden_size,
                                         cfg->num_experts_per_tok, y_perm, row_of_slot, topk_w, y));
}

moe_status_t moe_layer_forward(const moe_config_t* cfg, int64_t T, const void* x, const void* w_router,
                               const void* b_router, const moe_expert_weights_t* weights, void* y,
                               int32_t* topk_ids_out, float* topk_w_out, void* ws, size_t ws_bytes, void* stream) {
  moe_status_t s = check_cfg(cfg);
  if (s != MOE_OK) return s;
  if (!check_T(T, cfg->num_experts_per_tok)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!ptr_ok(x) || !ptr_ok(w_router) || !ptr_ok(b_router) || !ptr_ok(y) || !weights_ok(cfg, weights))
    return MOE_ERR_INVALID_ARG;
  if ((topk_ids_out != nullptr && !aligned16(topk_ids_out)) || (topk_w_out != nullptr && !aligned16(topk_w_out)))
    return MOE_ERR_INVALID_ARG;
  if ((s = check_variant(cfg)) != MOE_OK) return s;
  if (ws == nullptr || !aligned16(ws) || ws_bytes < layer_ws_bytes(cfg, T)) return MOE_ERR_WORKSPACE;
  Launch L;
  if (!get_launch(stream, &L)) return MOE_ERR_CUDA;
  if (cfg->wfmt == MOE_W_MXFP4_A8)
    return layer_forward_a8(cfg, L, T, x, w_router, b_router, weights, y, topk_ids_out, topk_w_out, ws);
  const Layout LY = layout(cfg, T);

  uint8_t* base = static_cast<uint8_t*>(ws);
  int32_t* ids = topk_ids_out ? topk_ids_out : reinterpret_cast<int32_t*>(base + LY.ids);
  float* w = topk_w_out ? topk_w_out : reinterpret_cast<float*>(base + LY.w);
  int32_t* eoff = reinterpret_cast<int32_t*>(base + LY.off);
  int32_t* ros = reinterpret_cast<int32_t*>(base + LY.ros);
  int32_t* sor = reinterpret_cast<int32_t*>(base + LY.sor);
  int32_t* pscr = reinterpret_cast<int32_t*>(base + LY.pscr);
  void* xperm = base + LY.xperm;
  void* h = base + LY.h;
  void* ys = base + LY.ys;
  void* ffn = base + LY.ffn;
  const bool bf16 = cfg->dtype == MOE_BF16;
  const int D = cfg->hidden_size, E = cfg->num_local_experts, k = cfg->num_experts_per_tok;

  if (LY.dl && moe::decode_layer_selected(bf16, T, k, E, D, cfg->intermediate_size)) {
    stage_mark(ST_ROUTER, true, L.stream);
    stage_mark(ST_ROUTER, false, L.stream);
    stage_mark(ST_GATEUP, true, L.stream);
    const moe_status_t st = cuda_status(moe::decode_layer(
        L, T, D, cfg->intermediate_size, E, k, x, w_router, b_router, to_internal(weights), cfg->swiglu_limit,
        cfg->swiglu_alpha, 0.0f, h_halves(cfg), !out_bf16(cfg), y, topk_ids_out, topk_w_out,
        reinterpret_cast<float*>(base + LY.dlog), reinterpret_cast<int*>(base + LY.dcnt),
        reinterpret_cast<float*>(base + LY.dpart), h, reinterpret_cast<float*>(base + LY.dys)));
    stage_mark(ST_GATEUP, false, L.stream);
    return st;
  }

  stage_mark(ST_ROUTER, true, L.stream);
  if (moe::router_topk(L, bf16, T, D, E, k, x, w_router, b_router, ids, w,
                       reinterpret_cast<float*>(base + LY.rpart)) != cudaSuccess)
    return MOE_ERR_CUDA;
  stage_mark(ST_ROUTER, false, L.stream);
  // with expert-GEMM variant 6 the single-CTA gate/up kernel gathers its A rows from x
  // (TMA gather4): the dispatch then builds the maps only, with no x_perm copy
  const bool gather = cfg->wfmt == MOE_W_DENSE && moe::gateup_gathers(bf16, T * k, E);
  const moe::GateupGather gx{x, sor, k, T};
  stage_mark(ST_DISPATCH, true, L.stream);
  if (moe::permute(L, bf16, T, D, E, k, ids, gather ? nullptr : x, eoff, ros, sor, gather ? nullptr : xperm, pscr) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  stage_mark(ST_DISPATCH, false, L.stream);
  s = run_experts(cfg, L, T, xperm, eoff, weights, h, ys, sor, w, ffn, gather ? &gx : nullptr);
  if (s != MOE_OK) return s;
  stage_mark(ST_COMBINE, true, L.stream);
  s = cuda_status(moe::combine_slots(L, out_bf16(cfg), T, D, k, ys, y));
  stage_mark(ST_COMBINE, false, L.stream);
  return s;
}

int32_t moe_mxfp8_scale_stride(int32_t K) { return K > 0 ? moe::mx8_sf_bytes_per_row(K) : -1; }

moe_status_t moe_quantize_mxfp8(int64_t rows, int32_t K, const void* x, uint8_t* xq, uint8_t* sf, void* stream) {
  if (rows < 0 || K <= 0 || K % 32 != 0 || K > (1 << 20) || rows > (int64_t(1) << 31)) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!ptr_ok(x) || !ptr_ok(xq) || !ptr_ok(sf)) return MOE_ERR_INVALID_ARG;
  Launch L;
  if (!get_launch(stream, &L)) return MOE_ERR_CUDA;
  return cuda_status(moe::mx8_quant_rows(L, rows, K, x, xq, sf));
}

moe_status_t moe_last_device_error(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  int bits = 0;
  if (moe::read_and_clear_device_error(&bits) != cudaSuccess) return MOE_ERR_CUDA;
  if (bits & moe::DEVERR_TIMEOUT) return MOE_ERR_TIMEOUT;
  if (bits & moe::DEVERR_BOUNDS) return MOE_ERR_DEVICE_BOUNDS;
  return MOE_OK;
}

void moe_set_stage_events(void* const* starts, void* const* stops, int32_t n) {
  std::lock_guard<std::mutex> g(g_ev_mu);
  for (int i = 0; i < kStages; ++i) {
    g_ev_start[i] = (starts != nullptr && i < n) ? static_cast<cudaEvent_t>(starts[i]) : nullptr;
    g_ev_stop[i] = (stops != nullptr && i < n) ? static_cast<cudaEvent_t>(stops[i]) : nullptr;
  }
}

uint64_t moe_launch_count(void) { return moe::g_launches.load(); }

moe_status_t moe_set_expert_gemm_variant(int32_t variant) {
  if (variant < 0 || variant > 7) return MOE_ERR_INVALID_ARG;
  moe::g_gemm_variant.store(variant);
  return MOE_OK;
}

void moe_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns == 0 ? 1000000000ull : ns); }

size_t moe_glm_router_workspace_size(const moe_config_t* cfg, int64_t T) {
  if (check_cfg(cfg) != MOE_OK || !check_T(T, cfg->num_experts_per_tok)) return size_t(-1);
  return moe::router_partial_bytes(T, cfg->num_local_experts);
}

size_t moe_glm_workspace_size(const moe_config_t* cfg, const moe_glm_params_t* p, int64_t T) {
  if (check_glm(cfg, p) != MOE_OK || !check_T(T, cfg->num_experts_per_tok)) return size_t(-1);
  return glm_layout(cfg, p, T).total;
}

moe_status_t moe_glm_router_topk(const moe_config_t* cfg, const moe_glm_params_t* p, int64_t T, const void* x,
                                 const void* w_router, int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes,
                                 void* stream) {
  moe_status_t s = check_glm(cfg, p);
  if (s != MOE_OK) return s;
  if (!check_T(T, cfg->num_experts_per_tok)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!ptr_ok(x) || !ptr_ok(w_router) || !ptr_ok(topk_ids) || !ptr_ok(topk_w)) return MOE_ERR_INVALID_ARG;
  if (p->e_score_correction_bias != nullptr && !aligned16(p->e_score_correction_bias)) return MOE_ERR_INVALID_ARG;
  if (ws == nullptr || !aligned16(ws) || ws_bytes < moe::router_partial_bytes(T, cfg->num_local_experts))
    return MOE_ERR_WORKSPACE;
  Launch L;
  if (!get_launch(stream, &L)) return MOE_ERR_CUDA;
  return cuda_status(moe::glm_router(L, cfg->dtype == MOE_BF16, T, cfg->hidden_size, cfg->num_local_experts,
                                     cfg->num_experts_per_tok, x, w_router, p->e_score_correction_bias,
                                     p->norm_topk_prob != 0, p->routed_scaling_factor, topk_ids, topk_w,
                                     static_cast<float*>(ws)));
}

moe_status_t moe_glm_layer_forward(const moe_config_t* cfg, const moe_glm_params_t* p, int64_t T, const void* x,
                                   const void* w_router, const moe_expert_weights_t* weights, void* y,
                                   int32_t* topk_ids_out, float* topk_w_out, void* ws, size_t ws_bytes,
                                   void* stream) {
  moe_status_t s = check_glm(cfg, p);
  if (s != MOE_OK) return s;
  if (!check_T(T, cfg->num_experts_per_tok)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  const int Fs = p->shared_intermediate_size;
  if (!ptr_ok(x) || !ptr_ok(w_router) || !ptr_ok(y) || weights == nullptr) return MOE_ERR_INVALID_ARG;
  if (!ptr_ok(weights->w_gate) || !ptr_ok(weights->w_up) || !ptr_ok(weights->w_down)) return MOE_ERR_INVALID_ARG;
  if (Fs > 0 && (!ptr_ok(p->ws_gate) || !ptr_ok(p->ws_up) || !ptr_ok(p->ws_down))) return MOE_ERR_INVALID_ARG;
  if (p->e_score_correction_bias != nullptr && !aligned16(p->e_score_correction_bias)) return MOE_ERR_INVALID_ARG;
  if ((topk_ids_out != nullptr && !aligned16(topk_ids_out)) || (topk_w_out != nullptr && !aligned16(topk_w_out)))
    return MOE_ERR_INVALID_ARG;
  if ((s = check_variant(cfg)) != MOE_OK) return s;
  const GlmLayout LY = glm_layout(cfg, p, T);
  if (ws == nullptr || !aligned16(ws) || ws_bytes < LY.total) return MOE_ERR_WORKSPACE;
  Launch L;
  if (!get_launch(stream, &L)) return MOE_ERR_CUDA;

  uint8_t* base = static_cast<uint8_t*>(ws);
  int32_t* ids = topk_ids_out ? topk_ids_out : reinterpret_cast<int32_t*>(base + LY.ids);
  float* w = topk_w_out ? topk_w_out : reinterpret_cast<float*>(base + LY.w);
  int32_t* eoff = reinterpret_cast<int32_t*>(base + LY.off);
  int32_t* ros = reinterpret_cast<int32_t*>(base + LY.ros);
  int32_t* sor = reinterpret_cast<int32_t*>(base + LY.sor);
  int32_t* pscr = reinterpret_cast<int32_t*>(base + LY.pscr);
  void* xperm = base + LY.xperm;
  void* h = base + LY.h;
  void* ys = base + LY.ys;
  void* zb = base + LY.zb;
  const bool bf16 = cfg->dtype == MOE_BF16;
  const int D = cfg->hidden_size, F = cfg->intermediate_size, E = cfg->num_local_experts,
            k = cfg->num_experts_per_tok;
  const int64_t R = T * k;
  const size_t es = elem_size(cfg);
  // SiLU(g) * u is the clipped SwiGLU with the gate floor at -inf, no upper clip and alpha = 1
  const float kInf = INFINITY;

  // zero biases for the expert GEMMs (the page's experts have none)
  size_t zb_elems = size_t(E) * (F > D ? F : D);
  if (size_t(Fs) > zb_elems) zb_elems = Fs;
  if (cudaMemsetAsync(zb, 0, zb_elems * es, L.stream) != cudaSuccess) return MOE_ERR_CUDA;

  if (moe::glm_router(L, bf16, T, D, E, k, x, w_router, p->e_score_correction_bias, p->norm_topk_prob != 0,
                      p->routed_scaling_factor, ids, w, reinterpret_cast<float*>(base + LY.rpart)) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (moe::permute(L, bf16, T, D, E, k, ids, x, eoff, ros, sor, xperm, pscr) != cudaSuccess) return MOE_ERR_CUDA;
  moe::ExpertWeights rw{};
  rw.w_gate = weights->w_gate;
  rw.w_up = weights->w_up;
  rw.w_down = weights->w_down;
  rw.b_gate = zb;
  rw.b_up = zb;
  rw.b_down = zb;
  const int hh = h_halves(cfg);
  if (moe::expert_gateup(L, bf16, R, D, F, E, xperm, eoff, rw, kInf, 1.0f, h, -kInf, hh) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (moe::expert_down(L, bf16, R, D, F, E, h, eoff, rw, sor, w, ys, hh) != cudaSuccess) return MOE_ERR_CUDA;
  void* ysh = nullptr;
  if (Fs > 0) {
    int32_t* soff = reinterpret_cast<int32_t*>(base + LY.soff);
    void* hs = base + LY.hs;
    ysh = base + LY.ysh;
    moe::ExpertWeights sw{};
    sw.w_gate = p->ws_gate;
    sw.w_up = p->ws_up;
    sw.w_down = p->ws_down;
    sw.b_gate = zb;
    sw.b_up = zb;
    sw.b_down = zb;
    int32_t* sid = reinterpret_cast<int32_t*>(base + LY.sid);
    float* sone = reinterpret_cast<float*>(base + LY.sone);
    if (moe::glm_shared_off(L, T, soff, sid, sone) != cudaSuccess) return MOE_ERR_CUDA;
    if (moe::expert_gateup(L, bf16, T, D, Fs, 1, x, soff, sw, kInf, 1.0f, hs, -kInf, hh) != cudaSuccess)
      return MOE_ERR_CUDA;
    // fp32 rows (identity slots, unit weights): the shared output is rounded once, with the sum
    if (moe::expert_down(L, bf16, T, D, Fs, 1, hs, soff, sw, sid, sone, ysh, hh) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return cuda_status(moe::combine_slots_shared(L, out_bf16(cfg), T, D, k, ys, ysh, y));
}

}  // extern "C"
