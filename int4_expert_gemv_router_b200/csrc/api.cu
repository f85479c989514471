// C-ABI entry points (include/moe.h): argument validation, workspace carving and the launch
// sequence of each call.  No kernel arithmetic lives here.
#include "../../include/moe.h"
#include "common.cuh"

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

namespace moe {

static thread_local std::string g_last_error;
static thread_local void* const* g_prof_events = nullptr;
static thread_local int g_prof_n = 0;

// Records the profiling event of kernel i (begin or end) if the hook is armed.
void prof_mark(int i, bool end, cudaStream_t s) {
  if (g_prof_events && i < g_prof_n) cudaEventRecord(static_cast<cudaEvent_t>(g_prof_events[2 * i + (end ? 1 : 0)]), s);
}

moe_status set_error(moe_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

moe_status cuda_fail(cudaError_t e, const char* what) {
  return set_error(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

static bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

moe_status check_shape(const moe_shape* s) {
  if (!s) return set_error(MOE_ERR_INVALID, "shape is NULL");
  if (s->group != kGroup) return set_error(MOE_ERR_INVALID, "group must be 64 (got %d)", s->group);
  if (s->bits != 4 && s->bits != 8) return set_error(MOE_ERR_INVALID, "bits must be 4 or 8 (got %d)", s->bits);
  if (s->hidden <= 0 || s->hidden % kGroup)
    return set_error(MOE_ERR_INVALID, "hidden must be a positive multiple of 64 (got %d)", s->hidden);
  if (s->inter <= 0 || s->inter % kGroup)
    return set_error(MOE_ERR_INVALID, "inter must be a positive multiple of 64 (got %d)", s->inter);
  if (s->shared_inter <= 0 || s->shared_inter % kGroup)
    return set_error(MOE_ERR_INVALID, "shared_inter must be a positive multiple of 64 (got %d)", s->shared_inter);
  if (s->n_experts < 1 || s->n_experts > kMaxExperts)
    return set_error(MOE_ERR_INVALID, "n_experts must be in [1, %d] (got %d)", kMaxExperts, s->n_experts);
  if (s->top_k < 1 || s->top_k > s->n_experts || s->top_k > kMaxTopK)
    return set_error(MOE_ERR_INVALID, "top_k must be in [1, min(E, %d)] (got %d)", kMaxTopK, s->top_k);
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_last_error(void) { return g_last_error.c_str(); }

const char* moe_version(void) { return "moe-b200 0.1 (sm_100a)"; }

moe_status moe_blob_layout(int32_t hidden, int32_t inter, int32_t bits, int32_t group, int64_t offsets[9],
                           int64_t* stride) {
  if (!offsets || !stride) return set_error(MOE_ERR_INVALID, "offsets/stride is NULL");
  if (group != kGroup) return set_error(MOE_ERR_INVALID, "group must be 64 (got %d)", group);
  if (bits != 4 && bits != 8) return set_error(MOE_ERR_INVALID, "bits must be 4 or 8 (got %d)", bits);
  if (hidden <= 0 || hidden % kGroup || inter <= 0 || inter % kGroup)
    return set_error(MOE_ERR_INVALID, "hidden and inter must be positive multiples of 64");
  const BlobLayout L = make_blob_layout(hidden, inter, bits);
  for (int i = 0; i < 9; ++i) offsets[i] = L.off[i];
  *stride = L.stride;
  return MOE_OK;
}

moe_status moe_workspace_size(const moe_shape* shape, int32_t T, size_t* bytes) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!bytes) return set_error(MOE_ERR_INVALID, "bytes is NULL");
  if (T < 1) return set_error(MOE_ERR_INVALID, "T must be >= 1 (got %d)", T);
  // one size serves every call on T tokens: the decode layout (T <= 8), the prefill layout,
  // and moe_group_pairs (which uses the prefill layout at any T)
  const size_t dec = make_ws_layout(T, shape->n_experts, shape->top_k, shape->inter, shape->shared_inter).total;
  const size_t pre = make_prefill_layout(T, shape->n_experts, shape->top_k, shape->hidden, shape->inter).total;
  *bytes = dec > pre ? dec : pre;
  return MOE_OK;
}

// Shapes whose many-token routing runs on the tensor cores (router GEMM + certified top-k).
static bool route_shape_many(const moe_shape* s) {
  return s->hidden % 128 == 0 && s->hidden <= 4096 && s->n_experts <= 512;
}

static moe_status fill_decode_args(const moe_shape* shape, int32_t T, void* ws, size_t ws_bytes, DecodeArgs* a) {
  memset(a, 0, sizeof *a);
  if (T < 1 || T > kMaxDecodeT)
    return set_error(MOE_ERR_UNSUPPORTED, "T must be in [1, %d] on the decode path (got %d)", kMaxDecodeT, T);
  if (!ws || !aligned(ws, kAlign)) return set_error(MOE_ERR_INVALID, "ws must be non-NULL and 256-byte aligned");
  const WsLayout W = make_ws_layout(T, shape->n_experts, shape->top_k, shape->inter, shape->shared_inter);
  if (ws_bytes < W.total)
    return set_error(MOE_ERR_INVALID, "ws_bytes %zu < required %zu", ws_bytes, W.total);
  char* b = static_cast<char*>(ws);
  a->H = shape->hidden;
  a->I = shape->inter;
  a->Is = shape->shared_inter;
  a->E = shape->n_experts;
  a->k = shape->top_k;
  a->T = T;
  a->L = make_blob_layout(shape->hidden, shape->inter, shape->bits);
  a->Ls = make_blob_layout(shape->hidden, shape->shared_inter, shape->bits);
  a->ctrl = reinterpret_cast<Ctrl*>(b + W.ctrl);
  a->logits = reinterpret_cast<double*>(b + W.logits);
  a->topk_idx = reinterpret_cast<int32_t*>(b + W.topk_idx);
  a->topk_w = reinterpret_cast<float*>(b + W.topk_w);
  a->gate = reinterpret_cast<float*>(b + W.gate);
  a->order = reinterpret_cast<int32_t*>(b + W.order);
  a->act_e = reinterpret_cast<int32_t*>(b + W.act_e);
  a->act_begin = reinterpret_cast<int32_t*>(b + W.act_begin);
  a->h = reinterpret_cast<float*>(b + W.h);
  a->hs = reinterpret_cast<float*>(b + W.hs);
  return MOE_OK;
}

moe_status moe_router_topk(const moe_shape* shape, const void* x, int32_t T, const void* w_router,
                           const float* router_bias, int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                           void* stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!x || !w_router || !topk_idx || !topk_w)
    return set_error(MOE_ERR_INVALID, "x, w_router, topk_idx and topk_w must be non-NULL");
  if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(topk_idx, 4) || !aligned(topk_w, 4) ||
      (router_bias && !aligned(router_bias, 4)))
    return set_error(MOE_ERR_INVALID, "x and w_router must be 16-byte aligned");
  if (T < 1) return set_error(MOE_ERR_INVALID, "T must be >= 1 (got %d)", T);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T > kMaxDecodeT && route_shape_many(shape)) {
    // many tokens: tensor-core logits with the certified exact recheck (the routing step of
    // the many-token layer forward)
    const int E = shape->n_experts, k = shape->top_k, H = shape->hidden;
    if (!ws || !aligned(ws, kAlign)) return set_error(MOE_ERR_INVALID, "ws must be non-NULL and 256-byte aligned");
    const PrefillLayout W = make_prefill_layout(T, E, k, H, shape->inter);
    if (ws_bytes < W.total) return set_error(MOE_ERR_INVALID, "ws_bytes %zu < required %zu", ws_bytes, W.total);
    char* b = static_cast<char*>(ws);
    PrefillArgs p{};
    p.T = T;
    p.E = E;
    p.k = k;
    p.H = H;
    p.I = shape->inter;
    p.x = static_cast<const uint16_t*>(x);
    p.wr = static_cast<const uint16_t*>(w_router);
    p.wsg = p.wr;  // the shared-gate logit is not needed here: its row is the first router row
    p.rbias = router_bias;
    p.route = true;
    p.ctrl = reinterpret_cast<Ctrl*>(b + W.ctrl);
    p.xnorm = reinterpret_cast<double*>(b + W.xnorm);
    p.wnorm = reinterpret_cast<double*>(b + W.wnorm);
    p.logits = reinterpret_cast<float*>(b + W.logits);
    p.topk_idx = topk_idx;
    p.topk_w = topk_w;
    p.gate = reinterpret_cast<float*>(b + W.gate);
    p.units_rt = reinterpret_cast<GemmUnit*>(b + W.units_rt);
    p.n_units = reinterpret_cast<int*>(b + W.n_units);
    GemmArgs& g = p.g;
    g.H = H;
    g.I = shape->inter;
    g.E = E;
    g.k = k;
    g.T = T;
    g.x = p.x;
    g.wr = p.wr;
    g.wsg = p.wsg;
    g.logits = p.logits;
    g.ctrl = p.ctrl;
    prof_mark(0, false, s);
    cudaError_t e = launch_prefill_route(p, s);
    if (e != cudaSuccess) return cuda_fail(e, "router launch");
    prof_mark(0, true, s);
    return MOE_OK;
  }
  // up to 8 tokens at a time on the decode router (fp64 sums of exact products)
  prof_mark(0, false, s);
  for (int32_t t0 = 0; t0 < T; t0 += kMaxDecodeT) {
    const int32_t Tc = T - t0 < kMaxDecodeT ? T - t0 : kMaxDecodeT;
    DecodeArgs a;
    if ((st = fill_decode_args(shape, Tc, ws, ws_bytes, &a)) != MOE_OK) return st;
    a.x = static_cast<const uint16_t*>(x) + (size_t)t0 * shape->hidden;
    a.wr = static_cast<const uint16_t*>(w_router);
    a.rbias = router_bias;
    // The shared-gate row is not needed here; point it at the first router row (its logit
    // lands in the workspace and is ignored).
    a.wsg = a.wr;
    a.topk_idx = topk_idx + (size_t)t0 * shape->top_k;
    a.topk_w = topk_w + (size_t)t0 * shape->top_k;
    cudaError_t e = launch_router_decode(a, false, s);
    if (e != cudaSuccess) return cuda_fail(e, "router launch");
  }
  prof_mark(0, true, s);
  return MOE_OK;
}

static moe_status run_fused_stack(const moe_shape* shape, int32_t T, const moe_layer_desc* L, int32_t n,
                                  const DecodeArgs& a, cudaStream_t s, float* out_partial = nullptr,
                                  int with_shared = 1) {
  static FusedArgs f;  // large (kMaxFusedLayers descriptors); filled per call under g_fused_mu
  static std::mutex g_fused_mu;
  std::lock_guard<std::mutex> lock(g_fused_mu);
  memset(&f, 0, sizeof f);
  f.H = shape->hidden;
  f.I = shape->inter;
  f.E = shape->n_experts;
  f.k = shape->top_k;
  f.T = T;
  f.bits = shape->bits;
  f.n_layers = n;
  f.L = a.L;
  f.ctrl = a.ctrl;
  f.logits = a.logits;
  f.h = a.h;
  f.hs = a.hs;
  for (int l = 0; l < n; ++l) {
    FusedLayer& d = f.layer[l];
    d.pool = L[l].pool;
    d.slot_table = L[l].slot_table;
    d.n_slots = L[l].n_slots;
    d.wr = static_cast<const uint16_t*>(L[l].w_router);
    d.rbias = L[l].router_bias;
    d.shared = L[l].shared_blob;
    d.wsg = static_cast<const uint16_t*>(L[l].w_shared_gate);
    d.x = static_cast<const uint16_t*>(L[l].x ? L[l].x : L[l - 1].out);
    d.residual = static_cast<const uint16_t*>(L[l].residual);
    d.out = static_cast<uint16_t*>(L[l].out);
    d.topk_idx_out = L[l].topk_idx_out;
    d.topk_w_out = L[l].topk_w_out;
    d.topk_idx_in = L[l].topk_idx_in;
    d.topk_w_in = L[l].topk_w_in;
    d.out_partial = out_partial;  // set only for single-layer partial calls
    d.with_shared = with_shared;
  }
  bool ok = true;
  prof_mark(0, false, s);
  cudaError_t e = launch_fused_decode(f, s, &ok);
  if (e != cudaSuccess) return cuda_fail(e, "fused decode launch");
  if (!ok) return set_error(MOE_ERR_UNSUPPORTED, "no fused decode kernel for this shape");
  prof_mark(0, true, s);
  return MOE_OK;
}

// Argument checks of one layer descriptor (everything but the shape).
static moe_status check_layer(const moe_shape* shape, const moe_layer_desc* d, bool first) {
  if (!d->pool || !d->slot_table || !d->shared_blob || !d->w_shared_gate || !d->out)
    return set_error(MOE_ERR_INVALID, "pool, slot_table, shared_blob, w_shared_gate and out must be non-NULL");
  if (first && !d->x) return set_error(MOE_ERR_INVALID, "the first layer needs x");
  if (!d->topk_idx_in && !d->w_router) return set_error(MOE_ERR_INVALID, "w_router is NULL and no topk_idx_in given");
  if (d->topk_idx_in && !d->topk_w_in) return set_error(MOE_ERR_INVALID, "topk_idx_in given without topk_w_in");
  if ((d->topk_idx_out == nullptr) != (d->topk_w_out == nullptr))
    return set_error(MOE_ERR_INVALID, "topk_idx_out and topk_w_out must both be given or both be NULL");
  if (d->n_slots < 1) return set_error(MOE_ERR_INVALID, "n_slots must be >= 1");
  if ((d->x && !aligned(d->x, 16)) || !aligned(d->out, 16) || (d->w_router && !aligned(d->w_router, 16)) ||
      !aligned(d->w_shared_gate, 16) || (d->residual && !aligned(d->residual, 16)))
    return set_error(MOE_ERR_INVALID, "x, out, w_router, w_shared_gate and residual must be 16-byte aligned");
  if (!aligned(d->pool, kAlign) || !aligned(d->shared_blob, kAlign))
    return set_error(MOE_ERR_INVALID, "pool and shared_blob must be 256-byte aligned");
  (void)shape;
  return MOE_OK;
}

// Many tokens: router GEMM + certified top-k, grouping, tcgen05 grouped GEMMs (prefill.cu).
static moe_status prefill_forward(const moe_shape* shape, const void* x, int32_t T, const void* w_router,
                                  const float* router_bias, const int32_t* topk_idx_in, const float* topk_w_in,
                                  const uint8_t* pool, const int32_t* slot_table, int64_t n_slots,
                                  const uint8_t* shared_blob, const void* w_shared_gate, const void* residual,
                                  void* out, int32_t* topk_idx_out, float* topk_w_out, void* ws, size_t ws_bytes,
                                  cudaStream_t s, float* partial_out = nullptr, int include_shared = 1) {
  if (!prefill_shape_supported(shape->hidden, shape->inter, shape->bits, shape->n_experts))
    return set_error(MOE_ERR_UNSUPPORTED,
                     "no prefill kernel for hidden=%d inter=%d bits=%d E=%d (hidden %% 128 == 0, E <= 512)",
                     shape->hidden, shape->inter, shape->bits, shape->n_experts);
  if (!ws || !aligned(ws, kAlign)) return set_error(MOE_ERR_INVALID, "ws must be non-NULL and 256-byte aligned");
  const int E = shape->n_experts, k = shape->top_k, H = shape->hidden, I = shape->inter;
  const PrefillLayout W = make_prefill_layout(T, E, k, H, I);
  if (ws_bytes < W.total) return set_error(MOE_ERR_INVALID, "ws_bytes %zu < required %zu", ws_bytes, W.total);
  char* b = static_cast<char*>(ws);
  PrefillArgs p{};
  p.T = T;
  p.E = E;
  p.k = k;
  p.H = H;
  p.I = I;
  p.x = static_cast<const uint16_t*>(x);
  p.wr = static_cast<const uint16_t*>(w_router);
  p.wsg = static_cast<const uint16_t*>(w_shared_gate);
  p.rbias = router_bias;
  p.residual = static_cast<const uint16_t*>(residual);
  // a partial forward (expert parallelism): the down products of this rank's experts (and the
  // shared expert's if included) are summed in fp32 straight into partial_out; no residual,
  // no rounding, no finalize
  p.out = partial_out ? nullptr : static_cast<uint16_t*>(out);
  p.no_shared = include_shared ? 0 : 1;
  p.route = (topk_idx_in == nullptr);
  p.ctrl = reinterpret_cast<Ctrl*>(b + W.ctrl);
  p.xnorm = reinterpret_cast<double*>(b + W.xnorm);
  p.wnorm = reinterpret_cast<double*>(b + W.wnorm);
  p.logits = reinterpret_cast<float*>(b + W.logits);
  if (topk_idx_in) {
    p.topk_idx = const_cast<int32_t*>(topk_idx_in);
    p.topk_w = const_cast<float*>(topk_w_in);
  } else if (topk_idx_out) {
    p.topk_idx = topk_idx_out;
    p.topk_w = topk_w_out;
  } else {
    p.topk_idx = reinterpret_cast<int32_t*>(b + W.topk_idx);
    p.topk_w = reinterpret_cast<float*>(b + W.topk_w);
  }
  p.gate = reinterpret_cast<float*>(b + W.gate);
  p.order = reinterpret_cast<int32_t*>(b + W.order);
  p.offsets = reinterpret_cast<int32_t*>(b + W.offsets);
  p.counts = reinterpret_cast<int32_t*>(b + W.counts);
  p.chunk_cnt = reinterpret_cast<int32_t*>(b + W.chunk_cnt);
  p.units_rt = reinterpret_cast<GemmUnit*>(b + W.units_rt);
  p.units_gu = reinterpret_cast<GemmUnit*>(b + W.units_gu);
  p.units_dn = reinterpret_cast<GemmUnit*>(b + W.units_dn);
  p.n_units = reinterpret_cast<int*>(b + W.n_units);
  p.acc = partial_out ? partial_out : reinterpret_cast<float*>(b + W.acc);
  p.h = reinterpret_cast<uint16_t*>(b + W.h);
  p.hs = reinterpret_cast<uint16_t*>(b + W.hs);
  p.xg = reinterpret_cast<uint16_t*>(b + W.xg);
  p.xp = reinterpret_cast<uint16_t*>(b + W.xp);
  p.perm = shape->bits == 4 ? 1 : 0;
  GemmArgs& g = p.g;
  g.H = H;
  g.I = I;
  g.E = E;
  g.k = k;
  g.T = T;
  g.pool = pool;
  g.slot_table = slot_table;
  g.n_slots = n_slots;
  g.shared = shared_blob;
  g.L = make_blob_layout(H, I, shape->bits);
  g.x = p.x;
  g.wr = p.wr;
  g.wsg = p.wsg;
  g.order = p.order;
  g.topk_w = p.topk_w;
  g.gate = p.gate;
  g.h = p.h;
  g.hs = p.hs;
  g.acc = p.acc;
  g.logits = p.logits;
  g.ctrl = p.ctrl;
  cudaError_t e = launch_prefill(p, shape->bits, s);
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  return MOE_OK;
}

moe_status moe_layer_forward(const moe_shape* shape, const void* x, int32_t T, const void* w_router,
                             const float* router_bias, const int32_t* topk_idx_in, const float* topk_w_in,
                             const uint8_t* pool, const int32_t* slot_table, int64_t n_slots,
                             const uint8_t* shared_blob, const void* w_shared_gate, const void* residual, void* out,
                             int32_t* topk_idx_out, float* topk_w_out, void* ws, size_t ws_bytes, void* stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (shape->shared_inter != shape->inter)
    return set_error(MOE_ERR_UNSUPPORTED, "this library needs shared_inter == inter (%d vs %d)", shape->shared_inter,
                     shape->inter);
  if (!decode_shape_supported(shape->hidden, shape->inter, shape->bits))
    return set_error(MOE_ERR_UNSUPPORTED,
                     "no decode kernel for hidden=%d inter=%d bits=%d (hidden: power of two in [256, 4096], "
                     "inter: power of two in [64, 1024])",
                     shape->hidden, shape->inter, shape->bits);
  if (!x || !pool || !slot_table || !shared_blob || !w_shared_gate || !out)
    return set_error(MOE_ERR_INVALID, "x, pool, slot_table, shared_blob, w_shared_gate and out must be non-NULL");
  if (!topk_idx_in && !w_router) return set_error(MOE_ERR_INVALID, "w_router is NULL and no topk_idx_in given");
  if (topk_idx_in && !topk_w_in) return set_error(MOE_ERR_INVALID, "topk_idx_in given without topk_w_in");
  if ((topk_idx_out == nullptr) != (topk_w_out == nullptr))
    return set_error(MOE_ERR_INVALID, "topk_idx_out and topk_w_out must both be given or both be NULL");
  if (n_slots < 1) return set_error(MOE_ERR_INVALID, "n_slots must be >= 1");
  if (!aligned(x, 16) || !aligned(out, 16) || (w_router && !aligned(w_router, 16)) ||
      !aligned(w_shared_gate, 16) || (residual && !aligned(residual, 16)))
    return set_error(MOE_ERR_INVALID, "x, out, w_router, w_shared_gate and residual must be 16-byte aligned");
  if (!aligned(pool, kAlign) || !aligned(shared_blob, kAlign))
    return set_error(MOE_ERR_INVALID, "pool and shared_blob must be 256-byte aligned");
  if (T > kMaxDecodeT)
    return prefill_forward(shape, x, T, w_router, router_bias, topk_idx_in, topk_w_in, pool, slot_table, n_slots,
                           shared_blob, w_shared_gate, residual, out, topk_idx_out, topk_w_out, ws, ws_bytes,
                           static_cast<cudaStream_t>(stream));
  DecodeArgs a;
  if ((st = fill_decode_args(shape, T, ws, ws_bytes, &a)) != MOE_OK) return st;
  a.x = static_cast<const uint16_t*>(x);
  a.wr = static_cast<const uint16_t*>(w_router);
  a.rbias = router_bias;
  a.wsg = static_cast<const uint16_t*>(w_shared_gate);
  a.pool = pool;
  a.slot_table = slot_table;
  a.n_slots = n_slots;
  a.shared_blob = shared_blob;
  a.residual = static_cast<const uint16_t*>(residual);
  a.out = static_cast<uint16_t*>(out);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (fused_shape_supported(shape->hidden, shape->inter, shape->bits, shape->n_experts)) {
    moe_layer_desc d{};
    d.x = x;
    d.w_router = w_router;
    d.router_bias = router_bias;
    d.topk_idx_in = topk_idx_in;
    d.topk_w_in = topk_w_in;
    d.pool = pool;
    d.slot_table = slot_table;
    d.n_slots = n_slots;
    d.shared_blob = shared_blob;
    d.w_shared_gate = w_shared_gate;
    d.residual = residual;
    d.out = out;
    d.topk_idx_out = topk_idx_out;
    d.topk_w_out = topk_w_out;
    return run_fused_stack(shape, T, &d, 1, a, s);
  }
  prof_mark(0, false, s);
  if (!topk_idx_in) {
    if (topk_idx_out) {
      a.topk_idx = topk_idx_out;
      a.topk_w = topk_w_out;
    }
    e = launch_router_decode(a, true, s);
    if (e != cudaSuccess) return cuda_fail(e, "router launch");
  } else {
    a.topk_idx = const_cast<int32_t*>(topk_idx_in);
    a.topk_w = const_cast<float*>(topk_w_in);
    e = launch_plan_decode(a, s);
    if (e != cudaSuccess) return cuda_fail(e, "plan launch");
  }
  prof_mark(0, true, s);
  bool ok = true;
  prof_mark(1, false, s);
  e = launch_gateup_decode(a, shape->bits, s, &ok);
  if (e != cudaSuccess) return cuda_fail(e, "gate/up launch");
  prof_mark(1, true, s);
  prof_mark(2, false, s);
  e = launch_down_decode(a, shape->bits, s, &ok);
  if (e != cudaSuccess) return cuda_fail(e, "down launch");
  prof_mark(2, true, s);
  return MOE_OK;
}

moe_status moe_layer_forward_partial(const moe_shape* shape, const void* x, int32_t T, const void* w_router,
                                     const float* router_bias, const int32_t* topk_idx_in, const float* topk_w_in,
                                     const uint8_t* pool, const int32_t* slot_table, int64_t n_slots,
                                     const uint8_t* shared_blob, const void* w_shared_gate, int32_t include_shared,
                                     float* partial_out, int32_t* topk_idx_out, float* topk_w_out, void* ws,
                                     size_t ws_bytes, void* stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (shape->shared_inter != shape->inter)
    return set_error(MOE_ERR_UNSUPPORTED, "this library needs shared_inter == inter");
  if (T < 1) return set_error(MOE_ERR_INVALID, "T must be >= 1 (got %d)", T);
  if (T <= kMaxDecodeT && !fused_shape_supported(shape->hidden, shape->inter, shape->bits, shape->n_experts))
    return set_error(MOE_ERR_UNSUPPORTED, "no fused decode kernel for hidden=%d inter=%d bits=%d E=%d",
                     shape->hidden, shape->inter, shape->bits, shape->n_experts);
  if (!partial_out || !aligned(partial_out, 16)) return set_error(MOE_ERR_INVALID, "partial_out must be non-NULL and 16-byte aligned");
  if (include_shared != 0 && include_shared != 1) return set_error(MOE_ERR_INVALID, "include_shared must be 0 or 1");
  if (T > kMaxDecodeT) {
    // many tokens: the prefill path over this rank's experts, summed into partial_out
    moe_layer_desc d{};
    d.x = x;
    d.w_router = w_router;
    d.router_bias = router_bias;
    d.topk_idx_in = topk_idx_in;
    d.topk_w_in = topk_w_in;
    d.pool = pool;
    d.slot_table = slot_table;
    d.n_slots = n_slots;
    d.shared_blob = shared_blob;
    d.w_shared_gate = w_shared_gate;
    d.out = partial_out;
    d.topk_idx_out = topk_idx_out;
    d.topk_w_out = topk_w_out;
    if ((st = check_layer(shape, &d, true)) != MOE_OK) return st;
    return prefill_forward(shape, x, T, w_router, router_bias, topk_idx_in, topk_w_in, pool, slot_table, n_slots,
                           shared_blob, w_shared_gate, nullptr, nullptr, topk_idx_out, topk_w_out, ws, ws_bytes,
                           static_cast<cudaStream_t>(stream), partial_out, include_shared);
  }
  moe_layer_desc d{};
  d.x = x;
  d.w_router = w_router;
  d.router_bias = router_bias;
  d.topk_idx_in = topk_idx_in;
  d.topk_w_in = topk_w_in;
  d.pool = pool;
  d.slot_table = slot_table;
  d.n_slots = n_slots;
  d.shared_blob = shared_blob;
  d.w_shared_gate = w_shared_gate;
  d.residual = nullptr;
  d.out = partial_out;  // checked for alignment only; the kernel writes partial_out
  d.topk_idx_out = topk_idx_out;
  d.topk_w_out = topk_w_out;
  if ((st = check_layer(shape, &d, true)) != MOE_OK) return st;
  DecodeArgs a;
  if ((st = fill_decode_args(shape, T, ws, ws_bytes, &a)) != MOE_OK) return st;
  return run_fused_stack(shape, T, &d, 1, a, static_cast<cudaStream_t>(stream), partial_out, include_shared);
}

moe_status moe_combine_partials(const float* const* partials, int32_t n_parts, int32_t T, int32_t hidden,
                                const void* residual, void* out, void* stream) {
  if (!partials || !out) return set_error(MOE_ERR_INVALID, "partials and out must be non-NULL");
  if (n_parts < 1 || n_parts > kMaxPartials)
    return set_error(MOE_ERR_INVALID, "n_parts must be in [1, %d] (got %d)", kMaxPartials, n_parts);
  if (T < 1 || hidden < 1) return set_error(MOE_ERR_INVALID, "T and hidden must be >= 1");
  PartialArgs p{};
  for (int i = 0; i < n_parts; ++i) {
    if (!partials[i] || !aligned(partials[i], 16)) return set_error(MOE_ERR_INVALID, "partial %d is NULL or misaligned", i);
    p.part[i] = partials[i];
  }
  if (!aligned(out, 16) || (residual && !aligned(residual, 16)))
    return set_error(MOE_ERR_INVALID, "out and residual must be 16-byte aligned");
  p.n = n_parts;
  p.count = (size_t)T * hidden;
  p.residual = static_cast<const uint16_t*>(residual);
  p.out = static_cast<uint16_t*>(out);
  cudaError_t e = launch_combine_partials(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "combine launch");
  return MOE_OK;
}

moe_status moe_stack_forward(const moe_shape* shape, int32_t T, const moe_layer_desc* layers, int32_t n_layers,
                             void* ws, size_t ws_bytes, void* stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!layers) return set_error(MOE_ERR_INVALID, "layers is NULL");
  if (n_layers < 1 || n_layers > kMaxFusedLayers)
    return set_error(MOE_ERR_INVALID, "n_layers must be in [1, %d] (got %d)", kMaxFusedLayers, n_layers);
  if (shape->shared_inter != shape->inter)
    return set_error(MOE_ERR_UNSUPPORTED, "this library needs shared_inter == inter");
  if (!decode_shape_supported(shape->hidden, shape->inter, shape->bits))
    return set_error(MOE_ERR_UNSUPPORTED, "no decode kernel for hidden=%d inter=%d bits=%d", shape->hidden,
                     shape->inter, shape->bits);
  for (int l = 0; l < n_layers; ++l)
    if ((st = check_layer(shape, &layers[l], l == 0)) != MOE_OK) return st;
  DecodeArgs a;
  if ((st = fill_decode_args(shape, T, ws, ws_bytes, &a)) != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (fused_shape_supported(shape->hidden, shape->inter, shape->bits, shape->n_experts))
    return run_fused_stack(shape, T, layers, n_layers, a, s);
  for (int l = 0; l < n_layers; ++l) {
    const moe_layer_desc& d = layers[l];
    st = moe_layer_forward(shape, d.x ? d.x : layers[l - 1].out, T, d.w_router, d.router_bias, d.topk_idx_in,
                           d.topk_w_in, d.pool, d.slot_table, d.n_slots, d.shared_blob, d.w_shared_gate, d.residual,
                           d.out, d.topk_idx_out, d.topk_w_out, ws, ws_bytes, stream);
    if (st != MOE_OK) return st;
  }
  return MOE_OK;
}

moe_status moe_group_pairs(const moe_shape* shape, int32_t T, const int32_t* topk_idx, int32_t* order,
                           int32_t* offsets, void* ws, size_t ws_bytes, void* stream) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (T < 1) return set_error(MOE_ERR_INVALID, "T must be >= 1 (got %d)", T);
  if (!topk_idx || !order || !offsets) return set_error(MOE_ERR_INVALID, "topk_idx, order and offsets must be non-NULL");
  if (shape->n_experts > 512) return set_error(MOE_ERR_UNSUPPORTED, "grouping supports E <= 512");
  if (!ws || !aligned(ws, kAlign)) return set_error(MOE_ERR_INVALID, "ws must be non-NULL and 256-byte aligned");
  const int E = shape->n_experts, k = shape->top_k;
  const PrefillLayout W = make_prefill_layout(T, E, k, shape->hidden, shape->inter);
  if (ws_bytes < W.total) return set_error(MOE_ERR_INVALID, "ws_bytes %zu < required %zu", ws_bytes, W.total);
  char* b = static_cast<char*>(ws);
  PrefillArgs p{};
  p.T = T;
  p.E = E;
  p.k = k;
  p.H = shape->hidden;
  p.I = shape->inter;
  p.ctrl = reinterpret_cast<Ctrl*>(b + W.ctrl);
  p.topk_idx = const_cast<int32_t*>(topk_idx);
  p.order = order;
  p.offsets = offsets;
  p.counts = reinterpret_cast<int32_t*>(b + W.counts);
  p.chunk_cnt = reinterpret_cast<int32_t*>(b + W.chunk_cnt);
  p.units_gu = reinterpret_cast<GemmUnit*>(b + W.units_gu);
  p.units_dn = reinterpret_cast<GemmUnit*>(b + W.units_dn);
  p.n_units = reinterpret_cast<int*>(b + W.n_units);
  cudaError_t e = launch_group(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "grouping launch");
  return MOE_OK;
}

moe_status moe_profile_events(void* const* events, int32_t n) {
  if (events && n < 0) return set_error(MOE_ERR_INVALID, "n must be >= 0");
  g_prof_events = events;
  g_prof_n = events ? n : 0;
  return MOE_OK;
}

namespace {
__global__ void k_set_u32(uint32_t* p, uint32_t v) { *p = v; }
}  // namespace

moe_status moe_ws_set_slot_wait(void* ws, uint32_t microseconds, void* stream) {
  if (!ws || !aligned(ws, kAlign)) return set_error(MOE_ERR_INVALID, "ws must be non-NULL and 256-byte aligned");
  Ctrl* c = static_cast<Ctrl*>(ws);
  k_set_u32<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(&c->slot_wait_us, microseconds);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "slot wait setting");
  return MOE_OK;
}

moe_status moe_ws_router_logits(const moe_shape* shape, int32_t T, void* ws, size_t ws_bytes, float** logits) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!ws || !logits) return set_error(MOE_ERR_INVALID, "ws and logits must be non-NULL");
  if (T <= kMaxDecodeT) return set_error(MOE_ERR_INVALID, "T must be > %d (the many-token layout)", kMaxDecodeT);
  const PrefillLayout W = make_prefill_layout(T, shape->n_experts, shape->top_k, shape->hidden, shape->inter);
  if (ws_bytes < W.total) return set_error(MOE_ERR_INVALID, "ws_bytes %zu < required %zu", ws_bytes, W.total);
  *logits = reinterpret_cast<float*>(static_cast<char*>(ws) + W.logits);
  return MOE_OK;
}

moe_status moe_ws_check(void* ws, void* stream, uint32_t* flags) {
  if (!ws || !flags) return set_error(MOE_ERR_INVALID, "ws and flags must be non-NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  uint32_t v = 0;
  e = cudaMemcpy(&v, ws, sizeof v, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "error word read");
  if (v) {
    const uint32_t zero = 0;
    e = cudaMemcpy(ws, &zero, sizeof zero, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "error word clear");
  }
  *flags = v;
  if (v) return set_error(MOE_ERR_DEVICE, "device error bits 0x%x", v);
  return MOE_OK;
}

}  // extern "C"
