// Internal declarations shared by the sm_100a kernels and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

namespace moe {

constexpr int kGroup = 64;      // quantisation group along the input dimension
constexpr int kAlign = 256;     // blob section / workspace alignment
constexpr int kMaxDecodeT = 8;  // tokens per call on the GEMV (decode) path
constexpr int kMaxTopK = 32;
constexpr int kMaxExperts = 1024;

// Slot-table entry of an expert whose blob is still being copied into its slot (a pool in
// overlap mode); the copy stream overwrites it with the slot once the blob has landed.
constexpr int32_t kSlotPending = -2;
// Slot-table entry of an expert that another rank holds (expert parallelism): the pair is
// left out of this rank's partial sum without an error.
constexpr int32_t kSlotRemote = -3;

// Device error-word bits (mirrors MOE_DEVERR_* in include/moe.h).
constexpr uint32_t kErrBadExpert = 0x1u;
constexpr uint32_t kErrBadSlot = 0x2u;
constexpr uint32_t kErrNonFinite = 0x4u;
constexpr uint32_t kErrTimeout = 0x8u;

// ---------------------------------------------------------------------------------------
// Fixed-stride expert blob: nine 256-byte aligned sections (gate/up/down codes, then
// gate scale, gate bias, up scale, up bias, down scale, down bias).
// ---------------------------------------------------------------------------------------
struct BlobLayout {
  int64_t off[9];
  int64_t stride;
};

inline int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

inline BlobLayout make_blob_layout(int H, int I, int bits) {
  BlobLayout L{};
  const int64_t codes_gu = (int64_t)I * H * bits / 8;
  const int64_t codes_d = (int64_t)H * I * bits / 8;
  const int64_t sb_gu = (int64_t)I * (H / kGroup) * 2;
  const int64_t sb_d = (int64_t)H * (I / kGroup) * 2;
  const int64_t size[9] = {codes_gu, codes_gu, codes_d, sb_gu, sb_gu, sb_gu, sb_gu, sb_d, sb_d};
  int64_t pos = 0;
  for (int i = 0; i < 9; ++i) {
    pos = round_up(pos, kAlign);
    L.off[i] = pos;
    pos += size[i];
  }
  L.stride = round_up(pos, kAlign);
  return L;
}

// ---------------------------------------------------------------------------------------
// Workspace: a control block, then fixed-size arrays, each 256-byte aligned.
// ---------------------------------------------------------------------------------------
struct Ctrl {
  uint32_t err;     // sticky MOE_DEVERR_* bits (cleared by moe_ws_check)
  uint32_t ticket;  // last-block-done counter of the router (always returns to 0)
  int32_t act_n;    // number of distinct routed experts of the current call
  int32_t n_valid;  // number of (token, k) pairs with a valid expert id
  uint32_t bar_count;  // fused decode kernel: grid-barrier arrivals (back to 0 at exit)
  uint32_t bar_gen;    // fused decode kernel: CTAs that have exited (back to 0 at exit)
  uint32_t slot_wait_us;  // bound of the fused decode kernel's waits for pending slot-table
                          // entries, microseconds (0: kWaitNs); a setting, not a counter
  uint32_t pad[57];
};
static_assert(sizeof(Ctrl) == 256, "ctrl block is 256 bytes");

struct WsLayout {
  size_t ctrl, logits, topk_idx, topk_w, gate, order, act_e, act_begin, h, hs, total;
};

inline WsLayout make_ws_layout(int T, int E, int k, int I, int Is) {
  WsLayout W{};
  size_t pos = 0;
  auto take = [&](size_t bytes) {
    size_t at = (size_t)round_up((int64_t)pos, kAlign);
    pos = at + bytes;
    return at;
  };
  W.ctrl = take(sizeof(Ctrl));
  W.logits = take(sizeof(double) * (size_t)T * (E + 1));
  W.topk_idx = take(sizeof(int32_t) * (size_t)T * k);
  W.topk_w = take(sizeof(float) * (size_t)T * k);
  W.gate = take(sizeof(float) * (size_t)T);
  W.order = take(sizeof(int32_t) * (size_t)T * k);
  W.act_e = take(sizeof(int32_t) * (size_t)T * k);
  W.act_begin = take(sizeof(int32_t) * ((size_t)T * k + 1));
  W.h = take(sizeof(float) * (size_t)T * k * I);
  W.hs = take(sizeof(float) * (size_t)T * Is);
  W.total = (size_t)round_up((int64_t)pos, kAlign);
  return W;
}

// Everything one decode-path layer call needs, as raw pointers.
struct DecodeArgs {
  int H, I, Is, E, k, T;
  const uint16_t* x;         // bf16 [T, H]
  const uint16_t* wr;        // bf16 [E, H]
  const float* rbias;        // fp32 [E] or null
  const uint16_t* wsg;       // bf16 [H]
  const uint8_t* pool;       // n_slots * stride
  const int32_t* slot_table; // [E]
  int64_t n_slots;
  const uint8_t* shared_blob;
  const uint16_t* residual;  // bf16 [T, H] or null
  uint16_t* out;             // bf16 [T, H]
  int32_t* topk_idx;         // [T, k]  (router output, or caller-given input)
  float* topk_w;             // [T, k]
  BlobLayout L, Ls;
  // workspace
  Ctrl* ctrl;
  double* logits;            // [T, E+1] (column E: shared-gate logit)
  float* gate;               // [T]
  int32_t* order;            // [T*k] pair numbers sorted by expert (stable)
  int32_t* act_e;            // [T*k] distinct experts, ascending
  int32_t* act_begin;        // [T*k+1] first sorted position of each distinct expert
  float* h;                  // [T*k, I]  SwiGLU intermediate per sorted pair
  float* hs;                 // [T, Is]   shared-expert intermediate per token
};

// Shared-memory carve of the fused kernel (byte offsets from the dynamic base), used by the
// host to size the launch and by the kernel to find its arrays.
struct FusedSmem {
  uint32_t xs4, xsum, partial, ids, pw, order, pos_of, act_e, act_slot, act_begin, gate, scratch, slot, topk, red,
      rbuf, rpart, total;
};
// Per-token top-k scratch of the fused kernel: 32 lane maxima (double + id), 64 candidates
// (double + id), a counter and the threshold lane.
constexpr int kTopkScratchBytes = 32 * 8 + 32 * 4 + 64 * 8 + 64 * 4 + 16;
// rr_max, rs_max: router rows and shared-expert rows one CTA stages for phase R.
__host__ __device__ inline FusedSmem fused_smem_layout(int T, int H, int I, int E, int bits, int k, int jmax,
                                                       int n_stages, int stage_bytes, int n_cons, int rr_max,
                                                       int rs_max) {
  FusedSmem m{};
  size_t off = (size_t)n_stages * stage_bytes;
  auto carve = [&](size_t bytes) {
    off = (off + 15) / 16 * 16;
    const uint32_t at = (uint32_t)off;
    off += bytes;
    return at;
  };
  const int CC = 128 / bits, NC = H / CC, TK = T * k;
  const int NCd = I / CC, NCLd = NCd < 32 ? NCd : 32;
  m.xs4 = carve((size_t)T * H * 4);
  m.xsum = carve((size_t)T * NC * 4);
  m.partial = carve((size_t)(TK + T) * jmax * 4);
  m.ids = carve((size_t)TK * 4);
  m.pw = carve((size_t)TK * 4);
  m.order = carve((size_t)TK * 4);
  m.pos_of = carve((size_t)TK * 4);
  m.act_e = carve((size_t)TK * 4);
  m.act_slot = carve((size_t)TK * 4);
  m.act_begin = carve((size_t)(TK + 1) * 4);
  m.gate = carve((size_t)T * 4);
  m.scratch = carve((size_t)5 * TK * 4);
  m.slot = carve((size_t)E * 4);
  m.topk = carve((size_t)T * kTopkScratchBytes);
  m.red = carve((size_t)n_cons * jmax * (NCLd + 1) * 4);
  const size_t rowg = 2 * (size_t)H * bits / 8 + 4 * (size_t)(H / kGroup) * 2;
  m.rbuf = carve((size_t)rr_max * H * 2 + (size_t)rs_max * rowg);
  m.rpart = carve((size_t)rr_max * 4 * T * 8);
  m.total = (uint32_t)((off + 127) / 128 * 128);
  return m;
}

// One layer of a fused decode stack (see decode_fused.cu).
struct FusedLayer {
  const uint8_t* pool;
  const int32_t* slot_table;
  int64_t n_slots;
  const uint16_t* wr;
  const float* rbias;
  const uint8_t* shared;
  const uint16_t* wsg;
  const uint16_t* x;
  const uint16_t* residual;
  uint16_t* out;
  int32_t* topk_idx_out;
  float* topk_w_out;
  const int32_t* topk_idx_in;
  const float* topk_w_in;
  float* out_partial;  // fp32 [T, H]: if set, the layer's partial sum goes here (no residual, no rounding)
  int with_shared;     // 1: the shared expert is part of this layer's sum
};
constexpr int kMaxFusedLayers = 64;

struct FusedArgs {
  int H, I, E, k, T, n_layers, bits;
  int n_stages, stage_bytes, jmax;
  int rr_max, rs_max;  // most router rows / shared-expert rows a CTA stages for phase R
  FusedSmem sm;        // shared-memory carve (host-computed)
  BlobLayout L;
  Ctrl* ctrl;
  double* logits;
  float* h;
  float* hs;
  FusedLayer layer[kMaxFusedLayers];
};

// ---------------------------------------------------------------------------------------
// Prefill path (prefill.cu)
// ---------------------------------------------------------------------------------------
constexpr int kModeRouter = 0, kModeGateUp = 1, kModeDown = 2;
constexpr int kPrefillN = 128;  // tokens (the MMA's M) per GEMM work unit
constexpr int kGroupChunk = 512;  // (token, k) pairs per CTA of the grouping kernels

// One tcgen05 GEMM work unit: expert e (-1: shared expert, -2: router), row tile mt, first
// column p0 (pair position, or token for the shared expert / router) and column count n.
struct GemmUnit {
  int e, mt, p0, n;
};

struct GemmArgs {
  int H, I, E, k, T;
  const uint8_t* pool;
  const int32_t* slot_table;
  int64_t n_slots;
  const uint8_t* shared;
  BlobLayout L;
  const uint16_t* x;    // bf16 [T, H]
  const uint16_t* wr;   // bf16 [E, H]
  const uint16_t* wsg;  // bf16 [H]
  const int32_t* order; // [T*k] pair numbers sorted by expert
  const float* topk_w;  // [T*k]
  const float* gate;    // [T]
  uint16_t* h;          // bf16 [T*k, I] per sorted pair
  uint16_t* hs;         // bf16 [T, I] shared expert
  float* acc;           // fp32 [T, H]
  float* logits;        // fp32 [T, E+1] (no bias)
  const GemmUnit* units;
  const int* n_units;
  Ctrl* ctrl;
  int n_rows;           // weight rows per work unit (the MMA's N): 128 or 256
  int perm;             // the gate/up epilogue writes h in k-octet order
  int sc_tma;           // 1: scales and biases arrive by TMA in chunks of 8 groups
  // TMA descriptors (filled by the launcher per GEMM): token rows (routed / shared
  // units), weight rows (router rows, or raw codes of the pool / of the shared blob), and
  // the scale + bias chunks (pool / shared blob)
  alignas(64) CUtensorMap map_tok;
  alignas(64) CUtensorMap map_tok2;
  alignas(64) CUtensorMap map_w;
  alignas(64) CUtensorMap map_w_shared;
  alignas(64) CUtensorMap map_sc;
  alignas(64) CUtensorMap map_sc_shared;
};

// Weight rows per GEMM work unit of the prefill path: gate/up units hold nI intermediate
// rows of both matrices (2*nI rows), down units NR output rows.
__host__ __device__ inline int prefill_gu_rows(int I) { return I % 128 == 0 ? 256 : 128; }
__host__ __device__ inline int prefill_dn_rows(int H) { return H % 256 == 0 ? 256 : 128; }

struct PrefillArgs {
  int T, E, k, H, I;
  const uint16_t* x;
  const uint16_t* wr;
  const uint16_t* wsg;
  const float* rbias;
  const uint16_t* residual;
  uint16_t* out;
  bool route;           // false: topk_idx / topk_w hold the caller's routing
  double* xnorm;        // [T]
  double* wnorm;        // [E+1]
  float* logits;
  int32_t* topk_idx;
  float* topk_w;
  float* gate;
  int32_t* order;
  int32_t* offsets;     // [E+1]
  int32_t* counts;      // [E]
  int32_t* chunk_cnt;   // [ceil(T*k / kGroupChunk)][E]: per-chunk counts, then exclusive sums
  GemmUnit* units_rt;
  GemmUnit* units_gu;
  GemmUnit* units_dn;
  int* n_units;         // [3]: gate/up, down, router
  float* acc;
  uint16_t* h;
  uint16_t* hs;
  uint16_t* xg;         // bf16 [T*k, H]: x rows in grouped pair order
  uint16_t* xp;         // bf16 [T, H]: x for the shared expert's gate/up (k-octet order, int4)
  int perm;             // int4: operands of the expert GEMMs in k-octet order (see prefill.cu)
  int no_shared;        // 1: the shared expert's work units are left out (a partial forward)
  Ctrl* ctrl;
  GemmArgs g;           // shared GEMM arguments (units filled per launch)
};

struct PrefillLayout {
  size_t ctrl, xnorm, wnorm, logits, topk_idx, topk_w, gate, order, offsets, counts, chunk_cnt, units_rt,
      units_gu, units_dn, n_units, acc, h, hs, xg, xp, total;
};

inline PrefillLayout make_prefill_layout(int T, int E, int k, int H, int I) {
  PrefillLayout W{};
  size_t pos = 0;
  auto take = [&](size_t bytes) {
    size_t at = (size_t)round_up((int64_t)pos, kAlign);
    pos = at + bytes;
    return at;
  };
  const size_t tiles = (size_t)E + ((size_t)T * k + kPrefillN - 1) / kPrefillN +
                       ((size_t)T + kPrefillN - 1) / kPrefillN + 1;
  const size_t rt_units = (size_t)((E + 1 + 127) / 128) * ((T + 127) / 128);
  W.ctrl = take(sizeof(Ctrl));
  W.xnorm = take(sizeof(double) * T);
  W.wnorm = take(sizeof(double) * (E + 1));
  W.logits = take(sizeof(float) * (size_t)T * (E + 1));
  W.topk_idx = take(sizeof(int32_t) * (size_t)T * k);
  W.topk_w = take(sizeof(float) * (size_t)T * k);
  W.gate = take(sizeof(float) * T);
  W.order = take(sizeof(int32_t) * (size_t)T * k);
  W.offsets = take(sizeof(int32_t) * (E + 1));
  W.counts = take(sizeof(int32_t) * E);
  W.chunk_cnt = take(sizeof(int32_t) * (size_t)E * (((size_t)T * k + kGroupChunk - 1) / kGroupChunk));
  W.units_rt = take(sizeof(GemmUnit) * rt_units);
  W.units_gu = take(sizeof(GemmUnit) * tiles * (I / 64));
  W.units_dn = take(sizeof(GemmUnit) * tiles * (H / 128));
  W.n_units = take(sizeof(int) * 4);
  W.acc = take(sizeof(float) * (size_t)T * H);
  W.h = take(2 * (size_t)T * k * I);
  W.hs = take(2 * (size_t)T * I);
  W.xg = take(2 * (size_t)T * k * H);
  W.xp = take(2 * (size_t)T * H);
  W.total = (size_t)round_up((int64_t)pos, kAlign);
  return W;
}

bool prefill_shape_supported(int H, int I, int bits, int E);
// Profiling hook of moe_profile_events (api.cu): event pair i around kernel group i.
void prof_mark(int i, bool end, cudaStream_t s);
cudaError_t launch_prefill(const PrefillArgs& p, int bits, cudaStream_t s);
cudaError_t launch_prefill_route(const PrefillArgs& p, cudaStream_t s);
cudaError_t launch_group(const PrefillArgs& p, cudaStream_t s);

// Sum of the expert-parallel ranks' fp32 partial outputs (fixed order) + residual -> bf16.
constexpr int kMaxPartials = 16;
struct PartialArgs {
  const float* part[kMaxPartials];
  int n;
  size_t count;               // T * H elements
  const uint16_t* residual;   // bf16 or null
  uint16_t* out;              // bf16
};
cudaError_t launch_combine_partials(const PartialArgs& p, cudaStream_t s);

// Kernel launchers (decode.cu).  Return cudaError_t of the launch.
cudaError_t launch_router_decode(const DecodeArgs& a, bool build_plan, cudaStream_t s);
cudaError_t launch_plan_decode(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_gateup_decode(const DecodeArgs& a, int bits, cudaStream_t s, bool* supported);
cudaError_t launch_down_decode(const DecodeArgs& a, int bits, cudaStream_t s, bool* supported);
bool decode_shape_supported(int H, int I, int bits);
// Fused decode stack (decode_fused.cu).
bool fused_shape_supported(int H, int I, int bits, int E);
cudaError_t launch_fused_decode(const FusedArgs& a, cudaStream_t s, bool* supported);

}  // namespace moe
