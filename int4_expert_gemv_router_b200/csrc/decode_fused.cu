// Fused persistent decode kernel: a stack of routed-MoE layers (T <= 8 tokens) in one
// cooperative launch on sm_100a.
//
// One CTA per SM, 16 warps: warps 0..14 compute, warp 15 streams weights.  Per layer:
//
//   phase R  router logits (E rows + the shared-gate row; fp64 sums of exact bf16 products)
//            and the shared expert's gate/up + SwiGLU rows, dealt round-robin over the CTAs
//            and their compute warps; activations staged once per CTA in shared memory.
//   -- grid barrier --
//   phase T  every CTA selects the top-k per token from the logits (the k-th best lane
//            maximum as a threshold, then ranking of the keys above it; ties to the lower
//            id), forms the softmax weights and the shared gate, and groups the (token, k)
//            pairs by expert.  CTA 0 writes the top-k.
//   phase G  the routed experts' gate/up rows, in blocks dealt round-robin over the CTAs,
//            stream into a shared-memory ring through cp.async.bulk (issued by the lanes of
//            warp 15, mbarrier transaction counts) and are reduced to h = silu(Wg x) * (Wu x);
//            right behind them the same warp streams this CTA's rows of every selected
//            expert's down matrix (and the shared expert's), so they are on chip before they
//            are needed.
//   -- grid barrier --
//   phase D  each CTA owns a slice of output rows: per expert one warp multiplies its staged
//            down rows with the expert's h (registers), the per-pair partial sums meet in
//            shared memory and are added in a fixed order (top-k slot order, then the shared
//            expert, then the residual) and rounded to bf16.
//   -- grid barrier --
//
// While a layer runs, warp 15 also prefetches the next layer's routing-independent rows
// (router matrix and shared expert) into L2 with cp.async.bulk.prefetch.
//
// The sums run in a fixed order, so the output bits do not depend on where experts sit in
// the pool.  Every wait (grid barrier, mbarrier) is bounded: on timeout the kernel sets
// MOE_DEVERR_TIMEOUT, lets its in-flight copies land and returns.
#include "common.cuh"
#include "kernels.cuh"
#include "sync.cuh"

namespace moe {
namespace {

constexpr int kFThreads = 512;
constexpr int kCons = 15;          // compute warps
constexpr int kConsThreads = kCons * 32;
constexpr int kProd = 15;          // streaming warp
constexpr int kMaxStages = 8;
constexpr int kFusedMaxE = 512;  // experts per layer on the fused path (larger E: unfused kernels)
constexpr int kLaneE = kFusedMaxE / 32;

constexpr int cgcd(int a, int b) { return b == 0 ? a : cgcd(b, a % b); }
constexpr int clcm(int a, int b) { return a / cgcd(a, b) * b; }

__device__ __forceinline__ void bar_cons() { asm volatile("bar.sync 1, %0;" ::"n"(kConsThreads) : "memory"); }

// Grid-wide barrier among the CTAs of a cooperative launch (called by one thread per CTA).
// bar_count only grows during a launch: barrier number b (0, 1, 2, ...) completes when it
// reaches (b + 1) * nblocks, so a barrier costs one atomic and the polls.  grid_exit()
// returns it to zero once every CTA has passed its last barrier.
// The arrival is an acq_rel atomic and the polls are acquire loads: the CTA's writes before
// the barrier (ordered before this thread's arrival by the CTA barrier that precedes it) are
// visible to every CTA that has seen the count complete, with no separate fence.
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ bool grid_barrier(Ctrl* c, uint32_t nblocks, uint32_t b) {
  const uint32_t target = (b + 1) * nblocks;
  const uint32_t arrived = atom_add_acq_rel(&c->bar_count, 1u) + 1;
  if (arrived >= target) return true;
  const unsigned long long t0 = now_ns();
  for (uint32_t it = 0;; ++it) {
    if (ld_acquire(&c->bar_count) >= target) return true;
    if ((it & 255u) == 255u && now_ns() - t0 > kWaitNs) {
      atomicOr(&c->err, kErrTimeout);
      return false;
    }
  }
}

// Called once per CTA after its last barrier: the last CTA out resets the barrier counters
// (no CTA reads bar_count any more by then).
__device__ void grid_exit(Ctrl* c, uint32_t nblocks) {
  __threadfence();
  if (atomicAdd(&c->bar_gen, 1u) + 1 == nblocks) {
    atomicExch(&c->bar_count, 0u);
    atomicExch(&c->bar_gen, 0u);
  }
}

// Key order of the top-k: larger logit first, ties to the lower id.
__device__ __forceinline__ bool key_better(double av, int ae, double bv, int be) {
  return av > bv || (av == bv && ae < be);
}

// Top-k of one token's logits by one warp, through shared memory instead of shuffle chains.
// Lane i (i < k) receives the i-th best key (sv, se): larger logit first, ties to the lower
// id.  The k-th best of the 32 lane maxima bounds the k-th best key from below; the keys at
// or above it (at least k, usually few) are ranked by counting; with more than 64 of them
// (many equal keys) k rounds of warp arg-max run instead.
__device__ __noinline__ void warp_topk(const double* lt, int E, int k, uint8_t* scratch, uint32_t* err,
                                       double& sv, int& se) {
  const int lane = threadIdx.x & 31;
  double* lmv = reinterpret_cast<double*>(scratch);          // [32]
  int* lme = reinterpret_cast<int*>(lmv + 32);               // [32]
  double* cv = reinterpret_cast<double*>(lme + 32);          // [64]
  int* ce = reinterpret_cast<int*>(cv + 64);                 // [64]
  int* cnt = ce + 64;                                        // [2]: candidates, threshold lane
  double v[kLaneE];
  double bv = -INFINITY;
  int be = 0x7fffffff;
  // all loads first (no side effects in between, so they are in flight together)
#pragma unroll
  for (int m = 0; m < kLaneE; ++m) {
    const int e = lane + 32 * m;
    v[m] = (e < E) ? __ldcg(lt + e) : -INFINITY;
  }
  bool nan_seen = false;
#pragma unroll
  for (int m = 0; m < kLaneE; ++m) {
    const int e = lane + 32 * m;
    if (!(v[m] == v[m])) {
      nan_seen = true;
      v[m] = -INFINITY;
    }
    if (e < E && key_better(v[m], e, bv, be)) {
      bv = v[m];
      be = e;
    }
  }
  if (nan_seen) atomicOr(err, kErrNonFinite);
  lmv[lane] = bv;
  lme[lane] = be;
  if (lane == 0) cnt[0] = 0;
  __syncwarp();
  int r = 0;
#pragma unroll 8
  for (int j = 0; j < 32; ++j) r += key_better(lmv[j], lme[j], bv, be) ? 1 : 0;
  if (r == k - 1 && be != 0x7fffffff) cnt[1] = lane;
  __syncwarp();
  const double thr_v = lmv[cnt[1]];
  const int thr_e = lme[cnt[1]];
#pragma unroll
  for (int m = 0; m < kLaneE; ++m) {
    const int e = lane + 32 * m;
    if (e < E && !key_better(thr_v, thr_e, v[m], e)) {
      const int pos = atomicAdd(&cnt[0], 1);
      if (pos < 64) {
        cv[pos] = v[m];
        ce[pos] = e;
      }
    }
  }
  __syncwarp();
  const int n = cnt[0];
  if (n <= 64) {
    double mv[2];
    int me[2], mr[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = lane + 32 * h;
      mv[h] = i < n ? cv[i] : -INFINITY;
      me[h] = i < n ? ce[i] : 0x7fffffff;
      mr[h] = 0;
    }
    for (int j = 0; j < n; ++j) {
      const double jv = cv[j];
      const int je = ce[j];
      mr[0] += key_better(jv, je, mv[0], me[0]) ? 1 : 0;
      mr[1] += key_better(jv, je, mv[1], me[1]) ? 1 : 0;
    }
    __syncwarp();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (lane + 32 * h < n && mr[h] < k) {
        lmv[mr[h]] = mv[h];
        lme[mr[h]] = me[h];
      }
    }
    __syncwarp();
    sv = lane < k ? lmv[lane] : -INFINITY;
    se = lane < k ? lme[lane] : 0x7fffffff;
    __syncwarp();
  } else {
    uint32_t taken = 0;
    sv = -INFINITY;
    se = 0x7fffffff;
    for (int rr = 0; rr < k; ++rr) {
      double rv = -INFINITY;
      int re = 0x7fffffff;
#pragma unroll
      for (int m = 0; m < kLaneE; ++m) {
        const int e = lane + 32 * m;
        if (e < E && !((taken >> m) & 1u) && key_better(v[m], e, rv, re)) {
          rv = v[m];
          re = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, rv, o);
        const int oe = __shfl_xor_sync(0xffffffffu, re, o);
        if (key_better(ov, oe, rv, re)) {
          rv = ov;
          re = oe;
        }
      }
      if (re != 0x7fffffff && (re & 31) == lane) taken |= 1u << (re >> 5);
      if (lane == rr) {
        sv = rv;
        se = re;
      }
    }
  }
}

// Rows per phase-G block: the CTAs' equal share of the rows in as few blocks of at most
// RG rows as it takes, rounded up to the granule gG.
__device__ __forceinline__ int gate_block_rows(int rows, int G, int RG, int gG) {
  if (rows <= 0) return gG;
  const int per_cta = (rows + G - 1) / G;
  const int n_blocks = (per_cta + RG - 1) / RG;
  const int br = (per_cta + n_blocks - 1) / n_blocks;
  return max(gG, (br + gG - 1) / gG * gG);
}

// Phase-R rows of CTA c (of G) in layer L: router rows [rr0, rr1) of the n_router = E + 1
// (the last one is the shared-gate row; only that one when the layer's routing is given) and
// shared-expert rows [sr0, sr1), each a contiguous range so that it is staged in a few copies.
struct RRange {
  int rr0, rr1, sr0, sr1, n_router;
};
__device__ __forceinline__ RRange r_ranges(const FusedLayer& L, int E, int I, int gG, int c, int G) {
  RRange r;
  r.n_router = (L.topk_idx_in ? 0 : E) + 1;
  r.rr0 = (int)((long long)c * r.n_router / G);
  r.rr1 = (int)((long long)(c + 1) * r.n_router / G);
  const int ngr = L.with_shared ? I / gG : 0;
  r.sr0 = (int)((long long)c * ngr / G) * gG;
  r.sr1 = (int)((long long)(c + 1) * ngr / G) * gG;
  return r;
}

template <int BITS, int H, int I, int TM>
__global__ void __launch_bounds__(kFThreads, 1) k_fused_decode(const __grid_constant__ FusedArgs a) {
  // ---- constants ----
  constexpr int CC = 128 / BITS, V4 = CC / 4;
  constexpr int NCg = H / CC, NCLg = NCg < 32 ? NCg : 32, RPWg = 32 / NCLg, CPLg = NCg / NCLg;
  constexpr int ROWBg = H * BITS / 8, NGg = H / kGroup, SRg = NGg * 2;
  constexpr int NCd = I / CC, NCLd = NCd < 32 ? NCd : 32, RPWd = 32 / NCLd, CPLd = NCd / NCLd;
  constexpr int ROWBd = I * BITS / 8, NGd = I / kGroup, SRd = NGd * 2;
  constexpr int gG = clcm(16 / cgcd(16, SRg), RPWg);
  constexpr int gD = clcm(16 / cgcd(16, SRd), RPWd);
  constexpr int ROWG_BYTES = 2 * ROWBg + 4 * SRg;  // one gate/up row with its scales
  constexpr int ROWD_BYTES = ROWBd + 2 * SRd;      // one down row with its scales
  // phase D: the RPWd lanes that share an h chunk; with two of them each loads half
  constexpr int HS = (RPWd == 2 && V4 % 2 == 0) ? 2 : 1, VH = V4 / HS;

  const int T = a.T, E = a.E, k = a.k, G = gridDim.x;
  // bound of the waits for pending slot-table entries (a blob copy that has not landed by
  // then is treated as failed: the expert is skipped and flagged)
  const unsigned long long slot_wait_ns = a.ctrl->slot_wait_us ? 1000ull * a.ctrl->slot_wait_us : kWaitNs;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NS = a.n_stages, SB = a.stage_bytes;
  const int RG = (SB / ROWG_BYTES) / gG * gG;  // gate/up rows per stage

  // ---- shared memory ----
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[kMaxStages], empty_bar[kMaxStages], plan_bar, rbar;
  __shared__ int s_act_n, s_n_valid, s_abort;
  uint8_t* ring = smem;
  uint8_t* rbuf = smem + a.sm.rbuf;                             // this CTA's phase-R rows
  uint8_t* rbuf_s = rbuf + (size_t)a.rr_max * H * 2;            // ... the shared-expert part
  double* rpart = reinterpret_cast<double*>(smem + a.sm.rpart);  // router-row quarter sums
  float4* xs4 = reinterpret_cast<float4*>(smem + a.sm.xs4);
  float* xsum = reinterpret_cast<float*>(smem + a.sm.xsum);
  float* partial = reinterpret_cast<float*>(smem + a.sm.partial);  // [(T*k + T) * jmax]
  const int TK = T * k;
#define P_IDS reinterpret_cast<int*>(smem + a.sm.ids)
#define P_PW reinterpret_cast<float*>(smem + a.sm.pw)
#define P_ORDER reinterpret_cast<int*>(smem + a.sm.order)
#define P_POS reinterpret_cast<int*>(smem + a.sm.pos_of)
#define P_ACTE reinterpret_cast<int*>(smem + a.sm.act_e)
#define P_SLOT reinterpret_cast<int*>(smem + a.sm.act_slot)
#define P_BEGIN reinterpret_cast<int*>(smem + a.sm.act_begin)
#define P_GATE reinterpret_cast<float*>(smem + a.sm.gate)
#define P_SCRATCH reinterpret_cast<int*>(smem + a.sm.scratch)
#define S_SLOT reinterpret_cast<int*>(smem + a.sm.slot)

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kCons);
    }
    mbar_init(&plan_bar, 1);
    mbar_init(&rbar, 1);
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  // This CTA's slice of output rows (phase D), in granules of gD rows.
  const int nGranD = H / gD;
  const int j0 = (int)((long long)blockIdx.x * nGranD / G) * gD;
  const int j1 = (int)((long long)(blockIdx.x + 1) * nGranD / G) * gD;
  const int nJ = j1 - j0;

  // =====================================================================================
  // streaming warp
  // =====================================================================================
  if (warp == kProd) {
    uint32_t q = 0;  // stage sequence number, shared convention with the compute warps
    bool ok = true;
    // The slot of distinct expert u of layer Lc.  An entry that was pending when phase X read
    // the table (the blob was still being copied) is polled until the copy stream has written
    // the slot; the result goes back to the plan, where the compute warps read it after the
    // stage's full barrier.  Whole warp; bounded (-1 and MOE_DEVERR_TIMEOUT after slot_wait_ns).
    // The entry is written by the copy stream (a stream memory operation after the blob's
    // copy), so it is read with system-scope acquire loads; the blob itself is then read by
    // cp.async.bulk, which goes through the async proxy: every lane orders its later bulk
    // copies after the acquire with a proxy fence (the warp barrier carries lane 0's acquire
    // to the other lanes first).
    const auto slot_of_unit = [&](const FusedLayer& L, int u) {
      int v = P_SLOT[u];
      if (v != kSlotPending) return v;
      if (lane == 0) {
        const int* entry = L.slot_table + P_ACTE[u];
        const unsigned long long t0 = now_ns();
        uint32_t ns = 64;
        for (;;) {
          v = ld_acquire_sys_s32(entry);
          if (v != kSlotPending) break;
          if (now_ns() - t0 > slot_wait_ns) {
            atomicOr(&a.ctrl->err, kErrTimeout);
            v = -1;
            break;
          }
          __nanosleep(ns);
          ns = ns < 1024 ? 2 * ns : 1024;
        }
        if (v != -1 && (v < 0 || v >= L.n_slots)) v = -1;
        if (v < 0) atomicOr(&a.ctrl->err, kErrBadSlot);
        P_SLOT[u] = v;
      }
      __syncwarp();
      fence_proxy_async_global();
      return __shfl_sync(0xffffffffu, v, 0);
    };
    // This CTA's phase-R rows of layer ln (its router rows, the shared-gate row if it holds
    // it, its shared-expert rows with their scales) copied into rbuf: at most eight bulk
    // copies, tracked on rbar.  pf: only an L2 prefetch of the same bytes.
    const auto issue_r = [&](int ln, bool pf) {
      const FusedLayer& Ln = a.layer[ln];
      const RRange R = r_ranges(Ln, E, I, gG, blockIdx.x, G);
      const int n_wr = max(0, min(R.rr1, R.n_router - 1) - R.rr0);  // rows of the router matrix
      const bool has_gate = R.rr1 == R.n_router && R.rr1 > R.rr0;
      const int ns = R.sr1 - R.sr0;
      if (!pf && lane == 0)
        mbar_expect_tx(&rbar, (uint32_t)((n_wr + (has_gate ? 1 : 0)) * H * 2 + ns * ROWG_BYTES));
      __syncwarp();
      if (lane == 0 && n_wr > 0) {
        if (pf) prefetch_l2(Ln.wr + (size_t)R.rr0 * H, n_wr * H * 2);
        else bulk_g2s(rbuf, Ln.wr + (size_t)R.rr0 * H, n_wr * H * 2, &rbar);
      }
      if (lane == 1 && has_gate) {
        if (pf) prefetch_l2(Ln.wsg, H * 2);
        else bulk_g2s(rbuf + (size_t)(R.n_router - 1 - R.rr0) * H * 2, Ln.wsg, H * 2, &rbar);
      }
      if (ns > 0 && lane >= 2 && lane < 8) {
        const int sec = lane - 2;
        const uint8_t* src = sec < 2 ? Ln.shared + a.L.off[sec] + (int64_t)R.sr0 * ROWBg
                                     : Ln.shared + a.L.off[1 + sec] + (int64_t)R.sr0 * SRg;
        const int bytes = sec < 2 ? ns * ROWBg : ns * SRg;
        if (pf) prefetch_l2(src, bytes);
        else bulk_g2s(rbuf_s + (sec < 2 ? sec * ns * ROWBg : 2 * ns * ROWBg + (sec - 2) * ns * SRg), src, bytes, &rbar);
      }
      __syncwarp();
    };
    // At one token phase R reads its rows from global memory (item i on CTA i % G; measured
    // faster there than staging them), and this warp only prefetches the next layer's rows
    // into L2; with several tokens the rows are staged in shared memory (issue_r).
    int n_r_issued = 0;  // rbar phases announced
    if constexpr (TM > 1) {
      issue_r(0, false);
      ++n_r_issued;
    }
    for (int l = 0; l < a.n_layers && ok; ++l) {
      const FusedLayer& Lc = a.layer[l];
      if constexpr (TM > 1) {
        // L2 prefetch of the next layer's phase-R rows (copied to shared memory later in this layer)
        if (l + 1 < a.n_layers) issue_r(l + 1, true);
      } else if (l + 1 < a.n_layers) {
        // L2 prefetch of the next layer's routing-independent rows this CTA's warps will read
        // (phase-R item i belongs to CTA i % G), one lane per item
        const FusedLayer& Ln = a.layer[l + 1];
        const int n_router = (Ln.topk_idx_in ? 0 : E) + 1;
        const int n_items = n_router + I / RPWg;
        for (int it = blockIdx.x + G * lane; it < n_items; it += G * 32) {
          if (it < n_router) {
            const bool gate_row = (it == n_router - 1);
            const uint16_t* row = gate_row ? Ln.wsg : Ln.wr + (size_t)it * H;
            prefetch_l2(row, H * 2);
          } else {
            const int r = (it - n_router) * RPWg;
            prefetch_l2(Ln.shared + a.L.off[0] + (int64_t)r * ROWBg, RPWg * ROWBg);
            prefetch_l2(Ln.shared + a.L.off[1] + (int64_t)r * ROWBg, RPWg * ROWBg);
          }
        }
      }
      // wait for this layer's plan
      if (!mbar_wait(&plan_bar, l & 1)) {
        ok = false;
        break;
      }
      if (*(volatile int*)&s_abort) break;
      const int act_n = s_act_n;
      // ---- phase G pieces ----
      // blocks of BR rows dealt round-robin over the CTAs (block b on CTA b % G), so that at
      // any moment the grid reads one contiguous stretch of the experts' rows; a block that
      // crosses into the next expert is two stages
      const int rows_g = act_n * I, BR = gate_block_rows(rows_g, G, RG, gG);
      for (int b0 = blockIdx.x * BR, b1 = min(b0 + BR, rows_g), f = b0; f < rows_g && ok;) {
        const int u = f / I, r0 = f - u * I;
        const int n = min(b1 - f, I - r0);
        const int s = q % NS;
        if (!mbar_wait(&empty_bar[s], ((q / NS) & 1) ^ 1)) {
          ok = false;
          break;
        }
        {
          // lane 0 announces the bytes, then lanes 0..5 issue the stage's six copies at once
          // (gate codes, up codes, then the four scale/bias sections)
          uint8_t* st = ring + (size_t)s * SB;
          const int slot = slot_of_unit(Lc, u);
          if (lane == 0) {
            if (slot < 0)
              mbar_arrive(&full_bar[s]);
            else
              mbar_expect_tx(&full_bar[s], (uint32_t)(n * ROWG_BYTES));
          }
          __syncwarp();
          if (slot >= 0 && lane < 6) {
            const uint8_t* b = Lc.pool + (int64_t)slot * a.L.stride;
            if (lane < 2)
              bulk_g2s(st + lane * n * ROWBg, b + a.L.off[lane] + (int64_t)r0 * ROWBg, n * ROWBg, &full_bar[s]);
            else
              bulk_g2s(st + 2 * n * ROWBg + (lane - 2) * n * SRg, b + a.L.off[lane + 1] + (int64_t)r0 * SRg,
                       n * SRg, &full_bar[s]);
          }
        }
        __syncwarp();
        ++q;
        f += n;
        if (f == b1) {
          b0 += G * BR;
          b1 = min(b0 + BR, rows_g);
          f = b0;
        }
      }
      // ---- phase D pieces: this CTA's down rows of every selected expert, then the shared one ----
      if (nJ > 0) {
        for (int u = 0; u < act_n; ++u) slot_of_unit(Lc, u);  // every pending slot settled
        __syncwarp();
        const int per_stage = SB / (nJ * ROWD_BYTES);
        const int n_units_d = act_n + (Lc.with_shared ? 1 : 0);  // the shared expert last
        for (int u = 0; u < n_units_d && ok;) {
          const int cnt = min(per_stage, n_units_d - u);
          const int s = q % NS;
          if (!mbar_wait(&empty_bar[s], ((q / NS) & 1) ^ 1)) {
            ok = false;
            break;
          }
          uint8_t* st = ring + (size_t)s * SB;
          if (lane == 0) {
            uint32_t bytes = 0;
            for (int z = 0; z < cnt; ++z) {
              const int uu = u + z;
              const int slot = (uu < act_n) ? P_SLOT[uu] : 0;
              if (uu < act_n && slot < 0) continue;
              bytes += nJ * ROWD_BYTES;
            }
            mbar_expect_tx(&full_bar[s], bytes);
          }
          __syncwarp();
          // three copies per expert (down codes, scales, biases), spread over the lanes
          for (int ci = lane; ci < 3 * cnt; ci += 32) {
            const int z = ci / 3, part = ci - 3 * z, uu = u + z;
            const uint8_t* b;
            if (uu < act_n) {
              const int slot = P_SLOT[uu];
              if (slot < 0) continue;
              b = Lc.pool + (int64_t)slot * a.L.stride;
            } else {
              b = Lc.shared;
            }
            uint8_t* d = st + (size_t)z * nJ * ROWD_BYTES;
            if (part == 0)
              bulk_g2s(d, b + a.L.off[2] + (int64_t)j0 * ROWBd, nJ * ROWBd, &full_bar[s]);
            else
              bulk_g2s(d + nJ * ROWBd + (part - 1) * nJ * SRd, b + a.L.off[6 + part] + (int64_t)j0 * SRd, nJ * SRd,
                       &full_bar[s]);
          }
          __syncwarp();
          ++q;
          u += cnt;
        }
      }
      // the next layer's phase-R rows: this CTA finished reading rbuf before the plan
      if (TM > 1 && ok && l + 1 < a.n_layers) {
        issue_r(l + 1, false);
        ++n_r_issued;
      }
    }
    if (!ok && lane == 0) {
      atomicOr(&a.ctrl->err, kErrTimeout);
      s_abort = 1;
    }
    // let every issued copy land before the CTA may exit
    if (lane == 0) {
      if (n_r_issued > 0) mbar_wait(&rbar, (uint32_t)(n_r_issued - 1) & 1);
      const uint32_t first = q > (uint32_t)NS ? q - NS : 0;
      for (uint32_t qq = first; qq < q; ++qq) mbar_wait(&full_bar[qq % NS], (qq / NS) & 1);
    }
    return;
  }

  // =====================================================================================
  // compute warps
  // =====================================================================================
  const int cw = warp;  // 0..14
  const int NW = G * kCons;  // compute warps of the grid (one-token phase R)
  uint32_t q = 0;
  uint32_t nb = 0;  // grid barriers passed in this launch
  bool ok = true;

  for (int l = 0; l < a.n_layers; ++l) {
    const FusedLayer& Lc = a.layer[l];
    const bool routed = (Lc.topk_idx_in == nullptr);

    // ---- stage x: chunk-interleaved, pre-scaled fp32 + chunk sums ----
    stage_vectors<BITS, H>(xs4, xsum, T, tid, kConsThreads, [&](int r, int i) {
      const uint2 raw = __ldcg(reinterpret_cast<const uint2*>(Lc.x + (size_t)r * H + i));
      return make_float4(bf_lo(raw.x), bf_hi(raw.x), bf_lo(raw.y), bf_hi(raw.y));
    });
    for (int e = tid; e < E; e += kConsThreads) S_SLOT[e] = __ldg(Lc.slot_table + e);
    bar_cons();

    // ---- phase R, one token: router rows, shared-gate row, shared gate/up rows from global ----
    if constexpr (TM == 1) {
      const int n_router = (routed ? E : 0) + 1;
      const int n_items = n_router + (Lc.with_shared ? I / RPWg : 0);
      for (int it = blockIdx.x + G * cw; it < n_items; it += NW) {  // item i: CTA i % G
        if (it < n_router) {
          const bool gate_row = (it == n_router - 1);
          const int e = gate_row ? E : it;
          const uint16_t* row = gate_row ? Lc.wsg : Lc.wr + (size_t)e * H;
          double acc = 0.0;
#pragma unroll 4
          for (int c8 = lane; c8 < H / 8; c8 += 32) {
            const uint4 w = ld_stream(row + c8 * 8);
            const float wv[8] = {bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y),
                                 bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w)};
            const int c = c8 / (CC / 8), v0 = (c8 % (CC / 8)) * 2;
            const float4 xa = xs4[(size_t)v0 * NCg + c];
            const float4 xb = xs4[(size_t)(v0 + 1) * NCg + c];
            const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
            double sp = 0.0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              // undo the staging scale (a power of two): the product stays exact
              const float xr = xv[i] * stage_unscale<BITS>(v0 * 4 + i);
              sp += (double)(wv[i] * xr);
            }
            acc += sp;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
          if (lane == 0) {
            if (!gate_row && Lc.rbias) acc += (double)Lc.rbias[e];
            a.logits[e] = acc;
          }
        } else {
          // shared expert gate/up row(s)
          const int r = (it - n_router) * RPWg + lane / NCLg;
          const int sub = lane % NCLg;
          const uint8_t* b = Lc.shared;
          float ag = 0.f, au = 0.f;
#pragma unroll 1
          for (int m = 0; m < CPLg; ++m) {
            const int c = sub + NCLg * m, g = c * CC / kGroup;
            const uint4 qg = ld_stream(b + a.L.off[0] + (int64_t)r * ROWBg + c * 16);
            const uint4 qu = ld_stream(b + a.L.off[1] + (int64_t)r * ROWBg + c * 16);
            const float sg = bf1(ld_u16(b + a.L.off[3] + (int64_t)r * SRg + g * 2));
            const float bg = bf1(ld_u16(b + a.L.off[4] + (int64_t)r * SRg + g * 2));
            const float su = bf1(ld_u16(b + a.L.off[5] + (int64_t)r * SRg + g * 2));
            const float bu = bf1(ld_u16(b + a.L.off[6] + (int64_t)r * SRg + g * 2));
            float dg, du;
            dot_chunk2<BITS>(qg, qu, xs4 + c, NCg, dg, du);
            const float xc = xsum[c];
            ag = fmaf(sg, dg, fmaf(bg, xc, ag));
            au = fmaf(su, du, fmaf(bu, xc, au));
          }
#pragma unroll
          for (int o = NCLg / 2; o > 0; o >>= 1) {
            ag += __shfl_xor_sync(0xffffffffu, ag, o);
            au += __shfl_xor_sync(0xffffffffu, au, o);
          }
          if (sub == 0) a.hs[r] = ag / (1.0f + expf(-ag)) * au;
        }
      }
    } else
    // ---- phase R: router rows, shared-gate row, shared gate/up rows (staged in rbuf) ----
    {
      const RRange R = r_ranges(Lc, E, I, gG, blockIdx.x, G);
      const int nrr = R.rr1 - R.rr0, ns = R.sr1 - R.sr0, nsi = ns / RPWg;
      // with several tokens a router row is split into nq column ranges on nq warps (their
      // fp64 sums added in a fixed order below), as far as the CTA's 15 warps go
      constexpr int NQ = (TM > 1 && (H / 8 / 4) % 32 == 0) ? 4 : 1;
      const int nq = (NQ == 4 && nrr * 4 + nsi <= kCons) ? 4 : (NQ == 4 && nrr * 2 + nsi <= kCons) ? 2 : 1;
      const int n_it = nrr * nq + nsi;
      if (cw < n_it && !mbar_wait(&rbar, l & 1)) {
        atomicOr(&a.ctrl->err, kErrTimeout);
        s_abort = 1;
      }
      for (int z = cw; z < n_it && !s_abort; z += kCons) {
        if (z < nrr * nq) {
          const int lr = z / nq, qq = z - lr * nq;
          const bool gate_row = (R.rr0 + lr == R.n_router - 1);
          const int e = gate_row ? E : R.rr0 + lr;
          const uint16_t* row = reinterpret_cast<const uint16_t*>(rbuf + (size_t)lr * H * 2);
          const int cq = H / 8 / nq;
          double acc[TM];
#pragma unroll
          for (int t = 0; t < TM; ++t) acc[t] = 0.0;
#pragma unroll 4
          for (int c8 = qq * cq + lane; c8 < (qq + 1) * cq; c8 += 32) {
            const uint4 w = *reinterpret_cast<const uint4*>(row + c8 * 8);
            const int c = c8 / (CC / 8), v0 = (c8 % (CC / 8)) * 2;
            // the weights times the inverse staging scales (powers of two: exact), so that
            // each product with a staged activation is the exact w * x
            const float wv[8] = {bf_lo(w.x) * stage_unscale<BITS>(v0 * 4 + 0), bf_hi(w.x) * stage_unscale<BITS>(v0 * 4 + 1),
                                 bf_lo(w.y) * stage_unscale<BITS>(v0 * 4 + 2), bf_hi(w.y) * stage_unscale<BITS>(v0 * 4 + 3),
                                 bf_lo(w.z) * stage_unscale<BITS>(v0 * 4 + 4), bf_hi(w.z) * stage_unscale<BITS>(v0 * 4 + 5),
                                 bf_lo(w.w) * stage_unscale<BITS>(v0 * 4 + 6), bf_hi(w.w) * stage_unscale<BITS>(v0 * 4 + 7)};
#pragma unroll
            for (int t = 0; t < TM; ++t) {
              if (t < T) {
                const float4 xa = xs4[((size_t)t * V4 + v0) * NCg + c];
                const float4 xb = xs4[((size_t)t * V4 + v0 + 1) * NCg + c];
                const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
                double s = 0.0;
#pragma unroll
                for (int i = 0; i < 8; ++i) s += (double)(wv[i] * xv[i]);
                acc[t] += s;
              }
            }
          }
#pragma unroll
          for (int t = 0; t < TM; ++t) {
            if (t < T) {
              double v = acc[t];
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
              if (lane == 0) {
                if (nq > 1) {
                  rpart[((size_t)lr * nq + qq) * T + t] = v;
                } else {
                  if (!gate_row && Lc.rbias) v += (double)Lc.rbias[e];
                  a.logits[(size_t)t * (E + 1) + e] = v;
                }
              }
            }
          }
        } else {
          // shared expert gate/up row(s): chunk by chunk, every token against each chunk
          const int rl = (z - nrr * nq) * RPWg + lane / NCLg;  // row within this CTA's range
          const int sub = lane % NCLg;
          const uint8_t* gq = rbuf_s + (size_t)rl * ROWBg;
          const uint8_t* uq = rbuf_s + (size_t)ns * ROWBg + rl * ROWBg;
          const uint8_t* sc = rbuf_s + 2 * (size_t)ns * ROWBg + rl * SRg;
          float ag[TM], au[TM];
#pragma unroll
          for (int t = 0; t < TM; ++t) ag[t] = au[t] = 0.f;
#pragma unroll 1
          for (int m = 0; m < CPLg; ++m) {
            const int c = sub + NCLg * m, g = c * CC / kGroup;
            const uint4 qg = *reinterpret_cast<const uint4*>(gq + c * 16);
            const uint4 qu = *reinterpret_cast<const uint4*>(uq + c * 16);
            const float sg = bf1(*reinterpret_cast<const uint16_t*>(sc + g * 2));
            const float bg = bf1(*reinterpret_cast<const uint16_t*>(sc + ns * SRg + g * 2));
            const float su = bf1(*reinterpret_cast<const uint16_t*>(sc + 2 * ns * SRg + g * 2));
            const float bu = bf1(*reinterpret_cast<const uint16_t*>(sc + 3 * ns * SRg + g * 2));
            if constexpr (TM == 1) {
              float dg, du;
              dot_chunk2<BITS>(qg, qu, xs4 + c, NCg, dg, du);
              const float xc = xsum[c];
              ag[0] = fmaf(sg, dg, fmaf(bg, xc, ag[0]));
              au[0] = fmaf(su, du, fmaf(bu, xc, au[0]));
            } else {
              // several tokens: each code pair becomes floats once and meets every token
              float2 gacc[TM], uacc[TM];
#pragma unroll
              for (int t = 0; t < TM; ++t) gacc[t] = uacc[t] = make_float2(0.f, 0.f);
#pragma unroll
              for (int wi = 0; wi < 4; ++wi) {
                float2 cg[4], cu[4];
                codes_of_word<BITS>(word_of(qg, wi), cg);
                codes_of_word<BITS>(word_of(qu, wi), cu);
#pragma unroll
                for (int t = 0; t < TM; ++t) {
                  if (t < T) {
                    const float4* xt = xs4 + (size_t)t * V4 * NCg + c;
                    if constexpr (BITS == 4) {
                      const float4 xa = xt[(2 * wi) * NCg], xb = xt[(2 * wi + 1) * NCg];
                      const float2 x01 = make_float2(xa.x, xa.y), x23 = make_float2(xa.z, xa.w);
                      const float2 x45 = make_float2(xb.x, xb.y), x67 = make_float2(xb.z, xb.w);
                      gacc[t] = ffma2(cg[3], x67, ffma2(cg[2], x45, ffma2(cg[1], x23, ffma2(cg[0], x01, gacc[t]))));
                      uacc[t] = ffma2(cu[3], x67, ffma2(cu[2], x45, ffma2(cu[1], x23, ffma2(cu[0], x01, uacc[t]))));
                    } else {
                      const float4 xa = xt[wi * NCg];
                      const float2 x01 = make_float2(xa.x, xa.y), x23 = make_float2(xa.z, xa.w);
                      gacc[t] = ffma2(cg[1], x23, ffma2(cg[0], x01, gacc[t]));
                      uacc[t] = ffma2(cu[1], x23, ffma2(cu[0], x01, uacc[t]));
                    }
                  }
                }
              }
#pragma unroll
              for (int t = 0; t < TM; ++t) {
                if (t < T) {
                  const float xc = xsum[t * NCg + c];
                  ag[t] = fmaf(sg, gacc[t].x + gacc[t].y, fmaf(bg, xc, ag[t]));
                  au[t] = fmaf(su, uacc[t].x + uacc[t].y, fmaf(bu, xc, au[t]));
                }
              }
            }
          }
#pragma unroll
          for (int t = 0; t < TM; ++t) {
            if (t < T) {
              float g2 = ag[t], u2 = au[t];
#pragma unroll
              for (int o = NCLg / 2; o > 0; o >>= 1) {
                g2 += __shfl_xor_sync(0xffffffffu, g2, o);
                u2 += __shfl_xor_sync(0xffffffffu, u2, o);
              }
              if (sub == 0) a.hs[(size_t)t * I + R.sr0 + rl] = g2 / (1.0f + expf(-g2)) * u2;
            }
          }
        }
      }
      if (nq > 1) {
        // the router rows' column-range sums, added in range order
        bar_cons();
        for (int i = tid; i < nrr * T; i += kConsThreads) {
          const int lr = i / T, t = i - lr * T;
          double v = 0.0;
          for (int qq = 0; qq < nq; ++qq) v += rpart[((size_t)lr * nq + qq) * T + t];
          const bool gate_row = (R.rr0 + lr == R.n_router - 1);
          const int e = gate_row ? E : R.rr0 + lr;
          if (!gate_row && Lc.rbias) v += (double)Lc.rbias[e];
          a.logits[(size_t)t * (E + 1) + e] = v;
        }
      }
    }
    bar_cons();
    if (tid == 0 && !grid_barrier(a.ctrl, G, nb)) s_abort = 1;
    ++nb;
    bar_cons();
    if (s_abort) ok = false;

    // ---- phase T: top-k, softmax, shared gate, grouping (every CTA) ----
    if (ok) {
      for (int t = cw; t < T; t += kCons) {
        const double* lt = a.logits + (size_t)t * (E + 1);
        if (routed) {
          double sv;
          int se;
          warp_topk(lt, E, k, smem + a.sm.topk + (size_t)t * kTopkScratchBytes, &a.ctrl->err, sv, se);
          // lanes 0..k-1 hold the selection in order
          const double v0 = __shfl_sync(0xffffffffu, sv, 0);
          const bool valid = lane < k && se != 0x7fffffff && sv != -INFINITY;
          const double ex = valid ? exp(sv - v0) : 0.0;
          double den = ex;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
          const int id = valid ? se : -1;
          if (lane < k) {
            if (!valid) atomicOr(&a.ctrl->err, kErrNonFinite);
            const float pw = valid ? (float)(ex / den) : 0.f;
            P_IDS[t * k + lane] = id;
            P_PW[t * k + lane] = pw;
            if (blockIdx.x == 0 && Lc.topk_idx_out) {
              Lc.topk_idx_out[t * k + lane] = id;
              Lc.topk_w_out[t * k + lane] = pw;
            }
          }
          if (T == 1) {
            // one token: the k ids are distinct, so this warp groups them itself (ranks by
            // shuffles) and the CTA skips the general grouping below
            // an expert held by another rank (expert parallelism) is left out like an
            // invalid id, without a flag: its term is that rank's
            const int key = lane < k ? ((id >= 0 && S_SLOT[id] != kSlotRemote) ? id : E) : 0x7fffffff;
            int rank = 0, before = 0;
            for (int j = 0; j < k; ++j) {
              const int kj = __shfl_sync(0xffffffffu, key, j);
              rank += (kj < key) || (kj == key && j < lane);
              before += kj < key;
            }
            const bool vld = lane < k && key < E;
            const unsigned vm = __ballot_sync(0xffffffffu, vld);
            if (lane < k) {
              P_ORDER[rank] = lane;
              P_POS[lane] = vld ? rank : -1;
            }
            if (vld) {  // every valid id is the first (and only) pair of its expert
              P_ACTE[before] = key;
              P_BEGIN[before] = before;
              const int slot = S_SLOT[key];
              const bool sok = (slot >= 0 && slot < Lc.n_slots) || slot == kSlotPending;
              if (!sok) atomicOr(&a.ctrl->err, kErrBadSlot);
              P_SLOT[before] = sok ? slot : -1;
            }
            if (lane == 0) {
              s_act_n = __popc(vm);
              s_n_valid = __popc(vm);
              P_BEGIN[__popc(vm)] = __popc(vm);
            }
          }
        } else if (lane < k) {
          P_IDS[t * k + lane] = Lc.topk_idx_in[t * k + lane];
          P_PW[t * k + lane] = Lc.topk_w_in[t * k + lane];
        }
      }
      // shared-expert gates on warps other than the top-k ones, in parallel with them
      for (int t = 0; t < T; ++t)
        if (cw == (T + t) % kCons && lane == 0) P_GATE[t] = (float)(1.0 / (1.0 + exp(-__ldcg(a.logits + (size_t)t * (E + 1) + E))));
    }
    bar_cons();
    // grouping: pairs sorted by (expert, pair number); invalid ids and experts held by another
    // rank left out (sorted last).  One warp ranks the T*k pairs by counting (each lane its
    // pairs against all keys, read as shared-memory broadcasts), then numbers the distinct
    // experts the same way: no CTA barrier inside, and the result does not depend on timing.
    if (ok && !(T == 1 && routed) && cw == 0) {
      int* key = P_SCRATCH;            // [TK] expert of pair i (E: left out)
      int* rnk = P_SCRATCH + TK;       // [TK] rank of pair i in (expert, pair) order
      int* first = P_SCRATCH + 3 * TK; // [TK] pair i is its expert's first
      for (int i = lane; i < TK; i += 32) {
        const int e = P_IDS[i];
        const bool valid = e >= 0 && e < E;
        if (!valid && blockIdx.x == 0) atomicOr(&a.ctrl->err, kErrBadExpert);
        key[i] = (valid && S_SLOT[e] != kSlotRemote) ? e : E;
      }
      __syncwarp();
      int nv = 0, an = 0;
      for (int i = lane; i < TK; i += 32) {
        const int ki = key[i];
        int r = 0;
        bool d = false;
        for (int j = 0; j < TK; ++j) {
          const int kj = key[j];
          r += (kj < ki) || (kj == ki && j < i);
          d = d || (kj == ki && j < i);
        }
        const bool f = !d && ki < E;
        rnk[i] = r;
        P_ORDER[r] = i;
        P_POS[i] = (ki < E) ? r : -1;
        first[i] = f ? 1 : 0;
        nv += ki < E;
        an += f;
      }
      __syncwarp();
      for (int i = lane; i < TK; i += 32) {
        if (!first[i]) continue;
        const int ki = key[i];
        int act = 0;  // distinct experts below this one
        for (int j = 0; j < TK; ++j) act += (first[j] && key[j] < ki);
        P_ACTE[act] = ki;
        P_BEGIN[act] = rnk[i];  // the first pair of an expert: its rank counts the pairs below
        const int slot = S_SLOT[ki];
        const bool sok = (slot >= 0 && slot < Lc.n_slots) || slot == kSlotPending;
        if (!sok) atomicOr(&a.ctrl->err, kErrBadSlot);
        P_SLOT[act] = sok ? slot : -1;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        nv += __shfl_xor_sync(0xffffffffu, nv, o);
        an += __shfl_xor_sync(0xffffffffu, an, o);
      }
      if (lane == 0) {
        s_act_n = an;
        s_n_valid = nv;
        P_BEGIN[an] = nv;
      }
    }
    bar_cons();
    if (tid == 0) mbar_arrive(&plan_bar);  // the streaming warp may issue this layer's pieces
    if (!ok) break;
    const int act_n = s_act_n, n_valid = s_n_valid;

    // ---- phase G: routed gate/up + SwiGLU from the ring ----
    {
      const int rows_g = act_n * I, BR = gate_block_rows(rows_g, G, RG, gG);
      const int sub = lane % NCLg, rsub = lane / NCLg;
      int done = 0;  // rows of this CTA already processed
      for (int b0 = blockIdx.x * BR, b1 = min(b0 + BR, rows_g), f = b0; f < rows_g;) {
        const int u = f / I, r0 = f - u * I;
        const int n = min(b1 - f, I - r0);
        const int s = q % NS;
        if (!mbar_wait(&full_bar[s], (q / NS) & 1)) {
          ok = false;
          atomicOr(&a.ctrl->err, kErrTimeout);
          break;
        }
        const uint8_t* st = ring + (size_t)s * SB;
        if (P_SLOT[u] >= 0) {
          const int pb = P_BEGIN[u], pe = P_BEGIN[u + 1];
          // row steps are dealt to warps round-robin over the CTA's whole row range
          const int step0 = done / RPWg;
          for (int step = (cw - step0 % kCons + kCons) % kCons; step < n / RPWg; step += kCons) {
            const int rl = step * RPWg + rsub;
            const uint8_t* gq = st + rl * ROWBg;
            const uint8_t* uq = st + n * ROWBg + rl * ROWBg;
            const uint8_t* sc = st + 2 * n * ROWBg + rl * SRg;
            for (int p = pb; p < pe; ++p) {
              const int t = P_ORDER[p] / k;
              float ag = 0.f, au = 0.f;
#pragma unroll 1
              for (int m = 0; m < CPLg; ++m) {
                const int c = sub + NCLg * m, g = c * CC / kGroup;
                const uint4 qg = *reinterpret_cast<const uint4*>(gq + c * 16);
                const uint4 qu = *reinterpret_cast<const uint4*>(uq + c * 16);
                float dg, du;
                dot_chunk2<BITS>(qg, qu, xs4 + (size_t)t * V4 * NCg + c, NCg, dg, du);
                const float xc = xsum[t * NCg + c];
                const float sg = bf1(*reinterpret_cast<const uint16_t*>(sc + g * 2));
                const float bg = bf1(*reinterpret_cast<const uint16_t*>(sc + n * SRg + g * 2));
                const float su = bf1(*reinterpret_cast<const uint16_t*>(sc + 2 * n * SRg + g * 2));
                const float bu = bf1(*reinterpret_cast<const uint16_t*>(sc + 3 * n * SRg + g * 2));
                ag = fmaf(sg, dg, fmaf(bg, xc, ag));
                au = fmaf(su, du, fmaf(bu, xc, au));
              }
#pragma unroll
              for (int o = NCLg / 2; o > 0; o >>= 1) {
                ag += __shfl_xor_sync(0xffffffffu, ag, o);
                au += __shfl_xor_sync(0xffffffffu, au, o);
              }
              if (sub == 0) a.h[(size_t)p * I + r0 + rl] = ag / (1.0f + expf(-ag)) * au;
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[s]);
        ++q;
        f += n;
        done += n;
        if (f == b1) {
          b0 += G * BR;
          b1 = min(b0 + BR, rows_g);
          f = b0;
        }
      }
    }
    bar_cons();
    if (tid == 0 && (!ok || !grid_barrier(a.ctrl, G, nb))) s_abort = 1;
    ++nb;
    bar_cons();
    if (s_abort) break;

    // ---- phase D: down rows j0..j1 of every selected expert and the shared expert ----
    if (nJ > 0) {
      // the first residual element this thread adds in the combine, loaded now
      float res_v = 0.f;
      if (Lc.residual && tid < T * nJ) res_v = bf1(__ldcg(Lc.residual + (size_t)(tid / nJ) * H + j0 + tid % nJ));
      const int per_stage = SB / (nJ * ROWD_BYTES);
      const int sub = lane % NCLd, rsub = lane / NCLd;
      float* red = reinterpret_cast<float*>(smem + a.sm.red) + (size_t)cw * a.jmax * (NCLd + 1);
      const int n_units_d = act_n + (Lc.with_shared ? 1 : 0);  // the shared expert last
      int it0 = 0;  // work items of the earlier stages
      for (int u0 = 0; u0 < n_units_d;) {
        const int cnt = min(per_stage, n_units_d - u0);
        const int s = q % NS;
        if (!mbar_wait(&full_bar[s], (q / NS) & 1)) {
          ok = false;
          atomicOr(&a.ctrl->err, kErrTimeout);
          break;
        }
        const uint8_t* st = ring + (size_t)s * SB;
        // work items: (expert of the stage, one of its token pairs), in stage order and dealt
        // to warps round-robin over the layer, so that an expert with many pairs (the shared
        // one has T) is spread over several warps.  At one token every expert has one pair:
        // the experts themselves are dealt (the same assignment, in a simpler loop).
        const auto n_pairs = [&](int u) { return u == act_n ? T : P_BEGIN[u + 1] - P_BEGIN[u]; };
        const auto do_item = [&](int z, int rem) {
          const int u = u0 + z;
          const bool shared = (u == act_n);
          const uint8_t* dq = st + (size_t)z * nJ * ROWD_BYTES;
          const uint8_t* ds = dq + nJ * ROWBd;
          const uint8_t* db = ds + nJ * SRd;
          const bool have = shared || P_SLOT[u] >= 0;
          const int p = (shared ? n_valid : P_BEGIN[u]) + rem;
          {
            int t;
            float w;
            const float* hsrc;
            if (!shared) {
              const int nn = P_ORDER[p];
              t = nn / k;
              w = P_PW[nn];
              hsrc = a.h + (size_t)p * I;
            } else {
              t = p - n_valid;
              w = P_GATE[t];
              hsrc = a.hs + (size_t)t * I;
            }
            (void)t;
            // this pair's h chunks in registers, pre-scaled like staged activations.  With two
            // lanes per chunk (lane, lane ^ NCLd) each loads one half and they swap halves.
            float4 hr[CPLd][V4];
            float hsum[CPLd];
#pragma unroll
            for (int m = 0; m < CPLd; ++m) {
              const int c = sub + NCLd * m;
              if constexpr (HS == 2) {
#pragma unroll
                for (int vv = 0; vv < VH; ++vv)
                  hr[m][vv] = __ldcg(reinterpret_cast<const float4*>(hsrc + c * CC + 4 * (rsub * VH + vv)));
#pragma unroll
                for (int vv = 0; vv < VH; ++vv) {
                  const float4 own = hr[m][vv];
                  const float4 oth = make_float4(__shfl_xor_sync(0xffffffffu, own.x, NCLd),
                                                 __shfl_xor_sync(0xffffffffu, own.y, NCLd),
                                                 __shfl_xor_sync(0xffffffffu, own.z, NCLd),
                                                 __shfl_xor_sync(0xffffffffu, own.w, NCLd));
                  hr[m][vv] = rsub ? oth : own;
                  hr[m][VH + vv] = rsub ? own : oth;
                }
              } else {
#pragma unroll
                for (int v = 0; v < V4; ++v) hr[m][v] = __ldcg(reinterpret_cast<const float4*>(hsrc + c * CC + 4 * v));
              }
              float sum = 0.f;
#pragma unroll
              for (int v = 0; v < V4; ++v) {
                const float4 f4 = hr[m][v];
                sum += (f4.x + f4.y) + (f4.z + f4.w);
                hr[m][v] = make_float4(f4.x * stage_scale<BITS>(4 * v), f4.y * stage_scale<BITS>(4 * v + 1),
                                       f4.z * stage_scale<BITS>(4 * v + 2), f4.w * stage_scale<BITS>(4 * v + 3));
              }
              hsum[m] = sum;
            }
            // per-lane partial dots of every row, then a fixed-order sum per row through
            // shared memory (no shuffle chain per row)
            for (int rs = 0; rs < nJ / RPWd; ++rs) {
              const int jl = rs * RPWd + rsub;
              float part = 0.f;
              if (have) {
#pragma unroll
                for (int m = 0; m < CPLd; ++m) {
                  const int c = sub + NCLd * m, g = c * CC / kGroup;
                  const uint4 qd = *reinterpret_cast<const uint4*>(dq + jl * ROWBd + c * 16);
                  const float sd = bf1(*reinterpret_cast<const uint16_t*>(ds + jl * SRd + g * 2));
                  const float bd = bf1(*reinterpret_cast<const uint16_t*>(db + jl * SRd + g * 2));
                  const float d = dot_chunk<BITS>(qd, hr[m], 1);
                  part = fmaf(sd, d, fmaf(bd, hsum[m], part));
                }
              }
              red[jl * (NCLd + 1) + sub] = part;
            }
            __syncwarp();
            for (int jl = lane; jl < nJ; jl += 32) {
              float sum = 0.f;
#pragma unroll
              for (int qq = 0; qq < NCLd; ++qq) sum += red[jl * (NCLd + 1) + qq];
              partial[(size_t)p * a.jmax + jl] = w * sum;
            }
            __syncwarp();
          }
        };
        int n_items = 0;
        if constexpr (TM == 1) {
          for (int z = (cw - u0 % kCons + kCons) % kCons; z < cnt; z += kCons)
            for (int rem = 0; rem < n_pairs(u0 + z); ++rem) do_item(z, rem);
          n_items = cnt;
        } else {
          for (int z = 0; z < cnt; ++z) n_items += n_pairs(u0 + z);
          for (int i = (cw - it0 % kCons + kCons) % kCons; i < n_items; i += kCons) {
            int z = 0, rem = i;
            while (rem >= n_pairs(u0 + z)) rem -= n_pairs(u0 + z++);
            do_item(z, rem);
          }
        }
        it0 += n_items;
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[s]);
        ++q;
        u0 += cnt;
      }
      bar_cons();
      // combine in a fixed order: top-k slots, then the shared expert, then the residual
      if (ok) {
        for (int i = tid; i < T * nJ; i += kConsThreads) {
          const int t = i / nJ, jl = i - t * nJ;
          float v = 0.f;
          for (int kk = 0; kk < k; ++kk) {
            const int p = P_POS[t * k + kk];
            if (p >= 0) v += partial[(size_t)p * a.jmax + jl];
          }
          if (Lc.with_shared) v += partial[(size_t)(n_valid + t) * a.jmax + jl];
          if (Lc.out_partial) {
            // expert parallelism: this rank's fp32 share of the sum; the ranks' shares are
            // added by an all-reduce and rounded once, with the residual, by the combine
            Lc.out_partial[(size_t)t * H + j0 + jl] = v;
          } else {
            if (Lc.residual) v += (i == tid) ? res_v : bf1(__ldcg(Lc.residual + (size_t)t * H + j0 + jl));
            Lc.out[(size_t)t * H + j0 + jl] = f2bf(v);
          }
        }
      }
    }
    bar_cons();
    if (tid == 0 && (!ok || !grid_barrier(a.ctrl, G, nb))) s_abort = 1;
    ++nb;
    bar_cons();
    if (s_abort) break;
  }
  // on an early exit make sure the streaming warp is not left waiting for a plan
  if (tid == 0 && s_abort) {
    s_abort = 1;
    mbar_arrive(&plan_bar);
  }
  if (tid == 0 && !s_abort) grid_exit(a.ctrl, G);
}

}  // namespace

static size_t fused_smem_bytes(const FusedArgs& a, int stages) {
  return fused_smem_layout(a.T, a.H, a.I, a.E, a.bits, a.k, a.jmax, stages, a.stage_bytes, kCons, a.rr_max,
                           a.rs_max).total;
}

template <int BITS, int H, int I, int TM>
static cudaError_t run_fused(FusedArgs a, cudaStream_t s) {
  static int n_sm = 0;
  if (!n_sm) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  }
  int max_smem = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  max_smem -= 2048;  // static shared memory and reserve
  // output-row slice of a CTA (granule gD rows)
  constexpr int CC = 128 / BITS, NCd = I / CC, NCLd = NCd < 32 ? NCd : 32, RPWd = 32 / NCLd;
  constexpr int SRd = (I / kGroup) * 2;
  constexpr int gD = clcm(16 / cgcd(16, SRd), RPWd);
  const int nGran = H / gD;
  a.jmax = ((nGran + n_sm - 1) / n_sm) * gD;
  // phase-R rows a CTA stages: its share of the E + 1 router rows and of the shared expert's
  // rows (in granules of gG rows)
  constexpr int NCg = H / CC, NCLg = NCg < 32 ? NCg : 32, RPWg = 32 / NCLg, SRg = (H / kGroup) * 2;
  constexpr int gG = clcm(16 / cgcd(16, SRg), RPWg);
  a.rr_max = (a.E + 1 + n_sm - 1) / n_sm;
  a.rs_max = ((I / gG + n_sm - 1) / n_sm) * gG;
  // ring stages of 32 KB, or 24 KB where that keeps four of them
  int stages = 2;
  for (int sb : {32768, 24576}) {
    a.stage_bytes = sb;
    stages = kMaxStages;
    while (stages > 2 && fused_smem_bytes(a, stages) > (size_t)max_smem) --stages;
    if (stages >= 4) break;
  }
  a.n_stages = stages;
  a.sm = fused_smem_layout(a.T, a.H, a.I, a.E, a.bits, a.k, a.jmax, stages, a.stage_bytes, kCons, a.rr_max,
                           a.rs_max);
  const size_t smem = a.sm.total;
  if (smem > (size_t)max_smem) return cudaErrorInvalidConfiguration;
  // one stage must hold one gate/up row and one expert's down slice
  if ((size_t)a.jmax * ((I * BITS / 8) + 2 * SRd) > (size_t)a.stage_bytes) return cudaErrorInvalidConfiguration;
  auto fn = k_fused_decode<BITS, H, I, TM>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int bps = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, fn, kFThreads, smem);
  if (e != cudaSuccess) return e;
  if (bps < 1) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_sm);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, a);
}

bool fused_shape_supported(int H, int I, int bits, int E) {
  return E <= kFusedMaxE && (bits == 4 || bits == 8) && ((H == 2048 && I == 512) || (H == 256 && I == 64) ||
                                      (H == 512 && I == 128) || (H == 1024 && I == 256) ||
                                      (H == 4096 && I == 1024));
}

cudaError_t launch_fused_decode(const FusedArgs& a, cudaStream_t s, bool* supported) {
  *supported = true;
#define MOE_FD(B, HH, II)                                            \
  if (a.bits == B && a.H == HH && a.I == II) {                       \
    if (a.T == 1) return run_fused<B, HH, II, 1>(a, s);              \
    return run_fused<B, HH, II, kMaxDecodeT>(a, s);                  \
  }
  MOE_FD(4, 2048, 512) MOE_FD(8, 2048, 512) MOE_FD(4, 256, 64) MOE_FD(8, 256, 64)
  MOE_FD(4, 512, 128) MOE_FD(8, 512, 128) MOE_FD(4, 1024, 256) MOE_FD(8, 1024, 256)
  MOE_FD(4, 4096, 1024) MOE_FD(8, 4096, 1024)
#undef MOE_FD
  *supported = false;
  return cudaSuccess;
}

}  // namespace moe
