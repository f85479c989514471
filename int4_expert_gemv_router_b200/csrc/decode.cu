// Decode-path kernels of the routed-MoE layer (T <= 8 tokens per call), sm_100a.
//
//   k_router   router GEMV (bf16 x bf16 products, exact in fp32, summed in fp64) over the
//              E expert rows plus the shared-gate row; the last CTA to finish selects the
//              top-k per token, applies the softmax over the selected logits, computes the
//              shared-expert gate and groups the (token, k) pairs by expert.
//   k_plan     the same grouping and shared gate when the caller supplies the top-k.
//   k_gateup   per (distinct expert, intermediate row): a = Wg.x, u = Wu.x over the packed
//              int4/int8 codes with the per-group bias folded in, h = silu(a) * u.
//   k_down     per output row j: sum over distinct experts of p * (Wd.h) plus the gated
//              shared expert and the residual, rounded to bf16.
//
// What they compute follows the Swiftlet pages («Paquets Swiftlet 80B Qwen dans Mac…»,
// paragraphs 5 and 9): router top-k of E experts per token, MLX-style affine group-64
// int4/int8 expert weights, a high-sparsity MoE with a shared expert.
//
// Inner-loop arithmetic.  For one row and one quantisation group g,
//     sum_i (s_g q_i + b_g) x_i = s_g * sum_i q_i x_i + b_g * X_g,   X_g = sum_{i in g} x_i,
// so codes are never dequantised: the kernels form sum q_i x_i and apply scale and bias once
// per 16-byte chunk.  A code q at bit position p of its 32-bit word is turned into the exact
// float q * 2^p by OR-ing the masked word into the mantissa of 2^23 and subtracting 2^23
// (p + 4 <= 23 keeps the value exact); the activation it multiplies was pre-scaled by
// 2^-p when it was staged in shared memory, so the product is exactly q * x.  Two codes go
// through one packed fp32x2 add and one packed fp32x2 FMA.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// ---------------------------------------------------------------------------------------
// Router dot product of one 8-element bf16 chunk of a weight row with staged x (fp32).
// Products of two bf16 values are exact in fp32; they are summed in fp64 in a fixed order.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ double router_chunk(const uint4& w, const float4& xa, const float4& xb) {
  double s = (double)(bf_lo(w.x) * xa.x);
  s += (double)(bf_hi(w.x) * xa.y);
  s += (double)(bf_lo(w.y) * xa.z);
  s += (double)(bf_hi(w.y) * xa.w);
  s += (double)(bf_lo(w.z) * xb.x);
  s += (double)(bf_hi(w.z) * xb.y);
  s += (double)(bf_lo(w.w) * xb.z);
  s += (double)(bf_hi(w.w) * xb.w);
  return s;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// x [T, H] bf16 -> shared fp32, router layout: chunk c (8 values) of token t as two float4 at
// xs[(t*2 + 0)*NCR + c] and xs[(t*2 + 1)*NCR + c].
__device__ __forceinline__ void stage_router_x(float4* xs, const uint16_t* x, int T, int H) {
  const int NCR = H / 8;
  for (int i = threadIdx.x; i < T * NCR; i += blockDim.x) {
    const int t = i / NCR, c = i - t * NCR;
    const uint4 raw = *reinterpret_cast<const uint4*>(x + (size_t)t * H + c * 8);
    xs[(t * 2 + 0) * NCR + c] = make_float4(bf_lo(raw.x), bf_hi(raw.x), bf_lo(raw.y), bf_hi(raw.y));
    xs[(t * 2 + 1) * NCR + c] = make_float4(bf_lo(raw.z), bf_hi(raw.z), bf_lo(raw.w), bf_hi(raw.w));
  }
}

// Logit of one row (E expert rows, or the shared-gate row) for token t, computed by one warp.
__device__ __forceinline__ double row_dot_warp(const uint16_t* row, const float4* xs, int t, int H) {
  const int NCR = H / 8, lane = threadIdx.x & 31;
  double acc = 0.0;
  for (int c = lane; c < NCR; c += 32) {
    const uint4 w = ld_stream(row + c * 8);
    acc += router_chunk(w, xs[(t * 2) * NCR + c], xs[(t * 2 + 1) * NCR + c]);
  }
  return warp_sum_d(acc);
}

// ---------------------------------------------------------------------------------------
// Grouping of the n = T*k (token, slot) pairs by expert (stable counting-sort semantics:
// pairs sorted by (expert, pair number)), for n <= blockDim.x.  Pairs whose id is outside
// [0, E) are flagged and left out.  Writes order, act_e, act_begin, ctrl->act_n, n_valid.
// ---------------------------------------------------------------------------------------
__device__ void build_plan_block(const int* ids, int n, const DecodeArgs& a) {
  __shared__ int s_key[kThreads];
  __shared__ int s_first[kThreads];
  const int i = threadIdx.x, E = a.E;
  int key = E;
  bool valid = false;
  if (i < n) {
    const int e = ids[i];
    valid = (e >= 0 && e < E);
    key = valid ? e : E;
    if (!valid) atomicOr(&a.ctrl->err, kErrBadExpert);
    s_key[i] = key;
  }
  __syncthreads();
  int rank = 0, first = 1;
  if (i < n) {
    for (int j = 0; j < n; ++j) {
      const int kj = s_key[j];
      rank += (kj < key) || (kj == key && j < i);
      if (kj == key && j < i) first = 0;
    }
    a.order[rank] = i;
    s_first[i] = (first && valid) ? 1 : 0;
  }
  __syncthreads();
  if (i < n && s_first[i]) {
    int act = 0;
    for (int j = 0; j < n; ++j) act += (s_first[j] && s_key[j] < key);
    a.act_e[act] = key;
    a.act_begin[act] = rank;
  }
  const int act_n = __syncthreads_count(i < n && s_first[i]);
  const int n_valid = __syncthreads_count(i < n && valid);
  if (i == 0) {
    a.act_begin[act_n] = n_valid;
    a.ctrl->act_n = act_n;
    a.ctrl->n_valid = n_valid;
  }
}

// ---------------------------------------------------------------------------------------
// K1: router
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads) k_router(const DecodeArgs a, int build_plan) {
  extern __shared__ float4 smem4[];
  __shared__ int s_ids[kMaxDecodeT * kMaxTopK];
  __shared__ int s_last;
  const int H = a.H, T = a.T, E = a.E, k = a.k;
  stage_router_x(smem4, a.x, T, H);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = gridDim.x * kWarps;
  const int NCR = H / 8;
  for (int e = blockIdx.x * kWarps + warp; e <= E; e += nw) {
    const uint16_t* row = (e < E) ? a.wr + (size_t)e * H : a.wsg;
    // Same per-token operation sequence as row_dot_warp (so the shared-gate logit is
    // bit-identical to the one k_plan computes), with the row read once for all tokens.
    double acc[kMaxDecodeT];
#pragma unroll
    for (int t = 0; t < kMaxDecodeT; ++t) acc[t] = 0.0;
    for (int c = lane; c < NCR; c += 32) {
      const uint4 w = ld_stream(row + c * 8);
#pragma unroll
      for (int t = 0; t < kMaxDecodeT; ++t)
        if (t < T) acc[t] += router_chunk(w, smem4[(t * 2) * NCR + c], smem4[(t * 2 + 1) * NCR + c]);
    }
#pragma unroll
    for (int t = 0; t < kMaxDecodeT; ++t) {
      if (t < T) {
        double l = warp_sum_d(acc[t]);
        if (lane == 0) {
          if (e < E && a.rbias) l += (double)a.rbias[e];
          a.logits[(size_t)t * (E + 1) + e] = l;
        }
      }
    }
  }
  // last CTA to finish does top-k, softmax, shared gate and grouping
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&a.ctrl->ticket, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int t = warp; t < T; t += kWarps) {
    const double* lt = a.logits + (size_t)t * (E + 1);
    double v[kMaxExperts / 32];
#pragma unroll
    for (int m = 0; m < kMaxExperts / 32; ++m) {
      const int e = lane + 32 * m;
      v[m] = (e < E) ? __ldcg(lt + e) : 0.0;
    }
    uint32_t taken = 0;
    double sel_v0 = 0.0, denom = 0.0;
    double my_v = 0.0;
    int my_e = -1;
    for (int r = 0; r < k; ++r) {
      double bv = 0.0;
      int be = 0x7fffffff;
#pragma unroll
      for (int m = 0; m < kMaxExperts / 32; ++m) {
        const int e = lane + 32 * m;
        if (e < E && !((taken >> m) & 1u) && (be == 0x7fffffff || v[m] > bv)) {
          if (v[m] == v[m]) {  // NaN never wins
            bv = v[m];
            be = e;
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        const bool better = (oe != 0x7fffffff) && (be == 0x7fffffff || ov > bv || (ov == bv && oe < be));
        if (better) {
          bv = ov;
          be = oe;
        }
      }
      if (be == 0x7fffffff || !isfinite(bv)) {
        if (lane == 0) atomicOr(&a.ctrl->err, kErrNonFinite);
        if (be == 0x7fffffff) be = -1;
      }
      if (be >= 0 && (be & 31) == lane) taken |= 1u << (be >> 5);
      if (r == 0) sel_v0 = bv;
      const double ex = (be >= 0) ? exp(bv - sel_v0) : 0.0;
      denom += ex;
      if (lane == r) {
        my_v = ex;
        my_e = be;
      }
    }
    // lane r holds slot r's numerator; write ids and weights
    if (lane < k) {
      a.topk_idx[t * k + lane] = my_e;
      a.topk_w[t * k + lane] = (float)(my_v / denom);
      s_ids[t * k + lane] = my_e;
    }
    if (lane == 0) a.gate[t] = (float)(1.0 / (1.0 + exp(-__ldcg(lt + E))));
  }
  __syncthreads();
  if (build_plan) build_plan_block(s_ids, T * k, a);
  if (threadIdx.x == 0) a.ctrl->ticket = 0u;
}

// Grouping + shared gate when the caller supplies the top-k (one CTA).
__global__ void __launch_bounds__(kThreads) k_plan(const DecodeArgs a) {
  extern __shared__ float4 smem4[];
  __shared__ int s_ids[kMaxDecodeT * kMaxTopK];
  const int H = a.H, T = a.T, k = a.k;
  stage_router_x(smem4, a.x, T, H);
  for (int i = threadIdx.x; i < T * k; i += blockDim.x) s_ids[i] = a.topk_idx[i];
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int t = warp; t < T; t += kWarps) {
    const double l = row_dot_warp(a.wsg, smem4, t, H);
    if (lane == 0) a.gate[t] = (float)(1.0 / (1.0 + exp(-l)));
  }
  build_plan_block(s_ids, T * k, a);
}

// ---------------------------------------------------------------------------------------
// K2: gate/up GEMV + SwiGLU.  Rows of all distinct routed experts, then the shared
// expert's rows, are split evenly over every warp of the grid; a warp handles RPW rows per
// step (RPW > 1 when a row is fewer than 32 chunks).
// ---------------------------------------------------------------------------------------
template <int BITS, int K>
__global__ void __launch_bounds__(kThreads) k_gateup(const DecodeArgs a) {
  constexpr int CC = 128 / BITS, NC = K / CC, NCL = NC < 32 ? NC : 32, RPW = 32 / NCL;
  constexpr int CPL = NC / NCL, V4 = CC / 4, ROWB = K * BITS / 8, NG = K / kGroup;
  extern __shared__ float4 smem4[];
  const int T = a.T;
  float4* xs4 = smem4;
  float* xsum = reinterpret_cast<float*>(smem4 + (size_t)T * V4 * NC);
  stage_vectors<BITS, K>(xs4, xsum, T, threadIdx.x, blockDim.x, [&](int r, int i) {
    const uint2 raw = *reinterpret_cast<const uint2*>(a.x + (size_t)r * K + i);
    return make_float4(bf_lo(raw.x), bf_hi(raw.x), bf_lo(raw.y), bf_hi(raw.y));
  });
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % NCL, rsub = lane / NCL;
  const int I = a.I, Is = a.Is;
  const int rows_routed = a.ctrl->act_n * I;
  const int steps = (rows_routed + Is) / RPW;
  const int W = gridDim.x * kWarps, gw = blockIdx.x * kWarps + warp;
  const int s0 = (int)((long long)gw * steps / W), s1 = (int)((long long)(gw + 1) * steps / W);
  for (int s = s0; s < s1; ++s) {
    const int f0 = s * RPW;
    const bool shared = f0 >= rows_routed;
    const uint8_t* blob;
    int r, pbeg, pend;
    if (!shared) {
      const int u = f0 / I;
      r = f0 - u * I + rsub;
      const int slot = a.slot_table[a.act_e[u]];
      if (slot < 0 || slot >= a.n_slots) {
        if (lane == 0) atomicOr(&a.ctrl->err, kErrBadSlot);
        continue;
      }
      blob = a.pool + (int64_t)slot * a.L.stride;
      pbeg = a.act_begin[u];
      pend = a.act_begin[u + 1];
    } else {
      r = f0 - rows_routed + rsub;
      blob = a.shared_blob;
      pbeg = 0;
      pend = T;
    }
    const uint8_t* gq = blob + a.L.off[0] + (int64_t)r * ROWB;
    const uint8_t* uq = blob + a.L.off[1] + (int64_t)r * ROWB;
    const uint16_t* gs = reinterpret_cast<const uint16_t*>(blob + a.L.off[3]) + r * NG;
    const uint16_t* gb = reinterpret_cast<const uint16_t*>(blob + a.L.off[4]) + r * NG;
    const uint16_t* us = reinterpret_cast<const uint16_t*>(blob + a.L.off[5]) + r * NG;
    const uint16_t* ub = reinterpret_cast<const uint16_t*>(blob + a.L.off[6]) + r * NG;
    uint4 qg[CPL], qu[CPL];
    float sg[CPL], bg[CPL], su[CPL], bu[CPL];
#pragma unroll
    for (int m = 0; m < CPL; ++m) {
      const int c = sub + NCL * m;
      qg[m] = ld_stream(gq + c * 16);
      qu[m] = ld_stream(uq + c * 16);
      const int g = c * CC / kGroup;
      sg[m] = bf1(ld_u16(gs + g));
      bg[m] = bf1(ld_u16(gb + g));
      su[m] = bf1(ld_u16(us + g));
      bu[m] = bf1(ld_u16(ub + g));
    }
    for (int p = pbeg; p < pend; ++p) {
      const int t = shared ? p : a.order[p] / a.k;
      const float4* xt = xs4 + (size_t)t * V4 * NC;
      const float* st = xsum + t * NC;
      float ag = 0.f, au = 0.f;
#pragma unroll
      for (int m = 0; m < CPL; ++m) {
        const int c = sub + NCL * m;
        float dg, du;
        dot_chunk2<BITS>(qg[m], qu[m], xt + c, NC, dg, du);
        const float xc = st[c];
        ag = fmaf(sg[m], dg, fmaf(bg[m], xc, ag));
        au = fmaf(su[m], du, fmaf(bu[m], xc, au));
      }
#pragma unroll
      for (int o = NCL / 2; o > 0; o >>= 1) {
        ag += __shfl_xor_sync(0xffffffffu, ag, o);
        au += __shfl_xor_sync(0xffffffffu, au, o);
      }
      if (sub == 0) {
        const float hv = ag / (1.0f + expf(-ag)) * au;
        if (shared)
          a.hs[(size_t)t * Is + r] = hv;
        else
          a.h[(size_t)p * I + r] = hv;
      }
    }
  }
}

// ---------------------------------------------------------------------------------------
// K3: down GEMV + top-k combine + gated shared expert + residual, one output row per
// NCL lanes.  Every routed pair's h (and each token's shared h) is staged in shared memory.
// The sum runs over distinct experts in ascending id, then the shared expert, in a fixed
// order, so the result does not depend on where the experts sit in the pool.
// ---------------------------------------------------------------------------------------
template <int BITS, int K, int TM>
__global__ void __launch_bounds__(kThreads) k_down(const DecodeArgs a) {
  constexpr int CC = 128 / BITS, NC = K / CC, NCL = NC < 32 ? NC : 32, RPW = 32 / NCL;
  constexpr int CPL = NC / NCL, V4 = CC / 4, ROWB = K * BITS / 8, NG = K / kGroup;
  extern __shared__ float4 smem4[];
  const int T = a.T, H = a.H, I = a.I;
  const int act_n = a.ctrl->act_n, nv = a.ctrl->n_valid;
  const int np = nv + T;
  float4* hs4 = smem4;
  float* hsum = reinterpret_cast<float*>(smem4 + (size_t)np * V4 * NC);
  stage_vectors<BITS, K>(hs4, hsum, np, threadIdx.x, blockDim.x, [&](int p, int i) {
    const float* src = (p < nv) ? a.h + (size_t)p * I : a.hs + (size_t)(p - nv) * I;
    return *reinterpret_cast<const float4*>(src + i);
  });
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % NCL, rsub = lane / NCL;
  const int steps = H / RPW;
  const int W = gridDim.x * kWarps, gw = blockIdx.x * kWarps + warp;
  const int s0 = (int)((long long)gw * steps / W), s1 = (int)((long long)(gw + 1) * steps / W);
  for (int s = s0; s < s1; ++s) {
    const int j = s * RPW + rsub;
    float acc[TM];
#pragma unroll
    for (int t = 0; t < TM; ++t) acc[t] = 0.f;
    for (int u = 0; u <= act_n; ++u) {
      const bool shared = (u == act_n);
      const uint8_t* blob;
      int pbeg, pend;
      if (!shared) {
        const int slot = a.slot_table[a.act_e[u]];
        if (slot < 0 || slot >= a.n_slots) {
          if (lane == 0) atomicOr(&a.ctrl->err, kErrBadSlot);
          continue;
        }
        blob = a.pool + (int64_t)slot * a.L.stride;
        pbeg = a.act_begin[u];
        pend = a.act_begin[u + 1];
      } else {
        blob = a.shared_blob;
        pbeg = nv;
        pend = nv + T;
      }
      const uint8_t* dq = blob + a.L.off[2] + (int64_t)j * ROWB;
      const uint16_t* ds = reinterpret_cast<const uint16_t*>(blob + a.L.off[7]) + j * NG;
      const uint16_t* db = reinterpret_cast<const uint16_t*>(blob + a.L.off[8]) + j * NG;
      uint4 q[CPL];
      float sd[CPL], bd[CPL];
#pragma unroll
      for (int m = 0; m < CPL; ++m) {
        const int c = sub + NCL * m;
        q[m] = ld_stream(dq + c * 16);
        const int g = c * CC / kGroup;
        sd[m] = bf1(ld_u16(ds + g));
        bd[m] = bf1(ld_u16(db + g));
      }
      for (int p = pbeg; p < pend; ++p) {
        int t;
        float w;
        if (!shared) {
          const int n = a.order[p];
          t = n / a.k;
          w = a.topk_w[n];
        } else {
          t = p - nv;
          w = a.gate[t];
        }
        const float4* hp = hs4 + (size_t)p * V4 * NC;
        const float* sp = hsum + p * NC;
        float part = 0.f;
#pragma unroll
        for (int m = 0; m < CPL; ++m) {
          const int c = sub + NCL * m;
          const float d = dot_chunk<BITS>(q[m], hp + c, NC);
          part = fmaf(sd[m], d, fmaf(bd[m], sp[c], part));
        }
        if constexpr (TM == 1) {
          acc[0] = fmaf(w, part, acc[0]);
        } else {
#pragma unroll
          for (int tt = 0; tt < TM; ++tt) acc[tt] = (tt == t) ? fmaf(w, part, acc[tt]) : acc[tt];
        }
      }
    }
#pragma unroll
    for (int tt = 0; tt < TM; ++tt) {
      if (tt < T) {
        float v = acc[tt];
#pragma unroll
        for (int o = NCL / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (sub == 0) {
          if (a.residual) v += bf1(a.residual[(size_t)tt * H + j]);
          a.out[(size_t)tt * H + j] = f2bf(v);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------------------
// launch helpers
// ---------------------------------------------------------------------------------------
int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <typename F>
cudaError_t prepare(F* fn, size_t smem, int* blocks_per_sm) {
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, fn, kThreads, smem);
}

template <int BITS, int K>
size_t gateup_smem(int T) {
  constexpr int CC = 128 / BITS, NC = K / CC;
  return (size_t)T * K * 4 + (size_t)T * NC * 4;
}

template <int BITS, int K>
cudaError_t run_gateup(const DecodeArgs& a, cudaStream_t s) {
  const size_t smem = gateup_smem<BITS, K>(a.T);
  int bps = 0;
  cudaError_t e = prepare(k_gateup<BITS, K>, smem, &bps);
  if (e != cudaSuccess) return e;
  if (bps < 1) return cudaErrorInvalidConfiguration;
  k_gateup<BITS, K><<<num_sms() * bps, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <int BITS, int K>
cudaError_t run_down(const DecodeArgs& a, cudaStream_t s) {
  constexpr int CC = 128 / BITS, NC = K / CC;
  const int np = a.T * a.k + a.T;  // upper bound of staged pairs
  const size_t smem = (size_t)np * K * 4 + (size_t)np * NC * 4;
  int bps = 0;
  cudaError_t e;
  if (a.T == 1) {
    e = prepare(k_down<BITS, K, 1>, smem, &bps);
    if (e != cudaSuccess) return e;
    if (bps < 1) return cudaErrorInvalidConfiguration;
    k_down<BITS, K, 1><<<num_sms() * bps, kThreads, smem, s>>>(a);
  } else {
    e = prepare(k_down<BITS, K, kMaxDecodeT>, smem, &bps);
    if (e != cudaSuccess) return e;
    if (bps < 1) return cudaErrorInvalidConfiguration;
    k_down<BITS, K, kMaxDecodeT><<<num_sms() * bps, kThreads, smem, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace

bool decode_shape_supported(int H, int I, int bits) {
  auto pow2_in = [](int v, int lo, int hi) { return v >= lo && v <= hi && (v & (v - 1)) == 0; };
  return (bits == 4 || bits == 8) && pow2_in(H, 256, 4096) && pow2_in(I, 64, 1024);
}

cudaError_t launch_router_decode(const DecodeArgs& a, bool build_plan, cudaStream_t s) {
  const size_t smem = (size_t)a.T * a.H * 4;
  cudaError_t e = cudaFuncSetAttribute(k_router, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int rows = a.E + 1;
  int blocks = (rows + kWarps - 1) / kWarps;
  if (blocks > 2 * num_sms()) blocks = 2 * num_sms();
  k_router<<<blocks, kThreads, smem, s>>>(a, build_plan ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_plan_decode(const DecodeArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)a.T * a.H * 4;
  cudaError_t e = cudaFuncSetAttribute(k_plan, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_plan<<<1, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gateup_decode(const DecodeArgs& a, int bits, cudaStream_t s, bool* supported) {
  *supported = true;
#define MOE_GU(B, K) \
  if (bits == B && a.H == K) return run_gateup<B, K>(a, s);
  MOE_GU(4, 256) MOE_GU(4, 512) MOE_GU(4, 1024) MOE_GU(4, 2048) MOE_GU(4, 4096)
  MOE_GU(8, 256) MOE_GU(8, 512) MOE_GU(8, 1024) MOE_GU(8, 2048) MOE_GU(8, 4096)
#undef MOE_GU
  *supported = false;
  return cudaSuccess;
}

cudaError_t launch_down_decode(const DecodeArgs& a, int bits, cudaStream_t s, bool* supported) {
  *supported = true;
#define MOE_DN(B, K) \
  if (bits == B && a.I == K) return run_down<B, K>(a, s);
  MOE_DN(4, 64) MOE_DN(4, 128) MOE_DN(4, 256) MOE_DN(4, 512) MOE_DN(4, 1024)
  MOE_DN(8, 64) MOE_DN(8, 128) MOE_DN(8, 256) MOE_DN(8, 512) MOE_DN(8, 1024)
#undef MOE_DN
  *supported = false;
  return cudaSuccess;
}

// out = bf16(sum of the partials in index order + residual): the combine of an
// expert-parallel layer after the partials have been summed across ranks (or, on one GPU,
// several ranks' partials summed here).
__global__ void k_combine_partials(const PartialArgs p) {
  const size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i >= p.count) return;
  if (i + 4 <= p.count) {
    float4 v = __ldg(reinterpret_cast<const float4*>(p.part[0] + i));
    for (int r = 1; r < p.n; ++r) {
      const float4 w = __ldg(reinterpret_cast<const float4*>(p.part[r] + i));
      v.x += w.x;
      v.y += w.y;
      v.z += w.z;
      v.w += w.w;
    }
    if (p.residual) {
      const uint2 rr = __ldg(reinterpret_cast<const uint2*>(p.residual + i));
      v.x += bf_lo(rr.x);
      v.y += bf_hi(rr.x);
      v.z += bf_lo(rr.y);
      v.w += bf_hi(rr.y);
    }
    uint2 o;
    o.x = (uint32_t)f2bf(v.x) | ((uint32_t)f2bf(v.y) << 16);
    o.y = (uint32_t)f2bf(v.z) | ((uint32_t)f2bf(v.w) << 16);
    *reinterpret_cast<uint2*>(p.out + i) = o;
  } else {
    for (size_t j = i; j < p.count; ++j) {
      float v = p.part[0][j];
      for (int r = 1; r < p.n; ++r) v += p.part[r][j];
      if (p.residual) v += bf1(p.residual[j]);
      p.out[j] = f2bf(v);
    }
  }
}

cudaError_t launch_combine_partials(const PartialArgs& p, cudaStream_t s) {
  const size_t n4 = (p.count + 3) / 4;
  k_combine_partials<<<(unsigned)((n4 + 255) / 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace moe
