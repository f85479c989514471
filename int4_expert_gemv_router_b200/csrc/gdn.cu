// Gated DeltaNet decode step (the linear-attention layers of the hybrid model), sm_100a.
//
// The pages: three quarters of the layers are Gated DeltaNet linear attention whose state
// has a fixed size whatever the context length («Paquets Swiftlet 80B Qwen dans Mac…»,
// paragraph 6; «Swiftlet: 在 Mac 和 iPhone 上執行…», section 技術譜系與正確性, which
// checks the Gated DeltaNet recurrence layer by layer).  One decode step of one sequence
// and one value head h, with the state S (d_v x d_k, fp32) mapping keys to values:
//
//     k^ = k / ||k||,  q^ = q / (||q|| sqrt(d_k))        (key head h / (H_v / H_k))
//     u  = S k^                                            (what the old state recalls)
//     S' = alpha S + beta (v - alpha u) k^T,  alpha = exp(g)
//     o  = S' q^
//
// i.e. S' = alpha S (I - beta k^ k^T) + beta v k^T, the gated delta rule.  Every row i of S
// is independent given k^ and q^ (u_i, the row update and o_i use row i only), so a warp
// owns whole rows: each lane holds d_k / 32 consecutive elements of a row in registers
// (one 16-byte load for d_k = 128), two warp sums give u_i and o_i, and the row is written
// back once.  A CTA covers 16, 32 or 64 rows of one (sequence, value head) (2, 4 or 8 per warp,
// all loaded at once): it normalises that head's k and q once, in shared memory.  The step reads and writes the state once: HBM bound,
// 2 * 4 * d_k * d_v bytes per (sequence, value head).
#include "../../include/moe.h"
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

struct GdnArgs {
  int B, Hk, Hv, dk, dv;
  float* S;              // [B, Hv, dv, dk]
  const uint16_t* q;     // bf16 [B, Hk, dk]
  const uint16_t* k;     // bf16 [B, Hk, dk]
  const uint16_t* v;     // bf16 [B, Hv, dv]
  const float* g;        // [B, Hv]
  const float* beta;     // [B, Hv]
  uint16_t* out;         // bf16 [B, Hv, dv]
};

namespace {

constexpr int kGdnWarps = 8;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// RPW rows per warp (2, 4 or 8), all loaded at once: the fewest that still fit the launch in
// one round of resident CTAs, so that every SM has as many bytes in flight as its rows give.
template <int DK, int RPW>
__global__ void __launch_bounds__(kGdnWarps * 32) k_gdn_step(const GdnArgs a) {
  constexpr int kGdnRowsPerWarp = RPW, kGdnRows = kGdnWarps * RPW;  // rows of S per CTA
  constexpr int EPL = DK / 32;  // elements of a row per lane
  static_assert(EPL == 2 || EPL == 4 || EPL == 8, "d_k of 64, 128 or 256");
  __shared__ float s_kq[2][DK];
  const int blocks_per_head = (a.dv + kGdnRows - 1) / kGdnRows;
  const int bh = blockIdx.x / blocks_per_head;  // b * Hv + h
  const int rb = blockIdx.x - bh * blocks_per_head;
  const int b = bh / a.Hv, h = bh - b * a.Hv;
  const int kh = h / (a.Hv / a.Hk);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* Sh = a.S + (size_t)bh * a.dv * DK;
  // the next kernel on the stream may start launching (it waits for this one where it must)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // the rows this warp owns, loaded first so that their latency overlaps the normalisation
  float row[kGdnRowsPerWarp][EPL];
  int ri[kGdnRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kGdnRowsPerWarp; ++r) {
    ri[r] = rb * kGdnRows + warp * kGdnRowsPerWarp + r;
    if (ri[r] < a.dv) {
      const float* src = Sh + (size_t)ri[r] * DK + lane * EPL;
      if constexpr (EPL % 4 == 0) {
#pragma unroll
        for (int e = 0; e < EPL; e += 4) {
          const float4 f = __ldcs(reinterpret_cast<const float4*>(src + e));
          row[r][e] = f.x;
          row[r][e + 1] = f.y;
          row[r][e + 2] = f.z;
          row[r][e + 3] = f.w;
        }
      } else {
        const float2 f = __ldcs(reinterpret_cast<const float2*>(src));
        row[r][0] = f.x;
        row[r][1] = f.y;
      }
    }
  }
  // Launched as a programmatic dependent (MOE_GDN_EARLY_STATE), the state rows above were read
  // while the kernel before may still run (the caller guarantees it does not write them);
  // from here on every read and write waits for it to have finished.  Without that launch
  // attribute the wait returns at once.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // k and q of this head's key head: warp 0 normalises k, warp 1 q (fp32 sums of squares)
  if (warp < 2) {
    const uint16_t* src = (warp == 0 ? a.k : a.q) + ((size_t)b * a.Hk + kh) * DK;
    float vals[EPL];
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      vals[e] = bf1(src[lane * EPL + e]);
      ss = fmaf(vals[e], vals[e], ss);
    }
    ss = warp_sum(ss);
    // 1 / max(||.||, 1e-6), and the query's 1/sqrt(d_k)
    float inv = 1.0f / fmaxf(sqrtf(ss), 1e-6f);
    if (warp == 1) inv *= rsqrtf((float)DK);
#pragma unroll
    for (int e = 0; e < EPL; ++e) s_kq[warp][lane * EPL + e] = vals[e] * inv;
  }
  __syncthreads();
  float kn[EPL], qn[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    kn[e] = s_kq[0][lane * EPL + e];
    qn[e] = s_kq[1][lane * EPL + e];
  }
  const float alpha = expf(a.g[bh]);
  const float beta = a.beta[bh];
#pragma unroll
  for (int r = 0; r < kGdnRowsPerWarp; ++r) {
    if (ri[r] >= a.dv) continue;  // the whole warp takes the same branch
    float u = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) u = fmaf(row[r][e], kn[e], u);
    u = warp_sum(u);
    const float vi = bf1(a.v[(size_t)bh * a.dv + ri[r]]);
    const float c = beta * (vi - alpha * u);
    float o = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      row[r][e] = fmaf(alpha, row[r][e], c * kn[e]);
      o = fmaf(row[r][e], qn[e], o);
    }
    o = warp_sum(o);
    float* dst = Sh + (size_t)ri[r] * DK + lane * EPL;
    if constexpr (EPL % 4 == 0) {
#pragma unroll
      for (int e = 0; e < EPL; e += 4)
        __stcs(reinterpret_cast<float4*>(dst + e), make_float4(row[r][e], row[r][e + 1], row[r][e + 2], row[r][e + 3]));
    } else {
      __stcs(reinterpret_cast<float2*>(dst), make_float2(row[r][0], row[r][1]));
    }
    if (lane == 0) a.out[(size_t)bh * a.dv + ri[r]] = f2bf(o);
  }
}

}  // namespace

// Rows per warp for a launch: the smallest of 2, 4, 8 whose CTAs (8 warps each) number at
// most four per SM, so that they are all resident at once (8 only while a row takes at most
// four registers per lane).
static int gdn_rows_per_warp(const GdnArgs& a, int n_sm) {
  const int max_rpw = a.dk <= 128 ? 8 : 4;
  for (int rpw = 2; rpw < max_rpw; rpw *= 2) {
    const long long ctas = (long long)a.B * a.Hv * ((a.dv + kGdnWarps * rpw - 1) / (kGdnWarps * rpw));
    if (ctas <= 4LL * n_sm) return rpw;
  }
  return max_rpw;
}

template <int RPW>
static cudaError_t launch_gdn_rpw(const GdnArgs& a, cudaStream_t s, bool early_state) {
  const int rows_cta = kGdnWarps * RPW;
  const int blocks = a.B * a.Hv * ((a.dv + rows_cta - 1) / rows_cta);
  void (*fn)(GdnArgs) = nullptr;
  switch (a.dk) {
    case 64: fn = k_gdn_step<64, RPW>; break;
    case 128: fn = k_gdn_step<128, RPW>; break;
    case 256: fn = k_gdn_step<256, RPW>; break;
    default: return cudaErrorInvalidValue;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(kGdnWarps * 32);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = early_state ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, fn, a);
}

cudaError_t launch_gdn_step(const GdnArgs& a, cudaStream_t s, bool early_state) {
  static int n_sm = 0;
  if (!n_sm) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (n_sm < 1) n_sm = 1;
  }
  switch (gdn_rows_per_warp(a, n_sm)) {
    case 2: return launch_gdn_rpw<2>(a, s, early_state);
    case 4: return launch_gdn_rpw<4>(a, s, early_state);
    default: return launch_gdn_rpw<8>(a, s, early_state);
  }
}

moe_status set_error(moe_status s, const char* fmt, ...);
moe_status cuda_fail(cudaError_t e, const char* what);

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_gdn_decode_step_ex(const moe_gdn_shape* shape, int32_t B, float* state, const void* q,
                                             const void* k, const void* v, const float* g, const float* beta,
                                             void* out, int32_t flags, void* stream) {
  if (flags & ~MOE_GDN_EARLY_STATE) return set_error(MOE_ERR_INVALID, "unknown flags 0x%x", flags);
  if (!shape) return set_error(MOE_ERR_INVALID, "shape is NULL");
  const int Hk = shape->n_k_heads, Hv = shape->n_v_heads, dk = shape->d_k, dv = shape->d_v;
  if (Hk < 1 || Hv < 1 || Hv % Hk) return set_error(MOE_ERR_INVALID, "n_v_heads must be a positive multiple of n_k_heads");
  if (dv < 1) return set_error(MOE_ERR_INVALID, "d_v must be >= 1");
  if (dk != 64 && dk != 128 && dk != 256) return set_error(MOE_ERR_UNSUPPORTED, "d_k must be 64, 128 or 256 (got %d)", dk);
  if (B < 1) return set_error(MOE_ERR_INVALID, "B must be >= 1 (got %d)", B);
  if (!state || !q || !k || !v || !g || !beta || !out)
    return set_error(MOE_ERR_INVALID, "state, q, k, v, g, beta and out must be non-NULL");
  if (((uintptr_t)state & 15) || ((uintptr_t)q & 15) || ((uintptr_t)k & 15) || ((uintptr_t)v & 1) ||
      ((uintptr_t)out & 1) || ((uintptr_t)g & 3) || ((uintptr_t)beta & 3))
    return set_error(MOE_ERR_INVALID, "state, q and k must be 16-byte aligned");
  const long long blocks = (long long)B * Hv * ((dv + 15) / 16);
  if (blocks > 0x7fffffffLL) return set_error(MOE_ERR_INVALID, "B * n_v_heads * d_v too large");
  GdnArgs a{B, Hk, Hv, dk, dv, state, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
            static_cast<const uint16_t*>(v), g, beta, static_cast<uint16_t*>(out)};
  cudaError_t e = launch_gdn_step(a, static_cast<cudaStream_t>(stream), (flags & MOE_GDN_EARLY_STATE) != 0);
  if (e != cudaSuccess) return cuda_fail(e, "gated delta step launch");
  return MOE_OK;
}

extern "C" moe_status moe_gdn_decode_step(const moe_gdn_shape* shape, int32_t B, float* state, const void* q,
                                          const void* k, const void* v, const float* g, const float* beta, void* out,
                                          void* stream) {
  return moe_gdn_decode_step_ex(shape, B, state, q, k, v, g, beta, out, 0, stream);
}
