// Prefill path of the routed-MoE layer (many tokens per call), sm_100a.
//
// The multi-token case the pages single out as the slow part («Swiftlet: 在 Mac 和 iPhone
// 上執行…», section 社群觀點: prefill is the bottleneck for long prompts).  With T·k pairs
// spread over E experts (about 80 tokens per expert at T = 4096, k = 10, E = 512) every
// expert sees a real matrix product, so the expert matmuls run on the tensor cores:
//
//   k_norms        ||x_t|| and ||w_e|| (fp64) for the routing error bound
//   k_gemm ROUTER  fp32 router logits on tcgen05 (bf16 x bf16 -> fp32 in TMEM)
//   k_route        top-k with certification: every expert whose fp32 logit is within the
//                  fp32 error bound of the k-th is recomputed exactly (fp64 sums of exact
//                  bf16 products) and the selection is made on the exact values; softmax
//                  over the selected logits; shared-expert gate
//   k_ghist, k_gscan, k_gplace
//                  stable counting sort of the (token, k) pairs by expert (per-chunk counts,
//                  one scan, per-chunk stable placement) and the list of GEMM work units
//                  (expert, row tile, token tile)
//   k_gemm GATEUP  per unit: [gate; up] rows of one expert (dequantised to bf16 in shared
//                  memory) x the expert's tokens (gathered), SwiGLU in the epilogue -> h
//   k_gemm DOWN    per unit: down rows x the expert's h, weighted scatter-add into an fp32
//                  accumulator (the shared expert is one more "expert" over all tokens)
//   k_finalize     out = bf16(acc + residual)
//
// GEMM kernel ("swap-AB": the weight rows are the MMA's M = 128, the tokens its N <= 128):
//   warp 0       TMEM allocation; lane 0 issues tcgen05.mma (kind::f16, cta_group::1)
//   warps 1..3   gather the tokens' activation rows with cp.async (zero rows beyond N)
//   warps 4..11  dequantise the weight rows (w = s*q + b, rounded to bf16) into shared memory;
//                the raw codes stream through a per-thread cp.async ring several stages ahead
//                and each unit's row scales and biases are copied to shared memory once
//   warps 12..15 epilogue: tcgen05.ld of the fp32 accumulator, then SwiGLU / scatter / store
// Operands are K-major with no swizzle: 8-row x 16-byte core matrices, k-octets 128 bytes
// apart (LBO) and 8-row groups 1024 bytes apart (SBO) for a 64-wide K stage.  A and B
// tiles have rings of their own (the B gather runs six stages ahead, its completion tracked
// by cp.async mbarrier arrivals); two TMEM accumulators of 128 columns let the epilogue of
// one unit overlap the next.
// Every wait is bounded; on timeout the kernel flags MOE_DEVERR_TIMEOUT, drains and frees
// its TMEM.
#include "common.cuh"
#include "kernels.cuh"
#include "sync.cuh"

#include <cuda_bf16.h>

namespace moe {
namespace {

constexpr int kKC = 64;                   // K per stage
constexpr int kNmax = kPrefillN;          // tokens per unit (MMA N)
constexpr int kABytes = 128 * kKC * 2;    // 16 KB
constexpr int kBBytes = kNmax * kKC * 2;  // 16 KB
constexpr int kBWarp0 = 1, kBWarps = 2;
constexpr int kAWarp0 = 3, kAWarps = 8;
constexpr int kEWarp0 = 11, kEWarps = 4;
constexpr int kGemmThreads = (kEWarp0 + kEWarps) * 32;  // 480
constexpr int kSBO = (kKC / 8) * 128;     // 1024
constexpr int kTmemCols = 2 * kNmax;      // two accumulators
constexpr int kRawBytes = 32 * 1024;      // cp.async ring of raw weight bytes (A producers)
constexpr int kAThreads = kAWarps * 32;
// raw bytes per A thread per stage, and ring depth, per mode / width
template <int BITS, int MODE>
struct RawRing {
  static constexpr int kBytes = BITS == 4 ? 16 : 32;
  static constexpr int kDepth = kRawBytes / (kAThreads * kBytes);
};
// A and B tile stages (16 KB each).  The dequantising modes also hold the raw ring and the
// unit's scales and biases (up to 32 KB at K = 4096), so they keep fewer A stages: the raw
// ring already runs kDepth stages ahead of the dequantisation.
template <int MODE>
struct StageCount {
  static constexpr int kA = MODE == kModeRouter ? 6 : 3;
  static constexpr int kB = 6;
};

__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((128u >> 4) & 0x3FFFu) << 16;   // LBO: next k-octet
  d |= (uint64_t)(((uint32_t)kSBO >> 4) & 0x3FFFu) << 32;  // SBO: next 8-row group
  d |= (uint64_t)1 << 46;                         // descriptor version (sm_100)
  return d;                                       // base offset 0, no swizzle
}

__device__ __forceinline__ uint32_t umma_idesc(int n) {
  // kind::f16: D fp32, A bf16, B bf16, both K-major, M = 128
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// arrival on an mbarrier once every cp.async this thread has issued so far has landed
// (.noinc: the arrival is one of the barrier's expected count)
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

// int8 codes -> bf16 on fp32 pairs: the code at bit position p becomes the exact float
// q*2^p by OR-ing it into the mantissa of 2^23 and subtracting 2^23; multiplying by s*2^-p
// (exact) then gives s*q, without integer-to-float instructions.  (bf16 has too few mantissa
// bits for the same trick on 8-bit codes.)
__device__ __forceinline__ float2 ffma2p(float2 a, float2 b, float2 c) {
  float2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(reinterpret_cast<unsigned long long&>(d))
      : "l"(reinterpret_cast<const unsigned long long&>(a)), "l"(reinterpret_cast<const unsigned long long&>(b)),
        "l"(reinterpret_cast<const unsigned long long&>(c)));
  return d;
}
__device__ __forceinline__ uint32_t dq2(uint32_t m0, uint32_t m1, float s0, float s1, float b) {
  const float2 v = codes2(m0, m1);  // exact q0*2^p0, q1*2^p1
  const float2 r = ffma2p(v, make_float2(s0, s1), make_float2(b, b));
  return pack_bf16(r.x, r.y);
}
// 8 int8 codes (two words, byte j at bits 8j) -> 8 bf16 values.
__device__ __forceinline__ uint4 dq8_int8(uint32_t w0, uint32_t w1, float s, float b) {
  const uint32_t h0 = w0 >> 16, h1 = w1 >> 16;
  const float s8 = s * 0x1p-8f;
  return make_uint4(dq2(w0 & 0xFFu, w0 & 0xFF00u, s, s8, b), dq2(h0 & 0xFFu, h0 & 0xFF00u, s, s8, b),
                    dq2(w1 & 0xFFu, w1 & 0xFF00u, s, s8, b), dq2(h1 & 0xFFu, h1 & 0xFF00u, s, s8, b));
}

// A-producer thread -> (tile row m, column half).  Lanes l and l ^ 8 share a row; the
// eight lanes of each quarter-warp take eight consecutive rows of one half, so that their
// 16-byte stores of a k-octet fill 128 contiguous bytes of the tile (no bank conflicts).
__device__ __forceinline__ void a_lane_map(int at, int& m, int& half) {
  const int w = at >> 5, l = at & 31;
  m = w * 16 + (l & 7) + ((l >> 4) << 3);
  half = (l >> 3) & 1;
}

// 8 int4 codes (one word, element j at bits 4j) -> 8 bf16 values round(s*q + b), on packed
// bf16 pairs.  OR-ing a code into the low mantissa bits of bf16 128.0 (0x4300) gives the
// exact value 128 + q; subtracting 128 is exact, and one fused multiply-add rounds s*q + b
// once.  Pairs come out as (q0, q4), (q1, q5), ... and are re-paired with byte permutes.
__device__ __forceinline__ uint32_t bf2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ uint4 dq8_int4_bf(uint32_t w, uint32_t s2, uint32_t b2) {
  constexpr uint32_t kMask = 0x000F000Fu, kBias = 0x43004300u;  // bf16 128.0 in both halves
  constexpr uint32_t kOne = 0x3F803F80u, kNeg128 = 0xC300C300u;  // bf16 1.0, -128.0
  uint32_t r[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t p = ((w >> (4 * i)) & kMask) | kBias;  // (128 + q_i, 128 + q_{i+4})
    r[i] = bf2_fma(bf2_fma(p, kOne, kNeg128), s2, b2);
  }
  return make_uint4(prmt(r[0], r[1], 0x5410u), prmt(r[2], r[3], 0x5410u), prmt(r[0], r[1], 0x7632u),
                    prmt(r[2], r[3], 0x7632u));
}

__device__ __forceinline__ int core_off(int row, int koct) {  // byte offset in a stage tile
  return (row >> 3) * kSBO + koct * 128 + (row & 7) * 16;
}

__device__ __forceinline__ bool wait_or_flag(uint64_t* bar, uint32_t parity, Ctrl* c) {
  if (mbar_wait_suspend(bar, parity)) return true;
  atomicOr(&c->err, kErrTimeout);
  return false;
}

// Every lane of a warp waits, and all take the same branch afterwards (a lane whose wait
// ran out would otherwise leave the others behind at the next __syncwarp).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Ctrl* c, int lane) {
  const bool ok = __all_sync(0xffffffffu, mbar_wait_suspend(bar, parity) ? 1 : 0);
  if (!ok && lane == 0) atomicOr(&c->err, kErrTimeout);
  return ok;
}

// ---------------------------------------------------------------------------------------
// GEMM kernel
// ---------------------------------------------------------------------------------------
template <int BITS, int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1) k_gemm(const __grid_constant__ GemmArgs a) {
  constexpr int kSA = StageCount<MODE>::kA, kSB = StageCount<MODE>::kB;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(8) uint64_t a_full[kSA], a_empty[kSA], b_full[kSB], b_empty[kSB], acc_full[2],
      acc_empty[2], drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_colt[kEWarps][kNmax];  // per epilogue warp (down): token of each column
  __shared__ float s_colw[kEWarps][kNmax];  // and its routing weight

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = (MODE == kModeDown) ? a.I : a.H;
  const int nK = K / kKC;
  const int n_units = *a.n_units;
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t b_area = smem_base + kSA * kABytes;

  if (tid == 0) {
    for (int s = 0; s < kSA; ++s) {
      // router rows are plain copies whose completion each A thread signals; dequantised
      // tiles are signalled once per A warp
      mbar_init(&a_full[s], MODE == kModeRouter ? kAThreads : kAWarps);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < kSB; ++s) {
      mbar_init(&b_full[s], kBWarps * 32);  // one cp.async-tracking arrival per B thread
      mbar_init(&b_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEWarps);
    }
    mbar_init(&drain, 1);
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"((uint32_t)kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      uint32_t q = 0;
      int it = 0;
      for (int u = blockIdx.x; u < n_units && !s_abort; u += gridDim.x, ++it) {
        const GemmUnit U = a.units[u];
        const int npad = (U.n + 15) & ~15;
        const uint32_t idesc = umma_idesc(npad);
        const int buf = it & 1;
        if (!wait_or_flag(&acc_empty[buf], ((it >> 1) & 1) ^ 1, a.ctrl)) {
          s_abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)buf * (uint32_t)kNmax;
        for (int kc = 0; kc < nK; ++kc, ++q) {
          const int sa = q % kSA, sb = q % kSB;
          if (!wait_or_flag(&a_full[sa], (q / kSA) & 1, a.ctrl) || !wait_or_flag(&b_full[sb], (q / kSB) & 1, a.ctrl)) {
            s_abort = 1;
            break;
          }
          // the tiles were written through the generic proxy (st.shared, cp.async)
          proxy_fence();
          tc_fence_after();
          const uint32_t a_base = smem_base + sa * kABytes;
          const uint32_t b_base = b_area + sb * kBBytes;
#pragma unroll
          for (int kk = 0; kk < kKC / 16; ++kk)
            umma_f16(d_tmem, umma_desc(a_base + kk * 256), umma_desc(b_base + kk * 256), idesc,
                     (kc > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&a_empty[sa]);
          umma_commit(&b_empty[sb]);
        }
        if (s_abort) break;
        umma_commit(&acc_full[buf]);
      }
      // every MMA this thread issued has completed once this commit arrives
      umma_commit(&drain);
      if (!mbar_wait(&drain, 0)) atomicOr(&a.ctrl->err, kErrTimeout);
    }
    __syncwarp();
  } else if (warp >= kBWarp0 && warp < kBWarp0 + kBWarps) {
    // ------------------------------ B gather (cp.async) ------------------------------
    // Thread bt copies columns bt and bt + 64 of the unit (one token or pair row each, 128
    // bytes per stage).  Each thread's copies of a stage are tracked by the stage's mbarrier
    // (an arrival that fires when they have landed), so the gather runs up to kSB stages ahead.
    const int bt = tid - kBWarp0 * 32;  // 0..63
    uint32_t q = 0;
    for (int u = blockIdx.x; u < n_units && !s_abort; u += gridDim.x) {
      const GemmUnit U = a.units[u];
      const int npad = (U.n + 15) & ~15;
      const uint16_t* src_base;
      int src_ld;
      if (MODE == kModeDown) {
        src_base = (U.e < 0) ? a.hs : a.h;
        src_ld = a.I;
      } else {
        src_base = a.x;
        src_ld = a.H;
      }
      // source row of each of the thread's two columns; nullptr: zero column (n >= U.n)
      const uint16_t* rows[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int n = bt + c * 64;
        int r = -1;
        if (n < U.n) r = (MODE == kModeGateUp && U.e >= 0) ? __ldg(a.order + U.p0 + n) / a.k : U.p0 + n;
        rows[c] = r < 0 ? nullptr : src_base + (size_t)r * src_ld;
      }
      bool stop = false;
      for (int kc = 0; kc < nK; ++kc, ++q) {
        const int sb = q % kSB;
        if (!warp_wait(&b_empty[sb], ((q / kSB) & 1) ^ 1, a.ctrl, lane)) {
          s_abort = 1;
          stop = true;
          break;
        }
        const uint32_t b_base = b_area + sb * kBBytes;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int n = bt + c * 64;
          if (n < npad) {  // columns beyond npad are not read by the MMA
            const uint16_t* src = rows[c] ? rows[c] + kc * kKC : a.x;
            const uint32_t d = b_base + core_off(n, 0);
#pragma unroll
            for (int j = 0; j < 8; ++j) cp_async16(d + j * 128, src + j * 8, rows[c] ? 16u : 0u);
          }
        }
        cp_async_arrive_noinc(&b_full[sb]);
      }
      if (stop) break;
    }
    cp_async_wait<0>();  // no copy may still be landing when the CTA leaves
  } else if (warp >= kAWarp0 && warp < kAWarp0 + kAWarps && MODE == kModeRouter) {
    // ------------------------------ A rows of the router (bf16, plain copies) ------------------------------
    int m, half;
    a_lane_map(tid - kAWarp0 * 32, m, half);
    uint32_t q = 0;
    for (int u = blockIdx.x; u < n_units && !s_abort; u += gridDim.x) {
      const GemmUnit U = a.units[u];
      const int e = U.mt * 128 + m;
      const uint16_t* row = e < a.E ? a.wr + (size_t)e * a.H : nullptr;
      bool stop = false;
      for (int kc = 0; kc < nK; ++kc, ++q) {
        const int sa = q % kSA;
        if (!warp_wait(&a_empty[sa], ((q / kSA) & 1) ^ 1, a.ctrl, lane)) {
          s_abort = 1;
          stop = true;
          break;
        }
        const uint32_t a_base = smem_base + sa * kABytes;
#pragma unroll
        for (int o = 0; o < 4; ++o) {
          const uint16_t* src = row ? row + kc * kKC + (half * 4 + o) * 8 : a.wsg;
          cp_async16(a_base + core_off(m, half * 4 + o), src, row ? 16u : 0u);
        }
        cp_async_arrive_noinc(&a_full[sa]);
      }
      if (stop) break;
    }
    cp_async_wait<0>();
  } else if (warp >= kAWarp0 && warp < kAWarp0 + kAWarps) {
    // ------------------------------ A producers (dequantise) ------------------------------
    // Raw weight bytes stream into a cp.async ring (kDepth stages ahead); each unit's row
    // scales and biases land once in shared memory (of the two threads of a row, half 0
    // copies the scales, half 1 the biases).  A thread only ever reads ring bytes it copied
    // itself; its partner's half of the scales becomes visible at the __syncwarp that
    // follows both threads' waits.
    using RR = RawRing<BITS, MODE>;
    constexpr int kDepth = RR::kDepth, kRB = RR::kBytes, kPieces = kRB / 16;
    const int at = tid - kAWarp0 * 32;  // 0..255
    int m, half;                        // tile row 0..127, which 32 columns of the stage
    a_lane_map(at, m, half);
    const int NG = K / kGroup;          // groups (= stages) per row
    const int sb_ld = 2 * NG + 8;       // uint16 per row of the scale area (16 bytes of padding)
    // ring: [slot][piece][thread][16 bytes], so a warp's accesses are 512 contiguous bytes
    uint8_t* raw_ring = smem + (size_t)kSA * kABytes + (size_t)kSB * kBBytes;
    uint8_t* my_raw = raw_ring + (size_t)at * 16;
    uint16_t* sb_area = reinterpret_cast<uint16_t*>(raw_ring + kRawBytes);  // [128][sb_ld]
    uint16_t* my_s = sb_area + (size_t)m * sb_ld;
    uint16_t* my_b = my_s + NG;
    uint32_t q = 0;
    for (int u = blockIdx.x; u < n_units && !s_abort; u += gridDim.x) {
      const GemmUnit U = a.units[u];
      // this thread's weight row (bytes of the row, its scales and biases)
      const uint8_t* src = nullptr;
      const uint8_t* sbsrc = nullptr;
      {
        const uint8_t* blob = nullptr;
        if (U.e < 0) {
          blob = a.shared;
        } else {
          const int slot = a.slot_table[U.e];
          if (slot < 0 || slot >= a.n_slots) atomicOr(&a.ctrl->err, kErrBadSlot);
          else blob = a.pool + (int64_t)slot * a.L.stride;
        }
        if (blob) {
          if (MODE == kModeGateUp) {
            const int r = U.mt * 64 + (m >> 1);
            const int up = m & 1;  // rows alternate gate, up of the same intermediate row
            src = blob + a.L.off[up ? 1 : 0] + (int64_t)r * (a.H * BITS / 8);
            sbsrc = blob + a.L.off[(up ? 5 : 3) + half] + (int64_t)r * NG * 2;
          } else {
            const int j = U.mt * 128 + m;
            src = blob + a.L.off[2] + (int64_t)j * (a.I * BITS / 8);
            sbsrc = blob + a.L.off[7 + half] + (int64_t)j * NG * 2;
          }
        }
      }
      const bool zero = (src == nullptr);
      auto issue = [&](int kc) {  // raw bytes of stage kc into ring slot kc % kDepth
        if (!zero && kc < nK) {
          const uint8_t* g = src + (size_t)kc * (kKC * BITS / 8) + half * kRB;
          const uint32_t d = smem_u32(my_raw + (size_t)(kc % kDepth) * kPieces * (kAThreads * 16));
#pragma unroll
          for (int o = 0; o < kPieces; ++o) cp_async16(d + o * (kAThreads * 16), g + o * 16, 16u);
        }
        cp_async_commit();  // one group per stage, empty past the end, so the counts stay uniform
      };
      // scales/biases of the row (one group with stage 0), then the first kDepth stages
      if (!zero) {
        uint16_t* dst = half ? my_b : my_s;
        if ((NG & 7) == 0) {  // rows of 16-byte multiples: 16-byte aligned in the blob and here
          for (int o = 0; o < NG * 2; o += 16) cp_async16(smem_u32(dst) + o, sbsrc + o, 16u);
        } else {  // narrow rows (small K): plain loads, visible after the first __syncwarp
          const uint16_t* g = reinterpret_cast<const uint16_t*>(sbsrc);
          for (int o = 0; o < NG; ++o) dst[o] = __ldg(g + o);
        }
      }
#pragma unroll 1
      for (int d = 0; d < kDepth; ++d) issue(d);
      bool stop = false;
      for (int kc = 0; kc < nK; ++kc, ++q) {
        const int sa = q % kSA;
        cp_async_wait<kDepth - 1>();  // this thread's bytes of stage kc have landed
        __syncwarp();                 // ... and the partner's half of the scales
        if (!warp_wait(&a_empty[sa], ((q / kSA) & 1) ^ 1, a.ctrl, lane)) {
          s_abort = 1;
          stop = true;
          break;
        }
        const uint8_t* rp = my_raw + (size_t)(kc % kDepth) * kPieces * (kAThreads * 16);
        uint4 rw[kPieces];
#pragma unroll
        for (int o = 0; o < kPieces; ++o)
          rw[o] = zero ? make_uint4(0, 0, 0, 0) : *reinterpret_cast<const uint4*>(rp + o * (kAThreads * 16));
        const uint32_t sbits = zero ? 0u : my_s[kc], bbits = zero ? 0u : my_b[kc];
        uint8_t* a_tile = smem + sa * kABytes;
        if (BITS == 4) {
          const uint32_t s2 = sbits | (sbits << 16), b2 = bbits | (bbits << 16);
          const uint32_t w4[4] = {rw[0].x, rw[0].y, rw[0].z, rw[0].w};
#pragma unroll
          for (int o = 0; o < 4; ++o)  // 4 k-octets of 8 values = this thread's 32 columns
            *reinterpret_cast<uint4*>(a_tile + core_off(m, half * 4 + o)) = dq8_int4_bf(w4[o], s2, b2);
        } else {
          const float sv = __uint_as_float(sbits << 16), bv = __uint_as_float(bbits << 16);
#pragma unroll
          for (int o = 0; o < 4; ++o) {
            const uint4 w = rw[o >> 1];
            const uint4 v = (o & 1) ? dq8_int8(w.z, w.w, sv, bv) : dq8_int8(w.x, w.y, sv, bv);
            *reinterpret_cast<uint4*>(a_tile + core_off(m, half * 4 + o)) = v;
          }
        }
        // the ring slot's bytes and this stage's scales are consumed (the stores above depend
        // on them): refill the slot, and let the partner go on to overwrite the scales
        __syncwarp();
        issue(kc + kDepth);
        proxy_fence();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[sa]);
      }
      if (stop) break;
    }
    cp_async_wait<0>();  // no copy may still be landing when the CTA leaves
  } else if (warp >= kEWarp0) {
    // ------------------------------ epilogue ------------------------------
    const int quad = warp & 3;       // TMEM lane quadrant of this warp
    const int m = quad * 32 + lane;  // accumulator row
    int it = 0;
    for (int u = blockIdx.x; u < n_units && !s_abort; u += gridDim.x, ++it) {
      const GemmUnit U = a.units[u];
      const int buf = it & 1;
      if (MODE == kModeDown) {
        // token and weight of every column, loaded while the unit's MMAs run
        for (int n = lane; n < U.n; n += 32) {
          int t;
          float w;
          if (U.e < 0) {
            t = U.p0 + n;
            w = __ldg(a.gate + t);
          } else {
            const int pair = __ldg(a.order + U.p0 + n);
            t = pair / a.k;
            w = __ldg(a.topk_w + pair);
          }
          s_colt[quad][n] = t;
          s_colw[quad][n] = w;
        }
        __syncwarp();
      }
      if (!warp_wait(&acc_full[buf], (it >> 1) & 1, a.ctrl, lane)) {
        s_abort = 1;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)buf * (uint32_t)kNmax;
      for (int c0 = 0; c0 < U.n; c0 += 8) {
        float v[8];
        tmem_ld8(taddr + c0, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int n = c0 + i;
          const float val = v[i];
          if (MODE == kModeGateUp) {
            const float other = __shfl_xor_sync(0xffffffffu, val, 1);
            if (n < U.n && !(m & 1)) {
              const float g = val, up = other;
              const float hv = g / (1.0f + expf(-g)) * up;
              const int r = U.mt * 64 + (m >> 1);
              uint16_t* dst = (U.e < 0) ? a.hs + (size_t)(U.p0 + n) * a.I : a.h + (size_t)(U.p0 + n) * a.I;
              dst[r] = f2bf(hv);
            }
          } else if (MODE == kModeDown) {
            if (n < U.n) {
              const int j = U.mt * 128 + m;
              atomicAdd(a.acc + (size_t)s_colt[quad][n] * a.H + j, s_colw[quad][n] * val);
            }
          } else {  // router logits (no bias)
            const int e = U.mt * 128 + m;
            if (n < U.n && e < a.E) a.logits[(size_t)(U.p0 + n) * (a.E + 1) + e] = val;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }

  // drain: every role has left its loop; make sure no MMA is still writing TMEM
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)kTmemCols));
  }
}

// ---------------------------------------------------------------------------------------
// norms for the routing error bound
// ---------------------------------------------------------------------------------------
__global__ void k_norms(const uint16_t* x, int T, int H, const uint16_t* wr, const uint16_t* wsg, int E,
                        double* xnorm, double* wnorm) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int rows = T + E + 1;
  if (warp >= rows) return;
  const uint16_t* row = warp < T ? x + (size_t)warp * H : (warp < T + E ? wr + (size_t)(warp - T) * H : wsg);
  double s = 0.0;
  for (int i = lane; i < H; i += 32) {
    const double v = (double)bf1(row[i]);
    s += v * v;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    if (warp < T) xnorm[warp] = sqrt(s);
    else wnorm[warp - T] = sqrt(s);
  }
}

// Exact-product fp64 dot of two bf16 rows by one warp (fixed order).
__device__ __forceinline__ double warp_dot_exact(const uint16_t* a, const uint16_t* b, int H) {
  const int lane = threadIdx.x & 31;
  double s = 0.0;
  for (int i = lane * 8; i < H; i += 256) {
    const uint4 va = *reinterpret_cast<const uint4*>(a + i);
    const uint4 vb = *reinterpret_cast<const uint4*>(b + i);
    s += (double)(bf_lo(va.x) * bf_lo(vb.x));
    s += (double)(bf_hi(va.x) * bf_hi(vb.x));
    s += (double)(bf_lo(va.y) * bf_lo(vb.y));
    s += (double)(bf_hi(va.y) * bf_hi(vb.y));
    s += (double)(bf_lo(va.z) * bf_lo(vb.z));
    s += (double)(bf_hi(va.z) * bf_hi(vb.z));
    s += (double)(bf_lo(va.w) * bf_lo(vb.w));
    s += (double)(bf_hi(va.w) * bf_hi(vb.w));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

// ---------------------------------------------------------------------------------------
// certified top-k: one warp per token
// ---------------------------------------------------------------------------------------
constexpr int kRouteCand = 96;

__global__ void __launch_bounds__(256) k_gate(PrefillArgs a) {
  const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + wl;
  if (t >= a.T) return;
  const double gl = warp_dot_exact(a.x + (size_t)t * a.H, a.wsg, a.H);
  if (lane == 0) a.gate[t] = (float)(1.0 / (1.0 + exp(-gl)));
}

__global__ void __launch_bounds__(256) k_route(PrefillArgs a) {
  __shared__ double s_cv[8][kRouteCand];
  __shared__ int s_ce[8][kRouteCand];
  __shared__ int s_cnt[8];
  const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + wl;
  if (t >= a.T) return;
  const int E = a.E, k = a.k, H = a.H;
  const float* lt = a.logits + (size_t)t * (E + 1);
  const uint16_t* xt = a.x + (size_t)t * H;
  // error bound of an fp32 sum of H exact products: |err| <= H * 2^-22 * ||x|| * ||w||
  const double cb = (double)H * 0x1p-22 * a.xnorm[t];
  // lower bound of the k-th best value: the k-th best lane maximum of (l - err)
  double lmax = -INFINITY;
  for (int e = lane; e < E; e += 32) {
    const double b = a.rbias ? (double)a.rbias[e] : 0.0;
    const double lo = (double)lt[e] + b - cb * a.wnorm[e];
    lmax = fmax(lmax, lo);
  }
  // k-th largest of the 32 lane maxima (rank by counting; ties resolved by lane id)
  int rank = 0;
  for (int j = 0; j < 32; ++j) {
    const double o = __shfl_sync(0xffffffffu, lmax, j);
    rank += (o > lmax || (o == lmax && j < lane)) ? 1 : 0;
  }
  const unsigned sel = __ballot_sync(0xffffffffu, rank == k - 1);
  const double thr = __shfl_sync(0xffffffffu, lmax, __ffs(sel) - 1);
  // candidates: upper bound reaches the threshold
  if (lane == 0) s_cnt[wl] = 0;
  __syncwarp();
  bool overflow = false;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    bool c = false;
    if (e < E) {
      const double b = a.rbias ? (double)a.rbias[e] : 0.0;
      c = ((double)lt[e] + b + cb * a.wnorm[e]) >= thr || !((double)lt[e] == (double)lt[e]);
    }
    const unsigned m = __ballot_sync(0xffffffffu, c);
    const int base = s_cnt[wl];
    if (c) {
      const int pos = base + __popc(m & ((1u << lane) - 1));
      if (pos < kRouteCand) s_ce[wl][pos] = e;
    }
    __syncwarp();
    if (lane == 0) s_cnt[wl] = base + __popc(m);
    __syncwarp();
  }
  int n = s_cnt[wl];
  if (n > kRouteCand) {
    overflow = true;  // recompute everything exactly (rare: many near-equal logits)
    n = E;
  }
  // exact values of the candidates (fp64 sums of exact products, fixed order)
  if (!overflow) {
    for (int i = 0; i < n; ++i) {
      const int e = s_ce[wl][i];
      const double v = warp_dot_exact(xt, a.wr + (size_t)e * H, H) + (a.rbias ? (double)a.rbias[e] : 0.0);
      if (lane == 0) s_cv[wl][i] = v;
    }
  }
  __syncwarp();
  // select the k best exact keys (value desc, id asc) by k rounds over the candidates
  double sv = -INFINITY;
  int se = 0x7fffffff;
  if (!overflow) {
    uint32_t taken[(kRouteCand + 31) / 32] = {0, 0, 0};
    for (int r = 0; r < k; ++r) {
      double bv = -INFINITY;
      int be = 0x7fffffff, bi = -1;
      for (int i = lane; i < n; i += 32) {
        if ((taken[i >> 5] >> (i & 31)) & 1u) continue;
        const double v = s_cv[wl][i];
        const int e = s_ce[wl][i];
        if (v > bv || (v == bv && e < be) || bi < 0) {
          if (v == v) {
            bv = v;
            be = e;
            bi = i;
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (oi >= 0 && (bi < 0 || ov > bv || (ov == bv && oe < be))) {
          bv = ov;
          be = oe;
          bi = oi;
        }
      }
      if (bi >= 0) taken[bi >> 5] |= 1u << (bi & 31);
      if (lane == r) {
        sv = bv;
        se = bi >= 0 ? be : 0x7fffffff;
      }
    }
  } else {
    // exact value of every expert, k rounds of warp arg-max
    uint32_t taken[kMaxExperts / 32] = {};
    for (int r = 0; r < k; ++r) {
      double bv = -INFINITY;
      int be = 0x7fffffff;
      for (int e = 0; e < E; ++e) {
        if ((taken[e >> 5] >> (e & 31)) & 1u) continue;
        const double v = warp_dot_exact(xt, a.wr + (size_t)e * H, H) + (a.rbias ? (double)a.rbias[e] : 0.0);
        if (v == v && (be == 0x7fffffff || v > bv || (v == bv && e < be))) {
          bv = v;
          be = e;
        }
      }
      if (be != 0x7fffffff) taken[be >> 5] |= 1u << (be & 31);
      if (lane == r) {
        sv = bv;
        se = be;
      }
    }
  }
  const double v0 = __shfl_sync(0xffffffffu, sv, 0);
  const bool valid = lane < k && se != 0x7fffffff;
  const double ex = valid ? exp(sv - v0) : 0.0;
  double den = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (lane < k) {
    if (!valid) atomicOr(&a.ctrl->err, kErrNonFinite);
    a.topk_idx[t * k + lane] = valid ? se : -1;
    a.topk_w[t * k + lane] = valid ? (float)(ex / den) : 0.f;
  }
  const double gl = warp_dot_exact(xt, a.wsg, H);
  if (lane == 0) a.gate[t] = (float)(1.0 / (1.0 + exp(-gl)));
}

// ---------------------------------------------------------------------------------------
// stable counting sort of the pairs by expert, and the GEMM work units.
//   k_ghist   per chunk of kGroupChunk pairs: its per-expert counts
//   k_gscan   per expert: exclusive sums over the chunks (in place), the expert's total;
//             offsets = exclusive scan of the totals; GEMM work units
//   k_gplace  per chunk: stable ranks (warp match + per-warp counts), order[slot] = pair
// Pair p of chunk c lands at offsets[e] + (pairs of e in chunks < c) + (pairs of e before it
// in chunk c): the pairs of one expert keep their pair-index order.
// ---------------------------------------------------------------------------------------
constexpr int kGroupThreads = 256;  // 8 warps; each takes kGroupChunk / 8 consecutive pairs
constexpr int kScanThreads = 1024;
static_assert(kGroupChunk % (kGroupThreads / 32 * 32) == 0, "chunk must split into whole warp rounds");

__global__ void __launch_bounds__(kGroupThreads) k_ghist(PrefillArgs a) {
  extern __shared__ int hsm[];  // [E]
  const int E = a.E, n = a.T * a.k;
  for (int e = threadIdx.x; e < E; e += kGroupThreads) hsm[e] = 0;
  __syncthreads();
  const int p0 = blockIdx.x * kGroupChunk;
#pragma unroll
  for (int j = 0; j < kGroupChunk / kGroupThreads; ++j) {
    const int p = p0 + j * kGroupThreads + threadIdx.x;
    if (p < n) {
      const int e = __ldg(a.topk_idx + p);
      if (e < 0 || e >= E) atomicOr(&a.ctrl->err, kErrBadExpert);
      else atomicAdd(&hsm[e], 1);
    }
  }
  __syncthreads();
  int* out = a.chunk_cnt + (size_t)blockIdx.x * E;
  for (int e = threadIdx.x; e < E; e += kGroupThreads) out[e] = hsm[e];
}

__global__ void __launch_bounds__(kScanThreads) k_gscan(PrefillArgs a) {
  __shared__ int cnt[kMaxExperts];
  __shared__ int off[kMaxExperts + 1];
  __shared__ int wsum[kScanThreads / 32];
  const int E = a.E, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n_chunks = (a.T * a.k + kGroupChunk - 1) / kGroupChunk;
  // per expert: running sum down the chunks (8 loads in flight per step)
  for (int e = threadIdx.x; e < E; e += kScanThreads) {
    int s = 0;
    for (int c0 = 0; c0 < n_chunks; c0 += 8) {
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = (c0 + j < n_chunks) ? a.chunk_cnt[(size_t)(c0 + j) * E + e] : 0;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (c0 + j < n_chunks) {
          a.chunk_cnt[(size_t)(c0 + j) * E + e] = s;
          s += v[j];
        }
    }
    cnt[e] = s;
  }
  __syncthreads();
  // exclusive scan of the totals (E <= 1024: one value per thread)
  {
    const int e = threadIdx.x;
    const int v = e < E ? cnt[e] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int wv = wsum[lane];
      int wi = wv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += y;
      }
      wsum[lane] = wi - wv;
    }
    __syncthreads();
    if (e < E) off[e] = wsum[warp] + incl - v;
    if (e == E - 1) off[E] = wsum[warp] + incl;
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= E; e += kScanThreads) {
    a.offsets[e] = off[e];
    if (e < E) a.counts[e] = cnt[e];
  }
  if (!a.units_gu) return;  // grouping only
  // work units: per expert, token tiles of <= kNmax pairs x row tiles; then the shared
  // expert.  Tile bases by an exclusive scan of the experts' tile counts.
  __syncthreads();
  int* tile_base = off;  // reuse after the offsets are out: [E + 1]
  __shared__ int offc[kMaxExperts];
  for (int e = threadIdx.x; e < E; e += kScanThreads) offc[e] = off[e];
  __syncthreads();
  {
    const int e = threadIdx.x;
    const int v = e < E ? (cnt[e] + kNmax - 1) / kNmax : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int wv = wsum[lane];
      int wi = wv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += y;
      }
      wsum[lane] = wi - wv;
    }
    __syncthreads();
    if (e < E) tile_base[e] = wsum[warp] + incl - v;
    if (e == E - 1) tile_base[E] = wsum[warp] + incl;
  }
  __syncthreads();
  const int mt_gu = a.I / 64, mt_dn = a.H / 128;
  for (int e = threadIdx.x; e < E; e += kScanThreads) {
    int tb = tile_base[e];
    for (int s0 = 0; s0 < cnt[e]; s0 += kNmax, ++tb) {
      const int nn = min(kNmax, cnt[e] - s0);
      for (int mt = 0; mt < mt_gu; ++mt) a.units_gu[tb * mt_gu + mt] = GemmUnit{e, mt, offc[e] + s0, nn};
      for (int mt = 0; mt < mt_dn; ++mt) a.units_dn[tb * mt_dn + mt] = GemmUnit{e, mt, offc[e] + s0, nn};
    }
  }
  const int tiles_r = tile_base[E];
  const int st_n = (a.T + kNmax - 1) / kNmax;
  for (int i = threadIdx.x; i < st_n * mt_gu; i += kScanThreads) {
    const int st = i / mt_gu, mt = i - st * mt_gu, t0 = st * kNmax;
    a.units_gu[(tiles_r + st) * mt_gu + mt] = GemmUnit{-1, mt, t0, min(kNmax, a.T - t0)};
  }
  for (int i = threadIdx.x; i < st_n * mt_dn; i += kScanThreads) {
    const int st = i / mt_dn, mt = i - st * mt_dn, t0 = st * kNmax;
    a.units_dn[(tiles_r + st) * mt_dn + mt] = GemmUnit{-1, mt, t0, min(kNmax, a.T - t0)};
  }
  if (threadIdx.x == 0) {
    a.n_units[0] = (tiles_r + st_n) * mt_gu;
    a.n_units[1] = (tiles_r + st_n) * mt_dn;
  }
}

__global__ void __launch_bounds__(kGroupThreads) k_gplace(PrefillArgs a) {
  extern __shared__ int wc[];  // [8][E]: per-warp counts, then per-warp running slots
  constexpr int kW = kGroupThreads / 32, kRounds = kGroupChunk / kGroupThreads;
  const int E = a.E, n = a.T * a.k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kW * E; i += kGroupThreads) wc[i] = 0;
  __syncthreads();
  // warp w takes pairs [p0 + w * 32 * kRounds, ... + 32 * kRounds), round by round
  const int pw = blockIdx.x * kGroupChunk + warp * 32 * kRounds;
  int ev[kRounds];
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const int p = pw + r * 32 + lane;
    const int e = p < n ? __ldg(a.topk_idx + p) : -1;
    ev[r] = (e >= 0 && e < E) ? e : -1;
  }
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const unsigned peers = __match_any_sync(0xffffffffu, ev[r]);
    if (ev[r] >= 0 && lane == __ffs(peers) - 1) wc[warp * E + ev[r]] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  const int* base = a.chunk_cnt + (size_t)blockIdx.x * E;
  for (int e = threadIdx.x; e < E; e += kGroupThreads) {
    int pos = a.offsets[e] + base[e];
#pragma unroll
    for (int w = 0; w < kW; ++w) {
      const int c = wc[w * E + e];
      wc[w * E + e] = pos;
      pos += c;
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const int e = ev[r];
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0) a.order[wc[warp * E + e] + __popc(peers & ((1u << lane) - 1))] = pw + r * 32 + lane;
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) wc[warp * E + e] += __popc(peers);
    __syncwarp();
  }
}

__global__ void k_finalize(const float* acc, const uint16_t* residual, uint16_t* out, size_t n) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = f2bf(acc[i] + (residual ? bf1(residual[i]) : 0.f));
}

__global__ void k_router_units(GemmUnit* units, int* n_units, int T, int E) {
  // E rows in tiles of 128 x tokens in tiles of 128 (the shared-expert gate logit is
  // computed exactly by k_route)
  const int mt_n = (E + 127) / 128;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int nt = (T + 127) / 128;
  if (i < mt_n * nt) {
    const int mt = i % mt_n, tt = i / mt_n;
    units[i] = GemmUnit{-2, mt, tt * 128, min(128, T - tt * 128)};
  }
  if (i == 0) *n_units = mt_n * nt;
}

template <int BITS, int MODE>
cudaError_t launch_gemm(const GemmArgs& g, int n_sm, cudaStream_t s) {
  const int K = (MODE == kModeDown) ? g.I : g.H;
  size_t smem = (size_t)StageCount<MODE>::kA * kABytes + (size_t)StageCount<MODE>::kB * kBBytes;
  if (MODE != kModeRouter) smem += kRawBytes + (size_t)128 * ((K / kGroup) * 4 + 16);
  auto fn = k_gemm<BITS, MODE>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  fn<<<n_sm, kGemmThreads, smem, s>>>(g);
  return cudaGetLastError();
}

}  // namespace

bool prefill_shape_supported(int H, int I, int bits, int E) {
  return (bits == 4 || bits == 8) && H % 128 == 0 && I % 64 == 0 && E <= 512 && H <= 4096 && I <= 4096;
}

cudaError_t launch_group(const PrefillArgs& p, cudaStream_t s) {
  const int n_chunks = (p.T * p.k + kGroupChunk - 1) / kGroupChunk;
  k_ghist<<<n_chunks, kGroupThreads, sizeof(int) * p.E, s>>>(p);
  k_gscan<<<1, kScanThreads, 0, s>>>(p);
  const size_t smem = sizeof(int) * (size_t)(kGroupThreads / 32) * p.E;
  k_gplace<<<n_chunks, kGroupThreads, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_prefill(const PrefillArgs& p, int bits, cudaStream_t s) {
  int dev = 0, n_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  const int T = p.T, E = p.E, H = p.H;
  cudaError_t e;
  // accumulator of the down products
  if ((e = cudaMemsetAsync(p.acc, 0, sizeof(float) * (size_t)T * H, s)) != cudaSuccess) return e;
  // norms, router logits, certified top-k
  prof_mark(0, false, s);
  {
    const int rows = T + E + 1;
    if (p.route) {
      k_norms<<<(rows * 32 + 255) / 256, 256, 0, s>>>(p.x, T, H, p.wr, p.wsg, E, p.xnorm, p.wnorm);
      const int mt_n = (E + 127) / 128, nt = (T + 127) / 128;
      k_router_units<<<(mt_n * nt + 255) / 256, 256, 0, s>>>(p.units_rt, p.n_units + 2, T, E);
      GemmArgs g = p.g;
      g.units = p.units_rt;
      g.n_units = p.n_units + 2;
      if ((e = (bits == 4 ? launch_gemm<4, kModeRouter>(g, n_sm, s) : launch_gemm<8, kModeRouter>(g, n_sm, s))) !=
          cudaSuccess)
        return e;
      k_route<<<(T + 7) / 8, 256, 0, s>>>(p);
    } else {
      k_gate<<<(T + 7) / 8, 256, 0, s>>>(p);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  prof_mark(0, true, s);
  // grouping and work units
  prof_mark(1, false, s);
  if ((e = launch_group(p, s)) != cudaSuccess) return e;
  prof_mark(1, true, s);
  // gate/up + SwiGLU, then down + scatter
  {
    GemmArgs g = p.g;
    g.units = p.units_gu;
    g.n_units = p.n_units;
    prof_mark(2, false, s);
    if ((e = (bits == 4 ? launch_gemm<4, kModeGateUp>(g, n_sm, s) : launch_gemm<8, kModeGateUp>(g, n_sm, s))) !=
        cudaSuccess)
      return e;
    prof_mark(2, true, s);
    g.units = p.units_dn;
    g.n_units = p.n_units + 1;
    prof_mark(3, false, s);
    if ((e = (bits == 4 ? launch_gemm<4, kModeDown>(g, n_sm, s) : launch_gemm<8, kModeDown>(g, n_sm, s))) !=
        cudaSuccess)
      return e;
    prof_mark(3, true, s);
  }
  const size_t n = (size_t)T * H;
  prof_mark(4, false, s);
  k_finalize<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p.acc, p.residual, p.out, n);
  prof_mark(4, true, s);
  return cudaGetLastError();
}

}  // namespace moe
