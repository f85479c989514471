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
//   k_ghist, k_gcol, k_gplace
//                  stable counting sort of the (token, k) pairs by expert (per-chunk counts,
//                  per-expert scans down the chunks, per-chunk stable placement) and the
//                  list of GEMM work units (expert, row tile, token tile)
//   k_permute      xg = the tokens' rows of x in grouped pair order (int4: in k-octet order,
//                  and xp = x in that order for the shared expert; see dq8_int4_bf)
//   k_gemm GATEUP  per unit: [gate; up] rows of one expert (dequantised to bf16 in shared
//                  memory) x the expert's rows of xg, SwiGLU in the epilogue -> h
//   k_gemm DOWN    per unit: down rows x the expert's h, weighted scatter-add into an fp32
//                  accumulator (the shared expert is one more "expert" over all tokens)
//   k_finalize     out = bf16(acc + residual) (8 elements per thread for aligned buffers)
//
// GEMM kernel (the unit's tokens are the MMA's M = 128 TMEM lanes, its weight rows the N <= 256
// columns; one kind::f16 MMA per 16-deep k-step):
//   warp 0        TMEM allocation; lane 0 issues tcgen05.mma (kind::f16, cta_group::1)
//   warp 1        token tiles by TMA (consecutive rows of x, of the expert-ordered copy xg,
//                 of h, hs)
//   warp 2        lane 0: raw codes by TMA (3-D / 4-D boxes over the pool) into a raw ring,
//                 with the scales and biases of every 8 stages; or router rows
//   warps 3..18   dequantise the codes (w = s*q + b, rounded to bf16) into the weight tile
//   warps 19..22  epilogue: tcgen05.ld of the fp32 accumulator, then SwiGLU / scatter / store
// Weight tiles written by the dequantising warps are K-major without swizzle (8-row x 16-byte
// core matrices, k-octets 128 bytes apart, 8-row groups 1024 bytes apart); tiles written by
// TMA (tokens, router rows) use the 128-byte swizzle.  Stage s holds one token and one weight
// tile, with one full barrier (TMA bytes plus the producers' arrivals) and one empty barrier
// (the MMA's commit); two TMEM accumulators of 256 columns let the epilogue of one unit
// overlap the next.  Every wait is bounded; on timeout the kernel flags MOE_DEVERR_TIMEOUT,
// drains and frees its TMEM.
#include "common.cuh"
#include "kernels.cuh"
#include "sync.cuh"

#include <cuda_bf16.h>

#include <algorithm>

namespace moe {
namespace {

constexpr int kKC = 64;                   // K per stage
constexpr int kTok = kPrefillN;           // tokens per unit: the MMA's M (128 TMEM lanes)
constexpr int kNMax = 256;                // weight rows per unit: the MMA's N
constexpr int kTBytes = kTok * kKC * 2;   // 16 KB: token tile of a stage
constexpr int kWBytes = kNMax * kKC * 2;  // 32 KB: weight tile of a stage (room for N = 256)
// warp roles
constexpr int kTLoadWarp = 1;             // token tiles by TMA
constexpr int kWLoadWarp = 2;             // lane 0: raw codes + scale chunks (or router rows) by TMA
constexpr int kDWarp0 = 3, kDWarps = 16;  // dequantisation: two groups of 8 warps, 256 weight rows each
constexpr int kDGroup = kDWarps / 2;      // warps per dequantising group (one stage each)
constexpr int kEWarp0 = 19, kEWarps = 4;  // epilogue
constexpr int kGemmThreads = (kEWarp0 + kEWarps) * 32;  // 736
constexpr int kSBO = (kKC / 8) * 128;     // 1024: 8-row group stride of a no-swizzle K-major tile
constexpr int kTmemCols = 2 * kNMax;      // two accumulators of up to 256 columns
constexpr int kTRows = 32;                // rows per token-tile load
constexpr int kStageMax = 6;
constexpr int kChunk = 8;                 // groups per scale chunk
constexpr int kChunkBytes = kNMax * 2 * kChunk * 2;  // 8 KB: scales + biases of 8 groups, 256 rows
constexpr int kSmemMax = 227 * 1024 - 8 * 1024;  // dynamic shared memory budget (static part aside)
// raw codes of one stage (256 weight rows x 64 codes), and how many stages are in flight
template <int BITS>
struct Raw {
  static constexpr int kRowBytes = kKC * BITS / 8;  // 32 or 64
  static constexpr int kBytes = kNMax * kRowBytes;  // 8 or 16 KB
};
constexpr int kRawMax = 8;  // raw stages in flight: what shared memory leaves, at most 8

// Position in a ring of n stages and the parity of its current pass.
struct Ring {
  int n, s = 0;
  uint32_t ph = 0;
  __device__ explicit Ring(int n_) : n(n_) {}
  __device__ void next() {
    if (++s == n) {
      s = 0;
      ph ^= 1;
    }
  }
};

// Shared-memory plan of one GEMM launch (host and device agree on it).  Stage s holds a
// token tile (16 KB) and a weight tile (up to 32 KB), with one full and one empty barrier.
struct GemmSmem {
  int n_st;            // stages
  int n_raw;           // raw-code stages in flight (dequantising modes)
  uint32_t w;          // byte offset of the weight tiles
  uint32_t raw, sc;    // byte offsets of the raw ring and the two scale-chunk slots
  uint32_t total;      // dynamic bytes, including 1 KB of alignment slack
};
template <int BITS, int MODE>
__host__ __device__ inline GemmSmem gemm_smem() {
  GemmSmem p{};
  const uint32_t wb = MODE == kModeRouter ? (uint32_t)(kTok * kKC * 2) : (uint32_t)kWBytes;
  const uint32_t budget = (uint32_t)kSmemMax - 1024u;
  if (MODE == kModeRouter) {
    const int n = (int)(budget / ((uint32_t)kTBytes + wb));
    p.n_st = n > kStageMax ? kStageMax : n;
    p.n_raw = 0;
  } else {
    // three stages of tiles, then as many raw stages as fit (the dequantisation runs behind
    // TMA latency otherwise), at least three
    const uint32_t rest = budget - 2u * kChunkBytes;
    p.n_st = 3;
    const int nr = (int)((rest - 3u * ((uint32_t)kTBytes + wb)) / (uint32_t)Raw<BITS>::kBytes);
    p.n_raw = nr > kRawMax ? kRawMax : nr;
    // A group waiting for raw stage s has converted s - 2 (the MMA has consumed s - 5), so the
    // slot's previous fill s - n_raw is known to have landed, and the parity wait cannot
    // mistake it for the fill it waits for, when n_raw >= 5 or n_raw is even (then s - n_raw
    // is one of the group's own earlier stages).  int8 leaves room for 3: use 2.
    if (p.n_raw < 5 && (p.n_raw & 1)) --p.n_raw;
  }
  p.w = (uint32_t)p.n_st * kTBytes;
  p.raw = p.w + (uint32_t)p.n_st * wb;
  p.sc = p.raw + (uint32_t)p.n_raw * Raw<BITS>::kBytes;
  p.total = p.sc + (MODE == kModeRouter ? 0u : 2u * kChunkBytes) + 1024u;
  return p;
}

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

// K-major operand with 128-byte swizzle (rows of 64 bf16 = 128 bytes, 16-byte chunks XOR-ed
// with the row's position in its 8-row group; the layout TMA writes with SWIZZLE_128B).  The
// k-step of one MMA (16 elements = 32 bytes) advances the start address; 8-row groups are
// 1024 bytes apart.  Tiles start on 1024-byte boundaries.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;                         // LBO (unused for swizzled K-major)
  d |= (uint64_t)((1024u >> 4) & 0x3FFFu) << 32;  // SBO: next 8-row group
  d |= (uint64_t)1 << 46;                         // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                         // layout: 128-byte swizzle
  return d;
}

// TMA loads into this CTA's shared memory, completing on an mbarrier (transaction bytes).
__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_4d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                       uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
      "[%6];" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
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

// 16 / 32 consecutive accumulator columns of this warp's 32 TMEM lanes (one row per thread)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
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

// 8 int4 codes (one word, element j at bits 4j) -> 8 bf16 values round(s*q + b), on packed
// bf16 pairs.  OR-ing a code into the low mantissa bits of bf16 128.0 (0x4300) gives the
// exact value 128 + q; subtracting 128 is exact, and one fused multiply-add rounds s*q + b
// once.  The pairs come out as (q0, q4), (q1, q5), (q2, q6), (q3, q7) and are stored in that
// order: the int4 expert GEMMs take both operands with every k-octet in the order
// 0, 4, 1, 5, 2, 6, 3, 7 (the token rows are written so by k_permute and by the gate/up
// epilogue, see perm_octet), which leaves each dot product unchanged and saves re-pairing
// the values with byte permutes here.
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
  return make_uint4(r[0], r[1], r[2], r[3]);
}
// Eight consecutive bf16 values (x0 .. x7) -> the k-octet order of the int4 GEMM operands:
// (x0, x4), (x1, x5), (x2, x6), (x3, x7).
__device__ __forceinline__ uint4 perm_octet(const uint4& v) {
  return make_uint4(prmt(v.x, v.z, 0x5410u), prmt(v.x, v.z, 0x7632u), prmt(v.y, v.w, 0x5410u),
                    prmt(v.y, v.w, 0x7632u));
}

__device__ __forceinline__ int core_off(int row, int koct) {  // byte offset in a stage tile
  return (row >> 3) * kSBO + koct * 128 + (row & 7) * 16;
}

__device__ __forceinline__ bool wait_or_flag(uint64_t* bar, uint32_t parity, Ctrl* c) {
  if (mbar_wait_suspend(bar, parity)) return true;
  atomicOr(&c->err, kErrTimeout);
  return false;
}

// The abort flag as the whole warp sees it (one value for all lanes, so that no lane
// leaves a loop whose other lanes go on to a __syncwarp).
__device__ __forceinline__ bool warp_aborted(const int* flag) {
  return __any_sync(0xffffffffu, *reinterpret_cast<const volatile int*>(flag) != 0);
}

// Bounded wait that sleeps between tries (32 ns doubling to 256 ns), so that a warp waiting
// for its next stage leaves the issue slots to the warps that are converting one.
__device__ __forceinline__ bool mbar_wait_backoff(uint64_t* b, uint32_t parity) {
  if (mbar_try_wait(b, parity)) return true;
  const unsigned long long t0 = now_ns();
  uint32_t ns = 32;
  for (;;) {
    __nanosleep(ns);
    if (mbar_try_wait(b, parity)) return true;
    if (now_ns() - t0 > kWaitNs) return false;
    ns = ns < 256 ? 2 * ns : 256;
  }
}
// Every lane of a warp waits, and all take the same branch afterwards (a lane whose wait
// ran out would otherwise leave the others behind at the next __syncwarp).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Ctrl* c, int lane) {
  const bool ok = __all_sync(0xffffffffu, mbar_wait_backoff(bar, parity) ? 1 : 0);
  if (!ok && lane == 0) atomicOr(&c->err, kErrTimeout);
  return ok;
}

// Wait (bounded) for the last stages a loader issued into a ring of n full barriers, so that
// no copy is still landing when the CTA leaves.  Normally the consumers have already waited
// for them and this returns at once; after an abort a phase may lack other arrivals, and
// the bound (far beyond any copy's latency) ends the wait.
__device__ __forceinline__ void drain_ring(uint64_t* full, int n, int issued, Ctrl* c) {
  for (int q = issued > n ? issued - n : 0; q < issued; ++q)
    if (!mbar_wait(&full[q % n], (uint32_t)((q / n) & 1))) {
      atomicOr(&c->err, kErrTimeout);
      return;
    }
}

// ---------------------------------------------------------------------------------------
// GEMM kernel
// ---------------------------------------------------------------------------------------
template <int BITS, int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1) k_gemm(const __grid_constant__ GemmArgs a) {
  constexpr int kRawB = Raw<BITS>::kBytes, kRowB = Raw<BITS>::kRowBytes;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kStageMax], empty[kStageMax], raw_full[kRawMax], raw_empty[kRawMax],
      chunk_full[2], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = (MODE == kModeDown) ? a.I : a.H;
  const int nK = K / kKC;
  const int NR = a.n_rows;  // weight rows per unit (the MMA's N): 128 or 256
  pdl_launch_dependents();
  const GemmSmem P = gemm_smem<BITS, MODE>();
  const uint32_t wbytes = MODE == kModeRouter ? (uint32_t)(kTok * kKC * 2) : (uint32_t)kWBytes;  // per stage
  // stage tiles start on 1024-byte boundaries (128-byte swizzle atoms)
  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (smem_base - smem_u32(smem_raw));
  const uint32_t w_area = smem_base + P.w;

  if (tid == 0) {
    for (int s = 0; s < P.n_st; ++s) {
      // full: the token loader's expect-tx arrival, plus the weight loader's (router rows by
      // TMA) or one arrival per warp of the dequantising group that owns the stage; empty: the
      // MMA's commit
      mbar_init(&full[s], MODE == kModeRouter ? 2 : kDGroup + 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < P.n_raw; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], kDGroup);
    }
    for (int c = 0; c < 2; ++c) mbar_init(&chunk_full[c], 1);
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
  // the setup above overlaps the kernel before; the work units and every input are its output
  pdl_wait();
  const int n_units = *a.n_units;
  const int my_units = n_units > (int)blockIdx.x ? (n_units - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp == 0) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      // D[token][row] += X[token][k] * W[row][k]: A = token tile (TMA, 128-byte swizzle),
      // B = weight tile (dequantised, no swizzle; router rows by TMA, 128-byte swizzle).
      // A stage or k-step moves only the descriptors' start addresses (bits 0..13 =
      // address >> 4; shared addresses stay below 256 KB, so nothing carries out).
      const uint64_t da0 = umma_desc_sw128(smem_base);
      const uint64_t db0 = MODE == kModeRouter ? umma_desc_sw128(w_area) : umma_desc(w_area);
      constexpr uint64_t kAStep = 32 >> 4;                                      // per k-step of 16
      constexpr uint64_t kBStep = MODE == kModeRouter ? (32 >> 4) : (256 >> 4);
      const uint32_t idesc = umma_idesc(NR);
      Ring r(P.n_st);
      int it = 0;
      for (int u = blockIdx.x; u < n_units && !s_abort; u += gridDim.x, ++it) {
        const int buf = it & 1;
        if (!wait_or_flag(&acc_empty[buf], ((it >> 1) & 1) ^ 1, a.ctrl)) {
          s_abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)buf * (uint32_t)kNMax;
        for (int kc = 0; kc < nK; ++kc, r.next()) {
          if (!wait_or_flag(&full[r.s], r.ph, a.ctrl)) {
            s_abort = 1;
            break;
          }
          // the dequantised tiles were written through the generic proxy (st.shared); each
          // writing thread fenced them to the async proxy before its arrival
          tc_fence_after();
          const uint64_t da = da0 + (uint64_t)(r.s * (kTBytes >> 4));
          const uint64_t db = db0 + (uint64_t)(r.s * (wbytes >> 4));
          umma_f16(d_tmem, da, db, idesc, kc > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < kKC / 16; ++kk) umma_f16(d_tmem, da + kk * kAStep, db + kk * kBStep, idesc, 1u);
          umma_commit(&empty[r.s]);
        }
        if (s_abort) break;
        umma_commit(&acc_full[buf]);
      }
      // every MMA this thread issued has completed once this commit arrives
      umma_commit(&drain);
      if (!mbar_wait(&drain, 0)) atomicOr(&a.ctrl->err, kErrTimeout);
    }
    __syncwarp();
  } else if (warp == kTLoadWarp) {
    // ------------------------------ token tiles (TMA) ------------------------------
    // A unit's tokens are consecutive rows of a bf16 matrix: x for the router and the shared
    // expert's gate/up, the expert-ordered copy xg for routed gate/up, h / hs for down.
    // Loads of kTRows rows, one per lane; rows beyond U.n belong to other units or lie
    // beyond the matrix (zero filled): their accumulator lanes are never read.
    Ring r(P.n_st);
    int issued = 0;
    for (int u = blockIdx.x; u < n_units && !warp_aborted(&s_abort); u += gridDim.x) {
      const GemmUnit U = a.units[u];
      const CUtensorMap* mt = (MODE != kModeRouter && U.e < 0) ? &a.map_tok2 : &a.map_tok;
      const int nrt = (U.n + kTRows - 1) / kTRows;
      const uint32_t bytes = (uint32_t)nrt * kTRows * 128u;
      bool stop = false;
      for (int kc = 0; kc < nK; ++kc, r.next()) {
        if (!warp_wait(&empty[r.s], r.ph ^ 1, a.ctrl, lane)) {
          stop = true;
          break;
        }
        if (lane == 0) mbar_expect_tx(&full[r.s], bytes);
        __syncwarp();  // the transaction count is registered before any load can land
        if (lane < nrt)
          tma_2d(smem_base + r.s * kTBytes + lane * kTRows * 128, mt, kc * kKC, U.p0 + lane * kTRows, &full[r.s]);
        ++issued;
      }
      if (stop) {
        s_abort = 1;
        break;
      }
    }
    if (lane == 0) drain_ring(full, P.n_st, issued, a.ctrl);
  } else if (warp == kWLoadWarp) {
    // ------------------------------ weight operand loads (TMA) ------------------------------
    // Router: NR router rows x 64 columns per stage straight into the weight tile.
    // Otherwise the stage's raw codes (NR rows x 64 codes) into the raw ring, and every 8
    // stages the scales and biases of those 8 groups (a scale chunk), for the dequantising
    // warps.  A unit whose expert has no valid slot reads an out-of-range slot, which TMA
    // fills with zeros (zero scales: it dequantises to 0).
    if (lane == 0) {
      Ring rr(MODE == kModeRouter ? P.n_st : P.n_raw);
      int issued = 0, chunks = 0;
      bool stop = false;
      // unit descriptors two units ahead and slots one unit ahead, so that the lookups'
      // latency is hidden behind the previous unit's loads
      auto unit_at = [&](int j) { return a.units[blockIdx.x + (size_t)j * gridDim.x]; };
      auto slot_of = [&](const GemmUnit& U) { return (MODE == kModeRouter || U.e < 0) ? 0 : a.slot_table[U.e]; };
      GemmUnit un1{}, un2{};
      int slot1 = 0;
      if (my_units > 0) {
        un1 = unit_at(0);
        slot1 = slot_of(un1);
      }
      if (my_units > 1) un2 = unit_at(1);
      const uint32_t raw_bytes = (uint32_t)NR * kRowB, chunk_bytes = (uint32_t)NR * 2 * kChunk * 2;
      for (int j = 0; j < my_units && !stop && !s_abort; ++j) {
        const GemmUnit U = un1;
        int slot = slot1;
        un1 = un2;
        if (j + 1 < my_units) slot1 = slot_of(un1);
        if (j + 2 < my_units) un2 = unit_at(j + 2);
        const CUtensorMap* mw = &a.map_w;
        const CUtensorMap* ms = &a.map_sc;
        if (MODE != kModeRouter) {
          if (U.e < 0) {
            mw = &a.map_w_shared;
            ms = &a.map_sc_shared;
            slot = 0;
          } else if (slot < 0 || slot >= a.n_slots) {
            atomicOr(&a.ctrl->err, kErrBadSlot);
            slot = (int)a.n_slots;  // out of range: zero fill
          }
        }
        const int row0 = MODE == kModeGateUp ? U.mt * (NR / 2) : U.mt * NR;
        for (int kc = 0; kc < nK; ++kc, rr.next()) {
          if (MODE == kModeRouter) {
            if (!wait_or_flag(&empty[rr.s], rr.ph ^ 1, a.ctrl)) {
              stop = true;
              break;
            }
            mbar_expect_tx(&full[rr.s], (uint32_t)NR * 128u);
            tma_2d(w_area + rr.s * wbytes, mw, kc * kKC, row0, &full[rr.s]);
          } else {
            if (!wait_or_flag(&raw_empty[rr.s], rr.ph ^ 1, a.ctrl)) {
              stop = true;
              break;
            }
            const bool chunk = a.sc_tma && (kc % kChunk) == 0;
            mbar_expect_tx(&raw_full[rr.s], raw_bytes);
            const uint32_t dst = smem_base + P.raw + rr.s * kRawB;
            if (MODE == kModeGateUp)  // [gate; up] x NR/2 rows of the row tile
              tma_4d(dst, mw, kc * kRowB, row0, 0, slot, &raw_full[rr.s]);
            else
              tma_3d(dst, mw, kc * kRowB, row0, slot, &raw_full[rr.s]);
            if (chunk) {  // [scale, bias] (x [gate, up]) x rows x 8 groups
              // its own barrier: the two dequantising groups read it from different stages
              mbar_expect_tx(&chunk_full[chunks & 1], chunk_bytes);
              tma_4d(smem_base + P.sc + (chunks & 1) * kChunkBytes, ms, kc, row0, 0, slot, &chunk_full[chunks & 1]);
              ++chunks;
            }
          }
          ++issued;
        }
      }
      if (stop) s_abort = 1;
      drain_ring(MODE == kModeRouter ? full : raw_full, MODE == kModeRouter ? P.n_st : P.n_raw, issued, a.ctrl);
      if (MODE != kModeRouter) drain_ring(chunk_full, 2, chunks, a.ctrl);
    }
    __syncwarp();
  } else if (warp >= kDWarp0 && warp < kDWarp0 + kDWarps && MODE != kModeRouter) {
    // ------------------------------ dequantisation ------------------------------
    // Two groups of eight warps take alternate stages (group 0 the even ones), so that two
    // stages are converted at once.  In its group, thread m turns the 64 codes of weight row m
    // into bf16 in the weight tile (eight consecutive rows per quarter-warp: each 16-byte store
    // of a k-octet fills 128 contiguous bytes, no bank conflicts).  Scales and biases come
    // from the stage's scale chunk (every 8 stages, by TMA) or, for rows of fewer than 8
    // groups, from global memory.
    const int grp = (warp - kDWarp0) / kDGroup;
    const int m = ((warp - kDWarp0) % kDGroup) * 32 + lane;  // weight row 0..255
    const bool active = m < NR;
    const int NG = K / kGroup;  // groups (= stages) per row
    const uint32_t raw_off = (uint32_t)m * kRowB;
    // position of row m's scale and bias in a chunk: [scale, bias](x [gate, up]) x rows x 8
    const int sec_rows = MODE == kModeGateUp ? NR / 2 : NR;
    const int sec = MODE == kModeGateUp && m >= NR / 2 ? 2 : 0;
    const int crow = MODE == kModeGateUp ? m % (NR / 2) : m;
    const uint32_t c_s = (uint32_t)((sec * sec_rows + crow) * kChunk), c_b = c_s + (uint32_t)(sec_rows * kChunk);
    // Raw-code reads go chunk by chunk (16 bytes) in an order rotated per lane, so that the
    // eight lanes of each quarter-warp read eight different bank groups (rows are 32 or 64
    // bytes apart: in plain order two or four of them would hit the same banks).
    constexpr int kRawChunks = kRowB / 16;
    const int rot = BITS == 4 ? (m >> 2) & 1 : (m >> 1) & 3;
    uint4 sv4 = make_uint4(0, 0, 0, 0), bv4 = make_uint4(0, 0, 0, 0);  // this row's chunk scales
    Ring ra(P.n_st), rr(P.n_raw);
    int g = 0;  // stage of the CTA's stream
    for (int j = 0; j < my_units && !warp_aborted(&s_abort); ++j) {
      // rows of fewer than 8 groups: this row's scales and biases straight from the blob
      const uint16_t *gs = nullptr, *gb = nullptr;
      if (!a.sc_tma && active) {
        const GemmUnit U = a.units[blockIdx.x + (size_t)j * gridDim.x];
        const uint8_t* blob = a.shared;
        if (U.e >= 0) {
          const int slot = a.slot_table[U.e];
          blob = (slot < 0 || slot >= a.n_slots) ? nullptr : a.pool + (int64_t)slot * a.L.stride;
        }
        if (blob) {
          if (MODE == kModeGateUp) {
            const int64_t r = (int64_t)(U.mt * (NR / 2) + crow) * NG * 2;
            gs = reinterpret_cast<const uint16_t*>(blob + a.L.off[m >= NR / 2 ? 5 : 3] + r);
            gb = reinterpret_cast<const uint16_t*>(blob + a.L.off[m >= NR / 2 ? 6 : 4] + r);
          } else {
            const int64_t r = (int64_t)(U.mt * NR + m) * NG * 2;
            gs = reinterpret_cast<const uint16_t*>(blob + a.L.off[7] + r);
            gb = reinterpret_cast<const uint16_t*>(blob + a.L.off[8] + r);
          }
        }
      }
      bool stop = false;
      for (int kc = 0; kc < nK; ++kc, ++g, ra.next(), rr.next()) {
        if ((g & 1) != grp) continue;  // the other group's stage
        if (!warp_wait(&raw_full[rr.s], rr.ph, a.ctrl, lane)) {
          stop = true;
          break;
        }
        uint32_t w[kRowB / 4];  // this thread's 64 codes, raw chunk (o + rot) % kRawChunks at w[4o..]
        uint32_t sbits = 0, bbits = 0;
        if (active) {
          const uint8_t* rp = smem + P.raw + rr.s * kRawB + raw_off;
#pragma unroll
          for (int o = 0; o < kRawChunks; ++o) {
            const uint4 v = *reinterpret_cast<const uint4*>(rp + ((o + rot) & (kRawChunks - 1)) * 16);
            w[4 * o + 0] = v.x;
            w[4 * o + 1] = v.y;
            w[4 * o + 2] = v.z;
            w[4 * o + 3] = v.w;
          }
          if (a.sc_tma) {
            // The rows of a chunk hold 8 groups (16 bytes): the group takes all 8 scales and
            // biases of its row at its first stage of the chunk (kc % 8 == grp; nK is a
            // multiple of 8 here, so kc and g have the same parity) and keeps them in
            // registers.  Chunk g / 8 sits in slot (g / 8) & 1, on that slot's
            // ((g / 8) >> 1)-th fill; the loader refills the slot (with chunk g / 8 + 2) only
            // after the release of raw stage 8 (g / 8 + 2) - n_raw > g, which comes after the
            // conversion of that stage and therefore after this read.
            if ((kc % kChunk) == grp) {
              if (!mbar_wait_backoff(&chunk_full[(g / kChunk) & 1], ((g / kChunk) >> 1) & 1)) {
                atomicOr(&a.ctrl->err, kErrTimeout);
                s_abort = 1;
              }
              const uint16_t* ch = reinterpret_cast<const uint16_t*>(smem + P.sc + ((g / kChunk) & 1) * kChunkBytes);
              sv4 = *reinterpret_cast<const uint4*>(ch + c_s);
              bv4 = *reinterpret_cast<const uint4*>(ch + c_b);
            }
            // group kc % 8 sits in word (kc % 8) / 2, half kc % 2 (= grp)
            const int q = (kc % kChunk) >> 1;
            const uint32_t sw = q == 0 ? sv4.x : q == 1 ? sv4.y : q == 2 ? sv4.z : sv4.w;
            const uint32_t bw = q == 0 ? bv4.x : q == 1 ? bv4.y : q == 2 ? bv4.z : bv4.w;
            sbits = (sw >> (16 * grp)) & 0xFFFFu;
            bbits = (bw >> (16 * grp)) & 0xFFFFu;
          } else if (gs) {
            sbits = __ldg(gs + kc);
            bbits = __ldg(gb + kc);
          }
        }
        if (!warp_wait(&empty[ra.s], ra.ph ^ 1, a.ctrl, lane)) {
          stop = true;
          break;
        }
        if (active) {
          // raw chunk c holds k-octets 4c .. 4c+3 (int4: one word each) or 2c, 2c+1 (int8: two
          // words each); k-octet j goes to core_off(m, j) = core_off(m, 0) + 128 j
          uint8_t* row_tile = smem + P.w + ra.s * kWBytes + core_off(m, 0);
          if (BITS == 4) {
            const uint32_t s2 = sbits | (sbits << 16), b2 = bbits | (bbits << 16);
#pragma unroll
            for (int o = 0; o < kRawChunks; ++o) {
              uint8_t* dst = row_tile + ((o + rot) & (kRawChunks - 1)) * 512;
#pragma unroll
              for (int i = 0; i < 4; ++i)
                *reinterpret_cast<uint4*>(dst + i * 128) = dq8_int4_bf(w[4 * o + i], s2, b2);
            }
          } else {
            const float sv = __uint_as_float(sbits << 16), bv = __uint_as_float(bbits << 16);
#pragma unroll
            for (int o = 0; o < kRawChunks; ++o) {
              uint8_t* dst = row_tile + ((o + rot) & (kRawChunks - 1)) * 256;
#pragma unroll
              for (int j = 0; j < 2; ++j)
                *reinterpret_cast<uint4*>(dst + j * 128) = dq8_int8(w[4 * o + 2 * j], w[4 * o + 2 * j + 1], sv, bv);
            }
          }
        }
        proxy_fence();
        __syncwarp();
        // The raw slot is released only here, once its codes have been used in the
        // conversion: with the release placed right after the loads into registers, the down
        // GEMM gave wrong outputs on the full prefill workload (the loader's next copy into
        // the slot reached codes that were still to be converted).  The scale chunk's slot is
        // refilled only after a later raw stage's release, so every read of a chunk also
        // precedes its refill by a whole conversion.
        if (lane == 0) {
          mbar_arrive(&full[ra.s]);
          mbar_arrive(&raw_empty[rr.s]);
        }
      }
      if (stop) {
        s_abort = 1;
        break;
      }
    }
  } else if (warp >= kEWarp0) {
    // ------------------------------ epilogue ------------------------------
    // This warp reads TMEM lanes 32*quad .. +31: the unit's tokens 32*quad + lane.
    const int quad = warp & 3;
    const int tok = quad * 32 + lane;
    int it = 0;
    for (int u = blockIdx.x; u < n_units && !warp_aborted(&s_abort); u += gridDim.x, ++it) {
      const GemmUnit U = a.units[u];
      const int buf = it & 1;
      const bool valid = tok < U.n;
      // down: the token this lane adds into and its weight, loaded while the MMAs run
      int t = 0;
      float wt = 0.f;
      if (MODE == kModeDown && valid) {
        if (U.e < 0) {
          t = U.p0 + tok;
          wt = __ldg(a.gate + t);
        } else {
          const int pair = __ldg(a.order + U.p0 + tok);
          t = pair / a.k;
          wt = __ldg(a.topk_w + pair);
        }
      }
      if (!warp_wait(&acc_full[buf], (it >> 1) & 1, a.ctrl, lane)) {
        s_abort = 1;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)buf * (uint32_t)kNMax;
      if (MODE == kModeGateUp) {
        // columns [0, NR/2) are gate rows, [NR/2, NR) the up rows of the same intermediate rows
        const int nI = NR / 2;
        uint16_t* hrow = ((U.e < 0) ? a.hs : a.h) + (size_t)(U.p0 + tok) * a.I + U.mt * nI;
        for (int c0 = 0; c0 < nI; c0 += 16) {
          float gv[16], uv[16];
          tmem_ld16(taddr + c0, gv);
          tmem_ld16(taddr + nI + c0, uv);
          if (valid) {
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              // silu(g) * up; h is rounded to bf16, far coarser than the fast exp / divide
              const float h0 = __fdividef(gv[2 * i], 1.0f + __expf(-gv[2 * i])) * uv[2 * i];
              const float h1 = __fdividef(gv[2 * i + 1], 1.0f + __expf(-gv[2 * i + 1])) * uv[2 * i + 1];
              pk[i] = pack_bf16(h0, h1);
            }
            uint4 o0 = make_uint4(pk[0], pk[1], pk[2], pk[3]), o1 = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            if (a.perm) {  // h is the down GEMM's token operand: k-octet order
              o0 = perm_octet(o0);
              o1 = perm_octet(o1);
            }
            reinterpret_cast<uint4*>(hrow + c0)[0] = o0;
            reinterpret_cast<uint4*>(hrow + c0)[1] = o1;
          }
        }
      } else if (MODE == kModeDown) {
        float* arow = a.acc + (size_t)t * a.H + U.mt * NR;
        for (int c0 = 0; c0 < NR; c0 += 32) {
          float v[32];
          tmem_ld32(taddr + c0, v);
          if (valid) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              atomicAdd(reinterpret_cast<float4*>(arow + c0) + i,
                        make_float4(wt * v[4 * i], wt * v[4 * i + 1], wt * v[4 * i + 2], wt * v[4 * i + 3]));
          }
        }
      } else {  // router logits (no bias)
        float* lrow = a.logits + (size_t)(U.p0 + tok) * (a.E + 1) + U.mt * NR;
        for (int c0 = 0; c0 < NR; c0 += 32) {
          float v[32];
          tmem_ld32(taddr + c0, v);
          if (valid) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (U.mt * NR + c0 + i < a.E) lrow[c0 + i] = v[i];
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
  pdl_launch_dependents();
  pdl_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int rows = T + E + 1;
  if (warp >= rows) return;
  const uint16_t* row = warp < T ? x + (size_t)warp * H : (warp < T + E ? wr + (size_t)(warp - T) * H : wsg);
  // 16-byte loads (rows are 16-byte aligned: the router GEMM reads x and w_r by TMA, the exact
  // dot products read w_sg 16 bytes at a time), eight partial sums per lane; the bound needs
  // the norm only to fp64 accuracy, not in a fixed order
  const uint4* r4 = reinterpret_cast<const uint4*>(row);
  double sp[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
  for (int i = lane; i < H / 8; i += 32) {
    const uint4 v = __ldg(r4 + i);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const double lo = (double)bf_lo(w4[j]), hi = (double)bf_hi(w4[j]);
      sp[2 * j] = fma(lo, lo, sp[2 * j]);
      sp[2 * j + 1] = fma(hi, hi, sp[2 * j + 1]);
    }
  }
  double s = ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    if (warp < T) xnorm[warp] = sqrt(s);
    else wnorm[warp - T] = sqrt(s);
  }
}

// Exact-product fp64 dot of two bf16 rows by one warp (fixed order).
// (eight partial sums per lane, so the additions are not one dependent chain; the order is
// fixed, and every product is exact, so the value differs from any other summation order
// only by fp64 rounding)
__device__ __forceinline__ double warp_dot_exact(const uint16_t* a, const uint16_t* b, int H) {
  const int lane = threadIdx.x & 31;
  double s[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
  for (int i = lane * 8; i < H; i += 256) {
    const uint4 va = *reinterpret_cast<const uint4*>(a + i);
    const uint4 vb = *reinterpret_cast<const uint4*>(b + i);
    s[0] += (double)(bf_lo(va.x) * bf_lo(vb.x));
    s[1] += (double)(bf_hi(va.x) * bf_hi(vb.x));
    s[2] += (double)(bf_lo(va.y) * bf_lo(vb.y));
    s[3] += (double)(bf_hi(va.y) * bf_hi(vb.y));
    s[4] += (double)(bf_lo(va.z) * bf_lo(vb.z));
    s[5] += (double)(bf_hi(va.z) * bf_hi(vb.z));
    s[6] += (double)(bf_lo(va.w) * bf_lo(vb.w));
    s[7] += (double)(bf_hi(va.w) * bf_hi(vb.w));
  }
  double t = ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  return t;
}

// ---------------------------------------------------------------------------------------
// certified top-k: one warp per token
// ---------------------------------------------------------------------------------------
constexpr int kRouteCand = 96;

__global__ void __launch_bounds__(256) k_gate(PrefillArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + wl;
  if (t >= a.T) return;
  const double gl = warp_dot_exact(a.x + (size_t)t * a.H, a.wsg, a.H);
  if (lane == 0) a.gate[t] = (float)(1.0 / (1.0 + exp(-gl)));
}

__global__ void __launch_bounds__(256) k_route(PrefillArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ double s_cl[8][kRouteCand];  // candidates' fp32 logits (with bias): the order key
  __shared__ double s_cu[8][kRouteCand];  // and their certified upper bounds
  __shared__ int s_ce[8][kRouteCand];
  __shared__ int s_ord[8][kRouteCand];
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
  // Exact values (fp64 sums of exact products, fixed order), lanes 0..k-1 keeping the best k
  // so far (value desc, id asc).  A candidate whose certified upper bound is below the k-th
  // kept exact value is skipped: its exact value is below every value of the final top k, so
  // the selection is the one over all candidates.  Normally the candidates come in decreasing
  // order of the fp32 logit; after an overflow every expert comes, in id order, under the
  // same test (at most E exact dots, most of them skipped once k are kept).
  double sv = -INFINITY;
  int se = 0x7fffffff;
  int cnt = 0;  // kept so far (<= k)
  const auto consider = [&](int e, double upper) {
    const double vk = __shfl_sync(0xffffffffu, sv, k - 1);
    if (cnt == k && upper < vk) return;
    const double v = warp_dot_exact(xt, a.wr + (size_t)e * H, H) + (a.rbias ? (double)a.rbias[e] : 0.0);
    if (!(v == v)) return;  // a NaN is never selected
    const bool before = lane < cnt && (sv > v || (sv == v && se < e));
    const int pos = __popc(__ballot_sync(0xffffffffu, before));
    if (pos >= k) return;
    const double pv = __shfl_up_sync(0xffffffffu, sv, 1);
    const int pe = __shfl_up_sync(0xffffffffu, se, 1);
    if (lane > pos) {
      sv = pv;
      se = pe;
    }
    if (lane == pos) {
      sv = v;
      se = e;
    }
    cnt = cnt < k ? cnt + 1 : k;
  };
  if (!overflow) {
    for (int i = lane; i < n; i += 32) {
      const int e = s_ce[wl][i];
      const double l = (double)lt[e] + (a.rbias ? (double)a.rbias[e] : 0.0);
      s_cl[wl][i] = (l == l) ? l : INFINITY;  // a NaN logit first (its exact value decides)
      s_cu[wl][i] = l + cb * a.wnorm[e];      // NaN for a NaN logit: never skipped
    }
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
      const double ki = s_cl[wl][i];
      int rank = 0;
      for (int j = 0; j < n; ++j) {
        const double kj = s_cl[wl][j];
        rank += (kj > ki || (kj == ki && j < i)) ? 1 : 0;
      }
      s_ord[wl][rank] = i;
    }
    __syncwarp();
    for (int r = 0; r < n; ++r) {
      const int i = s_ord[wl][r];
      consider(s_ce[wl][i], s_cu[wl][i]);
    }
  } else {
    for (int e = 0; e < E; ++e)
      consider(e, (double)lt[e] + (a.rbias ? (double)a.rbias[e] : 0.0) + cb * a.wnorm[e]);
  }
  if (lane >= cnt) {
    sv = -INFINITY;
    se = 0x7fffffff;
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
//   k_gcol    one warp per expert: exclusive sums of its counts down the chunks (in
//             place) and the expert's total
//   k_gplace  per chunk: offsets = exclusive scan of the totals; stable ranks (warp match
//             + per-warp counts); order[slot] = pair.  Chunk 0 also writes offsets, counts
//             and the GEMM work units.
// Pair p of chunk c lands at offsets[e] + (pairs of e in chunks < c) + (pairs of e before it
// in chunk c): the pairs of one expert keep their pair-index order.
// ---------------------------------------------------------------------------------------
constexpr int kGroupThreads = 256;  // 8 warps; each takes kGroupChunk / 8 consecutive pairs
static_assert(kGroupChunk % kGroupThreads == 0, "chunk must split into whole warp rounds");
static_assert(kMaxExperts <= 4 * kGroupThreads, "block scan takes 4 experts per thread");

// An expert whose slot-table entry marks it as held by another rank (expert parallelism):
// its pairs are left out of the grouping here, without an error; that rank computes them.
__device__ __forceinline__ bool remote_expert(const PrefillArgs& a, int e) {
  return a.g.slot_table && __ldg(a.g.slot_table + e) == kSlotRemote;
}

__global__ void __launch_bounds__(kGroupThreads) k_ghist(PrefillArgs a) {
  pdl_launch_dependents();
  pdl_wait();
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
      else if (!remote_expert(a, e)) atomicAdd(&hsm[e], 1);
    }
  }
  __syncthreads();
  int* out = a.chunk_cnt + (size_t)blockIdx.x * E;
  for (int e = threadIdx.x; e < E; e += kGroupThreads) out[e] = hsm[e];
}

__global__ void __launch_bounds__(1024) k_gcol(PrefillArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * 32 + (threadIdx.x >> 5);
  if (e >= a.E) return;
  const int E = a.E, nc = (a.T * a.k + kGroupChunk - 1) / kGroupChunk;
  int carry = 0;
  for (int c0 = 0; c0 < nc; c0 += 128) {
    int v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = c0 + j * 32 + lane;
      v[j] = c < nc ? a.chunk_cnt[(size_t)c * E + e] : 0;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int incl = v[j];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int c = c0 + j * 32 + lane;
      if (c < nc) a.chunk_cnt[(size_t)c * E + e] = carry + incl - v[j];
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  if (lane == 0) a.counts[e] = carry;
}

// Exclusive scan of val(0..E-1) over the block (kGroupThreads threads, 4 values each);
// out[0..E] (out[E] = total).  Every thread must call it.
template <class F>
__device__ void block_scan4(int E, F val, int* out, int* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int e0 = threadIdx.x * 4;
  int v[4], s = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    v[j] = (e0 + j < E) ? val(e0 + j) : 0;
    s += v[j];
  }
  int incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int wv = lane < kGroupThreads / 32 ? wsum[lane] : 0;
    int wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < kGroupThreads / 32) wsum[lane] = wi - wv;
    if (lane == kGroupThreads / 32 - 1) wsum[kGroupThreads / 32] = wi;
  }
  __syncthreads();
  int run = wsum[warp] + incl - s;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (e0 + j < E) out[e0 + j] = run;
    run += v[j];
  }
  if (threadIdx.x == 0) out[E] = wsum[kGroupThreads / 32];
  __syncthreads();
}

__global__ void __launch_bounds__(kGroupThreads) k_gplace(PrefillArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ int wc[];  // [8][E]: per-warp counts, then per-warp running slots
  __shared__ int s_off[kMaxExperts + 1];
  __shared__ int s_wsum[kGroupThreads / 32 + 1];
  constexpr int kW = kGroupThreads / 32, kRounds = kGroupChunk / kGroupThreads;
  const int E = a.E, n = a.T * a.k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kW * E; i += kGroupThreads) wc[i] = 0;
  block_scan4(E, [&](int e) { return a.counts[e]; }, s_off, s_wsum);
  // warp w takes pairs [pw, pw + 32 * kRounds), round by round
  const int pw = blockIdx.x * kGroupChunk + warp * 32 * kRounds;
  int ev[kRounds];
#pragma unroll
  for (int r = 0; r < kRounds; ++r) {
    const int p = pw + r * 32 + lane;
    const int e = p < n ? __ldg(a.topk_idx + p) : -1;
    ev[r] = (e >= 0 && e < E && !remote_expert(a, e)) ? e : -1;
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
    int pos = s_off[e] + base[e];
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
  // offsets (chunk 0), and the GEMM work units: per expert, token tiles of <= kTok pairs x
  // weight-row tiles; then the shared expert as one more expert over all tokens.  Every
  // chunk's CTA writes the units of experts e = chunk (mod chunks).
  if (blockIdx.x == 0)
    for (int e = threadIdx.x; e <= E; e += kGroupThreads) a.offsets[e] = s_off[e];
  if (!a.units_gu) return;  // grouping only
  __syncthreads();
  int* tile_base = wc;  // [E + 1], reused
  block_scan4(E, [&](int e) { return (a.counts[e] + kTok - 1) / kTok; }, tile_base, s_wsum);
  const int mt_gu = a.I / (prefill_gu_rows(a.I) / 2), mt_dn = a.H / prefill_dn_rows(a.H);
  for (int e = blockIdx.x + (int)gridDim.x * threadIdx.x; e < E; e += (int)gridDim.x * kGroupThreads) {
    int tb = tile_base[e];
    const int ce = a.counts[e];
    for (int s0 = 0; s0 < ce; s0 += kTok, ++tb) {
      const int nn = min(kTok, ce - s0);
      for (int mt = 0; mt < mt_gu; ++mt) a.units_gu[tb * mt_gu + mt] = GemmUnit{e, mt, s_off[e] + s0, nn};
      for (int mt = 0; mt < mt_dn; ++mt) a.units_dn[tb * mt_dn + mt] = GemmUnit{e, mt, s_off[e] + s0, nn};
    }
  }
  if (blockIdx.x != 0) return;
  const int tiles_r = tile_base[E];
  const int st_n = a.no_shared ? 0 : (a.T + kTok - 1) / kTok;  // the shared expert's token tiles
  for (int i = threadIdx.x; i < st_n * mt_gu; i += kGroupThreads) {
    const int st = i / mt_gu, mt = i - st * mt_gu, t0 = st * kTok;
    a.units_gu[(tiles_r + st) * mt_gu + mt] = GemmUnit{-1, mt, t0, min(kTok, a.T - t0)};
  }
  for (int i = threadIdx.x; i < st_n * mt_dn; i += kGroupThreads) {
    const int st = i / mt_dn, mt = i - st * mt_dn, t0 = st * kTok;
    a.units_dn[(tiles_r + st) * mt_dn + mt] = GemmUnit{-1, mt, t0, min(kTok, a.T - t0)};
  }
  if (threadIdx.x == 0) {
    a.n_units[0] = (tiles_r + st_n) * mt_gu;
    a.n_units[1] = (tiles_r + st_n) * mt_dn;
  }
}

// xg[p] = x[order[p] / k] for every grouped pair position p < offsets[E]: the routed gate/up
// GEMM then reads each expert's tokens as consecutive rows.  One warp per row.
__global__ void __launch_bounds__(256) k_permute(PrefillArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  // warps [0, T*k): xg row p (valid pairs only); with perm, warps [T*k, T*k + T): xp row t
  const int p = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int n_pairs = a.T * a.k;
  const uint4* src;
  uint4* dst;
  if (p < n_pairs) {
    if (p >= a.offsets[a.E]) return;
    src = reinterpret_cast<const uint4*>(a.x + (size_t)(__ldg(a.order + p) / a.k) * a.H);
    dst = reinterpret_cast<uint4*>(a.xg + (size_t)p * a.H);
  } else {
    if (!a.perm || p >= n_pairs + a.T) return;
    src = reinterpret_cast<const uint4*>(a.x + (size_t)(p - n_pairs) * a.H);
    dst = reinterpret_cast<uint4*>(a.xp + (size_t)(p - n_pairs) * a.H);
  }
  if (a.perm) {
    for (int i = lane; i < a.H / 8; i += 32) dst[i] = perm_octet(__ldg(src + i));
  } else {
    for (int i = lane; i < a.H / 8; i += 32) dst[i] = __ldg(src + i);
  }
}

__global__ void k_finalize(const float* acc, const uint16_t* residual, uint16_t* out, size_t n) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = f2bf(acc[i] + (residual ? bf1(residual[i]) : 0.f));
}
// The same, 8 elements per thread (two 16-byte loads of acc, one of the residual, one 16-byte
// store), grid-stride; for 16-byte aligned buffers.  acc is read for the last time: streaming
// loads.
__global__ void __launch_bounds__(256) k_finalize8(const float4* acc, const uint4* residual, uint4* out, size_t n8) {
  pdl_launch_dependents();
  pdl_wait();
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
    const float4 a0 = __ldcs(acc + 2 * i), a1 = __ldcs(acc + 2 * i + 1);
    const uint4 r = residual ? __ldcs(residual + i) : make_uint4(0, 0, 0, 0);
    uint4 o;
    o.x = (uint32_t)f2bf(a0.x + bf_lo(r.x)) | ((uint32_t)f2bf(a0.y + bf_hi(r.x)) << 16);
    o.y = (uint32_t)f2bf(a0.z + bf_lo(r.y)) | ((uint32_t)f2bf(a0.w + bf_hi(r.y)) << 16);
    o.z = (uint32_t)f2bf(a1.x + bf_lo(r.z)) | ((uint32_t)f2bf(a1.y + bf_hi(r.z)) << 16);
    o.w = (uint32_t)f2bf(a1.z + bf_lo(r.w)) | ((uint32_t)f2bf(a1.w + bf_hi(r.w)) << 16);
    out[i] = o;
  }
}

__global__ void k_router_units(GemmUnit* units, int* n_units, int T, int E) {
  pdl_launch_dependents();
  pdl_wait();
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

// Launches a kernel as a programmatic dependent of the kernel before it on the stream: it may
// start while that kernel finishes and waits for it (pdl_wait) before reading its results.
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*fn)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, std::forward<Args>(args)...);
}

template <int BITS, int MODE>
cudaError_t launch_gemm(const GemmArgs& g, int n_sm, cudaStream_t s) {
  const GemmSmem P = gemm_smem<BITS, MODE>();
  if (P.total > (uint32_t)kSmemMax || P.n_st < 2) return cudaErrorInvalidConfiguration;
  auto fn = k_gemm<BITS, MODE>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.total);
  if (e != cudaSuccess) return e;
  return launch_pdl(fn, dim3(n_sm), dim3(kGemmThreads), P.total, s, g);
}

// ---- TMA descriptors (host) ----
// The driver's encoder is looked up through the runtime, so the library does not link the
// driver library itself (it loads on machines without a GPU driver).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFn) nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}
cudaError_t encode_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const cuuint64_t* dims,
                       const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle sw) {
  const EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  const CUresult r = fn(m, dt, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}
// bf16 row-major [rows, cols] (row stride ld elements): boxes of 64 columns x box_rows rows,
// 128-byte swizzle (the operand layout of the MMAs)
cudaError_t map_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {ld * 2};
  const cuuint32_t box[2] = {64, box_rows};
  return encode_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}
// Raw gate/up codes of a pool (or one blob): bytes [slots][gate, up][I][H*b/8]; a box is one
// stage (64 codes) of nI rows of both matrices
cudaError_t map_codes_gu(CUtensorMap* m, const uint8_t* blob0, int64_t n_slots, const BlobLayout& L, int H, int I,
                         int bits, int nI) {
  const cuuint64_t dims[4] = {(cuuint64_t)H * bits / 8, (cuuint64_t)I, 2, (cuuint64_t)n_slots};
  const cuuint64_t strides[3] = {(cuuint64_t)H * bits / 8, (cuuint64_t)(L.off[1] - L.off[0]), (cuuint64_t)L.stride};
  const cuuint32_t box[4] = {(cuuint32_t)(kKC * bits / 8), (cuuint32_t)nI, 2, 1};
  return encode_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, blob0 + L.off[0], dims, strides, box,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
}
// Raw down codes: bytes [slots][H][I*b/8]; a box is one stage of NR rows
cudaError_t map_codes_dn(CUtensorMap* m, const uint8_t* blob0, int64_t n_slots, const BlobLayout& L, int H, int I,
                         int bits, int NR) {
  const cuuint64_t dims[3] = {(cuuint64_t)I * bits / 8, (cuuint64_t)H, (cuuint64_t)n_slots};
  const cuuint64_t strides[2] = {(cuuint64_t)I * bits / 8, (cuuint64_t)L.stride};
  const cuuint32_t box[3] = {(cuuint32_t)(kKC * bits / 8), (cuuint32_t)NR, 1};
  return encode_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, blob0 + L.off[2], dims, strides, box,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
}
// Scale / bias chunks: bf16 [slots][n_sec sections][rows][NG], the sections n_sec equally
// spaced blob sections starting at section `first` (gate/up: gate s, gate b, up s, up b;
// down: s, b); a box is 8 groups of box_rows rows of every section.  Needs NG % 8 == 0.
cudaError_t map_scales(CUtensorMap* m, const uint8_t* blob0, int64_t n_slots, const BlobLayout& L, int first,
                       int n_sec, int rows, int NG, int box_rows) {
  const cuuint64_t dims[4] = {(cuuint64_t)NG, (cuuint64_t)rows, (cuuint64_t)n_sec, (cuuint64_t)n_slots};
  const cuuint64_t strides[3] = {(cuuint64_t)NG * 2, (cuuint64_t)(L.off[first + 1] - L.off[first]),
                                 (cuuint64_t)L.stride};
  const cuuint32_t box[4] = {(cuuint32_t)kChunk, (cuuint32_t)box_rows, (cuuint32_t)n_sec, 1};
  return encode_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, blob0 + L.off[first], dims, strides, box,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
}

}  // namespace

bool prefill_shape_supported(int H, int I, int bits, int E) {
  return (bits == 4 || bits == 8) && H % 128 == 0 && I % 64 == 0 && E <= 512 && H <= 4096 && I <= 4096;
}

cudaError_t launch_group(const PrefillArgs& p, cudaStream_t s) {
  const int n_chunks = (p.T * p.k + kGroupChunk - 1) / kGroupChunk;
  cudaError_t e = launch_pdl(k_ghist, dim3(n_chunks), dim3(kGroupThreads), sizeof(int) * p.E, s, p);
  if (e == cudaSuccess) e = launch_pdl(k_gcol, dim3((p.E + 31) / 32), dim3(1024), 0, s, p);
  const size_t smem = sizeof(int) * (size_t)(kGroupThreads / 32) * p.E;
  if (e == cudaSuccess) e = launch_pdl(k_gplace, dim3(n_chunks), dim3(kGroupThreads), smem, s, p);
  return e;
}

// Norms, fp32 router logits on the tensor cores and the certified top-k of p.T tokens
// (p.route must be set): the routing step of the many-token path, also used alone by
// moe_router_topk.
static cudaError_t launch_route(const PrefillArgs& p, int n_sm, cudaStream_t s) {
  const int T = p.T, E = p.E, H = p.H;
  cudaError_t e;
  const int rows = T + E + 1;
  if ((e = launch_pdl(k_norms, dim3((rows * 32 + 255) / 256), dim3(256), 0, s, p.x, T, H, p.wr, p.wsg, E,
                      p.xnorm, p.wnorm)) != cudaSuccess)
    return e;
  const int mt_n = (E + 127) / 128, nt = (T + 127) / 128;
  if ((e = launch_pdl(k_router_units, dim3((mt_n * nt + 255) / 256), dim3(256), 0, s, p.units_rt, p.n_units + 2, T,
                      E)) != cudaSuccess)
    return e;
  GemmArgs g = p.g;
  g.units = p.units_rt;
  g.n_units = p.n_units + 2;
  g.n_rows = 128;
  g.sc_tma = 0;
  if ((e = map_bf16(&g.map_w, p.wr, E, H, H, 128)) != cudaSuccess) return e;
  if ((e = map_bf16(&g.map_tok, p.x, T, H, H, kTRows)) != cudaSuccess) return e;
  // the router GEMM reads bf16 rows only; the code width does not enter it
  if ((e = launch_gemm<4, kModeRouter>(g, n_sm, s)) != cudaSuccess) return e;
  return launch_pdl(k_route, dim3((T + 7) / 8), dim3(256), 0, s, p);
}

static int sm_count() {
  int dev = 0, n_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  return n_sm;
}

cudaError_t launch_prefill_route(const PrefillArgs& p, cudaStream_t s) { return launch_route(p, sm_count(), s); }

cudaError_t launch_prefill(const PrefillArgs& p, int bits, cudaStream_t s) {
  const int n_sm = sm_count();
  const int T = p.T, H = p.H;
  cudaError_t e;
  // accumulator of the down products
  if ((e = cudaMemsetAsync(p.acc, 0, sizeof(float) * (size_t)T * H, s)) != cudaSuccess) return e;
  // norms, router logits, certified top-k
  prof_mark(0, false, s);
  if (p.route) {
    if ((e = launch_route(p, n_sm, s)) != cudaSuccess) return e;
  } else {
    if ((e = launch_pdl(k_gate, dim3((T + 7) / 8), dim3(256), 0, s, p)) != cudaSuccess) return e;
  }
  prof_mark(0, true, s);
  // grouping and work units
  prof_mark(1, false, s);
  if ((e = launch_group(p, s)) != cudaSuccess) return e;
  if ((e = launch_pdl(k_permute, dim3((unsigned)((((size_t)T * p.k + (p.perm ? T : 0)) * 32 + 255) / 256)), dim3(256),
                      0, s, p)) != cudaSuccess)
    return e;
  prof_mark(1, true, s);
  // gate/up + SwiGLU, then down + scatter
  {
    GemmArgs g = p.g;
    g.units = p.units_gu;
    g.n_units = p.n_units;
    const int I = p.I;
    g.n_rows = prefill_gu_rows(I);
    g.sc_tma = (H / kGroup) % kChunk == 0;
    const int nI = g.n_rows / 2;
    if ((e = map_codes_gu(&g.map_w, g.pool, g.n_slots, g.L, H, I, bits, nI)) != cudaSuccess) return e;
    if ((e = map_codes_gu(&g.map_w_shared, g.shared, 1, g.L, H, I, bits, nI)) != cudaSuccess) return e;
    if (g.sc_tma) {
      if ((e = map_scales(&g.map_sc, g.pool, g.n_slots, g.L, 3, 4, I, H / kGroup, nI)) != cudaSuccess) return e;
      if ((e = map_scales(&g.map_sc_shared, g.shared, 1, g.L, 3, 4, I, H / kGroup, nI)) != cudaSuccess) return e;
    }
    if ((e = map_bf16(&g.map_tok, p.xg, (uint64_t)T * p.k, H, H, kTRows)) != cudaSuccess) return e;
    if ((e = map_bf16(&g.map_tok2, p.perm ? p.xp : p.x, T, H, H, kTRows)) != cudaSuccess) return e;
    g.perm = p.perm;
    prof_mark(2, false, s);
    if ((e = (bits == 4 ? launch_gemm<4, kModeGateUp>(g, n_sm, s) : launch_gemm<8, kModeGateUp>(g, n_sm, s))) !=
        cudaSuccess)
      return e;
    prof_mark(2, true, s);
    g.units = p.units_dn;
    g.n_units = p.n_units + 1;
    g.n_rows = prefill_dn_rows(H);
    g.sc_tma = (I / kGroup) % kChunk == 0;
    if ((e = map_codes_dn(&g.map_w, g.pool, g.n_slots, g.L, H, I, bits, g.n_rows)) != cudaSuccess) return e;
    if ((e = map_codes_dn(&g.map_w_shared, g.shared, 1, g.L, H, I, bits, g.n_rows)) != cudaSuccess) return e;
    if (g.sc_tma) {
      if ((e = map_scales(&g.map_sc, g.pool, g.n_slots, g.L, 7, 2, H, I / kGroup, g.n_rows)) != cudaSuccess) return e;
      if ((e = map_scales(&g.map_sc_shared, g.shared, 1, g.L, 7, 2, H, I / kGroup, g.n_rows)) != cudaSuccess) return e;
    }
    if ((e = map_bf16(&g.map_tok, p.h, (uint64_t)T * p.k, I, I, kTRows)) != cudaSuccess) return e;
    if ((e = map_bf16(&g.map_tok2, p.hs, T, I, I, kTRows)) != cudaSuccess) return e;
    prof_mark(3, false, s);
    if ((e = (bits == 4 ? launch_gemm<4, kModeDown>(g, n_sm, s) : launch_gemm<8, kModeDown>(g, n_sm, s))) !=
        cudaSuccess)
      return e;
    prof_mark(3, true, s);
  }
  const size_t n = (size_t)T * H;
  prof_mark(4, false, s);
  // a partial forward leaves its fp32 sum in acc (the caller's buffer): no finalize
  if (p.out) {
    const bool vec = n % 8 == 0 && (reinterpret_cast<uintptr_t>(p.acc) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(p.residual) & 15) == 0 && (reinterpret_cast<uintptr_t>(p.out) & 15) == 0;
    if (vec) {
      const size_t n8 = n / 8;
      const unsigned blocks = (unsigned)std::min<size_t>((n8 + 255) / 256, (size_t)n_sm * 8);
      e = launch_pdl(k_finalize8, dim3(blocks), dim3(256), 0, s, reinterpret_cast<const float4*>(p.acc),
                     reinterpret_cast<const uint4*>(p.residual), reinterpret_cast<uint4*>(p.out), n8);
    } else {
      e = launch_pdl(k_finalize, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, p.acc, p.residual, p.out, n);
    }
    if (e != cudaSuccess) return e;
  }
  prof_mark(4, true, s);
  return cudaSuccess;
}

}  // namespace moe
