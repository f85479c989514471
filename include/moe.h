/*
 * moe.h -- C ABI of the routed Mixture-of-Experts layer forward for NVIDIA B200 (sm_100a).
 *
 * What the layer computes (Swiftlet pages: «Paquets Swiftlet 80B Qwen dans Mac…»,
 * xix.ai, paragraphs 5 and 9; «Swiftlet: 在 Mac 和 iPhone 上執行 80B 與 35B Qwen 模型»,
 * agentlenshq.com, section 記憶體管理與權重串流; «Swiftlet — это Swift + Metal
 * рантайм…», news.bugfactory.tech, paragraph 3):
 *
 *   router   l[t,e] = sum_i x[t,i] * Wr[e,i] (+ b[e]); the k experts with the largest
 *            logits (ties: lower index first) are selected and weighted by a softmax
 *            over the k selected logits (weights sum to 1);
 *   experts  each selected expert is a SwiGLU MLP y = Wd (silu(Wg x) * (Wu x)) whose
 *            weights are MLX-style affine group-quantised codes (int4 or int8, group
 *            64 along the input dimension, bf16 scale and bias per group):
 *            w = scale * q + bias;
 *   shared   an always-on shared expert with the same blob format, scaled by
 *            sigmoid(w_sg . x);
 *   combine  out[t] = sum_k p[t,k] y_k + sigmoid(w_sg . x[t]) y_shared (+ residual[t]).
 *
 * Expert storage.  Every expert is one fixed-stride blob ("one read = one fetch"):
 * nine sections, each starting on a 256-byte boundary, in the order
 *   Wg.q [I, H*b/8], Wu.q [I, H*b/8], Wd.q [H, I*b/8]              (u8 codes)
 *   Wg.s, Wg.bias, Wu.s, Wu.bias [I, H/64], Wd.s, Wd.bias [H, I/64]  (bf16)
 * Codes are packed little-endian as MLX does: for int4, byte n of a row holds element
 * 2n in its low nibble and element 2n+1 in its high nibble; for int8 byte n is element
 * n.  A pool is n_slots blobs back to back; slot s starts at byte s * stride (64-bit
 * offsets).  slot_table[e] names the slot that holds expert e.
 *
 * Conventions for every call:
 *   - Pointers marked (dev) are device pointers, (host) are host pointers.  All device
 *     memory is owned by the caller; the library keeps no pointer after a call returns
 *     (except the pool object, which keeps the ones given to moe_pool_create).
 *   - bf16 tensors are passed as raw 16-bit patterns; all tensors are dense row-major.
 *   - Device pointers must be 16-byte aligned; the pool and blob pointers 256-byte
 *     aligned.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) and
 *     is asynchronous, except where a call says it synchronises.
 *   - Arguments are validated before anything is enqueued; a bad argument returns
 *     MOE_ERR_INVALID (or MOE_ERR_UNSUPPORTED for a valid shape this library has no
 *     kernel for) and enqueues nothing.  Nothing aborts or throws across this ABI.
 *     moe_last_error() gives a message for the calling thread's last failure.
 *   - Errors detected on the device (an expert id outside [0, E), a slot outside
 *     [0, n_slots), non-finite router logits) set bits in the workspace's error word
 *     and the offending term is skipped; read them with moe_ws_check().
 *   - The workspace must be zero-filled once before its first use; every call leaves
 *     its internal counters at zero again (after a MOE_DEVERR_TIMEOUT, zero it again).
 *     Calls that share a workspace must not run concurrently.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID = -1,      /* bad argument (null pointer, bad size, misalignment) */
  MOE_ERR_CUDA = -2,         /* a CUDA runtime call failed; see moe_last_error() */
  MOE_ERR_CAPACITY = -3,     /* a pool step needs more distinct experts than slots */
  MOE_ERR_NOT_RESIDENT = -4, /* reserved: an expert the call needs has no slot */
  MOE_ERR_UNSUPPORTED = -5,  /* valid request with no kernel in this library */
  MOE_ERR_TIMEOUT = -6,      /* a bounded device-side wait gave up */
  MOE_ERR_DEVICE = -7,       /* the device set an error bit (moe_ws_check) */
  MOE_ERR_IO = -8            /* the pool's backing file could not be opened or read */
} moe_status;

/* Device error-word bits (moe_ws_check). */
#define MOE_DEVERR_BAD_EXPERT 0x1u   /* a top-k expert id outside [0, E) was skipped   */
#define MOE_DEVERR_BAD_SLOT 0x2u     /* slot_table gave a slot outside [0, n_slots)     */
#define MOE_DEVERR_NONFINITE 0x4u    /* a router logit was NaN/Inf; top-k may be short  */
#define MOE_DEVERR_TIMEOUT 0x8u      /* a bounded device wait gave up                   */

typedef struct {
  int32_t hidden;       /* H: model width (multiple of 64)                                 */
  int32_t inter;        /* I: routed-expert intermediate width (multiple of 64)            */
  int32_t shared_inter; /* I_s: shared-expert intermediate width (this library: I_s == I)  */
  int32_t n_experts;    /* E: routed experts per layer (1..1024)                           */
  int32_t top_k;        /* k: experts per token (1..min(E, 32))                            */
  int32_t bits;         /* 4 or 8                                                          */
  int32_t group;        /* quantisation group along the input dimension: must be 64        */
} moe_shape;

/*
 * moe_blob_layout -- byte offsets of the nine sections of one expert blob and its stride.
 * Defines the fixed-stride blob ("one contiguous read per expert", «Swiftlet: 在 Mac 和
 * iPhone 上執行…», 記憶體管理與權重串流).  hidden/inter must be multiples of 64, bits 4 or
 * 8, group 64.  offsets (host, 9 entries) and stride (host) are written on success.
 */
MOE_API moe_status moe_blob_layout(int32_t hidden, int32_t inter, int32_t bits, int32_t group,
                           int64_t offsets[9], int64_t* stride);

/*
 * moe_workspace_size -- bytes of device workspace that moe_router_topk / moe_layer_forward
 * need for T tokens of this shape.  *bytes (host) is written on success.
 */
MOE_API moe_status moe_workspace_size(const moe_shape* shape, int32_t T, size_t* bytes);

/*
 * moe_router_topk -- router GEMV + softmax top-k (the per-layer router: «Paquets Swiftlet…»
 * paragraph 5, 10 of 512 / 8 of 256 experts per token).
 *   x           (dev) bf16 [T, H] activations
 *   w_router    (dev) bf16 [E, H]
 *   router_bias (dev) fp32 [E] or NULL: added to the logits before selection and softmax
 *   topk_idx    (dev) int32 [T, k] out: expert ids, logit descending, ties lower id first
 *   topk_w      (dev) fp32  [T, k] out: softmax over the k selected logits
 *   ws          (dev) workspace of ws_bytes >= moe_workspace_size(shape, T)
 * Any T >= 1.  Up to 8 tokens (and, in groups of 8, shapes the many-token router does not
 * cover): logits accumulated in fp64 from exact bf16*bf16 products.  More than 8 tokens with
 * hidden % 128 == 0, hidden <= 4096 and E <= 512: the router of the many-token layer
 * forward -- fp32 logits on the tensor cores, and every expert whose fp32 logit lies within
 * the fp32 error bound of the k-th is recomputed exactly before the selection and the
 * softmax.  Either way the selection is the exact-arithmetic selection except for logits
 * that tie to within fp64 rounding.  ws must hold moe_workspace_size(shape, T) bytes.
 */
MOE_API moe_status moe_router_topk(const moe_shape* shape, const void* x, int32_t T, const void* w_router,
                           const float* router_bias, int32_t* topk_idx, float* topk_w, void* ws,
                           size_t ws_bytes, void* stream);

/*
 * moe_layer_forward -- the routed-MoE layer forward for T tokens.
 *   x            (dev) bf16 [T, H]
 *   w_router     (dev) bf16 [E, H]      (unused when topk_idx_in != NULL)
 *   router_bias  (dev) fp32 [E] or NULL
 *   topk_idx_in  (dev) int32 [T, k] or NULL: precomputed routing (e.g. from moe_router_topk
 *                before moe_expert_pool_load); NULL routes inside this call
 *   topk_w_in    (dev) fp32 [T, k]: weights for topk_idx_in (required with it)
 *   pool         (dev) u8 [n_slots * stride] expert blobs; stride from moe_blob_layout
 *   slot_table   (dev) int32 [E]: slot of each expert; entries of experts that a call
 *                selects must be in [0, n_slots)
 *   n_slots      number of blobs in pool (bounds-checks slot_table on the device)
 *   shared_blob  (dev) u8 blob of the shared expert (layout with inter = I_s)
 *   w_shared_gate(dev) bf16 [H]: shared-expert gate, scale = sigmoid(w . x[t])
 *   residual     (dev) bf16 [T, H] or NULL: added to the output
 *   out          (dev) bf16 [T, H] out (round-to-nearest-even of the fp32 sum)
 *   topk_idx_out, topk_w_out (dev) [T, k] or NULL: the routing used (when routed inside)
 *   ws, ws_bytes workspace (see moe_workspace_size)
 * T: 1..8 runs the decode path (fused GEMV kernels): deterministic, the same inputs give
 * the same bits whichever slots the experts sit in.  T > 8 runs the many-token (prefill)
 * path: router on the tensor cores with every near-boundary logit recomputed exactly, the
 * pairs grouped by expert, and per-expert tcgen05 GEMMs on weights dequantised to bf16
 * (hidden % 128 == 0, E <= 512); its down products are summed with fp32 atomics, so the
 * last bits of out may vary from run to run.
 */
MOE_API moe_status moe_layer_forward(const moe_shape* shape, const void* x, int32_t T, const void* w_router,
                             const float* router_bias, const int32_t* topk_idx_in,
                             const float* topk_w_in, const uint8_t* pool, const int32_t* slot_table,
                             int64_t n_slots, const uint8_t* shared_blob, const void* w_shared_gate,
                             const void* residual, void* out, int32_t* topk_idx_out,
                             float* topk_w_out, void* ws, size_t ws_bytes, void* stream);

/*
 * One layer of a stack for moe_stack_forward (all pointers device pointers, as in
 * moe_layer_forward).  x may be NULL for layers after the first: the layer then reads the
 * previous layer's out.
 */
typedef struct {
  const void* x;                /* bf16 [T, H] layer input, or NULL (previous layer's out)   */
  const void* w_router;         /* bf16 [E, H] (unused when topk_idx_in != NULL)             */
  const float* router_bias;     /* fp32 [E] or NULL                                          */
  const int32_t* topk_idx_in;   /* int32 [T, k] or NULL (route inside)                       */
  const float* topk_w_in;       /* fp32 [T, k] (with topk_idx_in)                            */
  const uint8_t* pool;          /* u8 [n_slots * stride]                                     */
  const int32_t* slot_table;    /* int32 [E]                                                 */
  int64_t n_slots;
  const uint8_t* shared_blob;   /* shared-expert blob                                        */
  const void* w_shared_gate;    /* bf16 [H]                                                  */
  const void* residual;         /* bf16 [T, H] or NULL                                       */
  void* out;                    /* bf16 [T, H] out                                           */
  int32_t* topk_idx_out;        /* int32 [T, k] or NULL                                      */
  float* topk_w_out;            /* fp32 [T, k] or NULL                                       */
} moe_layer_desc;

/*
 * moe_stack_forward -- n_layers (1..64) routed-MoE layers in sequence, layer l+1 reading
 * layer l's output (decode: T = 1..8 tokens; the per-layer token decode loop of the pages,
 * «Swiftlet — это Swift + Metal рантайм…» paragraph 2, whose speed is bound by dispatch).
 *   layers (host) array of n_layers descriptors; every layer has the same shape.
 *   ws, ws_bytes as for moe_layer_forward (one workspace serves every layer).
 * Same results as calling moe_layer_forward once per layer.  For the shapes it supports
 * (hidden/inter 256/64, 512/128, 1024/256, 2048/512, 4096/1024; E <= 512) the whole stack
 * is one persistent cooperative kernel with grid-wide barriers between its phases; other
 * shapes run layer by layer.
 */
MOE_API moe_status moe_stack_forward(const moe_shape* shape, int32_t T, const moe_layer_desc* layers,
                                     int32_t n_layers, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_layer_forward_partial -- one rank's share of an expert-parallel layer (the routed
 * experts of a layer sharded over GPUs; the Swiftlet pages run one device and describe no
 * sharding, so this follows the plain reading of splitting the layer's experts, «Paquets
 * Swiftlet 80B Qwen dans Mac…», paragraph 5: 10 of 512 experts per token).
 * Arguments as moe_layer_forward, except:
 *   slot_table     (dev) int32 [E]: this rank's slots; -3 marks an expert that another rank
 *                  holds: its pairs are left out of this rank's sum (no error bit)
 *   include_shared 1: the shared expert's term is part of this rank's sum (one rank only)
 *   partial_out    (dev) fp32 [T, H] out: sum over this rank's selected experts of
 *                  p * y_e (+ sigmoid gate * y_shared if include_shared), no residual, not rounded
 * Every rank routes the same tokens and gets the same top-k (topk_idx_out), so the ranks'
 * partials add up to the layer; sum them (e.g. an NCCL all-reduce) and finish with
 * moe_combine_partials.  T <= 8: the fused decode kernel (shapes as moe_stack_forward);
 * T > 8: the prefill path, grouping only this rank's pairs and summing their down products
 * (and the shared expert's) into partial_out in fp32 (shapes as the prefill path:
 * hidden % 128 == 0, E <= 512).  Other shapes: MOE_ERR_UNSUPPORTED.
 */
MOE_API moe_status moe_layer_forward_partial(const moe_shape* shape, const void* x, int32_t T,
                                             const void* w_router, const float* router_bias,
                                             const int32_t* topk_idx_in, const float* topk_w_in,
                                             const uint8_t* pool, const int32_t* slot_table,
                                             int64_t n_slots, const uint8_t* shared_blob,
                                             const void* w_shared_gate, int32_t include_shared,
                                             float* partial_out, int32_t* topk_idx_out, float* topk_w_out,
                                             void* ws, size_t ws_bytes, void* stream);

/*
 * moe_combine_partials -- out = bf16_rne(partials[0] + ... + partials[n_parts-1] + residual),
 * summed in index order: the end of an expert-parallel layer.
 *   partials (host) array of n_parts (1..16) device pointers, each fp32 [T, H] (one pointer
 *            after an all-reduce has summed the ranks' partials in place)
 *   residual (dev) bf16 [T, H] or NULL;  out (dev) bf16 [T, H]
 */
MOE_API moe_status moe_combine_partials(const float* const* partials, int32_t n_parts, int32_t T,
                                        int32_t hidden, const void* residual, void* out, void* stream);

/*
 * moe_layer_forward_static -- moe_layer_forward for callers that cannot allocate device
 * memory.  The Swiftlet pages have no counterpart of this call.
 *
 * Some callers cannot call cudaMalloc: hosts that fix every device allocation up front
 * under a memory budget, code that runs where a new allocation would fail or stall the
 * device, and plain C callers with no device allocator of their own for scratch.  This call
 * takes the same inputs and outputs as moe_layer_forward (the caller still passes x, the
 * weights, the pool, the slot table and out) but no workspace.  Its scratch is one fixed
 * 1 MiB device array inside the library, which every GPU that loads the library holds
 * until the process exits; the call itself allocates nothing.
 *   - Shapes whose scratch need (moe_workspace_size) exceeds 1 MiB are rejected with
 *     MOE_ERR_INVALID and a message; T is limited to 1..8 as on the decode path.
 *   - The first call on each device looks up that device's scratch address (with the
 *     device current) and caches it; make that first call before any stream capture.
 *   - All calls share the one array, which keeps the last call's contents: each call
 *     clears the array's control block (on `stream`, before its kernels) and writes the
 *     rest before reading it.  Calls whose work overlaps on the GPU (other streams, other
 *     threads) race on the array and must not be issued.
 *   - Device-detected errors (bad slot or expert id) are skipped as in moe_layer_forward,
 *     but cannot be read back: the control block is cleared by the next call.
 *   - A device reset (cudaDeviceReset) gives the device a new context; the next call notices
 *     the change and looks the address up again (make that call outside stream capture too).
 *   - The control-block clear may already be enqueued when a later argument check fails;
 *     it touches only the library's own array.
 */
MOE_API moe_status moe_layer_forward_static(const moe_shape* shape, const void* x, int32_t T,
                                            const void* w_router, const float* router_bias,
                                            const int32_t* topk_idx_in, const float* topk_w_in,
                                            const uint8_t* pool, const int32_t* slot_table,
                                            int64_t n_slots, const uint8_t* shared_blob,
                                            const void* w_shared_gate, const void* residual,
                                            void* out, int32_t* topk_idx_out, float* topk_w_out,
                                            void* stream);

/*
 * moe_group_pairs -- stable counting sort of the T*k (token, slot) pairs by expert: the
 * grouping step of the many-token path (each expert then sees its tokens as one matrix;
 * «Swiftlet: 在 Mac 和 iPhone 上執行…», 社群觀點, on prefill).
 *   topk_idx (dev) int32 [T, k]; pair n = t*k + slot refers to topk_idx[n]
 *   order    (dev) int32 [T*k] out: pair numbers sorted by expert, ties in pair order
 *   offsets  (dev) int32 [E+1] out: pairs of expert e are order[offsets[e] .. offsets[e+1])
 *   ws, ws_bytes: workspace of moe_workspace_size(shape, T) bytes
 * Ids outside [0, E) are left out (MOE_DEVERR_BAD_EXPERT); then offsets[E] < T*k.  E <= 512.
 */
MOE_API moe_status moe_group_pairs(const moe_shape* shape, int32_t T, const int32_t* topk_idx, int32_t* order,
                                   int32_t* offsets, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_ws_check -- synchronise `stream`, read and clear the workspace's device error word.
 *   *flags (host) receives the MOE_DEVERR_* bits.  Returns MOE_ERR_DEVICE if any bit was
 *   set, MOE_OK otherwise.
 */
MOE_API moe_status moe_ws_check(void* ws, void* stream, uint32_t* flags);

/*
 * moe_ws_set_slot_wait -- how long the fused decode kernel waits for a slot-table entry that
 * is still pending (a pool in overlap mode marks each miss pending until its blob copy has
 * landed) before it treats the copy as failed: the expert is then skipped like an expert
 * with a bad slot, and MOE_DEVERR_TIMEOUT | MOE_DEVERR_BAD_SLOT are set.
 *   ws            (dev) workspace; the setting lives in its control block
 *   microseconds  the bound; 0 restores the default of 2 seconds
 * Enqueued on `stream` (one tiny kernel).  The setting stays with the workspace until changed
 * (moe_layer_forward_static clears its own control block every call, so it always uses the
 * default).  Failure detection by bounded waits: a copy that never lands ends in an error
 * bit, never in a hung kernel.
 */
MOE_API moe_status moe_ws_set_slot_wait(void* ws, uint32_t microseconds, void* stream);

/*
 * moe_ws_router_logits -- inspection hook: *logits (host) receives the device address, inside
 * ws, of the fp32 router logits [T, E+1] that the many-token router (moe_router_topk or
 * moe_layer_forward with T > 8) last left there: row t holds token t's logits without router
 * bias in columns 0..E-1 (column E is not written).  These are the tensor-core values before
 * the exact recheck; the selection never rests on them alone.  T > 8.
 */
MOE_API moe_status moe_ws_router_logits(const moe_shape* shape, int32_t T, void* ws, size_t ws_bytes,
                                        float** logits);

/* ------------------------------------------------------------------------------------ */
/* Gated DeltaNet decode step: the linear-attention layers that make up three quarters of */
/* the hybrid model's layers, each with a fixed-size recurrent state («Paquets Swiftlet 80B */
/* Qwen dans Mac…», paragraph 6; «Swiftlet: 在 Mac 和 iPhone 上執行…», 技術譜系與正確性). */
/* ------------------------------------------------------------------------------------ */
typedef struct {
  int32_t n_k_heads;  /* H_k: query/key heads                                              */
  int32_t n_v_heads;  /* H_v: value heads (a multiple of H_k; value head h reads key head   */
                      /*      h / (H_v / H_k))                                               */
  int32_t d_k;        /* key/query head width: 64, 128 or 256                                */
  int32_t d_v;        /* value head width                                                    */
} moe_gdn_shape;

/*
 * moe_gdn_decode_step -- one token of B sequences through the gated delta rule, per value
 * head (the pages print no formula; this is the rule that names the layer):
 *   k^ = k / ||k||,  q^ = q / (||q|| sqrt(d_k)),  alpha = exp(g)
 *   S' = alpha S + beta (v - alpha S k^) k^T   (= alpha S (I - beta k^ k^T) + beta v k^T)
 *   out = S' q^
 *   state (dev) fp32 [B, H_v, d_v, d_k], read and overwritten with S'
 *   q, k  (dev) bf16 [B, H_k, d_k];  v (dev) bf16 [B, H_v, d_v]
 *   g     (dev) fp32 [B, H_v] log decay (<= 0 for a decay);  beta (dev) fp32 [B, H_v]
 *   out   (dev) bf16 [B, H_v, d_v] (round to nearest even of the fp32 value)
 * The q/k/v projections, the gate activations and the output gate are the caller's.
 */
MOE_API moe_status moe_gdn_decode_step(const moe_gdn_shape* shape, int32_t B, float* state, const void* q,
                                       const void* k, const void* v, const float* g, const float* beta,
                                       void* out, void* stream);

/*
 * moe_gdn_decode_step_ex -- moe_gdn_decode_step with flags (0: the same call).
 *   MOE_GDN_EARLY_STATE: the step is launched as a programmatic dependent of the kernel
 *   before it on the stream and reads its state rows before that kernel has finished; it
 *   waits for that kernel only before reading q, k, v, g and beta and before writing
 *   anything.  The caller guarantees that the preceding kernel on the stream does not write
 *   this call's state (true of consecutive layers, each with its own state).  Everything
 *   else, ownership and errors as moe_gdn_decode_step.
 */
#define MOE_GDN_EARLY_STATE 1
MOE_API moe_status moe_gdn_decode_step_ex(const moe_gdn_shape* shape, int32_t B, float* state, const void* q,
                                          const void* k, const void* v, const float* g, const float* beta,
                                          void* out, int32_t flags, void* stream);

/* ------------------------------------------------------------------------------------ */
/* Bounded slot pool with LFU + recency eviction («Paquets Swiftlet…» paragraph 5;       */
/* «Swiftlet: 在 Mac 和 iPhone 上執行…», 記憶體管理與權重串流).  Misses are copied from   */
/* pinned host blobs with cudaMemcpyAsync on the pool's own side stream.                 */
/* ------------------------------------------------------------------------------------ */
typedef struct moe_pool moe_pool;

typedef struct {
  int64_t steps;      /* moe_expert_pool_load calls that succeeded                          */
  int64_t lookups;    /* distinct (step, expert) lookups                                    */
  int64_t hits;       /* lookups whose expert was resident                                  */
  int64_t misses;     /* lookups that loaded a blob                                         */
  int64_t evictions;  /* loads that replaced a resident expert                              */
  int64_t h2d_bytes;  /* bytes copied host -> device for misses                             */
} moe_pool_stats_t;

/*
 * moe_pool_create -- a pool of n_slots slots over caller memory.
 *   host_blobs (host, pinned) u8 [E * stride]: expert e's blob at byte e * stride
 *   dev_pool   (dev) u8 [n_slots * stride];  dev_slot_table (dev) int32 [E]
 * The slot table is initialised to -1 (no expert resident); the pool starts empty.
 * *out receives the handle (owned by the caller; free with moe_pool_destroy).
 * Creates one non-blocking side stream and two events.
 */
MOE_API moe_status moe_pool_create(const moe_shape* shape, int32_t n_slots, const uint8_t* host_blobs,
                           uint8_t* dev_pool, int32_t* dev_slot_table, moe_pool** out);

/*
 * moe_pool_create_file -- a pool whose misses are read from a file instead of host memory:
 * the storage tier of the pages, where a missed expert is one read of its fixed-stride blob
 * from the SSD, without mmap and without filling the page cache («Paquets Swiftlet…»,
 * paragraph 5; «Swiftlet: 在 Mac 和 iPhone 上執行…», 記憶體管理與權重串流).
 *   path   (host) a file holding E blobs back to back: expert e at byte e * stride
 *   flags  MOE_POOL_FILE_DIRECT: open with O_DIRECT (reads bypass the page cache; used when
 *          the stride is a multiple of 4096 and the file system accepts it, else buffered
 *          reads whose pages are released after each read)
 *   dev_pool, dev_slot_table, out: as for moe_pool_create.
 * Every moe_expert_pool_load then reads its misses with one pread per blob, up to 8 at once
 * on as many threads, into the pool's 8 pinned staging buffers, and copies each to its slot
 * on the side stream (in overlap mode each miss's slot-table entry is settled after its
 * copy, as for host blobs).  A blob that cannot be read leaves its slot empty and the load
 * returns MOE_ERR_IO; the table stays consistent.  MOE_ERR_IO also if the file cannot be
 * opened or is too short.  The file descriptor and buffers are released by moe_pool_destroy.
 */
#define MOE_POOL_FILE_DIRECT 0x1
MOE_API moe_status moe_pool_create_file(const moe_shape* shape, int32_t n_slots, const char* path, int32_t flags,
                                        uint8_t* dev_pool, int32_t* dev_slot_table, moe_pool** out);

/*
 * moe_expert_pool_load -- make every expert named in topk_idx (dev int32 [T, k], T >= 1)
 * resident.  A step with more than 8 tokens grows the pool's pinned id read-back buffer once
 * (one pinned host allocation).
 * SYNCHRONISES `stream` (the ids are needed on the host): copies the ids back, looks them
 * up (distinct ids in first-appearance order; hits refresh use count and last use), loads
 * each miss into the lowest empty slot, else evicts the slot with the smallest
 * (use count, last use step, slot index) among slots this step does not need, copies the
 * missed blobs and the updated slot table on the side stream, and makes `stream` wait for
 * them.  MOE_ERR_CAPACITY (nothing changed) if a step needs more distinct experts than
 * slots; MOE_ERR_INVALID for an id outside [0, E).  If a copy fails the slot is left
 * empty, the table stays consistent, and MOE_ERR_CUDA is returned.
 */
MOE_API moe_status moe_expert_pool_load(moe_pool* pool, const int32_t* topk_idx, int32_t T, void* stream);

/*
 * moe_pool_set_policy -- eviction policy of the next loads (for the eviction ablation):
 *   MOE_POOL_LFU_RECENCY (the pages' policy, the default): smallest (use count, last use, slot)
 *   MOE_POOL_LRU: smallest (last use, slot);  MOE_POOL_LFU: smallest (use count, slot)
 * among the slots whose expert the step does not need.  Host-side only; MOE_ERR_INVALID
 * for another value.
 */
enum { MOE_POOL_LFU_RECENCY = 0, MOE_POOL_LRU = 1, MOE_POOL_LFU = 2 };
MOE_API moe_status moe_pool_set_policy(moe_pool* pool, int32_t policy);

/*
 * moe_pool_set_overlap -- overlap mode of the next loads (0: off, the default).  Off, the
 * caller's stream waits until the step's misses have landed, then the layer forward runs.
 * On, moe_expert_pool_load uploads the slot table with every miss of the step marked
 * pending (-2), the caller's stream waits for that upload only, and each miss's blob copy is
 * followed on the side stream by a copy of its slot over the pending entry: the fused decode
 * kernel (moe_layer_forward / moe_stack_forward with T <= 8) starts at once, computes with the
 * resident experts and waits, per expert, for a pending entry to settle before it streams
 * that blob (the NEXT item of the Swiftlet pages' streaming design: compute on hits while the
 * misses are in flight).  Results are bit-identical to overlap off.  While overlap is on, the
 * slot table may hold -2 entries between a load and the end of the forward that follows it:
 * run that forward before the next load, and only the fused decode path may read the table.
 * MOE_ERR_UNSUPPORTED for shapes without a fused decode kernel.  Host-side only.
 */
MOE_API moe_status moe_pool_set_overlap(moe_pool* pool, int32_t on);

/* moe_pool_stats -- counters since creation (host struct). */
MOE_API moe_status moe_pool_stats(const moe_pool* pool, moe_pool_stats_t* stats);

/*
 * moe_pool_slot_table -- copy of the host mirror of the slot table (host int32 [E]) and of
 * the slot -> expert map (host int32 [n_slots]; either pointer may be NULL).
 */
MOE_API moe_status moe_pool_slot_table(const moe_pool* pool, int32_t* slot_of_expert, int32_t* expert_in_slot);

/*
 * moe_pool_inject_copy_failure -- test hook: the n-th blob copy from now (0 = the next one)
 * reports failure without being issued; -1 disarms.  Host-side only.
 */
MOE_API moe_status moe_pool_inject_copy_failure(moe_pool* pool, int64_t nth);

/* moe_pool_destroy -- waits for the side stream, releases the handle. NULL is a no-op. */
MOE_API void moe_pool_destroy(moe_pool* pool);

/*
 * moe_profile_events -- measurement hook.  While set (events != NULL), each
 * moe_layer_forward / moe_router_topk call on this thread records events[2*i] on its stream
 * just before its i-th kernel launch and events[2*i+1] just after it, for i < n
 * (decode, unfused: 0 router or grouping, 1 gate/up + SwiGLU, 2 down + combine; decode,
 * fused: 0 the persistent kernel; many tokens: 0 norms + router GEMM + certified top-k,
 * 1 grouping, 2 gate/up GEMM, 3 down GEMM, 4 final sum).  events are cudaEvent_t handles
 * owned by the caller.  Thread-local; NULL disables.
 */
MOE_API moe_status moe_profile_events(void* const* events, int32_t n);

/* Message of the calling thread's last failed call ("" if none). */
MOE_API const char* moe_last_error(void);

/* Library version string. */
MOE_API const char* moe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
