// Bounded expert slot pool with LFU + recency eviction (host side).
//
// The Swiftlet pages describe a bounded pool of slots that caches the popular routed
// experts, evicting with LFU combined with recency, and a fixed-stride container so that
// fetching one expert is a single read («Paquets Swiftlet 80B Qwen dans Mac…», paragraph
// 5; «Swiftlet: 在 Mac 和 iPhone 上執行 80B 與 35B Qwen 模型», section 記憶體管理與權重串流).
// Here the backing store is pinned host memory and a fetch is one cudaMemcpyAsync of one
// blob on the pool's side stream.
//
// Policy (the pages give only "LFU + recency"; this is the plain reading; LRU and pure LFU
// can be selected for the eviction ablation):
//   per slot: resident expert, use count (1 when loaded, +1 for every later step that uses
//   it), last-use step.  A step's distinct experts are looked up in first-appearance order;
//   hits refresh count and last use.  Misses are then loaded in the same order into the
//   lowest-numbered empty slot, else into the slot with the smallest
//   (count, last use, slot index) among slots whose expert the step does not need.
#include "../../include/moe.h"
#include "common.cuh"

#include <cuda.h>
#include <cuda_runtime.h>

#include <fcntl.h>
#include <sys/stat.h>
#include <unistd.h>

#include <cerrno>
#include <cstring>
#include <new>
#include <thread>
#include <vector>

namespace moe {
moe_status set_error(moe_status s, const char* fmt, ...);
moe_status cuda_fail(cudaError_t e, const char* what);
moe_status check_shape(const moe_shape* s);
}  // namespace moe

using namespace moe;

namespace {
// cuStreamWriteValue32 through the runtime's driver entry point (the library does not link
// libcuda): a 4-byte write done by the stream itself once its earlier work has finished,
// far cheaper than a 4-byte host-to-device copy.  Null if the driver does not offer it.
using WriteValue32Fn = CUresult (*)(CUstream, CUdeviceptr, cuuint32_t, unsigned int);
WriteValue32Fn write_value32_fn() {
  static WriteValue32Fn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuStreamWriteValue32", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (WriteValue32Fn) nullptr;
    return reinterpret_cast<WriteValue32Fn>(p);
  }();
  return fn;
}
}  // namespace

struct moe_pool {
  moe_shape shape;
  int32_t n_slots = 0;
  int64_t stride = 0;
  const uint8_t* host_blobs = nullptr;
  uint8_t* dev_pool = nullptr;
  int32_t* dev_slot_table = nullptr;
  std::vector<int32_t> slot_of;    // [E] slot of expert, -1 if not resident
  std::vector<int32_t> expert_in;  // [S] expert in slot, -1 if empty
  std::vector<int64_t> count;      // [S]
  std::vector<int64_t> last_use;   // [S]
  std::vector<uint8_t> needed;     // [E] scratch: expert needed by the current step
  int64_t step_no = 0;
  moe_pool_stats_t stats{};
  int32_t policy = MOE_POOL_LFU_RECENCY;
  bool overlap = false;            // forward may start before the misses have landed
  int64_t fail_at = -1;            // test hook: copies until an injected failure
  cudaStream_t side = nullptr;
  cudaEvent_t ready = nullptr;     // slot table + blobs of the last step are on the device
  bool ready_recorded = false;
  int32_t* h_ids = nullptr;        // pinned [h_ids_cap]: the step's ids read back
  int32_t h_ids_cap = 0;
  int32_t* h_table = nullptr;      // pinned [E]
  int32_t* h_final = nullptr;      // pinned [E]: the slot an overlap-mode miss resolves to
  // storage tier (moe_pool_create_file): misses are read from a file of fixed-stride blobs
  int fd = -1;
  bool direct = false;             // opened with O_DIRECT (no page cache)
  std::vector<uint8_t*> stage;     // pinned staging buffers, one blob each
  std::vector<cudaEvent_t> stage_ev;  // the copy out of each staging buffer has finished
  std::vector<bool> stage_busy;
};

namespace {
constexpr int kStageBufs = 8;  // blobs read from the file at once (one thread each)

struct Load {
  int32_t id, slot;
};

// Reads blob `id` (stride bytes at id * stride) into `dst`; false on an error or a short read.
bool read_blob(const moe_pool* p, int32_t id, uint8_t* dst) {
  int64_t done = 0;
  const int64_t off = (int64_t)id * p->stride;
  while (done < p->stride) {
    const ssize_t r = pread(p->fd, dst + done, (size_t)(p->stride - done), off + done);
    if (r < 0 && errno == EINTR) continue;
    if (r <= 0) return false;
    done += r;
  }
  // the blob is in the staging buffer now: do not let it take page-cache room from others
  if (!p->direct) posix_fadvise(p->fd, off, p->stride, POSIX_FADV_DONTNEED);
  return true;
}

// Overlap mode: the side stream writes the final slot of a miss over its pending entry once
// the blob copy before it has finished.
cudaError_t settle_entry(moe_pool* p, int32_t id) {
  const WriteValue32Fn wv = write_value32_fn();
  if (wv && wv(p->side, (CUdeviceptr)(p->dev_slot_table + id), (cuuint32_t)p->h_final[id], 0) == CUDA_SUCCESS)
    return cudaSuccess;
  return cudaMemcpyAsync(p->dev_slot_table + id, p->h_final + id, sizeof(int32_t), cudaMemcpyHostToDevice, p->side);
}

// The misses of a file-backed pool: in waves of kStageBufs, every blob of the wave is read
// by its own thread into a staging buffer (after the previous copy out of that buffer has
// finished), then copied to its slot on the side stream.  A blob that cannot be read leaves
// its slot empty (host state rolled back; ok[i] = 0).  With `settle` each miss's pending
// slot-table entry is written after its copy (or -1 for a failed read).  Returns the first
// CUDA error of a copy (the loads from that one on rolled back); reads do not raise one.
cudaError_t file_loads(moe_pool* p, const std::vector<Load>& loads, std::vector<char>& ok, bool settle) {
  ok.assign(loads.size(), 1);
  // On a CUDA error at load i0, the loads from i0 on keep no host state: their slots are left
  // empty and they stay non-resident, so that no later step counts them as hits on slots that
  // hold other weights (the next load uploads the whole table from the host mirror).
  const auto fail_from = [&](size_t i0, cudaError_t e) {
    for (size_t j = i0; j < loads.size(); ++j) {
      const Load& lr = loads[j];
      if (p->slot_of[lr.id] == lr.slot) {
        p->slot_of[lr.id] = -1;
        p->expert_in[lr.slot] = -1;
        p->stats.h2d_bytes -= p->stride;
      }
      p->h_final[lr.id] = -1;
      ok[j] = 0;
    }
    return e;
  };
  for (size_t w0 = 0; w0 < loads.size(); w0 += kStageBufs) {
    const size_t w1 = std::min(loads.size(), w0 + (size_t)kStageBufs);
    for (size_t i = w0; i < w1; ++i) {
      const int b = (int)(i - w0);
      if (p->stage_busy[b]) {
        cudaError_t e = cudaEventSynchronize(p->stage_ev[b]);
        if (e != cudaSuccess) return fail_from(w0, e);
        p->stage_busy[b] = false;
      }
    }
    std::vector<std::thread> readers;
    readers.reserve(w1 - w0);
    for (size_t i = w0; i < w1; ++i)
      readers.emplace_back([p, &loads, &ok, i, w0] { ok[i] = read_blob(p, loads[i].id, p->stage[i - w0]) ? 1 : 0; });
    for (auto& t : readers) t.join();
    for (size_t i = w0; i < w1; ++i) {
      const Load& ld = loads[i];
      const int b = (int)(i - w0);
      if (ok[i]) {
        cudaError_t e = cudaMemcpyAsync(p->dev_pool + (int64_t)ld.slot * p->stride, p->stage[b], (size_t)p->stride,
                                        cudaMemcpyHostToDevice, p->side);
        if (e == cudaSuccess) e = cudaEventRecord(p->stage_ev[b], p->side);
        if (e != cudaSuccess) return fail_from(i, e);
        p->stage_busy[b] = true;
      } else {
        p->slot_of[ld.id] = -1;
        p->expert_in[ld.slot] = -1;
        p->stats.h2d_bytes -= p->stride;
        p->h_final[ld.id] = -1;
      }
      if (settle) {
        cudaError_t e = settle_entry(p, ld.id);
        if (e != cudaSuccess) return fail_from(i, e);
      }
    }
  }
  return cudaSuccess;
}
}  // namespace

namespace {
moe_status pool_init(moe_pool* p, const moe_shape* shape, int32_t n_slots, const uint8_t* host_blobs,
                     uint8_t* dev_pool, int32_t* dev_slot_table);
}  // namespace

extern "C" {

moe_status moe_pool_create(const moe_shape* shape, int32_t n_slots, const uint8_t* host_blobs, uint8_t* dev_pool,
                           int32_t* dev_slot_table, moe_pool** out) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!out) return set_error(MOE_ERR_INVALID, "out is NULL");
  *out = nullptr;
  if (n_slots < 1) return set_error(MOE_ERR_INVALID, "n_slots must be >= 1");
  if (!host_blobs || !dev_pool || !dev_slot_table)
    return set_error(MOE_ERR_INVALID, "host_blobs, dev_pool and dev_slot_table must be non-NULL");
  if (((uintptr_t)dev_pool & 255) || ((uintptr_t)host_blobs & 15))
    return set_error(MOE_ERR_INVALID, "dev_pool must be 256-byte and host_blobs 16-byte aligned");
  cudaPointerAttributes attr{};
  if (cudaPointerGetAttributes(&attr, host_blobs) != cudaSuccess || attr.type != cudaMemoryTypeHost) {
    cudaGetLastError();
    return set_error(MOE_ERR_INVALID, "host_blobs must be pinned host memory (cudaHostAlloc / pin_memory)");
  }
  moe_pool* p = new (std::nothrow) moe_pool();
  if (!p) return set_error(MOE_ERR_INVALID, "out of host memory");
  st = pool_init(p, shape, n_slots, host_blobs, dev_pool, dev_slot_table);
  if (st != MOE_OK) return st;
  *out = p;
  return MOE_OK;
}

}  // extern "C"

namespace {
// The bookkeeping, side stream, events and pinned buffers every pool has; on failure the
// pool is destroyed.
moe_status pool_init(moe_pool* p, const moe_shape* shape, int32_t n_slots, const uint8_t* host_blobs,
                     uint8_t* dev_pool, int32_t* dev_slot_table) {
  p->shape = *shape;
  p->n_slots = n_slots;
  p->stride = make_blob_layout(shape->hidden, shape->inter, shape->bits).stride;
  p->host_blobs = host_blobs;
  p->dev_pool = dev_pool;
  p->dev_slot_table = dev_slot_table;
  const int E = shape->n_experts;
  p->slot_of.assign(E, -1);
  p->expert_in.assign(n_slots, -1);
  p->count.assign(n_slots, 0);
  p->last_use.assign(n_slots, -1);
  p->needed.assign(E, 0);
  cudaError_t e;
  if ((e = cudaStreamCreateWithFlags(&p->side, cudaStreamNonBlocking)) != cudaSuccess ||
      (e = cudaEventCreateWithFlags(&p->ready, cudaEventDisableTiming)) != cudaSuccess ||
      (e = cudaHostAlloc((void**)&p->h_ids, sizeof(int32_t) * kMaxDecodeT * kMaxTopK, cudaHostAllocDefault)) !=
          cudaSuccess ||
      (e = cudaHostAlloc((void**)&p->h_table, sizeof(int32_t) * E, cudaHostAllocDefault)) != cudaSuccess ||
      (e = cudaHostAlloc((void**)&p->h_final, sizeof(int32_t) * E, cudaHostAllocDefault)) != cudaSuccess) {
    moe_pool_destroy(p);
    return cuda_fail(e, "pool create");
  }
  p->h_ids_cap = kMaxDecodeT * kMaxTopK;
  for (int i = 0; i < E; ++i) p->h_table[i] = -1;
  e = cudaMemcpyAsync(dev_slot_table, p->h_table, sizeof(int32_t) * E, cudaMemcpyHostToDevice, p->side);
  if (e == cudaSuccess) e = cudaEventRecord(p->ready, p->side);
  if (e == cudaSuccess) e = cudaStreamSynchronize(p->side);
  if (e != cudaSuccess) {
    moe_pool_destroy(p);
    return cuda_fail(e, "pool slot table init");
  }
  p->ready_recorded = true;
  return MOE_OK;
}
}  // namespace

extern "C" {

moe_status moe_pool_create_file(const moe_shape* shape, int32_t n_slots, const char* path, int32_t flags,
                                uint8_t* dev_pool, int32_t* dev_slot_table, moe_pool** out) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!out) return set_error(MOE_ERR_INVALID, "out is NULL");
  *out = nullptr;
  if (!path) return set_error(MOE_ERR_INVALID, "path is NULL");
  if (flags & ~MOE_POOL_FILE_DIRECT) return set_error(MOE_ERR_INVALID, "unknown flags 0x%x", flags);
  if (n_slots < 1) return set_error(MOE_ERR_INVALID, "n_slots must be >= 1");
  if (!dev_pool || !dev_slot_table) return set_error(MOE_ERR_INVALID, "dev_pool and dev_slot_table must be non-NULL");
  if ((uintptr_t)dev_pool & 255) return set_error(MOE_ERR_INVALID, "dev_pool must be 256-byte aligned");
  const int64_t stride = make_blob_layout(shape->hidden, shape->inter, shape->bits).stride;
  // O_DIRECT needs block-aligned offsets and lengths: blob offsets are multiples of the stride
  bool direct = (flags & MOE_POOL_FILE_DIRECT) && stride % 4096 == 0;
  int fd = open(path, O_RDONLY | O_CLOEXEC | (direct ? O_DIRECT : 0));
  if (fd < 0 && direct) {  // a file system without O_DIRECT: buffered reads, page cache released
    direct = false;
    fd = open(path, O_RDONLY | O_CLOEXEC);
  }
  if (fd < 0) return set_error(MOE_ERR_IO, "cannot open %s: %s", path, strerror(errno));
  struct stat sb {};
  if (fstat(fd, &sb) != 0 || (int64_t)sb.st_size < stride * shape->n_experts) {
    close(fd);
    return set_error(MOE_ERR_IO, "%s holds %lld bytes, fewer than %d blobs of %lld", path, (long long)sb.st_size,
                     shape->n_experts, (long long)stride);
  }
  // the pool itself, without a host copy of the blobs
  moe_pool* p = new (std::nothrow) moe_pool();
  if (!p) {
    close(fd);
    return set_error(MOE_ERR_INVALID, "out of host memory");
  }
  p->fd = fd;
  p->direct = direct;
  const moe_status s2 = pool_init(p, shape, n_slots, nullptr, dev_pool, dev_slot_table);
  if (s2 != MOE_OK) return s2;  // pool_init released p (and closed fd)
  cudaError_t e = cudaSuccess;
  p->stage.assign(kStageBufs, nullptr);
  p->stage_ev.assign(kStageBufs, nullptr);
  p->stage_busy.assign(kStageBufs, false);
  for (int b = 0; b < kStageBufs && e == cudaSuccess; ++b) {
    e = cudaHostAlloc((void**)&p->stage[b], (size_t)stride, cudaHostAllocDefault);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->stage_ev[b], cudaEventDisableTiming);
  }
  if (e != cudaSuccess) {
    moe_pool_destroy(p);
    return cuda_fail(e, "staging buffers");
  }
  *out = p;
  return MOE_OK;
}

moe_status moe_expert_pool_load(moe_pool* p, const int32_t* topk_idx, int32_t T, void* stream) {
  if (!p || !topk_idx) return set_error(MOE_ERR_INVALID, "pool and topk_idx must be non-NULL");
  const int k = p->shape.top_k, E = p->shape.n_experts;
  if (T < 1) return set_error(MOE_ERR_INVALID, "T must be >= 1 (got %d)", T);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int n = T * k;
  if (n > p->h_ids_cap) {
    // a larger step than any before: grow the pinned read-back buffer (decode-sized steps
    // never reach this; the first many-token step pays one pinned allocation)
    int32_t* grown = nullptr;
    cudaError_t ea = cudaHostAlloc((void**)&grown, sizeof(int32_t) * (size_t)n, cudaHostAllocDefault);
    if (ea != cudaSuccess) return cuda_fail(ea, "pinned id buffer");
    cudaFreeHost(p->h_ids);
    p->h_ids = grown;
    p->h_ids_cap = n;
  }
  // The ids are needed on the host.  Synchronising the caller stream also guarantees that
  // every earlier forward on it has finished reading the slots this step may overwrite.
  cudaError_t e = cudaMemcpyAsync(p->h_ids, topk_idx, sizeof(int32_t) * n, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "top-k read-back");
  // The previous step's table upload reads h_table (and, in overlap mode, its per-miss entry
  // copies read h_final): let them finish before editing either.
  if (p->ready_recorded && (e = cudaEventSynchronize(p->ready)) != cudaSuccess) return cuda_fail(e, "pool event");
  if (p->overlap && (e = cudaStreamSynchronize(p->side)) != cudaSuccess) return cuda_fail(e, "pool side stream");
  // distinct ids in first-appearance order
  std::vector<int32_t> uniq;
  uniq.reserve(n);
  for (int i = 0; i < n; ++i) {
    const int32_t id = p->h_ids[i];
    if (id < 0 || id >= E) {
      for (int32_t u : uniq) p->needed[u] = 0;
      return set_error(MOE_ERR_INVALID, "expert id %d outside [0, %d)", id, E);
    }
    if (!p->needed[id]) {
      p->needed[id] = 1;
      uniq.push_back(id);
    }
  }
  if ((int)uniq.size() > p->n_slots) {
    for (int32_t u : uniq) p->needed[u] = 0;
    return set_error(MOE_ERR_CAPACITY, "step needs %zu distinct experts, pool has %d slots", uniq.size(),
                     p->n_slots);
  }
  const int64_t now = p->step_no;
  moe_status result = MOE_OK;
  std::vector<Load> loads;  // overlap mode: the misses, copied after the table upload
  for (int32_t id : uniq) {
    p->stats.lookups++;
    const int32_t sl = p->slot_of[id];
    if (sl >= 0) {
      p->stats.hits++;
      p->count[sl]++;
      p->last_use[sl] = now;
    }
  }
  for (int32_t id : uniq) {
    if (p->slot_of[id] >= 0) continue;
    p->stats.misses++;
    int32_t victim = -1;
    for (int32_t sl = 0; sl < p->n_slots; ++sl)
      if (p->expert_in[sl] < 0) {
        victim = sl;
        break;
      }
    bool evicting = false;
    if (victim < 0) {
      for (int32_t sl = 0; sl < p->n_slots; ++sl) {
        if (p->needed[p->expert_in[sl]]) continue;
        bool better;
        if (victim < 0) {
          better = true;
        } else if (p->policy == MOE_POOL_LRU) {
          better = p->last_use[sl] < p->last_use[victim];
        } else if (p->policy == MOE_POOL_LFU) {
          better = p->count[sl] < p->count[victim];
        } else {
          better = p->count[sl] < p->count[victim] ||
                   (p->count[sl] == p->count[victim] && p->last_use[sl] < p->last_use[victim]);
        }
        if (better) victim = sl;  // ascending scan keeps the lowest slot index on full ties
      }
      evicting = true;
    }
    if (evicting) {
      p->slot_of[p->expert_in[victim]] = -1;
      p->expert_in[victim] = -1;
      p->stats.evictions++;
    }
    bool failed = false;
    if (p->fail_at == 0) {
      failed = true;
      p->fail_at = -1;
    } else {
      if (p->fail_at > 0) p->fail_at--;
      if (p->overlap || p->fd >= 0) {
        loads.push_back({id, victim});  // copied below (overlap: after the table upload)
      } else {
        e = cudaMemcpyAsync(p->dev_pool + (int64_t)victim * p->stride, p->host_blobs + (int64_t)id * p->stride,
                            (size_t)p->stride, cudaMemcpyHostToDevice, p->side);
        failed = (e != cudaSuccess);
      }
    }
    if (failed) {
      // slot stays empty; the expert stays non-resident
      result = (e != cudaSuccess) ? cuda_fail(e, "blob copy") : set_error(MOE_ERR_CUDA, "blob copy failed (injected)");
      e = cudaSuccess;
      continue;
    }
    p->expert_in[victim] = id;
    p->slot_of[id] = victim;
    p->count[victim] = 1;
    p->last_use[victim] = now;
    p->stats.h2d_bytes += p->stride;
  }
  for (int32_t u : uniq) p->needed[u] = 0;
  if (p->fd >= 0 && !p->overlap) {
    // storage tier: the misses' blobs are read from the file (in waves of kStageBufs
    // parallel preads into pinned staging buffers) and copied to their slots; a failed read
    // leaves its slot empty before the table goes up
    std::vector<char> ok;
    e = file_loads(p, loads, ok, false);
    if (e != cudaSuccess) return cuda_fail(e, "blob copy from staging");
    for (size_t i = 0; i < loads.size(); ++i)
      if (!ok[i]) result = set_error(MOE_ERR_IO, "reading expert %d from the backing file failed", loads[i].id);
  }
  for (int i = 0; i < E; ++i) p->h_table[i] = p->slot_of[i];
  if (!p->overlap) {
    e = cudaMemcpyAsync(p->dev_slot_table, p->h_table, sizeof(int32_t) * E, cudaMemcpyHostToDevice, p->side);
    if (e == cudaSuccess) e = cudaEventRecord(p->ready, p->side);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, p->ready, 0);
    if (e != cudaSuccess) return cuda_fail(e, "slot table upload");
    p->ready_recorded = true;
    p->step_no++;
    if (result == MOE_OK) p->stats.steps++;
    return result;
  }
  // Overlap mode: the table goes up first with this step's misses marked pending, and the
  // caller's stream waits for that upload only.  Each miss's blob copy is then followed on
  // the side stream by a 4-byte copy of its slot over the pending entry; the fused decode
  // kernel waits for that entry before it streams the expert.
  for (const Load& ld : loads) {
    p->h_table[ld.id] = kSlotPending;
    p->h_final[ld.id] = ld.slot;
  }
  e = cudaMemcpyAsync(p->dev_slot_table, p->h_table, sizeof(int32_t) * E, cudaMemcpyHostToDevice, p->side);
  if (e == cudaSuccess) e = cudaEventRecord(p->ready, p->side);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, p->ready, 0);
  if (e != cudaSuccess) return cuda_fail(e, "slot table upload");
  p->ready_recorded = true;
  if (p->fd >= 0) {
    std::vector<char> ok;
    e = file_loads(p, loads, ok, true);
    if (e != cudaSuccess) return cuda_fail(e, "blob copy from staging");
    for (size_t i = 0; i < loads.size(); ++i)
      if (!ok[i]) result = set_error(MOE_ERR_IO, "reading expert %d from the backing file failed", loads[i].id);
    loads.clear();
  }
  for (size_t li = 0; li < loads.size(); ++li) {
    const Load& ld = loads[li];
    e = cudaMemcpyAsync(p->dev_pool + (int64_t)ld.slot * p->stride, p->host_blobs + (int64_t)ld.id * p->stride,
                        (size_t)p->stride, cudaMemcpyHostToDevice, p->side);
    if (e != cudaSuccess) {
      // the entry must still be settled, or the kernel would wait for it: not resident
      result = cuda_fail(e, "blob copy");
      p->h_final[ld.id] = -1;
      p->slot_of[ld.id] = -1;
      p->expert_in[ld.slot] = -1;
      p->stats.h2d_bytes -= p->stride;
    }
    const WriteValue32Fn wv = write_value32_fn();
    if (!wv || wv(p->side, (CUdeviceptr)(p->dev_slot_table + ld.id), (cuuint32_t)p->h_final[ld.id], 0) !=
                   CUDA_SUCCESS) {
      e = cudaMemcpyAsync(p->dev_slot_table + ld.id, p->h_final + ld.id, sizeof(int32_t), cudaMemcpyHostToDevice,
                          p->side);
      if (e != cudaSuccess) {
        // This entry and those of the loads not yet issued stay pending on the device.  Undo
        // them on the host, so that no later step counts them as hits on slots that hold
        // other weights; the next load uploads the whole table again from the host mirror.
        // The forward of this step must not run (its kernel would wait for the entries).
        for (size_t lj = li; lj < loads.size(); ++lj) {
          const Load& lr = loads[lj];
          if (p->slot_of[lr.id] == lr.slot) {
            p->slot_of[lr.id] = -1;
            p->expert_in[lr.slot] = -1;
            p->stats.h2d_bytes -= p->stride;
          }
          p->h_final[lr.id] = -1;
        }
        p->step_no++;
        return cuda_fail(e, "slot table entry");
      }
    }
  }
  p->step_no++;
  if (result == MOE_OK) p->stats.steps++;
  return result;
}

moe_status moe_pool_stats(const moe_pool* p, moe_pool_stats_t* stats) {
  if (!p || !stats) return set_error(MOE_ERR_INVALID, "pool and stats must be non-NULL");
  *stats = p->stats;
  return MOE_OK;
}

moe_status moe_pool_slot_table(const moe_pool* p, int32_t* slot_of_expert, int32_t* expert_in_slot) {
  if (!p) return set_error(MOE_ERR_INVALID, "pool is NULL");
  if (slot_of_expert) memcpy(slot_of_expert, p->slot_of.data(), sizeof(int32_t) * p->slot_of.size());
  if (expert_in_slot) memcpy(expert_in_slot, p->expert_in.data(), sizeof(int32_t) * p->expert_in.size());
  return MOE_OK;
}

moe_status moe_pool_set_policy(moe_pool* p, int32_t policy) {
  if (!p) return set_error(MOE_ERR_INVALID, "pool is NULL");
  if (policy != MOE_POOL_LFU_RECENCY && policy != MOE_POOL_LRU && policy != MOE_POOL_LFU)
    return set_error(MOE_ERR_INVALID, "unknown pool policy %d", policy);
  p->policy = policy;
  return MOE_OK;
}

moe_status moe_pool_set_overlap(moe_pool* p, int32_t on) {
  if (!p) return set_error(MOE_ERR_INVALID, "pool is NULL");
  if (on && !fused_shape_supported(p->shape.hidden, p->shape.inter, p->shape.bits, p->shape.n_experts))
    return set_error(MOE_ERR_UNSUPPORTED, "overlap mode needs a shape of the fused decode kernel");
  p->overlap = on != 0;
  return MOE_OK;
}

moe_status moe_pool_inject_copy_failure(moe_pool* p, int64_t nth) {
  if (!p) return set_error(MOE_ERR_INVALID, "pool is NULL");
  p->fail_at = nth < 0 ? -1 : nth;
  return MOE_OK;
}

void moe_pool_destroy(moe_pool* p) {
  if (!p) return;
  if (p->side) {
    cudaStreamSynchronize(p->side);
    cudaStreamDestroy(p->side);
  }
  if (p->ready) cudaEventDestroy(p->ready);
  if (p->h_ids) cudaFreeHost(p->h_ids);
  if (p->h_table) cudaFreeHost(p->h_table);
  if (p->h_final) cudaFreeHost(p->h_final);
  for (size_t i = 0; i < p->stage_ev.size(); ++i)
    if (p->stage_ev[i]) cudaEventDestroy(p->stage_ev[i]);
  for (size_t i = 0; i < p->stage.size(); ++i)
    if (p->stage[i]) cudaFreeHost(p->stage[i]);
  if (p->fd >= 0) close(p->fd);
  delete p;
}

}  // extern "C"
