// C ABI of the Muon step (declared in include/muon_ns.h).
//
// Host responsibilities only: argument validation, the plan (cached per
// shape table), the workspace, tensor maps for the bulk-tensor loads, the
// device copies of the per-call pointer tables (cached by content), and the
// ordered enqueue of the kernels on the caller's stream. All arithmetic of
// the step runs in the kernels of elementwise.cu, ns_tcgen05.cu and
// ns_fp32.cu.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <list>
#include <memory>
#include <string>
#include <vector>

#include "../../include/muon_ns.h"
#include "common.cuh"
#include "kernels.h"
#include "plan.h"

using namespace muon;

namespace {

thread_local std::string g_last_error;

int fail(int code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

#define MUON_CUDA_TRY(expr)                                                                 \
  do {                                                                                      \
    cudaError_t _e = (expr);                                                                \
    if (_e != cudaSuccess)                                                                  \
      return fail(_e == cudaErrorMemoryAllocation ? MUON_ERR_OOM : MUON_ERR_CUDA,           \
                  std::string(#expr) + ": " + cudaGetErrorString(_e));                     \
  } while (0)

// Restores the caller's current device on scope exit.
struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    ok = cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

// Builds the bytes of a table on a cache miss.
typedef int (*BlobBuilder)(const void* ctx, std::vector<unsigned char>& out);

// Device copies of the per-call pointer tables (matrix bindings, tensor maps
// of caller buffers), in a fixed ring of slots made once per plan.
//
// A call whose table bytes match a slot reuses it (nothing is uploaded). A
// call with new bytes takes the least recently used slot: it writes the bytes
// into that slot's pinned host staging (after that staging's previous upload
// has executed), makes the stream wait for the last work that read the slot
// (an event, so no host synchronisation), and uploads with one
// cudaMemcpyAsync on the call's stream. After a call's kernels are enqueued,
// every slot it used records a "used" event on the stream.
// Slots used while a stream is being captured are pinned: a graph keeps
// pointing at them, so they are never overwritten until the plan changes.
// A miss during capture is an error (the upload and the waits cannot be
// captured): run the call once uncaptured with the same pointers first.
class TableRing {
 public:
  ~TableRing() { release(); }

  // Frees everything (callers make sure no queued work uses the slots).
  void release() {
    for (Slot& s : slots_) {
      if (s.dev) cudaFree(s.dev);
      if (s.host) cudaFreeHost(s.host);
      if (s.copied) cudaEventDestroy(s.copied);
      if (s.used) cudaEventDestroy(s.used);
    }
    slots_.clear();
    cap_ = 0;
    tick_ = 0;
    in_call_.clear();
  }

  // Makes kSlots slots of at least `bytes` each (outside any capture).
  int reserve(size_t bytes) {
    bytes = std::max<size_t>(bytes, 256);
    if (!slots_.empty() && cap_ >= bytes) return MUON_OK;
    if (!slots_.empty()) {
      for (const Slot& s : slots_)
        if (s.pinned)
          return fail(MUON_ERR_INVALID_ARG, "pointer tables grew while a captured graph holds the old ones");
      // Growing: queued work may still read the old slots.
      cudaError_t e = cudaDeviceSynchronize();
      if (e != cudaSuccess) return fail(MUON_ERR_CUDA, std::string("table ring: ") + cudaGetErrorString(e));
      release();
    }
    slots_.resize(kSlots);
    for (Slot& s : slots_) {
      cudaError_t e = cudaMalloc(&s.dev, bytes);
      if (e == cudaSuccess) e = cudaHostAlloc(&s.host, bytes, cudaHostAllocDefault);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.copied, cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.used, cudaEventDisableTiming);
      if (e != cudaSuccess) {
        cudaGetLastError();
        release();
        return fail(e == cudaErrorMemoryAllocation ? MUON_ERR_OOM : MUON_ERR_CUDA,
                    std::string("table ring allocation: ") + cudaGetErrorString(e));
      }
    }
    cap_ = bytes;
    return MUON_OK;
  }

  // Device table for `key`; on a miss its bytes come from build(ctx) (or are
  // the key itself when build is NULL). Stream-ordered on `st`.
  int get(const void* key, size_t nkey, BlobBuilder build, const void* ctx, cudaStream_t st, void** out) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(st, &cs);
    if (e != cudaSuccess) return fail(MUON_ERR_CUDA, std::string("cudaStreamIsCapturing: ") + cudaGetErrorString(e));
    const bool capturing = cs != cudaStreamCaptureStatusNone;
    const unsigned char* k = static_cast<const unsigned char*>(key);
    for (size_t i = 0; i < slots_.size(); ++i) {
      Slot& s = slots_[i];
      if (s.filled && s.key.size() == nkey && std::memcmp(s.key.data(), k, nkey) == 0) {
        s.last = ++tick_;
        if (capturing) s.pinned = true;
        note_use(i);
        *out = s.dev;
        return MUON_OK;
      }
    }
    if (capturing)
      return fail(MUON_ERR_INVALID_ARG, "these pointers have no device tables yet and tables cannot be uploaded "
                                        "during stream capture: run the same call once before capturing it");
    std::vector<unsigned char> content;
    const unsigned char* src = k;
    size_t n = nkey;
    if (build) {
      int rc = build(ctx, content);
      if (rc) return rc;
      src = content.data();
      n = content.size();
    }
    int rc = reserve(n);
    if (rc) return rc;
    size_t victim = slots_.size();
    for (size_t i = 0; i < slots_.size(); ++i) {
      if (slots_[i].pinned || is_in_call(i)) continue;
      if (victim == slots_.size() || slots_[i].last < slots_[victim].last) victim = i;
    }
    if (victim == slots_.size())
      return fail(MUON_ERR_INVALID_ARG, "every pointer-table slot is pinned by a captured graph or used by this "
                                        "call; release the graphs (or change the plan) to free them");
    Slot& s = slots_[victim];
    if (s.filled) {
      // The staging's previous upload must have executed before it is
      // rewritten; the device copy waits for the slot's last readers.
      e = cudaEventSynchronize(s.copied);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(st, s.used, 0);
      if (e != cudaSuccess) return fail(MUON_ERR_CUDA, std::string("table ring: ") + cudaGetErrorString(e));
    }
    std::memcpy(s.host, src, n);
    e = cudaMemcpyAsync(s.dev, s.host, n, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaEventRecord(s.copied, st);
    if (e != cudaSuccess) return fail(MUON_ERR_CUDA, std::string("table upload: ") + cudaGetErrorString(e));
    s.key.assign(k, k + nkey);
    s.filled = true;
    s.last = ++tick_;
    note_use(victim);
    *out = s.dev;
    return MUON_OK;
  }

  // After a call's kernels are enqueued: the slots it used record that
  // point of the stream (skipped while capturing: those slots are pinned).
  int end_call(cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(st, &cs);
    int rc = MUON_OK;
    if (cs == cudaStreamCaptureStatusNone)
      for (size_t i : in_call_) {
        cudaError_t e = cudaEventRecord(slots_[i].used, st);
        if (e != cudaSuccess && rc == MUON_OK) rc = fail(MUON_ERR_CUDA, std::string("table ring: ") + cudaGetErrorString(e));
      }
    in_call_.clear();
    return rc;
  }

 private:
  struct Slot {
    std::vector<unsigned char> key;
    void* dev = nullptr;
    void* host = nullptr;        // pinned staging of the upload
    cudaEvent_t copied = nullptr;
    cudaEvent_t used = nullptr;
    unsigned long long last = 0;
    bool filled = false;
    bool pinned = false;
  };
  static constexpr int kSlots = 8;
  void note_use(size_t i) {
    if (!is_in_call(i)) in_call_.push_back(i);
  }
  bool is_in_call(size_t i) const { return std::find(in_call_.begin(), in_call_.end(), i) != in_call_.end(); }
  std::vector<Slot> slots_;
  size_t cap_ = 0;
  unsigned long long tick_ = 0;
  std::vector<size_t> in_call_;
};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2D bf16 row-major tensor (rows x cols, leading dimension ld elements),
// 128-byte swizzle, box of box_cols (inner) x box_rows.
int encode_map(TmapBlob* out, const void* base, int rows, int cols, int ld, int box_cols, int box_rows,
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  static_assert(sizeof(CUtensorMap) == sizeof(TmapBlob), "tensor map size");
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(reinterpret_cast<CUtensorMap*>(out), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
                   dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return MUON_OK;
}

// Maps of one X-layout buffer (m x n, ld): K-major 128- and 256-row boxes and
// the 64 x 64 M/N-major box.
int encode_x_triple(TmapBlob* out3, const void* base, const MatPlan& mp) {
  int rc;
  if ((rc = encode_map(out3 + MAP_K128, base, mp.m, mp.n, mp.ldx, 64, 128))) return rc;
  if ((rc = encode_map(out3 + MAP_K256, base, mp.m, mp.n, mp.ldx, 64, 256))) return rc;
  if ((rc = encode_map(out3 + MAP_MN, base, mp.m, mp.n, mp.ldx, 64, 64))) return rc;
  return MUON_OK;
}

// 32 x 32 store box with 64-byte swizzle (the epilogue's staging layout).
int encode_store_map(TmapBlob* out, const void* base, int rows, int cols, int ld) {
  return encode_map(out, base, rows, cols, ld, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

// A caller's fp32 parameter (dense rows x cols, cols % 4 == 0, 16-byte
// aligned): 32 x 32 boxes, 128-byte swizzle (a box row is 128 bytes).
int encode_p_map(TmapBlob* out, const float* base, int rows, int cols) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(reinterpret_cast<CUtensorMap*>(out), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base),
                   dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return MUON_OK;
}

}  // namespace

namespace muon {
void record_last_error(const std::string& msg) { g_last_error = msg; }
}  // namespace muon

// ---------------------------------------------------------------------------
// Handle
// ---------------------------------------------------------------------------

struct DevPlan {
  HostPlan hp;
  std::vector<int32_t> key;          // (m, n) per matrix
  void* ws = nullptr;
  size_t ws_size = 0;
  void* tables = nullptr;            // MatPlan[count] | prefix | tiles x3 | maps
  MatPlan* d_mats = nullptr;
  long long* d_prefix = nullptr;
  int4* d_tiles[3] = {nullptr, nullptr, nullptr};
  int* d_small = nullptr;
  TmapBlob* d_maps = nullptr;
  std::vector<MatPlan> mats;         // host copy with workspace pointers
  // Chunks for the pipelined host-buffer step: consecutive matrices with
  // about equal element counts, each with its own slice of every tile list.
  std::vector<int> chunk_bounds;                 // nchunks + 1
  int4* d_chunk_tiles[3] = {nullptr, nullptr, nullptr};
  std::vector<int> chunk_tile_off[3];            // nchunks + 1 each
  int* d_chunk_small = nullptr;
  std::vector<int> chunk_small_off;              // nchunks + 1
  double* partials = nullptr;                    // deterministic norm: one per K1 block
  void* gram_ws = nullptr;                       // Gram form: T and B1 per matrix
  GramBufs* d_gbufs = nullptr;                   // device table of T / B1 pointers
  TmapBlob* d_gmaps = nullptr;                   // device, kGramMapsPerMat per matrix
  void* staging = nullptr;                       // muon_step_host: kStagingSlots slots
  size_t staging_size = 0;
  size_t slot_bytes = 0;
  std::vector<int64_t> staging_off;              // count * 3: param, grad, momentum (within the slot)
  bool grouped = false;                          // chunks are the workspace cap's groups
  std::vector<TileRec> chunk_tiles_host[3];      // host copies of the per-chunk tile lists
  std::vector<int> chunk_small_host;
};

// Work of one enqueue: matrices [m0, m1), elementwise chunks [blk0, blk1),
// and the matching tile lists.
struct WorkRange {
  int m0 = 0, m1 = 0;
  long long blk0 = 0, blk1 = 0;
  const int4* tiles[3] = {nullptr, nullptr, nullptr};
  int ntiles[3] = {0, 0, 0};
  const int* small = nullptr;
  int nsmall = 0;
};

// Chunks of the pipelined host-buffer step: enough that the last chunk's
// compute and copy-out, which nothing overlaps, are a few percent of a step
// whose copies both ways keep PCIe busy.
constexpr int kHostChunks = 32;
constexpr int kStagingSlots = 3;    // staging slots in flight (H2D, compute, D2H)

struct muon_handle {
  int device = 0;
  muon_config cfg{};
  int num_sms = 0;
  DevStatus* status = nullptr;
  std::unique_ptr<DevPlan> plan;
  TableRing binds;     // MatBind tables of the calls
  TableRing in_maps;   // tensor maps of the callers' X inputs (stage call)
  TableRing subsets;   // tile lists restricted to the matrices with a gradient
  TableRing p_maps;    // tensor maps of the callers' parameters (update in the last combine)
  int last_launches = 0;
  // Per-launch timing (muon_profile_enable / muon_profile_read).
  std::vector<cudaEvent_t> prof_ev;   // 2 per slot
  std::vector<int> prof_kind;         // per slot
  int prof_slots = 0;                 // capacity in kernels
  int prof_used = 0;                  // kernels recorded so far
  int prof_calls_left = 0;            // calls that still record
  bool prof_this_call = false;
  // Pipelined host-buffer step: copy-in, compute and copy-out streams.
  cudaStream_t hs[3] = {nullptr, nullptr, nullptr};
  std::vector<cudaEvent_t> hev;       // 3 per chunk + 1
};

namespace {

void free_plan(DevPlan* p) {
  if (!p) return;
  cudaFree(p->ws);
  cudaFree(p->tables);
  cudaFree(p->staging);
  cudaFree(p->gram_ws);
  cudaFree(p->d_gbufs);
  cudaFree(p->partials);
}


int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

// Extra s x s buffers (T, B1), their pointer table and tensor maps for the
// Gram form of the iteration, for the matrices of the tile lists (the small
// path keeps its matrices on chip).
int ensure_gram_buffers(DevPlan& P) {
  if (P.gram_ws || P.d_gbufs) return MUON_OK;
  const int count = P.hp.count;
  std::vector<char> tiled((size_t)count, 1);
  for (int i : P.hp.small) tiled[(size_t)i] = 0;
  std::vector<int64_t> off((size_t)count * 2, -1);
  int64_t total = 0;
  // Groups of a capped plan run one after another: each lays out its own
  // buffers from offset 0.
  const std::vector<int>& groups = P.hp.groups;
  for (size_t gi = 0; gi + 1 < groups.size(); ++gi) {
    int64_t goff = 0;
    for (int i = groups[gi]; i < groups[gi + 1]; ++i)
      if (tiled[(size_t)i])
        for (int k = 0; k < 2; ++k) {
          off[(size_t)i * 2 + k] = goff;
          goff = align_up(goff + (int64_t)P.mats[i].s * P.mats[i].lds * 2, kRegionAlign);
        }
    total = std::max(total, goff);
  }
  if (total > 0) {
    cudaError_t e = cudaMalloc(&P.gram_ws, (size_t)total);
    if (e != cudaSuccess) {
      cudaGetLastError();
      P.gram_ws = nullptr;
      return fail(MUON_ERR_OOM, "Gram-form buffers of " + std::to_string(total) + " bytes failed to allocate");
    }
  }
  const size_t tab_bytes = align_up(sizeof(GramBufs) * (size_t)count, 256);
  const size_t map_bytes = sizeof(TmapBlob) * kGramMapsPerMat * (size_t)count;
  std::vector<unsigned char> host(tab_bytes + map_bytes, 0);
  GramBufs* gb = reinterpret_cast<GramBufs*>(host.data());
  TmapBlob* gm = reinterpret_cast<TmapBlob*>(host.data() + tab_bytes);
  char* base = static_cast<char*>(P.gram_ws);
  for (int i = 0; i < count; ++i) {
    if (!tiled[(size_t)i]) continue;
    const MatPlan& mp = P.mats[i];
    gb[i].t = base + off[(size_t)i * 2];
    gb[i].b1 = base + off[(size_t)i * 2 + 1];
    TmapBlob* m = gm + (size_t)i * kGramMapsPerMat;
    int rc;
    if ((rc = encode_map(m + 0, gb[i].t, mp.s, mp.s, mp.lds, 64, 128)) ||
        (rc = encode_map(m + 1, gb[i].t, mp.s, mp.s, mp.lds, 64, 256)) ||
        (rc = encode_map(m + 2, gb[i].b1, mp.s, mp.s, mp.lds, 64, 128)) ||
        (rc = encode_map(m + 3, gb[i].b1, mp.s, mp.s, mp.lds, 64, 256)) ||
        (rc = encode_store_map(m + 4, gb[i].t, mp.s, mp.s, mp.lds)) ||
        (rc = encode_store_map(m + 5, gb[i].b1, mp.s, mp.s, mp.lds)) ||
        (rc = encode_map(m + 6, gb[i].t, mp.s, mp.s, mp.lds, 64, 64)) ||
        (rc = encode_map(m + 7, gb[i].b1, mp.s, mp.s, mp.lds, 64, 64)))
      return rc;
  }
  void* d = nullptr;
  MUON_CUDA_TRY(cudaMalloc(&d, host.size()));
  P.d_gbufs = static_cast<GramBufs*>(d);
  MUON_CUDA_TRY(cudaMemcpy(d, host.data(), host.size(), cudaMemcpyHostToDevice));
  P.d_gmaps = reinterpret_cast<TmapBlob*>(static_cast<char*>(d) + tab_bytes);
  return MUON_OK;
}

constexpr int kProfMaxPerCall = 256;

// Marks the start of a call for the profiler.
void prof_call_begin(muon_handle* h) {
  h->prof_this_call = h->prof_calls_left > 0;
  if (h->prof_this_call) --h->prof_calls_left;
}

// Records the event before a kernel; returns the slot or -1.
int prof_before(muon_handle* h, int kind, cudaStream_t st) {
  if (!h->prof_this_call || h->prof_used >= h->prof_slots) return -1;
  const int slot = h->prof_used++;
  h->prof_kind[slot] = kind;
  cudaEventRecord(h->prof_ev[2 * slot], st);
  return slot;
}

void prof_after(muon_handle* h, int slot, cudaStream_t st) {
  if (slot >= 0) cudaEventRecord(h->prof_ev[2 * slot + 1], st);
}

void prof_free(muon_handle* h) {
  for (cudaEvent_t e : h->prof_ev) cudaEventDestroy(e);
  h->prof_ev.clear();
  h->prof_kind.clear();
  h->prof_slots = h->prof_used = h->prof_calls_left = 0;
  h->prof_this_call = false;
}

// Builds (or reuses) the plan, workspace, device tables and tensor maps for
// this shape table.
int ensure_plan(muon_handle* h, const int32_t* shapes, int count) {
  std::vector<int32_t> key((size_t)count * 2);
  for (int i = 0; i < count; ++i) {
    key[2 * i] = shapes[3 * i];
    key[2 * i + 1] = shapes[3 * i + 1];
  }
  if (h->plan && h->plan->key == key) return MUON_OK;

  auto np = std::make_unique<DevPlan>();
  std::string why;
  if (!build_plan(shapes, count, h->cfg.ns_precision, h->cfg.small_path != 0, h->cfg.cta_pair != 0, np->hp, why))
    return fail(MUON_ERR_INVALID_ARG, why);
  // Under a workspace cap the matrices run in groups that share one
  // workspace (consecutive matrices, each group as large as fits).
  if (h->cfg.workspace_cap_bytes &&
      !build_plan(shapes, count, h->cfg.ns_precision, h->cfg.small_path != 0, h->cfg.cta_pair != 0, np->hp, why,
                  (int64_t)h->cfg.workspace_cap_bytes))
    return fail(MUON_ERR_OOM, why);
  np->key = key;
  const HostPlan& hp = np->hp;

  // Drop the previous plan first (queued work may still use it).
  if (h->plan) {
    MUON_CUDA_TRY(cudaDeviceSynchronize());
    h->binds.release();
    h->in_maps.release();
    h->subsets.release();
    h->p_maps.release();
    free_plan(h->plan.get());
    h->plan.reset();
  }

  cudaError_t e = cudaMalloc(&np->ws, (size_t)hp.ws_bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MUON_ERR_OOM, "workspace allocation of " + std::to_string(hp.ws_bytes) + " bytes failed");
  }
  np->ws_size = (size_t)hp.ws_bytes;

  char* ws = static_cast<char*>(np->ws);
  np->mats = hp.mats;
  for (int i = 0; i < count; ++i) {
    MatPlan& mp = np->mats[i];
    mp.x0 = ws + hp.region_off[(size_t)i * 4 + 0];
    mp.x1 = ws + hp.region_off[(size_t)i * 4 + 1];
    mp.a = ws + hp.region_off[(size_t)i * 4 + 2];
    mp.b = ws + hp.region_off[(size_t)i * 4 + 3];
  }

  // Device tables, one allocation.
  const bool bf16 = h->cfg.ns_precision == MUON_NS_BF16;
  int64_t off = 0;
  const int64_t o_mats = off;  off = align_up(off + (int64_t)sizeof(MatPlan) * count, 256);
  const int64_t o_pref = off;  off = align_up(off + (int64_t)sizeof(long long) * (count + 1), 256);
  int64_t o_tiles[3];
  for (int p = 0; p < 3; ++p) {
    o_tiles[p] = off;
    off = align_up(off + (int64_t)sizeof(int4) * std::max<size_t>(hp.tiles[p].size(), 1), 256);
  }
  const int64_t o_small = off;
  off = align_up(off + (int64_t)sizeof(int) * std::max<size_t>(hp.small.size(), 1), 256);
  // Chunk partition and per-chunk slices of the tile lists: the cap's
  // groups when there are several (muon_step and muon_newton_schulz run them
  // one after another), else up to kHostChunks chunks of about equal element
  // counts for the pipelined host-buffer step.
  np->grouped = hp.groups.size() > 2;
  if (np->grouped) {
    np->chunk_bounds = hp.groups;
  } else {
    const int nch = std::min(count, kHostChunks);
    long long total = 0;
    for (int i = 0; i < count; ++i) total += np->mats[i].numel;
    np->chunk_bounds.assign(1, 0);
    long long cum = 0;
    for (int i = 0; i < count; ++i) {
      cum += np->mats[i].numel;
      const int made = (int)np->chunk_bounds.size() - 1;
      const int left_m = count - (i + 1), left_c = nch - (made + 1);
      if (made + 1 < nch && (cum * nch >= total * (long long)(made + 1) || left_m == left_c))
        np->chunk_bounds.push_back(i + 1);
    }
    np->chunk_bounds.push_back(count);
  }
  const int nch = (int)np->chunk_bounds.size() - 1;
  std::vector<int> chunk_of((size_t)count);
  for (int c = 0; c < nch; ++c)
    for (int i = np->chunk_bounds[c]; i < np->chunk_bounds[c + 1]; ++i) chunk_of[i] = c;
  std::vector<TileRec> chunk_tiles[3];
  for (int p = 0; p < 3; ++p) {
    np->chunk_tile_off[p].assign(1, 0);
    for (int c = 0; c < nch; ++c) {
      for (const TileRec& t : hp.tiles[p])
        if (chunk_of[t.mat] == c) chunk_tiles[p].push_back(t);
      np->chunk_tile_off[p].push_back((int)chunk_tiles[p].size());
    }
  }
  std::vector<int> chunk_small;
  np->chunk_small_off.assign(1, 0);
  for (int c = 0; c < nch; ++c) {
    for (int i : hp.small)
      if (chunk_of[i] == c) chunk_small.push_back(i);
    np->chunk_small_off.push_back((int)chunk_small.size());
  }
  int64_t o_ctiles[3];
  for (int p = 0; p < 3; ++p) {
    o_ctiles[p] = off;
    off = align_up(off + (int64_t)sizeof(int4) * std::max<size_t>(chunk_tiles[p].size(), 1), 256);
  }
  const int64_t o_csmall = off;
  off = align_up(off + (int64_t)sizeof(int) * std::max<size_t>(chunk_small.size(), 1), 256);
  const int64_t o_maps = off;
  if (bf16) off = align_up(off + (int64_t)sizeof(TmapBlob) * kMapsPerMat * count, 256);
  std::vector<unsigned char> host((size_t)off, 0);
  std::memcpy(host.data() + o_mats, np->mats.data(), sizeof(MatPlan) * count);
  std::memcpy(host.data() + o_pref, hp.prefix.data(), sizeof(long long) * (count + 1));
  for (int p = 0; p < 3; ++p) {
    int4* t = reinterpret_cast<int4*>(host.data() + o_tiles[p]);
    for (size_t k = 0; k < hp.tiles[p].size(); ++k)
      t[k] = make_int4(hp.tiles[p][k].mat, hp.tiles[p][k].ti, hp.tiles[p][k].tj, 0);
  }
  if (!hp.small.empty()) std::memcpy(host.data() + o_small, hp.small.data(), sizeof(int) * hp.small.size());
  for (int p = 0; p < 3; ++p) {
    int4* t = reinterpret_cast<int4*>(host.data() + o_ctiles[p]);
    for (size_t k = 0; k < chunk_tiles[p].size(); ++k)
      t[k] = make_int4(chunk_tiles[p][k].mat, chunk_tiles[p][k].ti, chunk_tiles[p][k].tj, 0);
  }
  if (!chunk_small.empty())
    std::memcpy(host.data() + o_csmall, chunk_small.data(), sizeof(int) * chunk_small.size());
  for (int p = 0; p < 3; ++p) np->chunk_tiles_host[p] = chunk_tiles[p];
  np->chunk_small_host = chunk_small;
  if (bf16) {
    TmapBlob* maps = reinterpret_cast<TmapBlob*>(host.data() + o_maps);
    for (int i = 0; i < count; ++i) {
      const MatPlan& mp = np->mats[i];
      TmapBlob* mm = maps + (size_t)i * kMapsPerMat;
      int rc;
      if ((rc = encode_x_triple(mm + MAP_X0, mp.x0, mp))) { free_plan(np.get()); return rc; }
      if ((rc = encode_x_triple(mm + MAP_X1, mp.x1, mp))) { free_plan(np.get()); return rc; }
      if ((rc = encode_map(mm + MAP_A_K128, mp.a, mp.s, mp.s, mp.lds, 64, 128))) { free_plan(np.get()); return rc; }
      if ((rc = encode_map(mm + MAP_A_K256, mp.a, mp.s, mp.s, mp.lds, 64, 256))) { free_plan(np.get()); return rc; }
      if ((rc = encode_map(mm + MAP_B_K128, mp.b, mp.s, mp.s, mp.lds, 64, 128))) { free_plan(np.get()); return rc; }
      if ((rc = encode_map(mm + MAP_B_K256, mp.b, mp.s, mp.s, mp.lds, 64, 256))) { free_plan(np.get()); return rc; }
      if ((rc = encode_map(mm + MAP_A_MN, mp.a, mp.s, mp.s, mp.lds, 64, 64))) { free_plan(np.get()); return rc; }
      if ((rc = encode_map(mm + MAP_B_MN, mp.b, mp.s, mp.s, mp.lds, 64, 64))) { free_plan(np.get()); return rc; }
      if ((rc = encode_store_map(mm + MAP_X0_ST, mp.x0, mp.m, mp.n, mp.ldx)) ||
          (rc = encode_store_map(mm + MAP_X1_ST, mp.x1, mp.m, mp.n, mp.ldx)) ||
          (rc = encode_store_map(mm + MAP_A_ST, mp.a, mp.s, mp.s, mp.lds)) ||
          (rc = encode_store_map(mm + MAP_B_ST, mp.b, mp.s, mp.s, mp.lds))) {
        free_plan(np.get());
        return rc;
      }
    }
  }
  e = cudaMalloc(&np->tables, (size_t)off);
  if (e != cudaSuccess) {
    cudaGetLastError();
    free_plan(np.get());
    return fail(MUON_ERR_OOM, "plan table allocation failed");
  }
  e = cudaMemcpy(np->tables, host.data(), (size_t)off, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    free_plan(np.get());
    return fail(MUON_ERR_CUDA, std::string("plan table upload: ") + cudaGetErrorString(e));
  }
  char* tb = static_cast<char*>(np->tables);
  np->d_mats = reinterpret_cast<MatPlan*>(tb + o_mats);
  np->d_prefix = reinterpret_cast<long long*>(tb + o_pref);
  for (int p = 0; p < 3; ++p) np->d_tiles[p] = reinterpret_cast<int4*>(tb + o_tiles[p]);
  np->d_small = reinterpret_cast<int*>(tb + o_small);
  for (int p = 0; p < 3; ++p) np->d_chunk_tiles[p] = reinterpret_cast<int4*>(tb + o_ctiles[p]);
  np->d_chunk_small = reinterpret_cast<int*>(tb + o_csmall);
  np->d_maps = bf16 ? reinterpret_cast<TmapBlob*>(tb + o_maps) : nullptr;
  if (h->cfg.deterministic) {
    const size_t nb = sizeof(double) * (size_t)std::max<long long>(hp.prefix[count], 1);
    if (cudaMalloc(reinterpret_cast<void**>(&np->partials), nb) != cudaSuccess) {
      cudaGetLastError();
      np->partials = nullptr;
      free_plan(np.get());
      return fail(MUON_ERR_OOM, "norm partials of " + std::to_string(nb) + " bytes failed to allocate");
    }
  }
  // Gram-form buffers are made with the plan so that a captured step never
  // allocates.
  if (bf16 && h->cfg.ns_algorithm == MUON_NS_GRAM) {
    const int rc = ensure_gram_buffers(*np);
    if (rc) { free_plan(np.get()); return rc; }
  }
  h->plan = std::move(np);
  return MUON_OK;
}

int check_ptr(const void* p, const char* what, int i) {
  if (p == nullptr) return fail(MUON_ERR_INVALID_ARG, std::string(what) + "[" + std::to_string(i) + "] is NULL");
  if (reinterpret_cast<uintptr_t>(p) % 16 != 0)
    return fail(MUON_ERR_INVALID_ARG, std::string(what) + "[" + std::to_string(i) + "] is not 16-byte aligned");
  return MUON_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

int check_common(muon_handle* h, const int32_t* shapes, int count) {
  if (h == nullptr) return fail(MUON_ERR_INVALID_ARG, "handle is NULL");
  if (shapes == nullptr) return fail(MUON_ERR_INVALID_ARG, "shapes is NULL");
  if (count < 1) return fail(MUON_ERR_INVALID_ARG, "count must be >= 1");
  for (int i = 0; i < count; ++i) {
    const int m = shapes[3 * i], n = shapes[3 * i + 1], fl = shapes[3 * i + 2];
    if (m < 1 || n < 1 || m > kMaxDim || n > kMaxDim)
      return fail(MUON_ERR_INVALID_ARG, "matrix " + std::to_string(i) + ": bad shape " + std::to_string(m) + " x " +
                                            std::to_string(n));
    if (fl & ~1) return fail(MUON_ERR_INVALID_ARG, "matrix " + std::to_string(i) + ": unknown flag bits");
  }
  return MUON_OK;
}

// Fills abc with ns_steps rows of (a, b, c): `rows` = 1 repeats one triple,
// `rows` = ns_steps gives one per step; NULL = the default triple.
int check_coeffs(const float* coeffs, int ns_steps, float* abc, int rows = 1) {
  if (ns_steps < 0 || ns_steps > kMaxNsSteps) return fail(MUON_ERR_INVALID_ARG, "ns_steps must be in [0, 64]");
  if (rows != 1 && rows != ns_steps)
    return fail(MUON_ERR_INVALID_ARG, "a coefficient table needs 1 or ns_steps rows");
  const float def[3] = {3.4445f, -4.7750f, 2.0315f};
  for (int t = 0; t < std::max(ns_steps, 1); ++t) {
    const float* c = coeffs ? coeffs + 3 * (rows == 1 ? 0 : t) : def;
    for (int k = 0; k < 3; ++k) {
      if (!std::isfinite(c[k])) return fail(MUON_ERR_INVALID_ARG, "coefficients must be finite");
      abc[3 * t + k] = c[k];
    }
  }
  return MUON_OK;
}

ElemLaunch elem_launch(const DevPlan& P, const MatBind* d_binds) {
  ElemLaunch L;
  L.plans = P.d_mats;
  L.binds = d_binds;
  L.prefix = P.d_prefix;
  L.count = P.hp.count;
  L.block_base = 0;
  L.nblocks = P.hp.prefix[P.hp.count];
  return L;
}

// Largest s of the matrices a range covers (an upper bound for its tile lists).
int range_max_s(const DevPlan& P, const WorkRange& R) {
  int s = 0;
  for (int i = R.m0; i < R.m1; ++i) s = std::max(s, P.mats[i].s);
  return s;
}

ElemLaunch elem_launch(const DevPlan& P, const MatBind* d_binds, const WorkRange& R) {
  ElemLaunch L = elem_launch(P, d_binds);
  L.block_base = R.blk0;
  L.nblocks = R.blk1 - R.blk0;
  return L;
}

WorkRange full_range(const DevPlan& P) {
  WorkRange R;
  R.m0 = 0;
  R.m1 = P.hp.count;
  R.blk0 = 0;
  R.blk1 = P.hp.prefix[P.hp.count];
  for (int p = 0; p < 3; ++p) {
    R.tiles[p] = P.d_tiles[p];
    R.ntiles[p] = (int)P.hp.tiles[p].size();
  }
  R.small = P.d_small;
  R.nsmall = (int)P.hp.small.size();
  return R;
}

WorkRange chunk_range(const DevPlan& P, int c) {
  WorkRange R;
  R.m0 = P.chunk_bounds[c];
  R.m1 = P.chunk_bounds[c + 1];
  R.blk0 = P.hp.prefix[R.m0];
  R.blk1 = P.hp.prefix[R.m1];
  for (int p = 0; p < 3; ++p) {
    R.tiles[p] = P.d_chunk_tiles[p] + P.chunk_tile_off[p][c];
    R.ntiles[p] = P.chunk_tile_off[p][c + 1] - P.chunk_tile_off[p][c];
  }
  R.small = P.d_chunk_small + P.chunk_small_off[c];
  R.nsmall = P.chunk_small_off[c + 1] - P.chunk_small_off[c];
  return R;
}

// Enqueue `ns_steps` Newton-Schulz iterations. The input of step 1 is
// `first_src`; intermediate results alternate X1, X0, X1, ...; the result of
// the last step goes to `last_dst` (or stays in the ping-pong buffers when
// last_dst < 0). *result receives the selector of the result buffer.
int enqueue_ns(muon_handle* h, const MatBind* d_binds, const std::vector<MatBind>& hbinds, const WorkRange& R,
               const TmapBlob* d_in_maps, const double* sumsq, int ns_steps, const float* abc, int first_src,
               int last_dst, cudaStream_t st, int* launches, int* result, const ApplyArgs* apply = nullptr,
               const TmapBlob* d_p_maps = nullptr) {
  DevPlan& P = *h->plan;
  const HostPlan& hp = P.hp;
  const bool bf16 = h->cfg.ns_precision == MUON_NS_BF16;
  if (bf16 && ns_steps > 0 && R.nsmall > 0) {
    // Matrices on the small path run every iteration in one launch and land
    // in the same buffer as the others' last step.
    NsSmallLaunch S;
    S.plans = P.d_mats;
    S.binds = d_binds;
    S.maps = P.d_maps;
    S.in_maps = d_in_maps;
    S.mats = R.small;
    S.nmats = R.nsmall;
    S.sumsq = sumsq;
    S.status = h->status;
    S.timeout_ns = (unsigned long long)(h->cfg.wait_timeout_s * 1e9);
    S.max_l = 0;
    for (int i : hp.small) S.max_l = std::max(S.max_l, P.mats[i].l);
    const int flips = h->cfg.ns_algorithm == MUON_NS_GRAM ? (ns_steps + 1) / 2 : ns_steps;
    const int final_sel = last_dst >= 0 ? last_dst : (flips % 2 == 1 ? BUF_X1 : BUF_X0);
    const int slot = prof_before(h, MUON_KERNEL_NS_SMALL, st);
    MUON_CUDA_TRY(launch_ns_small(S, ns_steps, first_src, final_sel, abc, st));
    prof_after(h, slot, st);
    ++*launches;
  }
  if (bf16 && h->cfg.ns_algorithm == MUON_NS_GRAM && ns_steps > 0) {
    // Gram form, segments of two steps (one of one at an odd end):
    //   A = X X^T; B0 = b0 A + c0 A^2;                       (GRAM, POLY)
    //   T = a0 A + B0 A; A = a0 T + T B0;                    (SYM, SYM)
    //   B1 = b1 A + c1 A^2;                                  (POLY)
    //   T = a1 B0 + a0 B1 + B1 B0;  X' = a0 a1 X + T X        (SYM, COMB)
    // a one-step segment is the plain step X' = a0 X + B0 X.
    int rc;
    if ((rc = ensure_gram_buffers(P))) return rc;
    NsLaunch L;
    L.plans = P.d_mats;
    L.binds = d_binds;
    L.maps = P.d_maps;
    L.in_maps = d_in_maps;
    L.sumsq = sumsq;
    L.status = h->status;
    L.grid = h->num_sms;
    L.timeout_ns = (unsigned long long)(h->cfg.wait_timeout_s * 1e9);
    L.gmaps = P.d_gmaps;
    L.gbufs = P.d_gbufs;
    L.tma_store = 1;
    L.max_s = range_max_s(P, R);
    auto run = [&](int phase, int src_sel, int dst_sel, int first, float a, float b, float c,
                   const PhaseSpec& spec) -> int {
      const int list = phase == PHASE_SYM ? PHASE_POLY : phase;
      L.tiles = R.tiles[list];
      L.ntiles = R.ntiles[list];
      if (L.ntiles == 0) return MUON_OK;
      const int kind = phase == PHASE_SYM ? MUON_KERNEL_NS_SYM : MUON_KERNEL_NS_GRAM + phase;
      const int slot = prof_before(h, kind, st);
      MUON_CUDA_TRY(launch_ns_phase_bf16(L, phase, src_sel, dst_sel, first, a, b, c, st, spec));
      prof_after(h, slot, st);
      ++*launches;
      return MUON_OK;
    };
    int src = first_src;
    bool first = true;
    for (int k = 0; k < ns_steps;) {
      const int len = std::min(2, ns_steps - k);
      const bool last = k + len == ns_steps;
      const int dst = (last && last_dst >= 0) ? last_dst : (src == BUF_X1 ? BUF_X0 : BUF_X1);
      const float* c0 = abc + 3 * k;
      PhaseSpec sp;
      if ((rc = run(PHASE_GRAM, src, dst, first, 0.f, 0.f, 0.f, sp))) return rc;
      sp.poly_out = SB_B;
      if ((rc = run(PHASE_POLY, src, dst, 0, 0.f, c0[1], c0[2], sp))) return rc;
      if (len == 2) {
        const float* c1 = abc + 3 * (k + 1);
        PhaseSpec s1;
        s1.sym_l = SB_B; s1.sym_r = SB_A; s1.sym_out = SB_T; s1.aux1 = SB_A; s1.e1 = c0[0];
        if ((rc = run(PHASE_SYM, src, dst, 0, 0.f, 0.f, 0.f, s1))) return rc;
        PhaseSpec s2;
        s2.sym_l = SB_T; s2.sym_r = SB_B; s2.sym_out = SB_A; s2.aux1 = SB_T; s2.e1 = c0[0];
        if ((rc = run(PHASE_SYM, src, dst, 0, 0.f, 0.f, 0.f, s2))) return rc;
        PhaseSpec s3;
        s3.poly_out = SB_B1;
        if ((rc = run(PHASE_POLY, src, dst, 0, 0.f, c1[1], c1[2], s3))) return rc;
        PhaseSpec s4;
        s4.sym_l = SB_B1; s4.sym_r = SB_B; s4.sym_out = SB_T;
        s4.aux1 = SB_B; s4.e1 = c1[0]; s4.aux2 = SB_B1; s4.e2 = c0[0];
        if ((rc = run(PHASE_SYM, src, dst, 0, 0.f, 0.f, 0.f, s4))) return rc;
        PhaseSpec s5;
        s5.comb_b = SB_T;
        if ((rc = run(PHASE_COMB, src, dst, first, c0[0] * c1[0], 0.f, 0.f, s5))) return rc;
      } else {
        PhaseSpec s5;
        s5.comb_b = SB_B;
        if ((rc = run(PHASE_COMB, src, dst, first, c0[0], 0.f, 0.f, s5))) return rc;
      }
      src = dst;
      first = false;
      k += len;
    }
    *result = src;
    return MUON_OK;
  }
  int src = first_src;
  for (int t = 1; t <= ns_steps; ++t) {
    const int dst = (t == ns_steps && last_dst >= 0) ? last_dst : (t % 2 == 1 ? BUF_X1 : BUF_X0);
    const int first = t == 1 ? 1 : 0;
    const float* c3 = abc + 3 * (t - 1);
    if (bf16) {
      NsLaunch L;
      L.plans = P.d_mats;
      L.binds = d_binds;
      L.maps = P.d_maps;
      L.in_maps = d_in_maps;
      L.sumsq = sumsq;
      L.status = h->status;
      L.grid = h->num_sms;
      L.timeout_ns = (unsigned long long)(h->cfg.wait_timeout_s * 1e9);
      L.tma_store = 1;
      L.max_s = range_max_s(P, R);
      for (int ph = 0; ph < 3; ++ph) {
        L.tiles = R.tiles[ph];
        L.ntiles = R.ntiles[ph];
        if (L.ntiles == 0) continue;
        // The step's last combine may carry the parameter update.
        if (apply && ph == PHASE_COMB && t == ns_steps) {
          L.apply = *apply;
          L.p_maps = d_p_maps;
        }
        const int slot = prof_before(h, MUON_KERNEL_NS_GRAM + ph, st);
        // a goes on the diagonal of B (POLY), so the combine adds no a X.
        const float a = ph == PHASE_COMB ? 0.0f : c3[0];
        if (hp.tile_m == kTileMPair)
          MUON_CUDA_TRY(launch_ns_phase_pair(L, ph, src, dst, first, a, c3[1], c3[2], st));
        else
          MUON_CUDA_TRY(launch_ns_phase_bf16(L, ph, src, dst, first, a, c3[1], c3[2], st));
        prof_after(h, slot, st);
        ++*launches;
      }
    } else {
      for (int i = R.m0; i < R.m1; ++i) {
        if (!hbinds[i].active) continue;
        const MatPlan& mp = P.mats[i];
        const float* s_ptr = static_cast<const float*>(sel_buf(mp, hbinds[i], src));
        float* d_ptr = static_cast<float*>(const_cast<void*>(sel_buf(mp, hbinds[i], dst)));
        for (int ph = PHASE_GRAM; ph <= PHASE_COMB; ++ph) {
          const int slot = prof_before(h, MUON_KERNEL_NS_FP32, st);
          MUON_CUDA_TRY(launch_ns_phase_fp32(mp, i, ph, s_ptr, d_ptr, sumsq, first, c3[0], c3[1], c3[2], st));
          prof_after(h, slot, st);
        }
        *launches += 3;
      }
    }
    src = dst;
  }
  *result = src;
  return MUON_OK;
}

// Validation of a full step's pointers: alignment and per-matrix overlap.
int check_step_ptrs(float* const* params, const void* const* grads, float* const* momenta, const int32_t* shapes,
                    int count) {
  if (!params || !grads || !momenta) return fail(MUON_ERR_INVALID_ARG, "params, grads and momenta arrays are required");
  int rc;
  for (int i = 0; i < count; ++i) {
    const size_t numel = (size_t)shapes[3 * i] * (size_t)shapes[3 * i + 1];
    const size_t gbytes = numel * ((shapes[3 * i + 2] & 1) ? 2 : 4);
    if ((rc = check_ptr(params[i], "params", i))) return rc;
    if ((rc = check_ptr(momenta[i], "momenta", i))) return rc;
    if (grads[i] && (rc = check_ptr(grads[i], "grads", i))) return rc;
    if (overlaps(params[i], numel * 4, momenta[i], numel * 4) ||
        (grads[i] && (overlaps(params[i], numel * 4, grads[i], gbytes) ||
                      overlaps(momenta[i], numel * 4, grads[i], gbytes))))
      return fail(MUON_ERR_INVALID_ARG, "matrix " + std::to_string(i) + ": params, grads and momenta overlap");
  }
  return MUON_OK;
}

int check_scalars(float lr, float beta, float wd) {
  if (!std::isfinite(lr) || !std::isfinite(wd)) return fail(MUON_ERR_INVALID_ARG, "lr and wd must be finite");
  if (!(beta >= 0.0f && beta < 1.0f)) return fail(MUON_ERR_INVALID_ARG, "beta must be in [0, 1)");
  return MUON_OK;
}

// Device pointer table of a step (cached by content).
int step_binds(muon_handle* h, float* const* params, const void* const* grads, float* const* momenta,
               const int32_t* shapes, int count, cudaStream_t st, std::vector<MatBind>& hb, const MatBind** db) {
  hb.assign((size_t)count, MatBind());
  for (int i = 0; i < count; ++i) {
    MatBind& b = hb[i];
    std::memset(&b, 0, sizeof(b));
    b.p = params[i];
    b.g = grads[i];
    b.mom = momenta[i];
    b.flags = shapes[3 * i + 2];
    b.active = grads[i] != nullptr;
  }
  void* d_binds = nullptr;
  int rc;
  if ((rc = h->binds.get(hb.data(), sizeof(MatBind) * count, nullptr, nullptr, st, &d_binds))) return rc;
  *db = static_cast<const MatBind*>(d_binds);
  return MUON_OK;
}

// Ends a call for the pointer-table rings on scope exit: every slot the call
// used records the point of `st` after its kernels.
struct CallTables {
  muon_handle* h;
  cudaStream_t st;
  ~CallTables() {
    h->binds.end_call(st);
    h->in_maps.end_call(st);
    h->subsets.end_call(st);
    h->p_maps.end_call(st);
  }
};

// Work ranges of a step: one per group of the plan (one group without a
// workspace cap). When some matrices have no gradient, the Newton-Schulz
// tile lists and the small-path list are restricted to the active matrices:
// the lists of every group, filtered, are one device table (kept in a ring
// keyed by the active mask), so a step over a few owned matrices (a round
// of layer-wise Muon) launches over their tiles only.
int step_ranges(muon_handle* h, const std::vector<MatBind>& hb, cudaStream_t st, std::vector<WorkRange>& out) {
  DevPlan& P = *h->plan;
  const int count = P.hp.count;
  const int nch = P.grouped ? (int)P.chunk_bounds.size() - 1 : 1;
  out.clear();
  for (int c = 0; c < nch; ++c) out.push_back(P.grouped ? chunk_range(P, c) : full_range(P));
  std::vector<unsigned char> mask((size_t)count);
  bool all = true;
  for (int i = 0; i < count; ++i) {
    mask[i] = hb[i].active ? 1 : 0;
    all = all && hb[i].active;
  }
  if (all) return MUON_OK;
  // Filtered lists, chunk by chunk: 3 tile lists (int4) then the small list
  // (int), each section 16-byte aligned.
  std::vector<size_t> sec_off((size_t)nch * 4 + 1, 0);
  std::vector<int> sec_n((size_t)nch * 4, 0);
  std::vector<unsigned char> bytes;
  auto put = [&](const void* src, size_t n) {
    const size_t at = bytes.size();
    bytes.resize(at + ((n + 15) / 16) * 16, 0);
    if (n) std::memcpy(bytes.data() + at, src, n);
  };
  for (int c = 0; c < nch; ++c) {
    for (int p = 0; p < 3; ++p) {
      const std::vector<TileRec>& src = P.grouped ? P.chunk_tiles_host[p] : P.hp.tiles[p];
      const int t0 = P.grouped ? P.chunk_tile_off[p][c] : 0;
      const int t1 = P.grouped ? P.chunk_tile_off[p][c + 1] : (int)src.size();
      std::vector<int4> f;
      for (int t = t0; t < t1; ++t)
        if (mask[src[t].mat]) f.push_back(make_int4(src[t].mat, src[t].ti, src[t].tj, 0));
      sec_off[(size_t)c * 4 + p] = bytes.size();
      sec_n[(size_t)c * 4 + p] = (int)f.size();
      put(f.data(), sizeof(int4) * f.size());
    }
    const std::vector<int>& ssrc = P.grouped ? P.chunk_small_host : P.hp.small;
    const int s0 = P.grouped ? P.chunk_small_off[c] : 0;
    const int s1 = P.grouped ? P.chunk_small_off[c + 1] : (int)ssrc.size();
    std::vector<int> f;
    for (int k = s0; k < s1; ++k)
      if (mask[ssrc[k]]) f.push_back(ssrc[k]);
    sec_off[(size_t)c * 4 + 3] = bytes.size();
    sec_n[(size_t)c * 4 + 3] = (int)f.size();
    put(f.data(), sizeof(int) * f.size());
  }
  if (bytes.empty()) bytes.resize(16, 0);
  struct Ctx {
    const std::vector<unsigned char>* b;
  } ctx{&bytes};
  auto build = [](const void* c, std::vector<unsigned char>& o) -> int {
    o = *static_cast<const Ctx*>(c)->b;
    return MUON_OK;
  };
  void* d = nullptr;
  int rc;
  if ((rc = h->subsets.get(mask.data(), mask.size(), build, &ctx, st, &d))) return rc;
  char* base = static_cast<char*>(d);
  for (int c = 0; c < nch; ++c) {
    WorkRange& R = out[c];
    for (int p = 0; p < 3; ++p) {
      R.tiles[p] = reinterpret_cast<const int4*>(base + sec_off[(size_t)c * 4 + p]);
      R.ntiles[p] = sec_n[(size_t)c * 4 + p];
    }
    R.small = reinterpret_cast<const int*>(base + sec_off[(size_t)c * 4 + 3]);
    R.nsmall = sec_n[(size_t)c * 4 + 3];
  }
  return MUON_OK;
}

// Momentum/norm/cast, Newton-Schulz and apply for the matrices of R.
// Tensor maps of the parameters for the update in the last combine, or
// NULL when the step applies O in a separate pass: other forms of the
// iteration, zero iterations, fused_apply off, an active matrix on the small
// path, or a parameter whose rows are not 16-byte aligned (n % 4 != 0 or an
// unaligned base) for the bulk copies.
int step_p_maps(muon_handle* h, float* const* params, const std::vector<MatBind>& hb, int ns_steps, cudaStream_t st,
                const TmapBlob** out) {
  *out = nullptr;
  const DevPlan& P = *h->plan;
  if (!h->cfg.fused_apply || h->cfg.ns_precision != MUON_NS_BF16 || h->cfg.ns_algorithm != MUON_NS_STANDARD ||
      P.hp.tile_m == kTileMPair || ns_steps <= 0)
    return MUON_OK;
  const int count = P.hp.count;
  std::vector<char> small((size_t)count, 0);
  for (int i : P.hp.small) small[i] = 1;
  for (int i = 0; i < count; ++i) {
    if (!hb[i].active) continue;
    if (small[i] || P.mats[i].n % 4 != 0 || (reinterpret_cast<uintptr_t>(params[i]) & 15u) != 0) return MUON_OK;
  }
  struct PCtx {
    float* const* p;
    const DevPlan* plan;
  } ctx{params, &P};
  auto build = [](const void* c, std::vector<unsigned char>& bytes) -> int {
    const PCtx& pc = *static_cast<const PCtx*>(c);
    const int n = pc.plan->hp.count;
    bytes.assign(sizeof(TmapBlob) * (size_t)n, 0);
    TmapBlob* maps = reinterpret_cast<TmapBlob*>(bytes.data());
    for (int i = 0; i < n; ++i) {
      const MatPlan& mp = pc.plan->mats[i];
      if (mp.n % 4 != 0 || (reinterpret_cast<uintptr_t>(pc.p[i]) & 15u) != 0) continue;   // never applied here
      const int rc = encode_p_map(maps + i, pc.p[i], mp.m, mp.n);
      if (rc) return rc;
    }
    return MUON_OK;
  };
  void* d = nullptr;
  int rc;
  if ((rc = h->p_maps.get(params, sizeof(float*) * (size_t)count, build, &ctx, st, &d))) return rc;
  *out = static_cast<const TmapBlob*>(d);
  return MUON_OK;
}

int enqueue_step_range(muon_handle* h, const MatBind* db, const std::vector<MatBind>& hb, const WorkRange& R,
                       float lr, float beta, int nesterov, float wd, int ns_steps, const float* abc, cudaStream_t st,
                       int* launches, const TmapBlob* d_p_maps) {
  DevPlan& P = *h->plan;
  double* sumsq = static_cast<double*>(P.ws);
  const bool fp32 = h->cfg.ns_precision == MUON_NS_FP32;
  int rc;
  MUON_CUDA_TRY(cudaMemsetAsync(sumsq + R.m0, 0, sizeof(double) * (size_t)(R.m1 - R.m0), st));
  const ElemLaunch EL = elem_launch(P, db, R);
  int slot = prof_before(h, MUON_KERNEL_MOMENTUM_NORM, st);
  MUON_CUDA_TRY(launch_momentum_norm(EL, BUF_X0, beta, nesterov ? 1 : 0, sumsq, P.partials, h->status,
                                     h->cfg.check_nonfinite, fp32, st));
  prof_after(h, slot, st);
  ++*launches;
  if (P.partials) {
    slot = prof_before(h, MUON_KERNEL_NORM_REDUCE, st);
    MUON_CUDA_TRY(launch_reduce_partials(EL, R.m0, R.m1, P.partials, sumsq, st));
    prof_after(h, slot, st);
    ++*launches;
  }
  int res = BUF_X0;
  // With parameter maps the last combine writes p' itself (step_p_maps says
  // when); otherwise O is stored and applied by a separate pass.
  ApplyArgs ap;
  ap.on = 1;
  ap.lr = lr;
  ap.wd = wd;
  ap.scale_mode = h->cfg.scale_mode;
  ap.extra_scale = h->cfg.extra_scale;
  if ((rc = enqueue_ns(h, db, hb, R, nullptr, sumsq, ns_steps, abc, BUF_X0, -1, st, launches, &res,
                       d_p_maps ? &ap : nullptr, d_p_maps)))
    return rc;
  if (d_p_maps) return MUON_OK;
  slot = prof_before(h, MUON_KERNEL_APPLY, st);
  MUON_CUDA_TRY(launch_apply(EL, res, lr, wd, h->cfg.scale_mode, h->cfg.extra_scale, ns_steps == 0 ? sumsq : nullptr,
                             fp32, st));
  prof_after(h, slot, st);
  ++*launches;
  return MUON_OK;
}

int step_impl(muon_handle* h, float* const* params, const void* const* grads, float* const* momenta,
              const int32_t* shapes, int count, float lr, float beta, int nesterov, float wd, int ns_steps,
              const float* abc, cudaStream_t st) {
  int rc;
  if ((rc = ensure_plan(h, shapes, count))) return rc;
  CallTables ct{h, st};
  std::vector<MatBind> hb;
  const MatBind* db = nullptr;
  if ((rc = step_binds(h, params, grads, momenta, shapes, count, st, hb, &db))) return rc;
  int launches = 0;
  prof_call_begin(h);
  DevPlan& P = *h->plan;
  std::vector<WorkRange> ranges;
  if ((rc = step_ranges(h, hb, st, ranges))) return rc;
  const TmapBlob* d_p_maps = nullptr;
  if ((rc = step_p_maps(h, params, hb, ns_steps, st, &d_p_maps))) return rc;
  // Groups under the workspace cap run one after another on the stream.
  for (const WorkRange& R : ranges)
    if ((rc = enqueue_step_range(h, db, hb, R, lr, beta, nesterov, wd, ns_steps, abc, st, &launches, d_p_maps)))
      return rc;
  (void)P;
  h->last_launches = launches;
  return MUON_OK;
}

}  // namespace

// ---------------------------------------------------------------------------
// Exported entry points
// ---------------------------------------------------------------------------

extern "C" {

const char* muon_last_error(void) { return g_last_error.c_str(); }

const char* muon_version(void) { return "muon_ns 0.1.0 (sm_100a)"; }

int muon_config_init(muon_config* cfg) {
  if (!cfg) return fail(MUON_ERR_INVALID_ARG, "cfg is NULL");
  cfg->scale_mode = MUON_SCALE_MOONLIGHT;
  cfg->extra_scale = 1.0f;
  cfg->ns_precision = MUON_NS_BF16;
  cfg->check_nonfinite = 0;
  cfg->num_sms = 0;
  cfg->workspace_cap_bytes = 0;
  cfg->wait_timeout_s = 2.0;
  cfg->small_path = 1;
  cfg->cta_pair = 0;
  cfg->ns_algorithm = MUON_NS_STANDARD;
  cfg->deterministic = 0;
  cfg->fused_apply = 1;
  return MUON_OK;
}

int muon_init(int device, const muon_config* cfg, muon_handle** out) {
  g_last_error.clear();
  if (!out) return fail(MUON_ERR_INVALID_ARG, "out is NULL");
  muon_config c;
  if (cfg) c = *cfg; else muon_config_init(&c);
  if (c.scale_mode < 0 || c.scale_mode > 3) return fail(MUON_ERR_INVALID_ARG, "unknown scale_mode");
  if (c.ns_precision != 0 && c.ns_precision != 1) return fail(MUON_ERR_INVALID_ARG, "unknown ns_precision");
  if (!std::isfinite(c.extra_scale)) return fail(MUON_ERR_INVALID_ARG, "extra_scale must be finite");
  if (!(c.wait_timeout_s > 0.0 && c.wait_timeout_s <= 600.0))
    return fail(MUON_ERR_INVALID_ARG, "wait_timeout_s must be in (0, 600]");
  if (c.num_sms < 0) return fail(MUON_ERR_INVALID_ARG, "num_sms must be >= 0");
  if (c.deterministic != 0 && c.deterministic != 1) return fail(MUON_ERR_INVALID_ARG, "deterministic must be 0 or 1");
  if (c.fused_apply != 0 && c.fused_apply != 1) return fail(MUON_ERR_INVALID_ARG, "fused_apply must be 0 or 1");
  if (c.ns_algorithm != MUON_NS_STANDARD && c.ns_algorithm != MUON_NS_GRAM)
    return fail(MUON_ERR_INVALID_ARG, "unknown ns_algorithm");
  if (c.ns_algorithm == MUON_NS_GRAM && (c.ns_precision != MUON_NS_BF16 || c.cta_pair))
    return fail(MUON_ERR_INVALID_ARG, "the Gram form runs in bf16 on single-CTA tiles (ns_precision 0, cta_pair 0)");
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
    cudaGetLastError();
    return fail(MUON_ERR_NO_DEVICE, "no CUDA device");
  }
  if (device < 0 || device >= ndev) return fail(MUON_ERR_INVALID_ARG, "device index out of range");
  cudaDeviceProp prop;
  MUON_CUDA_TRY(cudaGetDeviceProperties(&prop, device));
  if (prop.major != 10 || prop.minor != 0)
    return fail(MUON_ERR_UNSUPPORTED, std::string("device is sm_") + std::to_string(prop.major) +
                                          std::to_string(prop.minor) + "; this library is built for sm_100a");
  DeviceGuard g(device);
  if (!g.ok) return fail(MUON_ERR_CUDA, "cudaSetDevice failed");
  auto h = std::make_unique<muon_handle>();
  h->device = device;
  h->cfg = c;
  h->num_sms = c.num_sms > 0 ? std::min(c.num_sms, prop.multiProcessorCount) : prop.multiProcessorCount;
  MUON_CUDA_TRY(cudaMalloc(&h->status, sizeof(DevStatus)));
  MUON_CUDA_TRY(cudaMemset(h->status, 0, sizeof(DevStatus)));
  *out = h.release();
  return MUON_OK;
}

int muon_destroy(muon_handle* h) {
  if (!h) return MUON_OK;
  {
    DeviceGuard g(h->device);
    cudaDeviceSynchronize();
    h->binds.release();
    h->in_maps.release();
    h->subsets.release();
    h->p_maps.release();
    if (h->plan) free_plan(h->plan.get());
    prof_free(h);
    for (cudaEvent_t e : h->hev) cudaEventDestroy(e);
    for (int k = 0; k < 3; ++k)
      if (h->hs[k]) cudaStreamDestroy(h->hs[k]);
    cudaFree(h->status);
  }
  delete h;
  return MUON_OK;
}

int muon_step(muon_handle* h, float* const* params, const void* const* grads, float* const* momenta,
              const int32_t* shapes, int count, float lr, float beta, int nesterov, float wd, int ns_steps,
              const float* coeffs, void* stream) {
  g_last_error.clear();
  int rc;
  if ((rc = check_common(h, shapes, count))) return rc;
  if ((rc = check_step_ptrs(params, grads, momenta, shapes, count))) return rc;
  if ((rc = check_scalars(lr, beta, wd))) return rc;
  float abc[3 * kMaxNsSteps];
  if ((rc = check_coeffs(coeffs, ns_steps, abc))) return rc;
  DeviceGuard g(h->device);
  if (!g.ok) return fail(MUON_ERR_CUDA, "cudaSetDevice failed");
  return step_impl(h, params, grads, momenta, shapes, count, lr, beta, nesterov, wd, ns_steps, abc,
                   static_cast<cudaStream_t>(stream));
}

int muon_step_schedule(muon_handle* h, float* const* params, const void* const* grads, float* const* momenta,
                       const int32_t* shapes, int count, float lr, float beta, int nesterov, float wd, int ns_steps,
                       const float* coeff_table, int table_rows, void* stream) {
  g_last_error.clear();
  int rc;
  if ((rc = check_common(h, shapes, count))) return rc;
  if ((rc = check_step_ptrs(params, grads, momenta, shapes, count))) return rc;
  if ((rc = check_scalars(lr, beta, wd))) return rc;
  if (!coeff_table) return fail(MUON_ERR_INVALID_ARG, "coeff_table is required");
  float abc[3 * kMaxNsSteps];
  if ((rc = check_coeffs(coeff_table, ns_steps, abc, table_rows))) return rc;
  DeviceGuard g(h->device);
  if (!g.ok) return fail(MUON_ERR_CUDA, "cudaSetDevice failed");
  return step_impl(h, params, grads, momenta, shapes, count, lr, beta, nesterov, wd, ns_steps, abc,
                   static_cast<cudaStream_t>(stream));
}

int muon_qk_clip(muon_handle* h, float* const* weights, const int32_t* shapes, const float* const* s_max, int count,
                 float tau, void* stream) {
  g_last_error.clear();
  if (!h) return fail(MUON_ERR_INVALID_ARG, "handle is NULL");
  if (!weights || !shapes || !s_max || count < 1) return fail(MUON_ERR_INVALID_ARG, "weights, shapes, s_max, count");
  if (!(tau > 0.0f) || !std::isfinite(tau)) return fail(MUON_ERR_INVALID_ARG, "tau must be positive and finite");
  int rc;
  for (int i = 0; i < count; ++i) {
    const int rows = shapes[3 * i], cols = shapes[3 * i + 1], hr = shapes[3 * i + 2];
    if (rows < 1 || cols < 1 || hr < 1 || rows % hr)
      return fail(MUON_ERR_INVALID_ARG, "matrix " + std::to_string(i) + ": rows must be a positive multiple of head_rows");
    if ((rc = check_ptr(weights[i], "weights", i))) return rc;
    if (!s_max[i] || reinterpret_cast<uintptr_t>(s_max[i]) % 4)
      return fail(MUON_ERR_INVALID_ARG, "s_max[" + std::to_string(i) + "] is NULL or misaligned");
  }
  DeviceGuard g(h->device);
  if (!g.ok) return fail(MUON_ERR_CUDA, "cudaSetDevice failed");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int i = 0; i < count; ++i)
    MUON_CUDA_TRY(launch_qk_clip(weights[i], shapes[3 * i], shapes[3 * i + 1], shapes[3 * i + 2], s_max[i], tau, st));
  h->last_launches = count;
  return MUON_OK;
}

int muon_step_host(muon_handle* h, float* const* params, const void* const* grads, float* const* momenta,
                   const int32_t* shapes, int count, float lr, float beta, int nesterov, float wd, int ns_steps,
                   const float* coeffs, void* stream) {
  g_last_error.clear();
  int rc;
  if ((rc = check_common(h, shapes, count))) return rc;
  if (!params || !grads || !momenta) return fail(MUON_ERR_INVALID_ARG, "params, grads and momenta arrays are required");
  for (int i = 0; i < count; ++i)
    if (!params[i] || !momenta[i]) return fail(MUON_ERR_INVALID_ARG, "host params and momenta must be non-NULL");
  if ((rc = check_scalars(lr, beta, wd))) return rc;
  float abc[3 * kMaxNsSteps];
  if ((rc = check_coeffs(coeffs, ns_steps, abc))) return rc;
  DeviceGuard g(h->device);
  if (!g.ok) return fail(MUON_ERR_CUDA, "cudaSetDevice failed");
  if ((rc = ensure_plan(h, shapes, count))) return rc;
  DevPlan& P = *h->plan;
  const int nch = (int)P.chunk_bounds.size() - 1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // Staging: kStagingSlots slots, each holding one chunk's params, grads and
  // momenta (4 bytes per element each); chunk c uses slot c % kStagingSlots.
  if (!P.staging) {
    P.staging_off.assign((size_t)count * 3, 0);
    size_t slot = 0;
    for (int c = 0; c < nch; ++c) {
      int64_t off = 0;
      for (int i = P.chunk_bounds[c]; i < P.chunk_bounds[c + 1]; ++i)
        for (int k = 0; k < 3; ++k) {
          P.staging_off[(size_t)i * 3 + k] = off;
          off = align_up(off + P.mats[i].numel * 4, 256);
        }
      slot = std::max(slot, (size_t)off);
    }
    const int slots = std::min(nch, kStagingSlots);
    const size_t total = slot * (size_t)slots;
    cudaError_t e = cudaMalloc(&P.staging, total);
    if (e != cudaSuccess) {
      cudaGetLastError();
      P.staging = nullptr;
      return fail(MUON_ERR_OOM, "staging allocation of " + std::to_string(total) + " bytes failed");
    }
    P.staging_size = total;
    P.slot_bytes = slot;
  }
  for (int k = 0; k < 3; ++k)
    if (!h->hs[k]) MUON_CUDA_TRY(cudaStreamCreateWithFlags(&h->hs[k], cudaStreamNonBlocking));
  while ((int)h->hev.size() < 3 * nch + 1) {
    cudaEvent_t ev;
    MUON_CUDA_TRY(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
    h->hev.push_back(ev);
  }
  cudaEvent_t ev_begin = h->hev[3 * nch];
  auto ev_in = [&](int c) { return h->hev[3 * c]; };
  auto ev_comp = [&](int c) { return h->hev[3 * c + 1]; };
  auto ev_out = [&](int c) { return h->hev[3 * c + 2]; };

  // Device pointers of every matrix inside its chunk's slot.
  std::vector<float*> dp(count), dm(count);
  std::vector<const void*> dg(count);
  char* sb = static_cast<char*>(P.staging);
  for (int c = 0; c < nch; ++c) {
    char* slot = sb + (size_t)(c % kStagingSlots) * P.slot_bytes;
    for (int i = P.chunk_bounds[c]; i < P.chunk_bounds[c + 1]; ++i) {
      dp[i] = reinterpret_cast<float*>(slot + P.staging_off[(size_t)i * 3 + 0]);
      dg[i] = grads[i] ? slot + P.staging_off[(size_t)i * 3 + 1] : nullptr;
      dm[i] = reinterpret_cast<float*>(slot + P.staging_off[(size_t)i * 3 + 2]);
    }
  }
  CallTables ct{h, st};
  std::vector<MatBind> hb;
  const MatBind* db = nullptr;
  if ((rc = step_binds(h, dp.data(), dg.data(), dm.data(), shapes, count, st, hb, &db))) return rc;
  const TmapBlob* d_p_maps = nullptr;
  if ((rc = step_p_maps(h, dp.data(), hb, ns_steps, st, &d_p_maps))) return rc;

  cudaStream_t s_in = h->hs[0], s_comp = h->hs[1], s_out = h->hs[2];
  MUON_CUDA_TRY(cudaEventRecord(ev_begin, st));
  for (int k = 0; k < 3; ++k) MUON_CUDA_TRY(cudaStreamWaitEvent(h->hs[k], ev_begin, 0));
  int launches = 0;
  prof_call_begin(h);
  for (int c = 0; c < nch; ++c) {
    // Copy-in (after the slot's previous chunk has been copied out).
    if (c >= kStagingSlots) MUON_CUDA_TRY(cudaStreamWaitEvent(s_in, ev_out(c - kStagingSlots), 0));
    for (int i = P.chunk_bounds[c]; i < P.chunk_bounds[c + 1]; ++i) {
      if (!grads[i]) continue;
      const size_t numel = (size_t)P.mats[i].numel;
      const size_t gbytes = numel * ((shapes[3 * i + 2] & 1) ? 2 : 4);
      MUON_CUDA_TRY(cudaMemcpyAsync(dp[i], params[i], numel * 4, cudaMemcpyHostToDevice, s_in));
      MUON_CUDA_TRY(cudaMemcpyAsync(dm[i], momenta[i], numel * 4, cudaMemcpyHostToDevice, s_in));
      MUON_CUDA_TRY(cudaMemcpyAsync(const_cast<void*>(dg[i]), grads[i], gbytes, cudaMemcpyHostToDevice, s_in));
    }
    MUON_CUDA_TRY(cudaEventRecord(ev_in(c), s_in));
    // Compute.
    MUON_CUDA_TRY(cudaStreamWaitEvent(s_comp, ev_in(c), 0));
    if ((rc = enqueue_step_range(h, db, hb, chunk_range(P, c), lr, beta, nesterov, wd, ns_steps, abc, s_comp,
                                 &launches, d_p_maps)))
      return rc;
    MUON_CUDA_TRY(cudaEventRecord(ev_comp(c), s_comp));
    // Copy-out.
    MUON_CUDA_TRY(cudaStreamWaitEvent(s_out, ev_comp(c), 0));
    for (int i = P.chunk_bounds[c]; i < P.chunk_bounds[c + 1]; ++i) {
      if (!grads[i]) continue;
      const size_t numel = (size_t)P.mats[i].numel;
      MUON_CUDA_TRY(cudaMemcpyAsync(params[i], dp[i], numel * 4, cudaMemcpyDeviceToHost, s_out));
      MUON_CUDA_TRY(cudaMemcpyAsync(momenta[i], dm[i], numel * 4, cudaMemcpyDeviceToHost, s_out));
    }
    MUON_CUDA_TRY(cudaEventRecord(ev_out(c), s_out));
  }
  // The caller's stream resumes once every chunk is back in host memory.
  MUON_CUDA_TRY(cudaStreamWaitEvent(st, ev_out(nch - 1), 0));
  h->last_launches = launches;
  return MUON_OK;
}

int muon_momentum_norm(muon_handle* h, const void* const* grads, float* const* momenta, void* const* y,
                       double* sumsq, const int32_t* shapes, int count, float beta, int nesterov, void* stream) {
  g_last_error.clear();
  int rc;
  if ((rc = check_common(h, shapes, count))) return rc;
  if (!grads || !momenta || !y || !sumsq) return fail(MUON_ERR_INVALID_ARG, "grads, momenta, y and sumsq are required");
  if (reinterpret_cast<uintptr_t>(sumsq) % 8) return fail(MUON_ERR_INVALID_ARG, "sumsq must be 8-byte aligned");
  if (!(beta >= 0.0f && beta < 1.0f)) return fail(MUON_ERR_INVALID_ARG, "beta must be in [0, 1)");
  for (int i = 0; i < count; ++i) {
    if (!grads[i]) continue;
    if ((rc = check_ptr(grads[i], "grads", i)) || (rc = check_ptr(momenta[i], "momenta", i)) ||
        (rc = check_ptr(y[i], "y", i)))
      return rc;
  }
  DeviceGuard g(h->device);
  if (!g.ok) return fail(MUON_ERR_CUDA, "cudaSetDevice failed");
  if ((rc = ensure_plan(h, shapes, count))) return rc;
  DevPlan& P = *h->plan;
  std::vector<MatBind> hb((size_t)count);
  for (int i = 0; i < count; ++i) {
    std::memset(&hb[i], 0, sizeof(MatBind));
    hb[i].g = grads[i];
    hb[i].mom = momenta[i];
    hb[i].xout = y[i];
    hb[i].flags = shapes[3 * i + 2];
    hb[i].active = grads[i] != nullptr;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CallTables ct{h, st};
  void* d_binds = nullptr;
  if ((rc = h->binds.get(hb.data(), sizeof(MatBind) * count, nullptr, nullptr, st, &d_binds))) return rc;
  MUON_CUDA_TRY(cudaMemsetAsync(sumsq, 0, sizeof(double) * count, st));
  prof_call_begin(h);
  const ElemLaunch EL = elem_launch(P, static_cast<const MatBind*>(d_binds));
  int slot = prof_before(h, MUON_KERNEL_MOMENTUM_NORM, st);
  MUON_CUDA_TRY(launch_momentum_norm(EL, BUF_OUT, beta, nesterov ? 1 : 0, sumsq, P.partials, h->status,
                                     h->cfg.check_nonfinite, h->cfg.ns_precision == MUON_NS_FP32, st));
  prof_after(h, slot, st);
  h->last_launches = 1;
  if (P.partials) {
    slot = prof_before(h, MUON_KERNEL_NORM_REDUCE, st);
    MUON_CUDA_TRY(launch_reduce_partials(EL, 0, count, P.partials, sumsq, st));
    prof_after(h, slot, st);
    h->last_launches = 2;
  }
  return MUON_OK;
}

int muon_newton_schulz(muon_handle* h, const void* const* x_in, void* const* x_out, const double* sumsq,
                       const int32_t* shapes, int count, int ns_steps, const float* coeffs, void* stream) {
  g_last_error.clear();
  int rc;
  if ((rc = check_common(h, shapes, count))) return rc;
  if (!x_in || !x_out) return fail(MUON_ERR_INVALID_ARG, "x_in and x_out are required");
  float abc[3 * kMaxNsSteps];
  if ((rc = check_coeffs(coeffs, ns_steps, abc))) return rc;
  const size_t esz = h->cfg.ns_precision == MUON_NS_FP32 ? 4 : 2;
  for (int i = 0; i < count; ++i) {
    if ((rc = check_ptr(x_in[i], "x_in", i)) || (rc = check_ptr(x_out[i], "x_out", i))) return rc;
    const size_t bytes = (size_t)shapes[3 * i] * (size_t)round_up_i(shapes[3 * i + 1], 8) * esz;
    if (overlaps(x_in[i], bytes, x_out[i], bytes))
      return fail(MUON_ERR_INVALID_ARG, "matrix " + std::to_string(i) + ": x_in and x_out overlap");
  }
  DeviceGuard g(h->device);
  if (!g.ok) return fail(MUON_ERR_CUDA, "cudaSetDevice failed");
  if ((rc = ensure_plan(h, shapes, count))) return rc;
  DevPlan& P = *h->plan;
  std::vector<MatBind> hb((size_t)count);
  for (int i = 0; i < count; ++i) {
    std::memset(&hb[i], 0, sizeof(MatBind));
    hb[i].xin = x_in[i];
    hb[i].xout = x_out[i];
    hb[i].active = 1;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CallTables ct{h, st};
  void* d_binds = nullptr;
  if ((rc = h->binds.get(hb.data(), sizeof(MatBind) * count, nullptr, nullptr, st, &d_binds))) return rc;
  const MatBind* db = static_cast<const MatBind*>(d_binds);
  int launches = 0;
  prof_call_begin(h);
  if (ns_steps == 0) {
    const int slot = prof_before(h, MUON_KERNEL_SCALE_COPY, st);
    MUON_CUDA_TRY(launch_scale_copy(elem_launch(P, db), BUF_IN, BUF_OUT, sumsq, esz == 4, st));
    prof_after(h, slot, st);
    h->last_launches = 1;
    return MUON_OK;
  }
  const TmapBlob* d_in = nullptr;
  if (esz == 2) {
    // Tensor maps of the caller's inputs, cached by the pointer list (the
    // plan, hence every shape, is fixed while the cache lives).
    struct InCtx {
      const void* const* x_in;
      const DevPlan* plan;
    } ctx{x_in, &P};
    auto build = [](const void* c, std::vector<unsigned char>& out) -> int {
      const InCtx& ic = *static_cast<const InCtx*>(c);
      const int n = ic.plan->hp.count;
      out.assign(sizeof(TmapBlob) * kInMapsPerMat * (size_t)n, 0);
      TmapBlob* maps = reinterpret_cast<TmapBlob*>(out.data());
      for (int i = 0; i < n; ++i) {
        const int rc = encode_x_triple(maps + (size_t)i * kInMapsPerMat, ic.x_in[i], ic.plan->mats[i]);
        if (rc) return rc;
      }
      return MUON_OK;
    };
    void* dm = nullptr;
    if ((rc = h->in_maps.get(x_in, sizeof(void*) * (size_t)count, build, &ctx, st, &dm))) return rc;
    d_in = static_cast<const TmapBlob*>(dm);
  }
  int res = BUF_IN;
  if (P.grouped) {
    for (int c = 0; c + 1 < (int)P.chunk_bounds.size(); ++c)
      if ((rc = enqueue_ns(h, db, hb, chunk_range(P, c), d_in, sumsq, ns_steps, abc, BUF_IN, BUF_OUT, st, &launches,
                           &res)))
        return rc;
  } else if ((rc = enqueue_ns(h, db, hb, full_range(P), d_in, sumsq, ns_steps, abc, BUF_IN, BUF_OUT, st, &launches,
                              &res))) {
    return rc;
  }
  h->last_launches = launches;
  return MUON_OK;
}

int muon_apply(muon_handle* h, float* const* params, const void* const* o, const double* sumsq,
               const int32_t* shapes, int count, float lr, float wd, void* stream) {
  g_last_error.clear();
  int rc;
  if ((rc = check_common(h, shapes, count))) return rc;
  if (!params || !o) return fail(MUON_ERR_INVALID_ARG, "params and o are required");
  if (!std::isfinite(lr) || !std::isfinite(wd)) return fail(MUON_ERR_INVALID_ARG, "lr and wd must be finite");
  for (int i = 0; i < count; ++i) {
    if (!o[i]) continue;
    if ((rc = check_ptr(params[i], "params", i)) || (rc = check_ptr(o[i], "o", i))) return rc;
  }
  DeviceGuard g(h->device);
  if (!g.ok) return fail(MUON_ERR_CUDA, "cudaSetDevice failed");
  if ((rc = ensure_plan(h, shapes, count))) return rc;
  DevPlan& P = *h->plan;
  std::vector<MatBind> hb((size_t)count);
  for (int i = 0; i < count; ++i) {
    std::memset(&hb[i], 0, sizeof(MatBind));
    hb[i].p = params[i];
    hb[i].xin = o[i];
    hb[i].active = o[i] != nullptr;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CallTables ct{h, st};
  void* d_binds = nullptr;
  if ((rc = h->binds.get(hb.data(), sizeof(MatBind) * count, nullptr, nullptr, st, &d_binds))) return rc;
  prof_call_begin(h);
  const int slot = prof_before(h, MUON_KERNEL_APPLY, st);
  MUON_CUDA_TRY(launch_apply(elem_launch(P, static_cast<const MatBind*>(d_binds)), BUF_IN, lr, wd,
                             h->cfg.scale_mode, h->cfg.extra_scale, sumsq, h->cfg.ns_precision == MUON_NS_FP32, st));
  prof_after(h, slot, st);
  h->last_launches = 1;
  return MUON_OK;
}

int muon_plan_query(const int32_t* shapes, int count, int ns_precision, int plan_flags, int64_t* ws_bytes,
                    int64_t* region_offsets, int32_t* ntiles, int32_t* tiles, int64_t* chunk_prefix) {
  g_last_error.clear();
  if (plan_flags & ~(MUON_PLAN_SMALL_PATH | MUON_PLAN_CTA_PAIR)) return fail(MUON_ERR_INVALID_ARG, "unknown plan flags");
  HostPlan hp;
  std::string why;
  if (!build_plan(shapes, count, ns_precision, (plan_flags & MUON_PLAN_SMALL_PATH) != 0,
                  (plan_flags & MUON_PLAN_CTA_PAIR) != 0, hp, why))
    return fail(MUON_ERR_INVALID_ARG, why);
  if (ws_bytes) *ws_bytes = hp.ws_bytes;
  if (region_offsets) std::memcpy(region_offsets, hp.region_off.data(), sizeof(int64_t) * hp.region_off.size());
  if (ntiles) {
    for (int p = 0; p < 3; ++p) ntiles[p] = (int32_t)hp.tiles[p].size();
    ntiles[3] = (int32_t)hp.small.size();
  }
  if (tiles) {
    size_t k = 0;
    for (int p = 0; p < 3; ++p)
      for (const TileRec& t : hp.tiles[p]) {
        tiles[3 * k] = t.mat;
        tiles[3 * k + 1] = t.ti;
        tiles[3 * k + 2] = t.tj;
        ++k;
      }
    for (int i : hp.small) {
      tiles[3 * k] = i;
      tiles[3 * k + 1] = 0;
      tiles[3 * k + 2] = 0;
      ++k;
    }
  }
  if (chunk_prefix)
    for (int i = 0; i <= count; ++i) chunk_prefix[i] = hp.prefix[i];
  return MUON_OK;
}

int muon_workspace_size(muon_handle* h, const int32_t* shapes, int count, size_t* bytes) {
  g_last_error.clear();
  if (!h || !bytes) return fail(MUON_ERR_INVALID_ARG, "handle and bytes are required");
  HostPlan hp;
  std::string why;
  if (!build_plan(shapes, count, h->cfg.ns_precision, h->cfg.small_path != 0, h->cfg.cta_pair != 0, hp, why))
    return fail(MUON_ERR_INVALID_ARG, why);
  if (h->cfg.workspace_cap_bytes &&
      !build_plan(shapes, count, h->cfg.ns_precision, h->cfg.small_path != 0, h->cfg.cta_pair != 0, hp, why,
                  (int64_t)h->cfg.workspace_cap_bytes))
    return fail(MUON_ERR_OOM, why);
  *bytes = (size_t)hp.ws_bytes;
  return MUON_OK;
}

int muon_plan_groups(const int32_t* shapes, int count, int ns_precision, int plan_flags, size_t cap,
                     int32_t* ngroups, int32_t* group_bounds, int64_t* region_offsets, int64_t* ws_bytes) {
  g_last_error.clear();
  if (plan_flags & ~(MUON_PLAN_SMALL_PATH | MUON_PLAN_CTA_PAIR)) return fail(MUON_ERR_INVALID_ARG, "unknown plan flags");
  HostPlan hp;
  std::string why;
  const bool small = (plan_flags & MUON_PLAN_SMALL_PATH) != 0, pair = (plan_flags & MUON_PLAN_CTA_PAIR) != 0;
  if (!build_plan(shapes, count, ns_precision, small, pair, hp, why)) return fail(MUON_ERR_INVALID_ARG, why);
  if (cap && !build_plan(shapes, count, ns_precision, small, pair, hp, why, (int64_t)cap))
    return fail(MUON_ERR_OOM, why);
  const int ng = (int)hp.groups.size() - 1;
  if (ngroups) *ngroups = ng;
  if (group_bounds)
    for (int g = 0; g <= ng; ++g) group_bounds[g] = hp.groups[g];
  if (region_offsets) std::memcpy(region_offsets, hp.region_off.data(), sizeof(int64_t) * hp.region_off.size());
  if (ws_bytes) *ws_bytes = hp.ws_bytes;
  return MUON_OK;
}

int muon_workspace_ptr(muon_handle* h, void** base, size_t* bytes) {
  g_last_error.clear();
  if (!h || !base || !bytes) return fail(MUON_ERR_INVALID_ARG, "handle, base and bytes are required");
  *base = h->plan ? h->plan->ws : nullptr;
  *bytes = h->plan ? h->plan->ws_size : 0;
  return MUON_OK;
}

int muon_get_status(muon_handle* h, void* stream, int32_t* error_word, uint64_t* nonfinite_count) {
  g_last_error.clear();
  if (!h) return fail(MUON_ERR_INVALID_ARG, "handle is NULL");
  DeviceGuard g(h->device);
  MUON_CUDA_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  DevStatus s;
  MUON_CUDA_TRY(cudaMemcpy(&s, h->status, sizeof(s), cudaMemcpyDeviceToHost));
  MUON_CUDA_TRY(cudaMemset(h->status, 0, sizeof(DevStatus)));
  if (error_word) *error_word = s.error_word;
  if (nonfinite_count) *nonfinite_count = s.nonfinite;
  if (s.error_word) return fail(MUON_ERR_TIMEOUT, "a device-side wait expired (code " + std::to_string(s.error_word) + ")");
  if (s.nonfinite) return fail(MUON_ERR_NONFINITE, std::to_string(s.nonfinite) + " non-finite update entries");
  return MUON_OK;
}

int muon_profile_enable(muon_handle* h, int max_calls) {
  g_last_error.clear();
  if (!h) return fail(MUON_ERR_INVALID_ARG, "handle is NULL");
  if (max_calls < 0 || max_calls > 4096) return fail(MUON_ERR_INVALID_ARG, "max_calls must be in [0, 4096]");
  DeviceGuard g(h->device);
  MUON_CUDA_TRY(cudaDeviceSynchronize());
  prof_free(h);
  if (max_calls == 0) return MUON_OK;
  const int slots = max_calls * kProfMaxPerCall;
  h->prof_ev.assign((size_t)slots * 2, nullptr);
  h->prof_kind.assign((size_t)slots, 0);
  for (auto& e : h->prof_ev) {
    cudaError_t err = cudaEventCreate(&e);
    if (err != cudaSuccess) {
      e = nullptr;
      prof_free(h);
      return fail(MUON_ERR_CUDA, std::string("cudaEventCreate: ") + cudaGetErrorString(err));
    }
  }
  h->prof_slots = slots;
  h->prof_calls_left = max_calls;
  return MUON_OK;
}

int muon_profile_read(muon_handle* h, int32_t* kinds, float* ms, int max, int32_t* n) {
  g_last_error.clear();
  if (!h || !n) return fail(MUON_ERR_INVALID_ARG, "handle and n are required");
  DeviceGuard g(h->device);
  const int used = std::min(h->prof_used, std::max(max, 0));
  for (int k = 0; k < used; ++k) {
    MUON_CUDA_TRY(cudaEventSynchronize(h->prof_ev[2 * k + 1]));
    float t = 0.0f;
    MUON_CUDA_TRY(cudaEventElapsedTime(&t, h->prof_ev[2 * k], h->prof_ev[2 * k + 1]));
    if (kinds) kinds[k] = h->prof_kind[k];
    if (ms) ms[k] = t;
  }
  *n = used;
  const int calls = h->prof_slots / kProfMaxPerCall;
  h->prof_used = 0;
  h->prof_calls_left = calls;
  return MUON_OK;
}

int muon_last_launch_count(muon_handle* h, int32_t* launches) {
  if (!h || !launches) return fail(MUON_ERR_INVALID_ARG, "handle and launches are required");
  *launches = h->last_launches;
  return MUON_OK;
}

}  // extern "C"
