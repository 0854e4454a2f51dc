// Newton-Schulz stage for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc when they need this stage: a process
// whose device memory is entirely owned by its own pool allocator with a
// fixed budget (a cudaMalloc from outside the pool fails or steals from it),
// or a serving process that reserved its memory at start-up and must keep
// its device footprint fixed while it runs.
// muon_newton_schulz_noalloc serves them: it runs the same tensor-core
// Newton-Schulz kernels as muon_newton_schulz, but every byte of scratch it
// needs (the X ping-pong buffers, the Gram and polynomial matrices, the tile
// lists, the tensor maps and the status word) lives in one file-scope
// __device__ array of kNoallocScratchBytes. Every GPU that loads the library
// holds that array until the process exits.
//
// The host names the array only through the device address returned by
// cudaGetSymbolAddress, looked up once per device (the array's host-side
// name is a stand-in, not a device address). That set-up happens on the
// first call on each device, with that device current.
//
// Each call writes its tables (plans, tile lists, tensor maps) from host
// memory that lives only for the duration of the call, with a stream-ordered
// copy; a call on a stream that is being captured is therefore refused
// before anything is enqueued.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/muon_ns.h"
#include "common.cuh"
#include "kernels.h"
#include "plan.h"

namespace muon {
namespace {

constexpr size_t kNoallocScratchBytes = MUON_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;
constexpr double kNoallocWaitSeconds = 2.0;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

struct DeviceScratch {
  bool ready = false;
  unsigned char* base = nullptr;  // device address of g_noalloc_scratch
  int num_sms = 0;
};

std::mutex g_setup_mutex;
DeviceScratch g_scratch[kMaxDevices];

// Failures are reported through muon_last_error, like every entry point.
int noalloc_fail(int code, const std::string& msg) {
  record_last_error(msg);
  return code;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Device address of the scratch array on the current device (looked up once).
int scratch_for_current_device(DeviceScratch** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return noalloc_fail(MUON_ERR_NO_DEVICE, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return noalloc_fail(MUON_ERR_INVALID_ARG, "device index out of range");
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  DeviceScratch& ds = g_scratch[dev];
  if (!ds.ready) {
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return noalloc_fail(MUON_ERR_CUDA, std::string("cudaGetDeviceProperties: ") + cudaGetErrorString(e));
    if (prop.major != 10 || prop.minor != 0)
      return noalloc_fail(MUON_ERR_UNSUPPORTED, "device is not sm_100; this library is built for sm_100a");
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return noalloc_fail(MUON_ERR_CUDA, std::string("cudaGetSymbolAddress of the scratch array: ") +
                                             cudaGetErrorString(e));
    ds.base = static_cast<unsigned char*>(p);
    ds.num_sms = prop.multiProcessorCount;
    ds.ready = true;
  }
  *out = &ds;
  return MUON_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 row-major rows x cols (leading dimension ld), 128-byte swizzle.
int encode(TmapBlob* out, const void* base, int rows, int cols, int ld, int box_cols, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return noalloc_fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(reinterpret_cast<CUtensorMap*>(out), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
                   dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return noalloc_fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return MUON_OK;
}

int encode_x(TmapBlob* out3, const void* base, const MatPlan& mp) {
  int rc;
  if ((rc = encode(out3 + MAP_K128, base, mp.m, mp.n, mp.ldx, 64, 128))) return rc;
  if ((rc = encode(out3 + MAP_K256, base, mp.m, mp.n, mp.ldx, 64, 256))) return rc;
  return encode(out3 + MAP_MN, base, mp.m, mp.n, mp.ldx, 64, 64);
}

#define NOALLOC_CUDA_TRY(expr)                                                                            \
  do {                                                                                                    \
    cudaError_t _e = (expr);                                                                              \
    if (_e != cudaSuccess) return noalloc_fail(MUON_ERR_CUDA, std::string(#expr) + ": " + cudaGetErrorString(_e)); \
  } while (0)

}  // namespace
}  // namespace muon

using namespace muon;

extern "C" int muon_newton_schulz_noalloc(const void* const* x_in, void* const* x_out, const double* sumsq,
                                          const int32_t* shapes, int count, int ns_steps, const float* coeffs,
                                          int32_t* error_word, void* stream) {
  record_last_error(std::string());
  if (!x_in || !x_out) return noalloc_fail(MUON_ERR_INVALID_ARG, "x_in and x_out are required");
  if (ns_steps < 0 || ns_steps > 64) return noalloc_fail(MUON_ERR_INVALID_ARG, "ns_steps must be in [0, 64]");
  const float def[3] = {3.4445f, -4.7750f, 2.0315f};
  const float* abc = coeffs ? coeffs : def;
  for (int k = 0; k < 3; ++k)
    if (!std::isfinite(abc[k])) return noalloc_fail(MUON_ERR_INVALID_ARG, "coefficients must be finite");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(st, &cs);
    if (e != cudaSuccess) return noalloc_fail(MUON_ERR_CUDA, std::string("cudaStreamIsCapturing: ") + cudaGetErrorString(e));
    if (cs != cudaStreamCaptureStatusNone)
      return noalloc_fail(MUON_ERR_INVALID_ARG,
                          "muon_newton_schulz_noalloc uploads its tables from host memory that lives only during "
                          "the call; it is refused while the stream is being captured");
  }
  HostPlan hp;
  std::string why;
  if (!build_plan(shapes, count, 0, /*small_path=*/false, /*pair_tiles=*/false, hp, why)) return noalloc_fail(MUON_ERR_INVALID_ARG, why);
  for (int i = 0; i < count; ++i) {
    const void* a = x_in[i];
    const void* b = x_out[i];
    if (!a || !b) return noalloc_fail(MUON_ERR_INVALID_ARG, "x_in[" + std::to_string(i) + "] / x_out are NULL");
    if (reinterpret_cast<uintptr_t>(a) % 16 || reinterpret_cast<uintptr_t>(b) % 16)
      return noalloc_fail(MUON_ERR_INVALID_ARG, "matrix " + std::to_string(i) + ": pointers must be 16-byte aligned");
    const size_t bytes = (size_t)hp.mats[i].m * (size_t)hp.mats[i].ldx * 2;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    if (x < y + bytes && y < x + bytes)
      return noalloc_fail(MUON_ERR_INVALID_ARG, "matrix " + std::to_string(i) + ": x_in and x_out overlap");
  }

  // Layout of the scratch array: status | tables | workspace.
  size_t off = 256;                                   // DevStatus at 0
  const size_t o_mats = off;   off = align_up(off + sizeof(MatPlan) * count, 256);
  const size_t o_binds = off;  off = align_up(off + sizeof(MatBind) * count, 256);
  const size_t o_pref = off;   off = align_up(off + sizeof(long long) * (count + 1), 256);
  size_t o_tiles[3];
  for (int p = 0; p < 3; ++p) {
    o_tiles[p] = off;
    off = align_up(off + sizeof(int4) * (hp.tiles[p].size() + 1), 256);
  }
  const size_t o_maps = off;   off = align_up(off + sizeof(TmapBlob) * kMapsPerMat * count, 256);
  const size_t o_in = off;     off = align_up(off + sizeof(TmapBlob) * kInMapsPerMat * count, 1024);
  const size_t tables_end = off;
  const size_t o_ws = off;
  const size_t need = o_ws + (size_t)hp.ws_bytes;
  if (need > kNoallocScratchBytes)
    return noalloc_fail(MUON_ERR_INVALID_ARG,
                        "this shape table needs " + std::to_string(need) + " bytes of scratch; the static scratch of "
                        "muon_newton_schulz_noalloc holds " + std::to_string(kNoallocScratchBytes) +
                        " bytes (use muon_newton_schulz for larger sets)");

  DeviceScratch* ds = nullptr;
  int rc = scratch_for_current_device(&ds);
  if (rc) return rc;
  // Every matrix must live on the current device: its address goes into a
  // tensor map that this device's kernels read.
  int cur = -1;
  NOALLOC_CUDA_TRY(cudaGetDevice(&cur));
  for (int i = 0; i < count; ++i) {
    for (int k = 0; k < 2; ++k) {
      const void* ptr = k == 0 ? x_in[i] : static_cast<const void*>(x_out[i]);
      cudaPointerAttributes at;
      cudaError_t e = cudaPointerGetAttributes(&at, ptr);
      if (e != cudaSuccess) {
        cudaGetLastError();
        return noalloc_fail(MUON_ERR_INVALID_ARG, "matrix " + std::to_string(i) + ": pointer not known to CUDA");
      }
      if (at.type != cudaMemoryTypeDevice || at.device != cur)
        return noalloc_fail(MUON_ERR_INVALID_ARG, "matrix " + std::to_string(i) +
                                                      ": x_in and x_out must be device memory of the current device");
    }
  }
  unsigned char* base = ds->base;
  unsigned char* ws = base + o_ws;

  std::vector<unsigned char> host(tables_end, 0);
  MatPlan* mats = reinterpret_cast<MatPlan*>(host.data() + o_mats);
  MatBind* binds = reinterpret_cast<MatBind*>(host.data() + o_binds);
  for (int i = 0; i < count; ++i) {
    MatPlan mp = hp.mats[i];
    mp.x0 = ws + hp.region_off[(size_t)i * 4 + 0];
    mp.x1 = ws + hp.region_off[(size_t)i * 4 + 1];
    mp.a = ws + hp.region_off[(size_t)i * 4 + 2];
    mp.b = ws + hp.region_off[(size_t)i * 4 + 3];
    mats[i] = mp;
    MatBind mb;
    std::memset(&mb, 0, sizeof(mb));
    mb.xin = x_in[i];
    mb.xout = x_out[i];
    mb.active = 1;
    binds[i] = mb;
    TmapBlob* mm = reinterpret_cast<TmapBlob*>(host.data() + o_maps) + (size_t)i * kMapsPerMat;
    TmapBlob* im = reinterpret_cast<TmapBlob*>(host.data() + o_in) + (size_t)i * kInMapsPerMat;
    if ((rc = encode_x(mm + MAP_X0, mp.x0, mp)) || (rc = encode_x(mm + MAP_X1, mp.x1, mp)) ||
        (rc = encode(mm + MAP_A_K128, mp.a, mp.s, mp.s, mp.lds, 64, 128)) ||
        (rc = encode(mm + MAP_A_K256, mp.a, mp.s, mp.s, mp.lds, 64, 256)) ||
        (rc = encode(mm + MAP_B_K128, mp.b, mp.s, mp.s, mp.lds, 64, 128)) ||
        (rc = encode(mm + MAP_B_K256, mp.b, mp.s, mp.s, mp.lds, 64, 256)) ||
        (rc = encode(mm + MAP_A_MN, mp.a, mp.s, mp.s, mp.lds, 64, 64)) ||
        (rc = encode(mm + MAP_B_MN, mp.b, mp.s, mp.s, mp.lds, 64, 64)) || (rc = encode_x(im, x_in[i], mp)))
      return rc;
  }
  std::memcpy(host.data() + o_pref, hp.prefix.data(), sizeof(long long) * (count + 1));
  for (int p = 0; p < 3; ++p) {
    int4* t = reinterpret_cast<int4*>(host.data() + o_tiles[p]);
    for (size_t k = 0; k < hp.tiles[p].size(); ++k)
      t[k] = make_int4(hp.tiles[p][k].mat, hp.tiles[p][k].ti, hp.tiles[p][k].tj, 0);
  }

  DevStatus* status = reinterpret_cast<DevStatus*>(base);
  // The status word must start at zero; the tables are rewritten in full.
  // Both are stream-ordered after earlier calls on the same stream.
  NOALLOC_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(DevStatus), st));
  NOALLOC_CUDA_TRY(cudaMemcpyAsync(base + 256, host.data() + 256, tables_end - 256, cudaMemcpyHostToDevice, st));

  const MatPlan* d_mats = reinterpret_cast<const MatPlan*>(base + o_mats);
  const MatBind* d_binds = reinterpret_cast<const MatBind*>(base + o_binds);
  if (ns_steps == 0) {
    ElemLaunch EL;
    EL.plans = d_mats;
    EL.binds = d_binds;
    EL.prefix = reinterpret_cast<const long long*>(base + o_pref);
    EL.count = count;
    EL.block_base = 0;
    EL.nblocks = hp.prefix[count];
    NOALLOC_CUDA_TRY(launch_scale_copy(EL, BUF_IN, BUF_OUT, sumsq, false, st));
  } else {
    NsLaunch L;
    L.plans = d_mats;
    L.binds = d_binds;
    L.maps = reinterpret_cast<const TmapBlob*>(base + o_maps);
    L.in_maps = reinterpret_cast<const TmapBlob*>(base + o_in);
    L.sumsq = sumsq;
    L.status = status;
    L.grid = ds->num_sms;
    L.timeout_ns = (unsigned long long)(kNoallocWaitSeconds * 1e9);
    L.max_s = 0;
    for (int i = 0; i < count; ++i) L.max_s = std::max(L.max_s, hp.mats[i].s);
    int src = BUF_IN;
    for (int t = 1; t <= ns_steps; ++t) {
      const int dst = t == ns_steps ? BUF_OUT : (t % 2 == 1 ? BUF_X1 : BUF_X0);
      for (int ph = 0; ph < 3; ++ph) {
        L.tiles = reinterpret_cast<const int4*>(base + o_tiles[ph]);
        L.ntiles = (int)hp.tiles[ph].size();
        // a goes on the diagonal of B (POLY), so the combine adds no a X.
        const float a = ph == PHASE_COMB ? 0.0f : abc[0];
        NOALLOC_CUDA_TRY(launch_ns_phase_bf16(L, ph, src, dst, t == 1 ? 1 : 0, a, abc[1], abc[2], st));
      }
      src = dst;
    }
  }
  if (error_word)
    NOALLOC_CUDA_TRY(cudaMemcpyAsync(error_word, &status->error_word, sizeof(int32_t), cudaMemcpyDeviceToDevice, st));
  return MUON_OK;
}
