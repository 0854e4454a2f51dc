// Shared host/device definitions and sm_100a device helpers.
//
// Everything here is written for Blackwell (sm_100a): mbarriers with bounded
// waits, bulk-tensor (TMA) loads, and the tcgen05 tensor-core / tensor-memory
// instructions, all as inline PTX.
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace muon {

// A kernel's dynamic shared-memory limit is a per-device setting: raise it
// once on every device the process launches the kernel on.
template <typename Kernel>
inline cudaError_t ensure_dynamic_smem(Kernel kernel, int smem, std::atomic<unsigned long long>& done_mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit != 0 && (done_mask.load(std::memory_order_acquire) & bit) != 0) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess && bit != 0) done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}


// ---------------------------------------------------------------------------
// Plan-level and call-level per-matrix records (device resident).
// ---------------------------------------------------------------------------

// Geometry and workspace buffers of one matrix; built with the plan.
struct MatPlan {
  int m, n;          // p.shape = (fan-out, fan-in)
  int s, l;          // min(m, n), max(m, n)
  int tall;          // m > n: the iteration runs on X^T
  int ldx;           // leading dimension of X buffers (elements), round_up(n, 8)
  int lds;           // leading dimension of A and B (elements), round_up(s, 8)
  int pad_;
  long long numel;   // m * n
  void* x0;          // workspace X ping-pong buffers (m x ldx)
  void* x1;
  void* a;           // Gram A (s x lds)
  void* b;           // polynomial B (s x lds)
};

// Caller pointers of one matrix for one call.
struct MatBind {
  float* p;          // fp32 parameter (m x n, dense)
  const void* g;     // gradient (fp32 or bf16, dense); NULL = skip matrix
  float* mom;        // fp32 momentum (m x n, dense)
  const void* xin;   // caller X-layout input (stage entry points)
  void* xout;        // caller X-layout output (stage entry points)
  int flags;         // bit 0: gradient is bf16
  int active;        // 0 = skip this matrix everywhere
};

// Buffer selectors used by kernels to pick an X-layout buffer.
enum BufSel : int { BUF_X0 = 0, BUF_X1 = 1, BUF_IN = 2, BUF_OUT = 3 };

__host__ __device__ inline const void* sel_buf(const MatPlan& mp, const MatBind& mb, int sel) {
  return sel == BUF_X0 ? mp.x0 : sel == BUF_X1 ? mp.x1 : sel == BUF_IN ? mb.xin : (const void*)mb.xout;
}

// Per-handle device status block.
struct DevStatus {
  int error_word;                   // first expired wait's code, 0 = none
  int pad_;
  unsigned long long nonfinite;     // non-finite u entries seen
};

// Codes written to the error word.
enum WaitCode : int {
  WAIT_OK = 0,
  WAIT_TMA_EMPTY = 1,     // producer waiting for a free stage
  WAIT_TMA_FULL = 2,      // MMA issuer waiting for loaded operands
  WAIT_ACC_EMPTY = 3,     // MMA issuer waiting for a drained accumulator
  WAIT_ACC_FULL = 4,      // epilogue waiting for a finished accumulator
  WAIT_DRAIN = 5          // clean-up wait after an abort
};

constexpr int kElemChunk = 8192;  // elements per block in the elementwise kernels
constexpr int kMaxNsSteps = 64;   // Newton-Schulz iterations per call
constexpr double kNormEps = 1e-7; // added to ||u||_F before dividing

__host__ __device__ inline long long ceil_div_ll(long long a, long long b) { return (a + b - 1) / b; }
__host__ __device__ inline int round_up_i(int a, int b) { return (a + b - 1) / b * b; }

#if defined(__CUDACC__)

// ---------------------------------------------------------------------------
// Small device helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 1/(sqrt(sumsq) + eps) in double, or 1 when there is no norm.
__device__ __forceinline__ double inv_norm(const double* sumsq, int mat) {
  if (sumsq == nullptr) return 1.0;
  return 1.0 / (sqrt(sumsq[mat]) + kNormEps);
}

// Shape-dependent update scale of an m x n matrix ("Why Muon Works",
// configuration block; "About Muon: Why Not Adam", the program's
// 0.2 sqrt(max(m, n))) times the caller's extra factor.
__device__ __forceinline__ float update_scale_dev(int m, int n, int mode, float extra) {
  double s;
  const double dm = m, dn = n;
  switch (mode) {
    case 0: s = 0.2 * sqrt(dm > dn ? dm : dn); break;          // Moonlight
    case 1: s = sqrt((dm / dn) > 1.0 ? (dm / dn) : 1.0); break; // Jordan
    case 2: s = sqrt(dm / dn); break;                          // Bernstein
    default: s = 1.0; break;
  }
  return (float)(s * (double)extra);
}

// 1 - lr wd, rounded the same way wherever the update is applied.
__device__ __forceinline__ float apply_decay(float lr, float wd) { return __fsub_rn(1.0f, __fmul_rn(lr, wd)); }

// Multiplier of O in p' = p (1 - lr wd) - step O: lr times the update scale,
// times inv = 1/(||u|| + eps) when O was not normalised (zero iterations).
__device__ __forceinline__ float apply_step(float lr, int m, int n, int mode, float extra, double inv) {
  return (float)((double)lr * (double)update_scale_dev(m, n, mode, extra) * inv);
}

// One entry of the update from an fp32 O value: O is rounded to bf16 first,
// so the result is bitwise that of the separate apply pass, which reads the
// stored bf16 O.
__device__ __forceinline__ float apply_one(float p, float o, float decay, float step) {
  return fmaf(p, decay, -step * __bfloat162float(__float2bfloat16_rn(o)));
}

// ---------------------------------------------------------------------------
// mbarrier (shared::cta) with bounded waits
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Same test, but a thread whose phase is still incomplete may sleep up to
// `suspend_ns` in the instruction (it wakes when the phase completes), so
// waiting warps do not spin.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t suspend_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(suspend_ns)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete. Gives up when the
// shared error word is set by anyone, or after `timeout_ns` nanoseconds, in
// which case it records `code` in the error word. Returns false on give-up.
// try_wait itself suspends the thread for a short, hardware-defined time
// while the phase is incomplete, so the loop does not spin hot; the timer is
// a register read every try, the shared error word (one global address for
// every waiting warp on the GPU) is read at most every 20 microseconds.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int* err,
                                                  uint64_t timeout_ns, int code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  uint64_t next_check = t0 + 20000;
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    const uint64_t t = global_timer_ns();
    if (t - t0 > timeout_ns) {
      atomicCAS(err, 0, code);
      return false;
    }
    if (t >= next_check) {
      if (*reinterpret_cast<volatile int*>(err) != 0) return false;
      next_check = t + 20000;
    }
  }
}

// Wait with only a time limit (used while draining after an abort: the
// outstanding copy or MMA must land before the CTA frees its resources).
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > timeout_ns) return false;
  }
  return true;
}

// ---------------------------------------------------------------------------
// Bulk-tensor (TMA) loads: 2D tile, global -> shared::cta, completion on an
// mbarrier. The tensor map lives in global memory (written by the host before
// launch). No multicast.
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tma_prefetch_desc(const void* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Tile store, shared::cta -> global, tracked by this thread's bulk async
// groups. Elements outside the tensor map's extent are not written.
__device__ __forceinline__ void tma_store_2d(const void* map, const void* smem_src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(smem_src)), "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until all of this thread's bulk groups have completed.
__device__ __forceinline__ void bulk_wait_group_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (bulk copies) issued after the next synchronisation.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Tile load by one CTA of a cta_group::2 pair: the data lands in this CTA's
// shared memory, the completion is counted on the mbarrier at
// `bar_cluster_addr` (a shared::cluster address, here the leader CTA's).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const void* map, uint32_t bar_cluster_addr, int x,
                                                 int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster_addr)
      : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory allocation, MMA, commit, loads and fences.
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_slot)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive (once) on an mbarrier when all previously issued tcgen05 async ops
// of this thread have completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i gets lane (base+i).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// ---------------------------------------------------------------------------
// Thread-block clusters of two CTAs (the tcgen05 cta_group::2 pair)
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_count_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}

// shared::cluster address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_shared_rank(const void* p, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(p)), "r"(rank));
  return out;
}

// Arrive on an mbarrier given by its shared::cluster address (another CTA's).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_slot)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem of both CTAs] (+)= A * B^T over the CTA pair: M = 256 (128 rows of A
// in each CTA's shared memory), N up to 256 (N/2 rows of B in each CTA).
__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the mbarrier at the same offset in every CTA of `cta_mask`
// when all previously issued tcgen05 ops of this thread have completed.
__device__ __forceinline__ void tc_commit_pair_multicast(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

// Shared-memory matrix descriptor for tcgen05.mma (SWIZZLE_128B layouts).
//   start: shared address of the first element (16-byte units in the field)
//   lbo  : leading-dimension byte offset; sbo: stride-dimension byte offset
// K-major tiles: rows of 128 bytes, 8-row swizzle atoms of 1024 bytes,
//   sbo = 1024, lbo unused (1). MN-major tiles: 64-element (128-byte) rows
//   along M/N, 8 K-rows per 1024-byte atom; lbo = stride between 64-element
//   M/N chunks, sbo = stride between 8-row K groups.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;            // descriptor version for sm_100
  d |= (uint64_t)2u << 61;            // layout: SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4)                         // D format: f32
         | (1u << 7)                       // A format: bf16
         | (1u << 10)                      // B format: bf16
         | ((uint32_t)a_mn_major << 15)    // A major: 0 = K, 1 = MN
         | ((uint32_t)b_mn_major << 16)    // B major
         | ((uint32_t)(N >> 3) << 17)      // N / 8
         | ((uint32_t)(M >> 4) << 24);     // M / 16
}

#endif  // __CUDACC__

}  // namespace muon
