// Small-matrix Newton-Schulz path: the whole iteration on chip.
//
// For a matrix with s = min(m, n) <= 128 and l = max(m, n) <= 512 one CTA
// keeps X in shared memory, forms A = X X^T (or X^T X), B = aI + bA + cA^2
// (a added to the diagonal in fp32 before B's rounding, as the tiled
// kernels do) and X <- BX (or XB) on the tensor cores with the accumulators in
// tensor memory, and runs all ns_steps iterations in one launch ("About
// Muon: Why Not Adam", sections "The lemma that makes it possible" and "The
// whole thing, in about forty lines"). Only the input and the final result
// cross HBM.
//
// Shared-memory images (128-byte swizzle, rows of 64 bf16, 8-row atoms of
// 1 KiB; element (r, c) of an image lives in 64-column chunk c/64, row r,
// 16-byte unit ((c % 64)/8) ^ (r % 8)):
//   X : row-major X in 64-column chunks. Wide (m <= n): 128 rows (rows >= m
//       are zero), ceil(n/64) chunks. Tall: round_up(m, 128) rows, 2 chunks.
//       The same bytes serve every GEMM: as K-major rows of X (wide Gram,
//       tall combine) and as M/N-major columns of X (tall Gram, wide
//       combine).
//   A, B : 128 x 128, two 64-column chunks, K-major (A and B are symmetric).
// Padding rows / columns are zero and stay zero through the iteration.
//
// One CTA of 128 threads per matrix: thread 0 issues the bulk-tensor loads
// and the tcgen05.mma instructions; all four warps run the epilogues (warp
// w reads tensor-memory lanes 32w..32w+31, i.e. output rows). Every wait is
// bounded; on expiry the error word is set, the outstanding copy or MMA is
// drained, tensor memory is freed and the CTA returns.
//
// Two sizes of the kernel: the general one (X up to 128 x 512 or 512 x 128:
// 192 KiB of shared memory and all 512 tensor-memory columns, one CTA per
// SM), and a compact one for calls whose small matrices all have
// max(m, n) <= 128 (X image 32 KiB, 96 KiB in all, 256 columns: the Gram
// accumulator in columns 0..127 is dead once the polynomial's epilogue has
// read it, and the combine reuses them), so two CTAs share an SM and hide
// each other's phase latencies.
#include "common.cuh"
#include "kernels.h"

namespace muon {

namespace {

constexpr int kThreads = 128;
constexpr int kABytes = 128 * 128 * 2;  // A image (two 16 KiB chunks)
constexpr int kChunk = 128 * 128;       // one 64-column chunk of a 128-row image

// kXBytes: X image capacity; kTmemCols: tensor-memory columns of the CTA.
template <int kXBytes>
struct __align__(1024) SmallSmem {
  uint8_t x[kXBytes];
  uint8_t a[kABytes];
  uint8_t b[kABytes];
  uint64_t load_bar;
  uint64_t mma_bar;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr int kXFull = 128 * 1024, kTmemFull = 512;      // X up to 128 x 512 / 512 x 128
constexpr int kXCompact = 32 * 1024, kTmemCompact = 256;  // X up to 128 x 128

struct SmallArgs {
  NsSmallLaunch L;
  int ns_steps, src_sel, final_sel;
  float coef[kMaxNsSteps][3];   // (a, b, c) of every step
};

__device__ __forceinline__ uint32_t swz(int r, int c, int chunk_stride) {
  return (uint32_t)((c >> 6) * chunk_stride + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1));
}

__device__ __forceinline__ void sts_row32(uint8_t* img, int r, int c0, int cs, const float (&o)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 raw;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(o[8 * q + 2 * i], o[8 * q + 2 * i + 1]);
    *reinterpret_cast<uint4*>(img + swz(r, c0 + 8 * q, cs)) = raw;
  }
}

__device__ __forceinline__ float bf16r(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

template <int kXBytes, int kTmemCols, int kMinBlocks>
__global__ void __launch_bounds__(kThreads, kMinBlocks) ns_small_kernel(const __grid_constant__ SmallArgs args) {
  extern __shared__ uint8_t smem_raw[];
  SmallSmem<kXBytes>& sm =
      *reinterpret_cast<SmallSmem<kXBytes>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const NsSmallLaunch& L = args.L;
  const int mat = L.mats[blockIdx.x];
  const MatPlan mp = L.plans[mat];
  const MatBind mb = L.binds[mat];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int* err = &L.status->error_word;
  const uint64_t tmo = L.timeout_ns;
  const uint64_t drain_tmo = tmo > 500000000ull ? tmo : 500000000ull;
  if (!mb.active) return;

  const bool tall = mp.tall != 0;
  const int x_rows = tall ? round_up_i(mp.m, 128) : 128;
  const int x_chunks = tall ? 2 : (mp.n + 63) / 64;
  const int x_cs = x_rows * 128;                    // bytes per 64-column chunk of X
  const uint32_t xs = smem_u32(sm.x), as = smem_u32(sm.a), bs = smem_u32(sm.b);

  if (tid == 0) {
    mbar_init(&sm.load_bar, 1);
    mbar_init(&sm.mma_bar, 1);
    fence_barrier_init();
    sm.abort_flag = 0;
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // Zero the A and B images once: their padding must read as zero.
  for (int i = tid * 16; i < 2 * kABytes; i += kThreads * 16)
    *reinterpret_cast<uint4*>(sm.a + i) = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // Load X (zero fill outside m x n).
  const TmapBlob* xmaps = args.src_sel == BUF_IN ? L.in_maps + (size_t)mat * kInMapsPerMat
                                                 : L.maps + (size_t)mat * kMapsPerMat +
                                                       (args.src_sel == BUF_X0 ? MAP_X0 : MAP_X1);
  uint32_t load_phase = 0, mma_phase = 0;
  bool ok = true;
  if (tid == 0) {
    const int row_blocks = x_rows / 128;
    mbar_arrive_expect_tx(&sm.load_bar, (uint32_t)(x_chunks * row_blocks * kChunk));
    for (int j = 0; j < x_chunks; ++j)
      for (int rb = 0; rb < row_blocks; ++rb)
        tma_load_2d(sm.x + j * x_cs + rb * kChunk, xmaps + MAP_K128, &sm.load_bar, 64 * j, 128 * rb);
  }
  // All threads wait for the load; the decision to stop is made uniformly.
  {
    const bool w = mbar_wait_bounded(&sm.load_bar, load_phase, err, tmo, WAIT_TMA_FULL);
    if (__syncthreads_or(!w)) {
      if (tid == 0) mbar_wait_drain(&sm.load_bar, load_phase, drain_tmo);
      ok = false;
    }
  }

  const double alpha = inv_norm(L.sumsq, mat);
  for (int t = 1; t <= args.ns_steps && ok; ++t) {
    const bool first = t == 1;
    const bool last = t == args.ns_steps;
    const float ca = args.coef[t - 1][0], cb = args.coef[t - 1][1], cc = args.coef[t - 1][2];

    // ---------------- Gram: TMEM columns [0, 128) ----------------
    if (tid == 0) {
      tc_fence_after();
      if (!tall) {   // A = X X^T, K = the columns of X
        const uint32_t idesc = umma_idesc_bf16(128, 128, 0, 0);
        for (int k = 0; k < x_chunks * 4; ++k) {
          const uint64_t d = umma_desc_sw128(xs + (k >> 2) * x_cs + (k & 3) * 32, 16, 1024);
          tc_mma_bf16(tmem, d, d, idesc, k != 0);
        }
      } else {       // A = X^T X, K = the rows of X; both operands M/N-major
        const uint32_t idesc = umma_idesc_bf16(128, 128, 1, 1);
        for (int k = 0; k < x_rows / 16; ++k) {
          const uint64_t d = umma_desc_sw128(xs + k * 2048, (uint32_t)x_cs, 1024);
          tc_mma_bf16(tmem, d, d, idesc, k != 0);
        }
      }
      tc_commit(&sm.mma_bar);
    }
    {
      const bool w = mbar_wait_bounded(&sm.mma_bar, mma_phase, err, tmo, WAIT_ACC_FULL);
      if (__syncthreads_or(!w)) {
        if (tid == 0) mbar_wait_drain(&sm.mma_bar, mma_phase, drain_tmo);
        ok = false;
        break;
      }
      mma_phase ^= 1u;
    }
    tc_fence_after();
    const float sc_gram = first ? (float)(alpha * alpha) : 1.0f;
    const int row = warp * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
    for (int c0 = 0; c0 < 128; c0 += 32) {
      float v[32];
      tmem_ld_32x32b_x32(lane_base + (uint32_t)c0, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= sc_gram;
      sts_row32(sm.a, row, c0, kChunk, v);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---------------- Polynomial: TMEM columns [128, 256) ----------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = umma_idesc_bf16(128, 128, 0, 0);
      for (int k = 0; k < 8; ++k) {
        const uint64_t d = umma_desc_sw128(as + (k >> 2) * kChunk + (k & 3) * 32, 16, 1024);
        tc_mma_bf16(tmem + 128, d, d, idesc, k != 0);
      }
      tc_commit(&sm.mma_bar);
    }
    {
      const bool w = mbar_wait_bounded(&sm.mma_bar, mma_phase, err, tmo, WAIT_ACC_FULL);
      if (__syncthreads_or(!w)) {
        if (tid == 0) mbar_wait_drain(&sm.mma_bar, mma_phase, drain_tmo);
        ok = false;
        break;
      }
      mma_phase ^= 1u;
    }
    tc_fence_after();
#pragma unroll 1
    for (int c0 = 0; c0 < 128; c0 += 32) {
      float av[32], pv[32];
      tmem_ld_32x32b_x32(lane_base + (uint32_t)c0, av);          // A (fp32, before rounding)
      tmem_ld_32x32b_x32(lane_base + 128u + (uint32_t)c0, pv);   // A A
      // B + a I: the chunk whose columns are this warp's rows holds the
      // diagonal, lane i at column i.
      const int dcol = (c0 == warp * 32 && row < mp.s) ? lane : -1;
#pragma unroll
      for (int i = 0; i < 32; ++i) pv[i] = fmaf(cb, bf16r(av[i] * sc_gram), cc * pv[i]) + (i == dcol ? ca : 0.0f);
      sts_row32(sm.b, row, c0, kChunk, pv);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---------------- Combine ----------------
    if (tid == 0) {
      tc_fence_after();
      if (!tall) {   // D = B X: M = 128 rows of B, N = columns of X (<= 256 per MMA), K = 128
        for (int p = 0; p * 4 < x_chunks; ++p) {
          const int nch = min(4, x_chunks - 4 * p);
          const uint32_t idesc = umma_idesc_bf16(128, 64 * nch, 0, 1);
          for (int k = 0; k < 8; ++k) {
            const uint64_t da = umma_desc_sw128(bs + (k >> 2) * kChunk + (k & 3) * 32, 16, 1024);
            const uint64_t db = umma_desc_sw128(xs + 4 * p * x_cs + k * 2048, (uint32_t)x_cs, 1024);
            tc_mma_bf16(tmem + (uint32_t)(256 * p), da, db, idesc, k != 0);
          }
        }
      } else {       // D = X B: M = rows of X in blocks of 128, N = 128, K = 128
        const uint32_t idesc = umma_idesc_bf16(128, 128, 0, 0);
        for (int mb = 0; mb < x_rows / 128; ++mb) {
          for (int k = 0; k < 8; ++k) {
            const uint64_t da = umma_desc_sw128(xs + (k >> 2) * x_cs + mb * kChunk + (k & 3) * 32, 16, 1024);
            const uint64_t db = umma_desc_sw128(bs + (k >> 2) * kChunk + (k & 3) * 32, 16, 1024);
            tc_mma_bf16(tmem + (uint32_t)(128 * mb), da, db, idesc, k != 0);
          }
        }
      }
      tc_commit(&sm.mma_bar);
    }
    {
      const bool w = mbar_wait_bounded(&sm.mma_bar, mma_phase, err, tmo, WAIT_ACC_FULL);
      if (__syncthreads_or(!w)) {
        if (tid == 0) mbar_wait_drain(&sm.mma_bar, mma_phase, drain_tmo);
        ok = false;
        break;
      }
      mma_phase ^= 1u;
    }
    tc_fence_after();
    const float sc = first ? (float)alpha : 1.0f;
    __nv_bfloat16* gdst = last ? static_cast<__nv_bfloat16*>(const_cast<void*>(sel_buf(mp, mb, args.final_sel)))
                               : nullptr;
    const int blocks = tall ? x_rows / 128 : 1;
    const int cols = tall ? 128 : x_chunks * 64;
    for (int blk = 0; blk < blocks; ++blk) {
      const int r = blk * 128 + row;        // row of X
#pragma unroll 1
      for (int c0 = 0; c0 < cols; c0 += 32) {
        float v[32];
        tmem_ld_32x32b_x32(lane_base + (uint32_t)(blk * 128 + c0), v);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= sc;
        if (!last) {
          sts_row32(sm.x, r, c0, x_cs, v);
        } else if (r < mp.m && c0 < mp.n) {
          __nv_bfloat16* dst = gdst + (size_t)r * mp.ldx + c0;
          if (c0 + 32 <= mp.n) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 raw;
              __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
              for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[8 * q + 2 * i], v[8 * q + 2 * i + 1]);
              reinterpret_cast<uint4*>(dst)[q] = raw;
            }
          } else {
            for (int i = 0; i < 32 && c0 + i < mp.n; ++i) dst[i] = __float2bfloat16_rn(v[i]);
          }
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

int ns_small_smem_bytes() { return (int)sizeof(SmallSmem<kXFull>) + 1024; }

cudaError_t launch_ns_small(const NsSmallLaunch& L, int ns_steps, int src_sel, int final_sel, const float* abc,
                            cudaStream_t st) {
  if (L.nmats <= 0 || ns_steps <= 0) return cudaSuccess;
  if (ns_steps > kMaxNsSteps) return cudaErrorInvalidValue;
  SmallArgs args;
  args.L = L;
  args.ns_steps = ns_steps;
  args.src_sel = src_sel;
  args.final_sel = final_sel;
  for (int t = 0; t < ns_steps; ++t)
    for (int k = 0; k < 3; ++k) args.coef[t][k] = abc[3 * t + k];
  if (L.max_l <= 128) {
    static std::atomic<unsigned long long> attr_done{0};
    const int smem = (int)sizeof(SmallSmem<kXCompact>) + 1024;
    auto kern = ns_small_kernel<kXCompact, kTmemCompact, 2>;
    const cudaError_t e = ensure_dynamic_smem(kern, smem, attr_done);
    if (e != cudaSuccess) return e;
    kern<<<L.nmats, kThreads, smem, st>>>(args);
  } else {
    static std::atomic<unsigned long long> attr_done{0};
    const int smem = ns_small_smem_bytes();
    auto kern = ns_small_kernel<kXFull, kTmemFull, 1>;
    const cudaError_t e = ensure_dynamic_smem(kern, smem, attr_done);
    if (e != cudaSuccess) return e;
    kern<<<L.nmats, kThreads, smem, st>>>(args);
  }
  return cudaGetLastError();
}

}  // namespace muon
