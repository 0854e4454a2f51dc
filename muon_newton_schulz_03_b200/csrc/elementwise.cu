// Elementwise stages of the Muon step, grouped over all matrices of a call.
//
// K1 "momentum_norm": momentum EMA, Nesterov blend, per-matrix sum of squares
//    of the update direction u, and the cast of u to the Newton-Schulz input.
//    ("About Muon: Why Not Adam", section "The whole thing, in about forty
//    lines": buf.lerp_(grad, 1 - mu), grad.lerp(buf, mu), the cast and the
//    Frobenius norm that Newton-Schulz divides by; Nesterov: "Por que AdamW
//    ...", section "Momentum: recordar el paso anterior".)
// K4 "apply": decoupled weight decay and the scaled orthogonalised update
//    (same program: p.mul_(1 - lr*wd), p.add_(O, alpha=-lr*scale); the scale
//    families from "How Do We Turn It Into a Real Optimizer?" and "The
//    spectral ball gives UV^T").
// K0 "scale_copy": out = alpha * in (the zero-iteration Newton-Schulz stage).
//
// All three are HBM-bound: each thread block takes kElemChunk consecutive
// elements of one matrix (block -> matrix by binary search over the chunk
// prefix), loads and stores are 16-byte vectors when a row length is a
// multiple of 8, and the sum of squares is reduced thread -> warp -> block
// with one double-precision atomic per block.
#include "common.cuh"
#include "kernels.h"

namespace muon {

namespace {

constexpr int kThreads = 256;
constexpr int kVec = 8;                                   // elements per vector step
constexpr int kIters = kElemChunk / (kThreads * kVec);    // 4
static_assert(kIters * kThreads * kVec == kElemChunk, "chunk must tile evenly");

__device__ __forceinline__ int find_matrix(const long long* prefix, int count, long long block) {
  int lo = 0, hi = count;  // prefix[lo] <= block < prefix[hi]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (__ldg(prefix + mid) <= block) lo = mid; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ void load8_f32(const float* p, float (&v)[8]) {
  float4 a = __ldcs(reinterpret_cast<const float4*>(p));
  float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void store8_f32(float* p, const float (&v)[8]) {
  __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
  __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(v[4], v[5], v[6], v[7]));
}

__device__ __forceinline__ void load8_bf16(const __nv_bfloat16* p, float (&v)[8]) {
  uint4 raw = __ldcs(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ void store8_bf16(__nv_bfloat16* p, const float (&v)[8]) {
  uint4 raw;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = raw;
}

__device__ __forceinline__ double block_sum(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  if (warp == 0) {
    t = lane < (kThreads / 32) ? red[lane] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  }
  return t;  // valid in thread 0
}

__device__ __forceinline__ unsigned block_count(unsigned v, unsigned* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  unsigned t = 0;
  if (warp == 0) {
    t = lane < (kThreads / 32) ? red[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  }
  return t;
}

// Momentum, Nesterov blend and u for one element (fp32, the lerp forms).
__device__ __forceinline__ float momentum_u(float g, float& m, float beta, float one_minus_beta, int nesterov) {
  const float mn = fmaf(beta, m, one_minus_beta * g);   // beta*m + (1-beta)*g
  m = mn;
  return nesterov ? fmaf(beta, mn - g, g) : mn;          // g + beta*(m' - g)
}

template <bool kFp32Out>
__global__ void __launch_bounds__(kThreads) k1_momentum_norm(
    const MatPlan* __restrict__ plans, const MatBind* __restrict__ binds, const long long* __restrict__ prefix,
    int count, long long block_base, int ysel, float beta, int nesterov, double* __restrict__ sumsq,
    double* __restrict__ partials, DevStatus* status, int check_nonfinite) {
  __shared__ double red[kThreads / 32];
  __shared__ unsigned redc[kThreads / 32];
  const long long blk = (long long)blockIdx.x + block_base;
  const int mat = find_matrix(prefix, count, blk);
  const MatBind mb = binds[mat];
  if (!mb.active || mb.g == nullptr) return;
  const MatPlan mp = plans[mat];
  const long long e0 = (blk - prefix[mat]) * (long long)kElemChunk;
  const long long e1 = min(e0 + (long long)kElemChunk, mp.numel);
  const float omb = 1.0f - beta;
  void* ybase = const_cast<void*>(sel_buf(mp, mb, ysel));
  const bool g_bf16 = (mb.flags & 1) != 0;

  double acc = 0.0;
  unsigned bad = 0;
  if ((mp.n % kVec) == 0 && e1 - e0 == kElemChunk) {
    // Whole chunk, dense X layout: the loads of vector step it + 1 are issued
    // before the stores of step it, so each thread keeps two steps in flight.
    const long long eb = e0 + (long long)threadIdx.x * kVec;
    float g[2][8], m[2][8];
    auto load = [&](int it, int b) {
      const long long e = eb + (long long)it * kThreads * kVec;
      if (g_bf16) load8_bf16(static_cast<const __nv_bfloat16*>(mb.g) + e, g[b]);
      else load8_f32(static_cast<const float*>(mb.g) + e, g[b]);
      load8_f32(mb.mom + e, m[b]);
    };
    load(0, 0);
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
      const int b = it & 1;
      if (it + 1 < kIters) load(it + 1, b ^ 1);
      const long long e = eb + (long long)it * kThreads * kVec;
      float u[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        u[i] = momentum_u(g[b][i], m[b][i], beta, omb, nesterov);
        acc += (double)u[i] * (double)u[i];
        if (check_nonfinite) bad += !isfinite(u[i]);
      }
      store8_f32(mb.mom + e, m[b]);
      if (kFp32Out) store8_f32(static_cast<float*>(ybase) + e, u);
      else store8_bf16(static_cast<__nv_bfloat16*>(ybase) + e, u);
    }
  } else if ((mp.n % kVec) == 0) {
    // ldx == n: the X layout is dense, element e maps to offset e.
    for (int it = 0; it < kIters; ++it) {
      const long long e = e0 + ((long long)it * kThreads + threadIdx.x) * kVec;
      if (e >= e1) break;
      float g[8], m[8], u[8];
      if (g_bf16) load8_bf16(static_cast<const __nv_bfloat16*>(mb.g) + e, g);
      else load8_f32(static_cast<const float*>(mb.g) + e, g);
      load8_f32(mb.mom + e, m);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        u[i] = momentum_u(g[i], m[i], beta, omb, nesterov);
        acc += (double)u[i] * (double)u[i];
        if (check_nonfinite) bad += !isfinite(u[i]);
      }
      store8_f32(mb.mom + e, m);
      if (kFp32Out) store8_f32(static_cast<float*>(ybase) + e, u);
      else store8_bf16(static_cast<__nv_bfloat16*>(ybase) + e, u);
    }
  } else {
    for (long long e = e0 + threadIdx.x; e < e1; e += kThreads) {
      const float g = g_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(mb.g)[e])
                             : static_cast<const float*>(mb.g)[e];
      float m = mb.mom[e];
      const float u = momentum_u(g, m, beta, omb, nesterov);
      mb.mom[e] = m;
      acc += (double)u * (double)u;
      if (check_nonfinite) bad += !isfinite(u);
      const long long r = e / mp.n, c = e - r * mp.n;
      const long long off = r * mp.ldx + c;
      if (kFp32Out) static_cast<float*>(ybase)[off] = u;
      else static_cast<__nv_bfloat16*>(ybase)[off] = __float2bfloat16_rn(u);
    }
  }
  const double tot = block_sum(acc, red);
  if (threadIdx.x == 0) {
    if (partials != nullptr) partials[blk] = tot;   // fixed-order sum later
    else atomicAdd(sumsq + mat, tot);
  }
  if (check_nonfinite) {
    __syncthreads();
    const unsigned nb = block_count(bad, redc);
    if (threadIdx.x == 0 && nb) atomicAdd(&status->nonfinite, (unsigned long long)nb);
  }
}

// Deterministic norm: one warp per matrix adds that matrix's per-block
// partial sums in a fixed order (lane-strided, then a fixed shuffle tree).
__global__ void __launch_bounds__(kThreads) k1b_reduce_partials(const MatBind* __restrict__ binds,
                                                                const long long* __restrict__ prefix, int m0,
                                                                int m1, const double* __restrict__ partials,
                                                                double* __restrict__ sumsq) {
  const int mat = m0 + (int)((blockIdx.x * (unsigned)kThreads + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (mat >= m1) return;
  const MatBind mb = binds[mat];
  if (!mb.active || mb.g == nullptr) return;
  const long long b0 = prefix[mat], b1 = prefix[mat + 1];
  double v = 0.0;
  for (long long b = b0 + lane; b < b1; b += 32) v += partials[b];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) sumsq[mat] = v;
}

template <bool kFp32In>
__global__ void __launch_bounds__(kThreads) k4_apply(const MatPlan* __restrict__ plans,
                                                     const MatBind* __restrict__ binds,
                                                     const long long* __restrict__ prefix, int count,
                                                     long long block_base, int osel, float lr, float wd,
                                                     int scale_mode, float extra_scale,
                                                     const double* __restrict__ sumsq) {
  const long long blk = (long long)blockIdx.x + block_base;
  const int mat = find_matrix(prefix, count, blk);
  const MatBind mb = binds[mat];
  if (!mb.active) return;
  const MatPlan mp = plans[mat];
  const void* obase = sel_buf(mp, mb, osel);
  if (obase == nullptr) return;
  const long long e0 = (blk - prefix[mat]) * (long long)kElemChunk;
  const long long e1 = min(e0 + (long long)kElemChunk, mp.numel);
  const float decay = apply_decay(lr, wd);
  const float step = apply_step(lr, mp.m, mp.n, scale_mode, extra_scale, inv_norm(sumsq, mat));
  if ((mp.n % kVec) == 0 && e1 - e0 == kElemChunk) {
    // Whole chunk: two vector steps in flight per thread, as in K1.
    const long long eb = e0 + (long long)threadIdx.x * kVec;
    float p[2][8], o[2][8];
    auto load = [&](int it, int b) {
      const long long e = eb + (long long)it * kThreads * kVec;
      load8_f32(mb.p + e, p[b]);
      if (kFp32In) load8_f32(static_cast<const float*>(obase) + e, o[b]);
      else load8_bf16(static_cast<const __nv_bfloat16*>(obase) + e, o[b]);
    };
    load(0, 0);
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
      const int b = it & 1;
      if (it + 1 < kIters) load(it + 1, b ^ 1);
      const long long e = eb + (long long)it * kThreads * kVec;
#pragma unroll
      for (int i = 0; i < 8; ++i) p[b][i] = fmaf(p[b][i], decay, -step * o[b][i]);
      store8_f32(mb.p + e, p[b]);
    }
  } else if ((mp.n % kVec) == 0) {
    for (int it = 0; it < kIters; ++it) {
      const long long e = e0 + ((long long)it * kThreads + threadIdx.x) * kVec;
      if (e >= e1) break;
      float p[8], o[8];
      load8_f32(mb.p + e, p);
      if (kFp32In) load8_f32(static_cast<const float*>(obase) + e, o);
      else load8_bf16(static_cast<const __nv_bfloat16*>(obase) + e, o);
#pragma unroll
      for (int i = 0; i < 8; ++i) p[i] = fmaf(p[i], decay, -step * o[i]);
      store8_f32(mb.p + e, p);
    }
  } else {
    for (long long e = e0 + threadIdx.x; e < e1; e += kThreads) {
      const long long r = e / mp.n, c = e - r * mp.n;
      const long long off = r * mp.ldx + c;
      const float o = kFp32In ? static_cast<const float*>(obase)[off]
                              : __bfloat162float(static_cast<const __nv_bfloat16*>(obase)[off]);
      mb.p[e] = fmaf(mb.p[e], decay, -step * o);
    }
  }
}

template <bool kFp32>
__global__ void __launch_bounds__(kThreads) k0_scale_copy(const MatPlan* __restrict__ plans,
                                                          const MatBind* __restrict__ binds,
                                                          const long long* __restrict__ prefix, int count,
                                                          long long block_base, int isel, int osel,
                                                          const double* __restrict__ sumsq) {
  const long long blk = (long long)blockIdx.x + block_base;
  const int mat = find_matrix(prefix, count, blk);
  const MatBind mb = binds[mat];
  if (!mb.active) return;
  const MatPlan mp = plans[mat];
  const void* in = sel_buf(mp, mb, isel);
  void* out = const_cast<void*>(sel_buf(mp, mb, osel));
  const float alpha = (float)inv_norm(sumsq, mat);
  const long long e0 = (blk - prefix[mat]) * (long long)kElemChunk;
  const long long e1 = min(e0 + (long long)kElemChunk, mp.numel);
  for (long long e = e0 + threadIdx.x; e < e1; e += kThreads) {
    const long long r = e / mp.n, c = e - r * mp.n;
    const long long off = r * mp.ldx + c;
    if (kFp32) static_cast<float*>(out)[off] = alpha * static_cast<const float*>(in)[off];
    else
      static_cast<__nv_bfloat16*>(out)[off] =
          __float2bfloat16_rn(alpha * __bfloat162float(static_cast<const __nv_bfloat16*>(in)[off]));
  }
}

// QK-Clip ("The Optimizer Wars", MuonClip): after the update, the rows of
// head h of W_q or W_k are multiplied by sqrt(gamma_h), gamma_h =
// min(1, tau / S_max^h), so the head's q.k logits shrink by gamma_h.
__global__ void __launch_bounds__(kThreads) k5_qk_clip(float* __restrict__ w, long long rows, long long cols,
                                                       int head_rows, const float* __restrict__ s_max, float tau) {
  const long long n = rows * cols;
  for (long long e = (long long)blockIdx.x * kThreads + threadIdx.x; e < n; e += (long long)gridDim.x * kThreads) {
    const long long r = e / cols;
    const float s = s_max[r / head_rows];
    if (s > tau) w[e] *= sqrtf(tau / s);     // false for NaN: no clip
  }
}

}  // namespace

cudaError_t launch_qk_clip(float* w, long long rows, long long cols, int head_rows, const float* s_max, float tau,
                           cudaStream_t st) {
  const long long n = rows * cols;
  if (n <= 0) return cudaSuccess;
  long long blocks = (n + kThreads - 1) / kThreads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  k5_qk_clip<<<(unsigned)blocks, kThreads, 0, st>>>(w, rows, cols, head_rows, s_max, tau);
  return cudaGetLastError();
}

cudaError_t launch_momentum_norm(const ElemLaunch& L, int ysel, float beta, int nesterov, double* sumsq,
                                 double* partials, DevStatus* status, int check_nonfinite, bool fp32_out,
                                 cudaStream_t st) {
  if (L.nblocks <= 0) return cudaSuccess;
  if (fp32_out)
    k1_momentum_norm<true><<<(unsigned)L.nblocks, kThreads, 0, st>>>(L.plans, L.binds, L.prefix, L.count,
                                                                      L.block_base, ysel, beta, nesterov, sumsq,
                                                                      partials, status, check_nonfinite);
  else
    k1_momentum_norm<false><<<(unsigned)L.nblocks, kThreads, 0, st>>>(L.plans, L.binds, L.prefix, L.count,
                                                                       L.block_base, ysel, beta, nesterov, sumsq,
                                                                       partials, status, check_nonfinite);
  return cudaGetLastError();
}

cudaError_t launch_reduce_partials(const ElemLaunch& L, int m0, int m1, const double* partials, double* sumsq,
                                   cudaStream_t st) {
  if (m1 <= m0) return cudaSuccess;
  const int warps_per_block = kThreads / 32;
  const unsigned grid = (unsigned)((m1 - m0 + warps_per_block - 1) / warps_per_block);
  k1b_reduce_partials<<<grid, kThreads, 0, st>>>(L.binds, L.prefix, m0, m1, partials, sumsq);
  return cudaGetLastError();
}

cudaError_t launch_apply(const ElemLaunch& L, int osel, float lr, float wd, int scale_mode, float extra_scale,
                         const double* sumsq, bool fp32_in, cudaStream_t st) {
  if (L.nblocks <= 0) return cudaSuccess;
  if (fp32_in)
    k4_apply<true><<<(unsigned)L.nblocks, kThreads, 0, st>>>(L.plans, L.binds, L.prefix, L.count, L.block_base, osel, lr, wd,
                                                             scale_mode, extra_scale, sumsq);
  else
    k4_apply<false><<<(unsigned)L.nblocks, kThreads, 0, st>>>(L.plans, L.binds, L.prefix, L.count, L.block_base, osel, lr, wd,
                                                              scale_mode, extra_scale, sumsq);
  return cudaGetLastError();
}

cudaError_t launch_scale_copy(const ElemLaunch& L, int isel, int osel, const double* sumsq, bool fp32,
                              cudaStream_t st) {
  if (L.nblocks <= 0) return cudaSuccess;
  if (fp32)
    k0_scale_copy<true><<<(unsigned)L.nblocks, kThreads, 0, st>>>(L.plans, L.binds, L.prefix, L.count, L.block_base, isel, osel,
                                                                  sumsq);
  else
    k0_scale_copy<false><<<(unsigned)L.nblocks, kThreads, 0, st>>>(L.plans, L.binds, L.prefix, L.count, L.block_base, isel,
                                                                   osel, sumsq);
  return cudaGetLastError();
}

}  // namespace muon
