// fp32 debug Newton-Schulz: plain FFMA tiled GEMMs with fused epilogues
// (Gram with the alpha^2 fold, bA + cA^2, alpha (aX + BX): the program's own
// grouping, where the bf16 kernels put a on the diagonal of B instead),
// launched once per matrix and phase. Full (not symmetric) outputs. Performance is not a goal; the arithmetic is fp32 with
// fp32 accumulation so the result can be held to a tight tolerance against
// the float64 oracle.
#include "common.cuh"
#include "kernels.h"

namespace muon {

namespace {

constexpr int TM = 64, TN = 64, TK = 16;
constexpr int kThreads = 256;

// C[i][j] = sum_k opA(i, k) * opB(k, j), opA(i,k) = A[i*ars + k*acs],
// opB(k,j) = B[k*brs + j*bcs]; then the phase epilogue.
__global__ void __launch_bounds__(kThreads) ffma_phase_kernel(const float* __restrict__ A, long long ars,
                                                              long long acs, const float* __restrict__ B,
                                                              long long brs, long long bcs, int M, int N, int K,
                                                              int phase, float* __restrict__ out, int ldo,
                                                              const float* __restrict__ aux, int ldaux,
                                                              const double* __restrict__ sumsq, int mat, int first,
                                                              float a, float b, float c) {
  __shared__ float As[TK][TM + 1];
  __shared__ float Bs[TK][TN + 1];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int i0 = blockIdx.y * TM, j0 = blockIdx.x * TN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += TK) {
    for (int idx = threadIdx.x; idx < TK * TM; idx += kThreads) {
      const int kk = idx / TM, ii = idx % TM;
      const int gi = i0 + ii, gk = k0 + kk;
      As[kk][ii] = (gi < M && gk < K) ? A[gi * ars + gk * acs] : 0.0f;
    }
    for (int idx = threadIdx.x; idx < TK * TN; idx += kThreads) {
      const int kk = idx / TN, jj = idx % TN;
      const int gj = j0 + jj, gk = k0 + kk;
      Bs[kk][jj] = (gj < N && gk < K) ? B[gk * brs + gj * bcs] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) av[r] = As[kk][ty * 4 + r];
#pragma unroll
      for (int q = 0; q < 4; ++q) bv[q] = Bs[kk][tx * 4 + q];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[r][q] = fmaf(av[r], bv[q], acc[r][q]);
    }
    __syncthreads();
  }
  float sc = 1.0f;
  if (first) {
    const double al = inv_norm(sumsq, mat);
    sc = (float)(phase == PHASE_GRAM ? al * al : al);
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = i0 + ty * 4 + r;
    if (i >= M) continue;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = j0 + tx * 4 + q;
      if (j >= N) continue;
      float o;
      if (phase == PHASE_GRAM) o = acc[r][q] * sc;
      else if (phase == PHASE_POLY) o = fmaf(b, aux[(long long)i * ldaux + j], c * acc[r][q]);
      else o = sc * fmaf(a, aux[(long long)i * ldaux + j], acc[r][q]);
      out[(long long)i * ldo + j] = o;
    }
  }
}

}  // namespace

// One phase of one matrix. `mp` is the host copy of the matrix record; the
// fold factor alpha = 1/(sqrt(sumsq[mat]) + eps) of the first step is read
// on the device.
cudaError_t launch_ns_phase_fp32(const MatPlan& mp, int mat, int phase, const float* src, float* dst,
                                 const double* sumsq, int first, float a, float b, float c, cudaStream_t st) {
  const float* X = src;
  const float* Am = static_cast<const float*>(mp.a);
  const float* Bm = static_cast<const float*>(mp.b);
  const long long ldx = mp.ldx, lds = mp.lds;
  dim3 block(kThreads);
  if (phase == PHASE_GRAM) {
    const int M = mp.s, N = mp.s, K = mp.l;
    dim3 grid((N + TN - 1) / TN, (M + TM - 1) / TM);
    if (!mp.tall)  // A[i][j] = sum_k X[i][k] X[j][k]
      ffma_phase_kernel<<<grid, block, 0, st>>>(X, ldx, 1, X, 1, ldx, M, N, K, phase, static_cast<float*>(mp.a),
                                                mp.lds, nullptr, 0, sumsq, mat, first, a, b, c);
    else           // A[i][j] = sum_k X[k][i] X[k][j]
      ffma_phase_kernel<<<grid, block, 0, st>>>(X, 1, ldx, X, ldx, 1, M, N, K, phase, static_cast<float*>(mp.a),
                                                mp.lds, nullptr, 0, sumsq, mat, first, a, b, c);
  } else if (phase == PHASE_POLY) {
    const int M = mp.s, N = mp.s, K = mp.s;
    dim3 grid((N + TN - 1) / TN, (M + TM - 1) / TM);
    ffma_phase_kernel<<<grid, block, 0, st>>>(Am, lds, 1, Am, lds, 1, M, N, K, phase, static_cast<float*>(mp.b),
                                              mp.lds, Am, mp.lds, sumsq, mat, 0, a, b, c);
  } else {
    const int M = mp.m, N = mp.n, K = mp.s;
    dim3 grid((N + TN - 1) / TN, (M + TM - 1) / TM);
    if (!mp.tall)  // X'[r][c] = sc (a X[r][c] + sum_k B[r][k] X[k][c])
      ffma_phase_kernel<<<grid, block, 0, st>>>(Bm, lds, 1, X, ldx, 1, M, N, K, phase, dst, mp.ldx, X, mp.ldx, sumsq,
                                                mat, first, a, b, c);
    else           // X'[r][c] = sc (a X[r][c] + sum_k X[r][k] B[k][c])
      ffma_phase_kernel<<<grid, block, 0, st>>>(X, ldx, 1, Bm, lds, 1, M, N, K, phase, dst, mp.ldx, X, mp.ldx, sumsq,
                                                mat, first, a, b, c);
  }
  return cudaGetLastError();
}

}  // namespace muon
