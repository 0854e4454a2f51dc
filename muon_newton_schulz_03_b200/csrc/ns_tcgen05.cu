// Newton-Schulz phases on the 5th-generation tensor cores (sm_100a).
//
// One quintic step ("About Muon: Why Not Adam", sections "The lemma that
// makes it possible" and "The whole thing, in about forty lines") is three
// grouped launches of this persistent kernel over all matrices of a call:
//   GRAM : A = X X^T            (wide, X is s x l)   or  X^T X  (tall)
//   POLY : B = a I + b A + c A A   (A symmetric)
//   COMB : X' = B X             (wide)               or  X B  (tall;
//                                                         B is symmetric)
// so that X' = a X + (b A + c A^2) X: a sits on B's diagonal, added in fp32
// before B's one bf16 rounding, and the combine is a bare product whose
// epilogue reads nothing but the accumulator. (The Gram form, which runs the
// polynomial with a = 0, asks the combine for a X itself: a != 0 there.)
// Gram and polynomial outputs are symmetric: only tiles on or right of the
// 256-block diagonal are computed and stored, so a symmetric buffer holds its
// upper 256-block triangle (diagonal blocks whole). Its lower part is the
// mirror image of the upper, taken at load time: a consumer that needs a
// K-block below the diagonal block of its operand rows loads it transposed
// (M/N-major boxes) from the stored block above the diagonal, and the MMA
// takes that K-block with M/N-major operand layout. Tall matrices (m > n) are
// never transposed in memory: the Gram reads X with M/N-major operand tiles,
// and the combine computes X B instead of B X^T.
// The Frobenius normalisation X0 = Y/(||u|| + eps) of the first step is
// folded into its epilogues: A0 = alpha^2 Y Y^T and X1 = alpha B0 Y.
//
// Structure of one CTA (192 threads, one CTA per SM, persistent over a
// static round-robin tile list):
//   warp 0     : bulk-tensor (TMA) producer, 4-stage shared-memory ring
//   warp 1     : tensor-memory allocator and single-thread tcgen05.mma issuer
//   warps 2..5 : epilogue; tcgen05.ld of a 128 x 256 fp32 accumulator,
//                fused polynomial, bf16 round-to-nearest-even stores
// Two accumulators in tensor memory (2 x 256 columns) let the epilogue of
// one tile overlap the main loop of the next.
// Every wait is bounded: on expiry the error word is set, every role stops,
// in-flight copies and MMAs are drained and tensor memory is freed.
#include <cmath>
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace muon {

namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int kStages = 4;
constexpr int kABytes = BM * BK * 2;            // 16 KiB
constexpr int kBBytes = BN * BK * 2;            // 32 KiB
constexpr int kStageBytes = kABytes + kBBytes;  // 48 KiB
constexpr int kMnChunkBytes = 64 * BK * 2;      // one 64 (M/N) x 64 (K) box, 8 KiB
constexpr int kThreads = 192;
constexpr int kTmemCols = 2 * BN;               // two fp32 accumulators
constexpr int kOutBox = 32;                     // bulk-store box: 32 rows x 32 columns
constexpr int kOutStageBytes = kOutBox * kOutBox * 2;
constexpr int kAuxTmaMinK = 2048;               // combine tiles with K >= this read X by bulk loads
// A polynomial launch whose matrices all have s below this takes b A on the
// tensor cores (short tiles: the epilogue, not the MMA, is the critical
// path); longer ones read A through bulk loads in the epilogue.
constexpr int kIdentMaxS = 2048;

struct __align__(1024) SmemLayout {
  uint8_t stage[kStages][kStageBytes];
  // Epilogue staging, per epilogue warp: two 32 x 32 bf16 output blocks for
  // bulk stores and two blocks for bulk loads of the auxiliary operand
  // (64-byte rows, 64-byte swizzle). A polynomial launch that takes b A on
  // the tensor cores holds its two scaled 64 x 64 identities in the 16 KiB
  // of auxiliary blocks instead (128-byte swizzle; 1024-byte aligned).
  uint8_t ostage[4][2][kOutStageBytes];
  uint8_t auxstage[4][2][kOutStageBytes];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint64_t aux_full[4][2];   // per epilogue warp: bulk loads of the combine's X blocks
  uint32_t tmem_base;
};

struct NsArgs {
  NsLaunch L;
  int phase, src_sel, dst_sel, first;
  float a, b, c;
  PhaseSpec spec;
  // Polynomial launches with c != 0 over short matrices (s < kIdentMaxS):
  // B = c (A A + q A) + a I, q = b / c split into two bf16 values (hi + lo)
  // whose scaled identities the MMA multiplies A by.
  int poly_ident;
  uint32_t ident_bits;   // bf16 bits of hi (low half) and lo (high half)
  int ident_parts;       // identities to apply: 0 when b == 0, 1 when lo == 0, else 2
};

constexpr int kIdentBytes = 64 * BK * 2;   // one 64 x 64 bf16 identity, 8 KiB

// Everything a role needs to know about one tile.
struct TileJob {
  int mat, ti, tj;
  int kblocks;
  const void* map_a;
  const void* map_b;
  int a_mn, b_mn;      // operand majorness: 0 = K-major, 1 = M/N-major
  int a_coord, b_coord;  // K-major: first row; M/N-major: first M/N index
  // Operand rows from a symmetric buffer (upper 256-block triangle stored):
  // K-blocks left of the rows' diagonal block come transposed through the
  // 64 x 64 map.
  int a_sym, b_sym;
  const void* map_a_mn;
  const void* map_b_mn;
};

// K-block kb of operand rows starting at r0 of a symmetric buffer is below
// the stored triangle (its 256-column block lies left of the rows' 256-block).
__device__ __forceinline__ bool below_stored(int r0, int kb) { return (kb * BK) / 256 < r0 / 256; }

__device__ __forceinline__ const TmapBlob* src_maps(const NsLaunch& L, int mat, int src_sel) {
  if (src_sel == BUF_IN) return L.in_maps + (size_t)mat * kInMapsPerMat;
  return L.maps + (size_t)mat * kMapsPerMat + (src_sel == BUF_X0 ? MAP_X0 : MAP_X1);
}

// Tensor map of an s x s buffer: K-major box of 128 rows (or 256).
__device__ __forceinline__ const TmapBlob* sym_map(const NsLaunch& L, int mat, int id, bool rows256) {
  if (id == SB_A) return L.maps + (size_t)mat * kMapsPerMat + (rows256 ? MAP_A_K256 : MAP_A_K128);
  if (id == SB_B) return L.maps + (size_t)mat * kMapsPerMat + (rows256 ? MAP_B_K256 : MAP_B_K128);
  return L.gmaps + (size_t)mat * kGramMapsPerMat + (id == SB_T ? 0 : 2) + (rows256 ? 1 : 0);
}

// 64 x 64 map of an s x s buffer (transposed loads of the missing triangle).
__device__ __forceinline__ const TmapBlob* sym_map_mn(const NsLaunch& L, int mat, int id) {
  if (id == SB_A) return L.maps + (size_t)mat * kMapsPerMat + MAP_A_MN;
  if (id == SB_B) return L.maps + (size_t)mat * kMapsPerMat + MAP_B_MN;
  return L.gmaps + (size_t)mat * kGramMapsPerMat + (id == SB_T ? 6 : 7);
}

__device__ __forceinline__ __nv_bfloat16* sym_ptr(const NsLaunch& L, const MatPlan& mp, int mat, int id) {
  if (id == SB_A) return static_cast<__nv_bfloat16*>(mp.a);
  if (id == SB_B) return static_cast<__nv_bfloat16*>(mp.b);
  if (id == SB_T) return static_cast<__nv_bfloat16*>(L.gbufs[mat].t);
  if (id == SB_B1) return static_cast<__nv_bfloat16*>(L.gbufs[mat].b1);
  return nullptr;
}

// Store map (32 x 32 box) of an s x s buffer.
__device__ __forceinline__ const TmapBlob* sym_store_map(const NsLaunch& L, int mat, int id) {
  if (id == SB_A) return L.maps + (size_t)mat * kMapsPerMat + MAP_A_ST;
  if (id == SB_B) return L.maps + (size_t)mat * kMapsPerMat + MAP_B_ST;
  return L.gmaps + (size_t)mat * kGramMapsPerMat + (id == SB_T ? 4 : 5);
}

// Byte offset of the 16-byte group `q` of row `r` in a 32 x 32 bf16 block
// with 64-byte rows and the 64-byte swizzle of the bulk-tensor unit (the
// group index is XORed with bits 1..2 of the row).
__device__ __forceinline__ uint32_t sw64_offset(int r, int q) {
  return (uint32_t)(r * 64 + ((q ^ ((r >> 1) & 3)) << 4));
}

__device__ __forceinline__ TileJob decode(const NsArgs& A, const int4 t, const MatPlan& mp) {
  TileJob j;
  j.mat = t.x;
  j.ti = t.y;
  j.tj = t.z;
  j.a_sym = j.b_sym = 0;
  j.map_a_mn = j.map_b_mn = nullptr;
  const TmapBlob* own = A.L.maps + (size_t)j.mat * kMapsPerMat;
  if (A.phase == PHASE_GRAM) {
    const TmapBlob* xs = src_maps(A.L, j.mat, A.src_sel);
    j.kblocks = (mp.l + BK - 1) / BK;
    if (!mp.tall) {  // A[i][j] = sum_k X[i][k] X[j][k]
      j.map_a = xs + MAP_K128; j.a_mn = 0; j.a_coord = j.ti * BM;
      j.map_b = xs + MAP_K256; j.b_mn = 0; j.b_coord = j.tj * BN;
    } else {         // A[i][j] = sum_k X[k][i] X[k][j]
      j.map_a = xs + MAP_MN; j.a_mn = 1; j.a_coord = j.ti * BM;
      j.map_b = xs + MAP_MN; j.b_mn = 1; j.b_coord = j.tj * BN;
    }
  } else if (A.phase == PHASE_POLY) {  // (A A)[i][j] = sum_k A[i][k] A[j][k]
    j.kblocks = (mp.s + BK - 1) / BK;
    j.map_a = own + MAP_A_K128; j.a_mn = 0; j.a_coord = j.ti * BM;
    j.map_b = own + MAP_A_K256; j.b_mn = 0; j.b_coord = j.tj * BN;
    j.a_sym = j.b_sym = 1;
    j.map_a_mn = j.map_b_mn = own + MAP_A_MN;
  } else if (A.phase == PHASE_SYM) {   // (L R)[i][j] = sum_k L[i][k] R[j][k], R symmetric
    j.kblocks = (mp.s + BK - 1) / BK;
    j.map_a = sym_map(A.L, j.mat, A.spec.sym_l, false); j.a_mn = 0; j.a_coord = j.ti * BM;
    j.map_b = sym_map(A.L, j.mat, A.spec.sym_r, true);  j.b_mn = 0; j.b_coord = j.tj * BN;
    j.a_sym = j.b_sym = 1;
    j.map_a_mn = sym_map_mn(A.L, j.mat, A.spec.sym_l);
    j.map_b_mn = sym_map_mn(A.L, j.mat, A.spec.sym_r);
  } else {
    const TmapBlob* xs = src_maps(A.L, j.mat, A.src_sel);
    j.kblocks = (mp.s + BK - 1) / BK;
    if (!mp.tall) {  // (B X)[r][c] = sum_k B[r][k] X[k][c]
      j.map_a = sym_map(A.L, j.mat, A.spec.comb_b, false); j.a_mn = 0; j.a_coord = j.ti * BM;
      j.map_b = xs + MAP_MN;      j.b_mn = 1; j.b_coord = j.tj * BN;
      j.a_sym = 1;
      j.map_a_mn = sym_map_mn(A.L, j.mat, A.spec.comb_b);
    } else {         // (X B)[r][c] = sum_k X[r][k] B[c][k]
      j.map_a = xs + MAP_K128;    j.a_mn = 0; j.a_coord = j.ti * BM;
      j.map_b = sym_map(A.L, j.mat, A.spec.comb_b, true); j.b_mn = 0; j.b_coord = j.tj * BN;
      j.b_sym = 1;
      j.map_b_mn = sym_map_mn(A.L, j.mat, A.spec.comb_b);
    }
  }
  return j;
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float (&o)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 raw;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(o[8 * q + 2 * i], o[8 * q + 2 * i + 1]);
    reinterpret_cast<uint4*>(dst)[q] = raw;
  }
}

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* src, float (&o)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 raw = reinterpret_cast<const uint4*>(src)[q];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      o[8 * q + 2 * i] = f.x;
      o[8 * q + 2 * i + 1] = f.y;
    }
  }
}

// 32 consecutive bf16 of one row, as raw 16-byte groups; entries past the
// last column (or of a row past the last row) read as zero.
__device__ __forceinline__ void load_aux_chunk(const __nv_bfloat16* row_ptr, int col0, int cols, bool row_ok,
                                               uint4 (&r)[4]) {
  if (row_ok && col0 + 32 <= cols) {
    const uint4* p = reinterpret_cast<const uint4*>(row_ptr + col0);
#pragma unroll
    for (int q = 0; q < 4; ++q) r[q] = p[q];
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c0 = col0 + 8 * q + 2 * i;
        const uint32_t lo = (row_ok && c0 < cols) ? (uint32_t)__bfloat16_as_ushort(row_ptr[c0]) : 0u;
        const uint32_t hi = (row_ok && c0 + 1 < cols) ? (uint32_t)__bfloat16_as_ushort(row_ptr[c0 + 1]) : 0u;
        w[i] = lo | (hi << 16);
      }
      r[q] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

__device__ __forceinline__ void unpack_bf16x32(const uint4 (&r)[4], float (&o)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r[q]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      o[8 * q + 2 * i] = f.x;
      o[8 * q + 2 * i + 1] = f.y;
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) ns_phase_kernel(const __grid_constant__ NsArgs args) {
  extern __shared__ uint8_t smem_raw[];
  SmemLayout& sm = *reinterpret_cast<SmemLayout*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const NsLaunch& L = args.L;
  int* err = &L.status->error_word;
  const uint64_t tmo = L.timeout_ns;
  // Clean-up waits get at least half a second whatever the wait limit.
  const uint64_t drain_tmo = tmo > 500000000ull ? tmo : 500000000ull;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], 4);
    }
    mbar_init(&sm.drain, 1);
    for (int w = 0; w < 4; ++w)
      for (int b = 0; b < 2; ++b) mbar_init(&sm.aux_full[w][b], 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  const bool ident = args.phase == PHASE_POLY && args.poly_ident != 0;
  if (ident && warp >= 2) {
    // hi I and lo I as 64 x 64 K-major tiles in the 128-byte swizzle of the
    // operand loads: thread e writes row e % 64 of tile e / 64 (element
    // (r, k) sits in 16-byte unit (k / 8) ^ (r % 8) of row r).
    const int e = (int)threadIdx.x - 64;
    const int r = e & 63;
    const uint32_t bits = (e >> 6) ? (args.ident_bits >> 16) : (args.ident_bits & 0xffffu);
    uint8_t* rowp = &sm.auxstage[0][0][0] + (e >> 6) * kIdentBytes + r * 128;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint32_t w[4];
#pragma unroll
      for (int h = 0; h < 4; ++h)
        w[h] = ((q ^ (r & 7)) == (r >> 3) && ((r & 7) >> 1) == h) ? bits << (16 * (r & 1)) : 0u;
      *reinterpret_cast<uint4*>(rowp + q * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sm.tmem_base;
  // Launched as a programmatic dependent of the previous kernel on the
  // stream: everything above may overlap that kernel's last CTAs; nothing it
  // wrote is read before this wait (which returns once it has completed and
  // its memory operations are visible).
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------------------------
    // Producer
    // ------------------------------------------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0;            // bit s: stage s has been filled at least once
      uint32_t last_parity = 0;      // bit s: parity of the last fill of stage s
      bool ok = true;
      for (int t = blockIdx.x; t < L.ntiles && ok; t += gridDim.x) {
        const int4 tile = L.tiles[t];
        if (!L.binds[tile.x].active) continue;
        const MatPlan mp = L.plans[tile.x];
        const TileJob j = decode(args, tile, mp);
        for (int kb = 0; kb < j.kblocks; ++kb) {
          if (!mbar_wait_bounded(&sm.empty[stage], phase ^ 1u, err, tmo, WAIT_TMA_EMPTY)) { ok = false; break; }
          mbar_arrive_expect_tx(&sm.full[stage], kStageBytes);
          uint8_t* sa = sm.stage[stage];
          uint8_t* sb = sa + kABytes;
          const int k0 = kb * BK;
          const bool ta = j.a_sym && below_stored(j.a_coord, kb);   // mirrored K-block
          const bool tb = j.b_sym && below_stored(j.b_coord, kb);
          if (!j.a_mn && !ta) {
            tma_load_2d(sa, j.map_a, &sm.full[stage], k0, j.a_coord);
          } else {
            const void* ma = ta ? j.map_a_mn : j.map_a;
#pragma unroll
            for (int c = 0; c < BM / 64; ++c)
              tma_load_2d(sa + c * kMnChunkBytes, ma, &sm.full[stage], j.a_coord + 64 * c, k0);
          }
          if (!j.b_mn && !tb) {
            tma_load_2d(sb, j.map_b, &sm.full[stage], k0, j.b_coord);
          } else {
            const void* mb = tb ? j.map_b_mn : j.map_b;
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
              tma_load_2d(sb + c * kMnChunkBytes, mb, &sm.full[stage], j.b_coord + 64 * c, k0);
          }
          armed |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // Let every copy this thread started land before the CTA exits.
        for (int s = 0; s < kStages; ++s)
          if (armed & (1u << s)) mbar_wait_drain(&sm.full[s], (last_parity >> s) & 1u, drain_tmo);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------
    // MMA issuer
    // ------------------------------------------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued = false;
      const uint32_t ident_base = smem_u32(&sm.auxstage[0][0][0]);
      for (int t = blockIdx.x; t < L.ntiles && ok; t += gridDim.x) {
        const int4 tile = L.tiles[t];
        if (!L.binds[tile.x].active) continue;
        const MatPlan mp = L.plans[tile.x];
        const TileJob j = decode(args, tile, mp);
        if (!mbar_wait_bounded(&sm.acc_empty[acc], acc_phase ^ 1u, err, tmo, WAIT_ACC_EMPTY)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < j.kblocks; ++kb) {
          if (!mbar_wait_bounded(&sm.full[stage], phase, err, tmo, WAIT_TMA_FULL)) { ok = false; break; }
          tc_fence_after();
          // Majorness of this K-block's operands (mirrored K-blocks of a
          // symmetric buffer arrive M/N-major, as the producer loaded them).
          const int amn = j.a_mn | (j.a_sym && below_stored(j.a_coord, kb) ? 1 : 0);
          const int bmn = j.b_mn | (j.b_sym && below_stored(j.b_coord, kb) ? 1 : 0);
          const uint32_t idesc = umma_idesc_bf16(BM, BN, amn, bmn);
          const uint32_t sa = smem_u32(sm.stage[stage]);
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int k16 = 0; k16 < BK / 16; ++k16) {
            const uint64_t da = amn ? umma_desc_sw128(sa + k16 * 2048, kMnChunkBytes, 1024)
                                    : umma_desc_sw128(sa + k16 * 32, 16, 1024);
            const uint64_t db = bmn ? umma_desc_sw128(sb + k16 * 2048, kMnChunkBytes, 1024)
                                    : umma_desc_sw128(sb + k16 * 32, 16, 1024);
            tc_mma_bf16(d_tmem, da, db, idesc, (kb | k16) != 0);
          }
          if (ident && (kb * BK) / BN == j.tj) {
            // q A on the 64 output columns equal to this K-block's indices:
            // D[:, k - tj*256] += A[:, k] (hi + lo), N = 64.
            const uint32_t d_sub = d_tmem + (uint32_t)(kb * BK - j.tj * BN);
            const uint32_t idesc64 = umma_idesc_bf16(BM, 64, amn, 0);
            for (int part = 0; part < args.ident_parts; ++part) {
#pragma unroll
              for (int k16 = 0; k16 < BK / 16; ++k16) {
                const uint64_t da = amn ? umma_desc_sw128(sa + k16 * 2048, kMnChunkBytes, 1024)
                                        : umma_desc_sw128(sa + k16 * 32, 16, 1024);
                const uint64_t di = umma_desc_sw128(ident_base + (uint32_t)(part * kIdentBytes + k16 * 32), 16, 1024);
                tc_mma_bf16(d_sub, da, di, idesc64, 1);
              }
            }
          }
          issued = true;
          tc_commit(&sm.empty[stage]);      // frees the stage once these MMAs finish
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&sm.acc_full[acc]);       // accumulator ready for the epilogue
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok && issued) {
        tc_commit(&sm.drain);
        mbar_wait_drain(&sm.drain, 0, drain_tmo);
      }
    }
  } else {
    // ------------------------------------------------------------------
    // Epilogue (warps 2..5): warp w reads tensor-memory lanes 32*(w%4)..+31
    // ------------------------------------------------------------------
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    int obuf = 0;   // staging block pair used by this warp's next chunk
    // The last combine of a step may update the parameters in place of
    // storing O (ApplyArgs): p' = p (1 - lr wd) - lr scale O, O rounded to
    // bf16 first, p moved in 32 x 32 fp32 blocks by bulk copies through this
    // warp's two staging regions (the output blocks and the auxiliary
    // blocks, 4 KiB each, both unused by that launch otherwise).
    const bool apply = args.phase == PHASE_COMB && L.apply.on != 0;
    const float decay = apply ? apply_decay(L.apply.lr, L.apply.wd) : 1.0f;
    const bool tma_out = L.tma_store != 0 && !(args.phase == PHASE_COMB && args.dst_sel == BUF_OUT) && !apply;
    // The combine reads X a second time only when it adds a X itself
    // (a != 0, the Gram form); the plain iteration puts a on the diagonal of
    // B in the polynomial's epilogue, so its combine is the bare product.
    const bool comb_ax = args.phase == PHASE_COMB && args.a != 0.0f;
    // The auxiliary operand of the polynomial (A, when it does not take b A
    // on the tensor cores) and of the combine (X) comes through bulk-tensor
    // loads of 32 x 32 blocks into this warp's two auxiliary buffers when it
    // is a workspace buffer with a 32 x 32 map: always for the polynomial,
    // and for the combine when its main loop is long (K = s >= kAuxTmaMinK).
    // A per-lane row load touches 32 cache lines per instruction; on short
    // combine tiles the bulk loads wait behind the producer's operand loads
    // in the same copy engine instead.
    const bool aux_tma_phase = L.tma_store != 0 &&
                               ((args.phase == PHASE_POLY && !ident) || (comb_ax && args.src_sel != BUF_IN));
    uint32_t aux_parity = 0;    // bit b: parity of the next wait on aux_full[quarter][b]
    uint32_t aux_pending = 0;   // bit b: a load into buffer b has not been waited for
    for (int t = blockIdx.x; t < L.ntiles; t += gridDim.x) {
      const int4 tile = L.tiles[t];
      const MatBind mb = L.binds[tile.x];
      if (!mb.active) continue;
      const MatPlan mp = L.plans[tile.x];

      // Everything that does not need the accumulator is set up before
      // waiting for it, and the first chunk of the auxiliary operand is
      // already on its way.
      const int ti = tile.y, tj = tile.z;
      const int phase = args.phase;
      int rows, cols, ld;
      __nv_bfloat16* out;
      const __nv_bfloat16* aux = nullptr;
      const __nv_bfloat16* aux2 = nullptr;
      int aux_ld = 0;
      float sc = 1.0f;
      if (phase == PHASE_GRAM) {
        rows = cols = mp.s; ld = mp.lds; out = static_cast<__nv_bfloat16*>(mp.a);
        if (args.first) { const double al = inv_norm(L.sumsq, tile.x); sc = (float)(al * al); }
      } else if (phase == PHASE_POLY) {
        rows = cols = mp.s; ld = mp.lds; out = sym_ptr(L, mp, tile.x, args.spec.poly_out);
        if (ident) sc = args.c;   // the accumulator holds A A + q A
        else { aux = static_cast<const __nv_bfloat16*>(mp.a); aux_ld = mp.lds; }
      } else if (phase == PHASE_SYM) {
        rows = cols = mp.s; ld = mp.lds; out = sym_ptr(L, mp, tile.x, args.spec.sym_out);
        aux = sym_ptr(L, mp, tile.x, args.spec.aux1); aux2 = sym_ptr(L, mp, tile.x, args.spec.aux2);
        aux_ld = mp.lds;
      } else {
        rows = mp.m; cols = mp.n; ld = mp.ldx;
        out = static_cast<__nv_bfloat16*>(const_cast<void*>(sel_buf(mp, mb, args.dst_sel)));
        if (comb_ax) { aux = static_cast<const __nv_bfloat16*>(sel_buf(mp, mb, args.src_sel)); aux_ld = mp.ldx; }
        if (args.first) sc = (float)inv_norm(L.sumsq, tile.x);
      }
      // Symmetric outputs are stored as computed (upper 256-block triangle);
      // their consumers read the blocks below it transposed.
      const TmapBlob* st_map = nullptr;
      if (tma_out) {
        if (phase == PHASE_GRAM) st_map = sym_store_map(L, tile.x, SB_A);
        else if (phase == PHASE_POLY) st_map = sym_store_map(L, tile.x, args.spec.poly_out);
        else if (phase == PHASE_SYM) st_map = sym_store_map(L, tile.x, args.spec.sym_out);
        else st_map = L.maps + (size_t)tile.x * kMapsPerMat + (args.dst_sel == BUF_X0 ? MAP_X0_ST : MAP_X1_ST);
      }
      const int warp_row0 = ti * BM + quarter * 32;
      const float e1 = args.spec.e1, e2 = args.spec.e2;
      const int row = ti * BM + row_in_tile;
      const bool row_ok = row < rows;
      const uint32_t t_base = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
      const float ca = args.a, cb = args.b, cc = args.c;
      const __nv_bfloat16* aux_row = aux != nullptr ? aux + (size_t)row * aux_ld : nullptr;
      uint4 xa[4], xb[4];   // packed bf16 auxiliary values of the current and the next chunk
      const bool aux_tma = aux_tma_phase && (phase == PHASE_POLY || mp.s >= kAuxTmaMinK);
      const TmapBlob* aux_map =
          !aux_tma ? nullptr
          : L.maps + (size_t)tile.x * kMapsPerMat +
                (phase == PHASE_POLY ? MAP_A_ST : (args.src_sel == BUF_X0 ? MAP_X0_ST : MAP_X1_ST));
      // Bulk load of the auxiliary block of chunk `c` into buffer c & 1
      // (issued by lane 0 after every lane has finished reading that buffer).
      auto aux_issue = [&](int c) {
        const int b = c & 1;
        __syncwarp();   // every lane has read the buffer's previous block
        if (lane == 0) {
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&sm.aux_full[quarter][b], kOutStageBytes);
          tma_load_2d(sm.auxstage[quarter][b], aux_map, &sm.aux_full[quarter][b], tj * BN + c * 32, warp_row0);
        }
        aux_pending |= 1u << b;
      };
      if (apply) {
        const TmapBlob* pm = L.p_maps + tile.x;
        const float step = apply_step(L.apply.lr, mp.m, mp.n, L.apply.scale_mode, L.apply.extra_scale, 1.0);
        const int nch = min(BN / 32, (cols - tj * BN + 31) / 32);   // chunks holding a column of the matrix
        uint8_t* const pbuf[2] = {&sm.ostage[quarter][0][0], &sm.auxstage[quarter][0][0]};
        // Bulk load of p's block for chunk c into buffer c & 1, once that
        // buffer's previous block has been stored (read by the copy engine)
        // and read by every lane.
        auto p_load = [&](int c) {
          const int b = c & 1;
          if (lane == 0) bulk_wait_group_read<0>();
          __syncwarp();
          if (lane == 0) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&sm.aux_full[quarter][b], 32 * 32 * 4);
            tma_load_2d(pbuf[b], pm, &sm.aux_full[quarter][b], tj * BN + c * 32, warp_row0);
          }
          aux_pending |= 1u << b;
        };
        p_load(0);
        if (!mbar_wait_bounded(&sm.acc_full[acc], acc_phase, err, tmo, WAIT_ACC_FULL)) break;
        tc_fence_after();
        bool ok = true;
        for (int c = 0; c < nch; ++c) {
          if (c + 1 < nch) p_load(c + 1);
          float v[32];
          tmem_ld_32x32b_x32(t_base + (uint32_t)(c * 32), v);
          const int b = c & 1;
          if (!mbar_wait_bounded(&sm.aux_full[quarter][b], (aux_parity >> b) & 1u, err, tmo, WAIT_ACC_FULL)) {
            ok = false;
            break;
          }
          aux_parity ^= 1u << b;
          aux_pending &= ~(1u << b);
          // This lane's row of the block: 128 bytes, 16-byte unit u at unit
          // u ^ (row % 8) (128-byte swizzle of the copy engine).
          uint8_t* rowp = pbuf[b] + lane * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            float4* q = reinterpret_cast<float4*>(rowp + ((u ^ (lane & 7)) << 4));
            float4 pv = *q;
            pv.x = apply_one(pv.x, v[4 * u + 0] * sc, decay, step);
            pv.y = apply_one(pv.y, v[4 * u + 1] * sc, decay, step);
            pv.z = apply_one(pv.z, v[4 * u + 2] * sc, decay, step);
            pv.w = apply_one(pv.w, v[4 * u + 3] * sc, decay, step);
            *q = pv;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (warp_row0 < rows) tma_store_2d(pm, pbuf[b], tj * BN + c * 32, warp_row0);
            bulk_commit_group();
          }
        }
        if (!ok) break;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.acc_empty[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        continue;
      }
      if (aux_tma) {
        aux_issue(0);
      } else if (aux_row != nullptr) {
        load_aux_chunk(aux_row, tj * BN, cols, row_ok, xa);
      }

      if (!mbar_wait_bounded(&sm.acc_full[acc], acc_phase, err, tmo, WAIT_ACC_FULL)) break;
      tc_fence_after();

      // One 32-column chunk: returns false past the last column.
      auto chunk = [&](int ch, uint4 (&cur)[4], uint4 (&nxt)[4]) -> bool {
        const int col0 = tj * BN + ch * 32;
        if (col0 >= cols) return false;                // warp-uniform
        if (aux_tma) {
          if (ch + 1 < BN / 32 && col0 + 32 < cols) aux_issue(ch + 1);
        } else if (aux_row != nullptr && ch + 1 < BN / 32 && col0 + 32 < cols) {
          load_aux_chunk(aux_row, col0 + 32, cols, row_ok, nxt);
        }
        float v[32];
        tmem_ld_32x32b_x32(t_base + (uint32_t)(ch * 32), v);
        const bool full_chunk = col0 + 32 <= cols;
        float o[32];
        if (aux_tma) {
          // This lane's row of the block, from the swizzled shared copy.
          const int b = ch & 1;
          if (!mbar_wait_bounded(&sm.aux_full[quarter][b], (aux_parity >> b) & 1u, err, tmo, WAIT_ACC_FULL))
            return false;
          aux_parity ^= 1u << b;
          aux_pending &= ~(1u << b);
          const uint8_t* ab = sm.auxstage[quarter][b];
#pragma unroll
          for (int q = 0; q < 4; ++q) cur[q] = *reinterpret_cast<const uint4*>(ab + sw64_offset(lane, q));
        }
        if (aux_row == nullptr) {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = v[i] * sc;
        } else {
          float x[32];
          unpack_bf16x32(cur, x);
          if (phase == PHASE_SYM) {
            if (aux2 != nullptr) {
              float y[32];
              if (row_ok && full_chunk) {
                load_bf16x32(aux2 + (size_t)row * aux_ld + col0, y);
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  y[i] = (row_ok && col0 + i < cols) ? __bfloat162float(aux2[(size_t)row * aux_ld + col0 + i])
                                                     : 0.0f;
              }
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = fmaf(e1, x[i], fmaf(e2, y[i], v[i]));
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = fmaf(e1, x[i], v[i]);
            }
          } else if (phase == PHASE_POLY) {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = fmaf(cb, x[i], cc * v[i]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = sc * fmaf(ca, x[i], v[i]);
          }
        }
        if (phase == PHASE_POLY) {
          // B + a I: the chunk whose columns are this warp's rows holds the
          // diagonal, lane i at column i.
          const int dcol = col0 == warp_row0 ? lane : -1;
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] += i == dcol ? ca : 0.0f;
        }
        if (tma_out) {
          // Stage the 32 x 32 block in shared memory and write it with a bulk
          // store; the tensor map clips rows and columns beyond the matrix.
          uint8_t* dbuf = sm.ostage[quarter][obuf];
          if (lane == 0) bulk_wait_group_read<1>();   // the block used two chunks ago is free
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 raw;
            __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
            for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(o[8 * q + 2 * i], o[8 * q + 2 * i + 1]);
            *reinterpret_cast<uint4*>(dbuf + sw64_offset(lane, q)) = raw;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (warp_row0 < rows) tma_store_2d(st_map, dbuf, col0, warp_row0);
            bulk_commit_group();
          }
          obuf ^= 1;
          return true;
        }
        if (row_ok) {
          __nv_bfloat16* dst = out + (size_t)row * ld + col0;
          if (full_chunk) {
            store_bf16x32(dst, o);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (col0 + i < cols) dst[i] = __float2bfloat16_rn(o[i]);
          }
        }
        return true;
      };
      // Chunks in pairs so that the two auxiliary buffers stay in registers.
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ch += 2) {
        if (!chunk(ch, xa, xb)) break;
        if (!chunk(ch + 1, xb, xa)) break;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    // Bulk stores read this CTA's shared memory: let them finish; loads that
    // were issued but not waited for (after an abort) must land too.
    if ((tma_out || apply) && lane == 0) bulk_wait_group_all();
    if (lane == 0)
      for (int b = 0; b < 2; ++b)
        if (aux_pending & (1u << b)) mbar_wait_drain(&sm.aux_full[quarter][b], (aux_parity >> b) & 1u, drain_tmo);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

int ns_bf16_smem_bytes() { return (int)sizeof(SmemLayout) + 1024; }

namespace {

// Round-to-nearest-even bf16 bits of a finite float.
uint32_t bf16_bits_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, sizeof(u));
  u += 0x7fffu + ((u >> 16) & 1u);
  return u >> 16;
}

float bf16_bits_value(uint32_t h) {
  const uint32_t u = h << 16;
  float f;
  std::memcpy(&f, &u, sizeof(f));
  return f;
}

// The polynomial takes q A = (b / c) A on the tensor cores while |q| stays
// this small: the accumulator then holds A A + q A with entries a few times
// those of A A, so its fp32 rounding stays far below the bf16 rounding of B.
constexpr double kIdentMaxRatio = 64.0;

}  // namespace

cudaError_t launch_ns_phase_bf16(const NsLaunch& L, int phase, int src_sel, int dst_sel, int first, float a,
                                 float b, float c, cudaStream_t st, const PhaseSpec& spec) {
  if (L.ntiles <= 0) return cudaSuccess;
  static std::atomic<unsigned long long> attr_done{0};
  const int smem = ns_bf16_smem_bytes();
  {
    const cudaError_t e = ensure_dynamic_smem(ns_phase_kernel, smem, attr_done);
    if (e != cudaSuccess) return e;
  }
  NsArgs args;
  args.L = L;
  args.phase = phase;
  args.src_sel = src_sel;
  args.dst_sel = dst_sel;
  args.first = first;
  args.a = a;
  args.b = b;
  args.c = c;
  args.spec = spec;
  args.poly_ident = 0;
  args.ident_bits = 0;
  args.ident_parts = 1;
  if (phase == PHASE_POLY && c != 0.0f && L.max_s < kIdentMaxS) {
    const double q = (double)b / (double)c;
    if (std::isfinite(q) && std::fabs(q) <= kIdentMaxRatio) {
      const uint32_t hi = bf16_bits_rne((float)q);
      const uint32_t lo = bf16_bits_rne((float)(q - (double)bf16_bits_value(hi)));
      args.poly_ident = 1;
      args.ident_bits = hi | (lo << 16);
      args.ident_parts = (hi & 0x7fffu) == 0 ? 0 : (lo & 0x7fffu) != 0 ? 2 : 1;   // b = 0: A A alone
    }
  }
  const int grid = L.grid < L.ntiles ? L.grid : L.ntiles;
  // Programmatic stream serialization: this launch may begin while the
  // previous kernel's last CTAs finish; the kernel waits for it before its
  // first dependent read (griddepcontrol.wait).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, ns_phase_kernel, args);
}

}  // namespace muon
