// Newton-Schulz phases on CTA pairs (tcgen05 cta_group::2), 256 x 256 tiles.
//
// Same three phases as ns_tcgen05.cu ("About Muon: Why Not Adam", sections
// "The lemma that makes it possible" and "The whole thing, in about forty
// lines"): GRAM A = X X^T (or X^T X), POLY B = aI + bA + cA^2, COMB X' = BX
// (or XB), with the normalisation folded into the first step's
// epilogues. Here each output tile is 256 x 256 and belongs to a cluster of
// two CTAs on neighbouring SMs: CTA r holds rows 128r..128r+127 of the
// tile's A operand and N-rows 128r..128r+127 of its B operand in its own
// shared memory, and one tcgen05.mma.cta_group::2 (M = 256, N = 256) from
// the leader CTA multiplies the pair's operands into both CTAs' tensor
// memories (each CTA receives its 128 rows). Per SM, operand traffic from L2
// and through shared memory is two thirds of the 128 x 256 single-CTA tile.
// The symmetric Gram and polynomial outputs list only tiles on or right of
// the diagonal (TJ >= TI) and mirror the strictly upper ones.
//
// Roles per CTA (192 threads, one CTA per SM, persistent over the tile list
// with a static stride of the cluster count):
//   warp 0    : bulk-tensor producer for this CTA's halves, 6-stage ring; the
//               copies of both CTAs complete on the leader's `full` barrier,
//               which the leader arms for both halves
//   warp 1    : leader: tcgen05.mma issuer; peer: waits for the final drain
//   warps 2-5 : epilogue of this CTA's 128 rows, then one arrive on the
//               leader's accumulator-empty barrier
// The leader's commits reach both CTAs (CTA-mask multicast commit). Every
// wait is bounded; on expiry the error word is set and every role stops;
// the leader waits for the copies of every stage it armed (which covers the
// peer's copies of those stages), the peer gives its last copies a bounded
// grace period, the leader drains its MMAs, the pair meets at a cluster
// barrier and frees tensor memory.
#include "common.cuh"
#include "kernels.h"

namespace muon {

namespace {

constexpr int BM = 256, BN = 256, BK = 64;   // pair tile
constexpr int kHalf = 128;                   // rows of A and of B per CTA
constexpr int kStages = 6;
constexpr int kHalfBytes = kHalf * BK * 2;   // 16 KiB
constexpr int kStageBytes = 2 * kHalfBytes;  // A half + B half
constexpr int kMnChunkBytes = 64 * BK * 2;   // one 64 x 64 M/N-major box
constexpr int kThreads = 192;
constexpr int kTmemCols = 2 * BN;            // two 256-column fp32 accumulators
constexpr int kOutStageBytes = 32 * 32 * 2;  // one 32 x 32 bf16 bulk-store block

struct __align__(1024) PairSmem {
  uint8_t stage[kStages][kStageBytes];
  // Epilogue staging for bulk stores: per epilogue warp two direct and two
  // transposed 32 x 32 blocks (64-byte rows, 64-byte swizzle).
  uint8_t ostage[4][4][kOutStageBytes];
  uint64_t full[kStages];      // leader only: both CTAs' copies of the stage landed
  uint64_t empty[kStages];     // MMAs reading the stage are done (both CTAs)
  uint64_t acc_full[2];        // accumulator ready (both CTAs)
  uint64_t acc_empty[2];       // leader only: both CTAs drained it
  uint64_t drain;              // all MMAs of the leader done (both CTAs)
  uint32_t tmem_base;
};

struct PairArgs {
  NsLaunch L;
  int phase, src_sel, dst_sel, first;
  float a, b, c;
};

struct PairJob {
  int kblocks;
  const void* map_a;
  const void* map_b;
  int a_mn, b_mn;
  int a_coord, b_coord;        // this CTA's first row (K-major) or M/N index (M/N-major)
};

__device__ __forceinline__ const TmapBlob* src_maps_pair(const NsLaunch& L, int mat, int src_sel) {
  if (src_sel == BUF_IN) return L.in_maps + (size_t)mat * kInMapsPerMat;
  return L.maps + (size_t)mat * kMapsPerMat + (src_sel == BUF_X0 ? MAP_X0 : MAP_X1);
}

__device__ __forceinline__ PairJob decode_pair(const PairArgs& A, const int4 t, const MatPlan& mp, int rank) {
  PairJob j;
  const int mat = t.x;
  const int ra = t.y * BM + rank * kHalf;   // this CTA's rows of the A operand
  const int rb = t.z * BN + rank * kHalf;   // this CTA's rows of the B operand
  const TmapBlob* own = A.L.maps + (size_t)mat * kMapsPerMat;
  if (A.phase == PHASE_GRAM) {
    const TmapBlob* xs = src_maps_pair(A.L, mat, A.src_sel);
    j.kblocks = (mp.l + BK - 1) / BK;
    if (!mp.tall) {
      j.map_a = xs + MAP_K128; j.a_mn = 0;
      j.map_b = xs + MAP_K128; j.b_mn = 0;
    } else {
      j.map_a = xs + MAP_MN; j.a_mn = 1;
      j.map_b = xs + MAP_MN; j.b_mn = 1;
    }
  } else if (A.phase == PHASE_POLY) {
    j.kblocks = (mp.s + BK - 1) / BK;
    j.map_a = own + MAP_A_K128; j.a_mn = 0;
    j.map_b = own + MAP_A_K128; j.b_mn = 0;
  } else {
    const TmapBlob* xs = src_maps_pair(A.L, mat, A.src_sel);
    j.kblocks = (mp.s + BK - 1) / BK;
    if (!mp.tall) {   // B X: rows of B, columns of X
      j.map_a = own + MAP_B_K128; j.a_mn = 0;
      j.map_b = xs + MAP_MN;      j.b_mn = 1;
    } else {          // X B: rows of X, rows of B (B symmetric)
      j.map_a = xs + MAP_K128;    j.a_mn = 0;
      j.map_b = own + MAP_B_K128; j.b_mn = 0;
    }
  }
  j.a_coord = ra;
  j.b_coord = rb;
  return j;
}

// Byte offset of 16-byte group q of row r in a 32 x 32 bf16 block with
// 64-byte rows under the bulk-tensor unit's 64-byte swizzle.
__device__ __forceinline__ uint32_t sw64_off(int r, int q) {
  return (uint32_t)(r * 64 + ((q ^ ((r >> 1) & 3)) << 4));
}

__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const float (&o)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 raw;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(o[8 * q + 2 * i], o[8 * q + 2 * i + 1]);
    reinterpret_cast<uint4*>(dst)[q] = raw;
  }
}

__device__ __forceinline__ void load_row32(const __nv_bfloat16* src, float (&o)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 raw = reinterpret_cast<const uint4*>(src)[q];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      o[8 * q + 2 * i] = f.x;
      o[8 * q + 2 * i + 1] = f.y;
    }
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    ns_pair_kernel(const __grid_constant__ PairArgs args) {
  extern __shared__ uint8_t smem_raw[];
  PairSmem& sm = *reinterpret_cast<PairSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = (int)cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = (int)cluster_id_x();
  const int ncl = (int)cluster_count_x();
  const NsLaunch& L = args.L;
  int* err = &L.status->error_word;
  const uint64_t tmo = L.timeout_ns;
  const uint64_t drain_tmo = tmo > 500000000ull ? tmo : 500000000ull;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);                // the leader's expect_tx for both halves
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], 8);           // 4 epilogue warps in each CTA
    }
    mbar_init(&sm.drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&sm.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();          // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------
    // Producer (both CTAs): this CTA's halves of A and B
    // ------------------------------------------------------------------
    if (lane == 0) {
      const uint32_t leader_full0 = map_shared_rank(&sm.full[0], 0);
      int stage = 0;
      uint32_t phase = 0, armed = 0, last_parity = 0;
      bool ok = true, issued = false;
      for (int t = cid; t < L.ntiles && ok; t += ncl) {
        const int4 tile = L.tiles[t];
        if (!L.binds[tile.x].active) continue;
        const MatPlan mp = L.plans[tile.x];
        const PairJob j = decode_pair(args, tile, mp, rank);
        for (int kb = 0; kb < j.kblocks; ++kb) {
          if (!mbar_wait_bounded(&sm.empty[stage], phase ^ 1u, err, tmo, WAIT_TMA_EMPTY)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&sm.full[stage], 2 * kStageBytes);
          const uint32_t bar = leader_full0 + (uint32_t)(stage * sizeof(uint64_t));
          uint8_t* sa = sm.stage[stage];
          uint8_t* sb = sa + kHalfBytes;
          const int k0 = kb * BK;
          if (!j.a_mn) {
            tma_load_2d_pair(sa, j.map_a, bar, k0, j.a_coord);
          } else {
            tma_load_2d_pair(sa, j.map_a, bar, j.a_coord, k0);
            tma_load_2d_pair(sa + kMnChunkBytes, j.map_a, bar, j.a_coord + 64, k0);
          }
          if (!j.b_mn) {
            tma_load_2d_pair(sb, j.map_b, bar, k0, j.b_coord);
          } else {
            tma_load_2d_pair(sb, j.map_b, bar, j.b_coord, k0);
            tma_load_2d_pair(sb + kMnChunkBytes, j.map_b, bar, j.b_coord + 64, k0);
          }
          issued = true;
          armed |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok && issued) {
        if (leader) {
          // Every stage the leader armed counts both CTAs' copies.
          for (int s = 0; s < kStages; ++s)
            if (armed & (1u << s)) mbar_wait_drain(&sm.full[s], (last_parity >> s) & 1u, drain_tmo);
        } else {
          // The peer cannot observe the leader's barrier: give its copies in
          // flight a bounded grace period (bulk copies finish in microseconds).
          const uint64_t t0 = global_timer_ns();
          while (global_timer_ns() - t0 < 200000ull) __nanosleep(1000);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      if (leader) {
        // --------------------------------------------------------------
        // MMA issuer (leader)
        // --------------------------------------------------------------
        int stage = 0, acc = 0;
        uint32_t phase = 0, acc_phase = 0;
        bool ok = true;
        for (int t = cid; t < L.ntiles && ok; t += ncl) {
          const int4 tile = L.tiles[t];
          if (!L.binds[tile.x].active) continue;
          const MatPlan mp = L.plans[tile.x];
          const PairJob j = decode_pair(args, tile, mp, 0);
          if (!mbar_wait_bounded(&sm.acc_empty[acc], acc_phase ^ 1u, err, tmo, WAIT_ACC_EMPTY)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
          const uint32_t idesc = umma_idesc_bf16(BM, BN, j.a_mn, j.b_mn);
          for (int kb = 0; kb < j.kblocks; ++kb) {
            if (!mbar_wait_bounded(&sm.full[stage], phase, err, tmo, WAIT_TMA_FULL)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = smem_u32(sm.stage[stage]);
            const uint32_t sb = sa + kHalfBytes;
#pragma unroll
            for (int k16 = 0; k16 < BK / 16; ++k16) {
              const uint64_t da = j.a_mn ? umma_desc_sw128(sa + k16 * 2048, kMnChunkBytes, 1024)
                                         : umma_desc_sw128(sa + k16 * 32, 16, 1024);
              const uint64_t db = j.b_mn ? umma_desc_sw128(sb + k16 * 2048, kMnChunkBytes, 1024)
                                         : umma_desc_sw128(sb + k16 * 32, 16, 1024);
              tc_mma_bf16_pair(d_tmem, da, db, idesc, (kb | k16) != 0);
            }
            tc_commit_pair_multicast(&sm.empty[stage], 0x3);
            if (++stage == kStages) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          tc_commit_pair_multicast(&sm.acc_full[acc], 0x3);
          if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
        // Always: one last commit so both CTAs can tell every MMA is done.
        tc_commit_pair_multicast(&sm.drain, 0x3);
        mbar_wait_drain(&sm.drain, 0, drain_tmo);
      } else {
        // Peer: the leader's final commit also reaches this CTA; wait for it
        // so no MMA still reads this CTA's memory when it leaves.
        mbar_wait_drain(&sm.drain, 0, drain_tmo);
      }
    }
  } else {
    // ------------------------------------------------------------------
    // Epilogue (both CTAs): warp w reads tensor-memory lanes 32*(w%4)..+31
    // ------------------------------------------------------------------
    const int quarter = warp & 3;
    const int row_in_half = quarter * 32 + lane;
    const uint32_t leader_acc_empty0 = map_shared_rank(&sm.acc_empty[0], 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    int obuf = 0;
    const bool tma_out = L.tma_store != 0 && !(args.phase == PHASE_COMB && args.dst_sel == BUF_OUT);
    for (int t = cid; t < L.ntiles; t += ncl) {
      const int4 tile = L.tiles[t];
      const MatBind mb = L.binds[tile.x];
      if (!mb.active) continue;
      const MatPlan mp = L.plans[tile.x];
      if (!mbar_wait_bounded(&sm.acc_full[acc], acc_phase, err, tmo, WAIT_ACC_FULL)) break;
      tc_fence_after();

      const int ti = tile.y, tj = tile.z;
      const int phase = args.phase;
      int rows, cols, ld;
      __nv_bfloat16* out;
      const __nv_bfloat16* aux = nullptr;
      int aux_ld = 0;
      float sc = 1.0f;
      if (phase == PHASE_GRAM) {
        rows = cols = mp.s; ld = mp.lds; out = static_cast<__nv_bfloat16*>(mp.a);
        if (args.first) { const double al = inv_norm(L.sumsq, tile.x); sc = (float)(al * al); }
      } else if (phase == PHASE_POLY) {
        rows = cols = mp.s; ld = mp.lds; out = static_cast<__nv_bfloat16*>(mp.b);
        aux = static_cast<const __nv_bfloat16*>(mp.a); aux_ld = mp.lds;
      } else {
        rows = mp.m; cols = mp.n; ld = mp.ldx;
        out = static_cast<__nv_bfloat16*>(const_cast<void*>(sel_buf(mp, mb, args.dst_sel)));
        // a X only when a is not already on the diagonal of B
        if (args.a != 0.0f) { aux = static_cast<const __nv_bfloat16*>(sel_buf(mp, mb, args.src_sel)); aux_ld = mp.ldx; }
        if (args.first) sc = (float)inv_norm(L.sumsq, tile.x);
      }
      const bool mirror = (phase != PHASE_COMB) && (tj > ti);
      const TmapBlob* own_maps = L.maps + (size_t)tile.x * kMapsPerMat;
      const TmapBlob* st_map = phase == PHASE_GRAM ? own_maps + MAP_A_ST
                               : phase == PHASE_POLY ? own_maps + MAP_B_ST
                               : own_maps + (args.dst_sel == BUF_X0 ? MAP_X0_ST : MAP_X1_ST);
      const int warp_row0 = ti * BM + rank * kHalf + quarter * 32;
      const int row = ti * BM + rank * kHalf + row_in_half;
      const bool row_ok = row < rows;
      const uint32_t t_base = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
      const float ca = args.a, cb = args.b, cc = args.c;

#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        const int col0 = tj * BN + ch * 32;
        if (col0 >= cols) break;                       // warp-uniform
        float v[32];
        tmem_ld_32x32b_x32(t_base + (uint32_t)(ch * 32), v);
        const bool full_chunk = col0 + 32 <= cols;
        float o[32];
        if (aux == nullptr) {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = v[i] * sc;
        } else {
          float x[32];
          if (row_ok && full_chunk) {
            load_row32(aux + (size_t)row * aux_ld + col0, x);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              x[i] = (row_ok && col0 + i < cols) ? __bfloat162float(aux[(size_t)row * aux_ld + col0 + i]) : 0.0f;
          }
          if (phase == PHASE_POLY) {
            const int dcol = col0 == warp_row0 ? lane : -1;   // B + a I: this warp's diagonal chunk
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = fmaf(cb, x[i], cc * v[i]) + (i == dcol ? ca : 0.0f);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = sc * fmaf(ca, x[i], v[i]);
          }
        }
        if (tma_out) {
          uint8_t* dbuf = sm.ostage[quarter][obuf];
          uint8_t* mbuf = sm.ostage[quarter][2 + obuf];
          if (lane == 0) bulk_wait_group_read<1>();   // the pair used two chunks ago is free
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 raw;
            __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
            for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(o[8 * q + 2 * i], o[8 * q + 2 * i + 1]);
            *reinterpret_cast<uint4*>(dbuf + sw64_off(lane, q)) = raw;
          }
          if (mirror) {
            const uint32_t in_group = (uint32_t)(lane & 7) * 2;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              *reinterpret_cast<__nv_bfloat16*>(mbuf + sw64_off(j, lane >> 3) + in_group) = __float2bfloat16_rn(o[j]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (warp_row0 < rows) {
              tma_store_2d(st_map, dbuf, col0, warp_row0);
              if (mirror) tma_store_2d(st_map, mbuf, warp_row0, col0);
            }
            bulk_commit_group();
          }
          obuf ^= 1;
          continue;
        }
        if (row_ok) {
          __nv_bfloat16* dst = out + (size_t)row * ld + col0;
          if (full_chunk) {
            store_row32(dst, o);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (col0 + i < cols) dst[i] = __float2bfloat16_rn(o[i]);
          }
        }
        if (mirror && row_ok) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (col0 + i < cols) out[(size_t)(col0 + i) * ld + row] = __float2bfloat16_rn(o[i]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_acc_empty0 + (uint32_t)(acc * sizeof(uint64_t)));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (tma_out && lane == 0) bulk_wait_group_all();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();          // no CTA leaves while the pair's MMAs may touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace

int ns_pair_smem_bytes() { return (int)sizeof(PairSmem) + 1024; }

// Number of CTA pairs that can be resident at once (some GPCs hold an odd
// number of SMs, so it can be below half the SM count); a persistent grid
// larger than this would run its last clusters in a second wave.
int pair_clusters_resident(int smem) {
  static int cached = -1;
  if (cached >= 0) return cached;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, (const void*)ns_pair_kernel, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = 0;
  }
  cached = n;
  return cached;
}

cudaError_t launch_ns_phase_pair(const NsLaunch& L, int phase, int src_sel, int dst_sel, int first, float a,
                                 float b, float c, cudaStream_t st) {
  if (L.ntiles <= 0) return cudaSuccess;
  static std::atomic<unsigned long long> attr_done{0};
  const int smem = ns_pair_smem_bytes();
  {
    const cudaError_t e = ensure_dynamic_smem(ns_pair_kernel, smem, attr_done);
    if (e != cudaSuccess) return e;
  }
  PairArgs args;
  args.L = L;
  args.phase = phase;
  args.src_sel = src_sel;
  args.dst_sel = dst_sel;
  args.first = first;
  args.a = a;
  args.b = b;
  args.c = c;
  int max_pairs = L.grid / 2;
  const int resident = pair_clusters_resident(smem);
  if (resident > 0 && resident < max_pairs) max_pairs = resident;
  const int pairs = max_pairs < L.ntiles ? max_pairs : L.ntiles;
  ns_pair_kernel<<<2 * (pairs > 0 ? pairs : 1), kThreads, smem, st>>>(args);
  return cudaGetLastError();
}

int ns_pair_clusters_resident() { return pair_clusters_resident(ns_pair_smem_bytes()); }

}  // namespace muon
