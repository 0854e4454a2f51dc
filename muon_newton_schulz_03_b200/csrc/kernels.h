// Host-side launch interfaces of the CUDA kernels (internal to the library).
#pragma once

#include <cstdint>
#include <string>
#include <cuda_runtime.h>

#include "common.cuh"

namespace muon {

// Grouped elementwise launch: one block per chunk of kElemChunk elements.
struct ElemLaunch {
  const MatPlan* plans = nullptr;     // device
  const MatBind* binds = nullptr;     // device
  const long long* prefix = nullptr;  // device, count + 1 entries
  int count = 0;
  long long block_base = 0;           // first chunk of the launch (0 for a whole set)
  long long nblocks = 0;              // chunks in the launch (prefix[count] for a whole set)
};

// partials == nullptr: one double atomic per block into sumsq; else each
// block stores its partial at partials[block] and launch_reduce_partials
// adds them per matrix in a fixed order (bitwise reproducible norms).
cudaError_t launch_momentum_norm(const ElemLaunch& L, int ysel, float beta, int nesterov, double* sumsq,
                                 double* partials, DevStatus* status, int check_nonfinite, bool fp32_out,
                                 cudaStream_t st);
cudaError_t launch_reduce_partials(const ElemLaunch& L, int m0, int m1, const double* partials, double* sumsq,
                                   cudaStream_t st);
cudaError_t launch_apply(const ElemLaunch& L, int osel, float lr, float wd, int scale_mode, float extra_scale,
                         const double* sumsq, bool fp32_in, cudaStream_t st);
// QK-Clip: rows of head h scaled by sqrt(tau / s_max[h]) when s_max[h] > tau.
cudaError_t launch_qk_clip(float* w, long long rows, long long cols, int head_rows, const float* s_max, float tau,
                           cudaStream_t st);

cudaError_t launch_scale_copy(const ElemLaunch& L, int isel, int osel, const double* sumsq, bool fp32,
                              cudaStream_t st);

// Newton-Schulz phases. PHASE_SYM is the product of two symmetric s x s
// buffers used by the Gram form of the iteration.
enum NsPhase : int { PHASE_GRAM = 0, PHASE_POLY = 1, PHASE_COMB = 2, PHASE_SYM = 3 };

// The s x s buffers of a matrix: the Gram A and polynomial B of the plan,
// and T and B1, used only by the Gram form.
enum SymBuf : int { SB_A = 0, SB_B = 1, SB_T = 2, SB_B1 = 3, SB_NONE = -1 };

struct GramBufs {
  void* t;
  void* b1;
};
// T (K-major 128- and 256-row boxes), B1 (same), then the 32 x 32 store
// boxes of T and B1.
// Gram-form maps per matrix: T K128, T K256, B1 K128, B1 K256, T store,
// B1 store, T 64 x 64 (M/N-major loads), B1 64 x 64.
constexpr int kGramMapsPerMat = 8;

// Operands and epilogue of one launch beyond the phase itself.
struct PhaseSpec {
  int poly_out = SB_B;                 // POLY: where B = aI + bA + cA^2 goes (a = 0 in the Gram form)
  int sym_l = SB_A, sym_r = SB_A;      // SYM: D = L R (both symmetric)
  int sym_out = SB_T;
  int aux1 = SB_NONE, aux2 = SB_NONE;  // SYM: out = D + e1 aux1 + e2 aux2
  float e1 = 0.0f, e2 = 0.0f;
  int comb_b = SB_B;                   // COMB: left operand (SB_B or SB_T)
};

// Tensor maps of one matrix (bf16 path). Each CUtensorMap is 128 bytes and
// must be 64-byte aligned in global memory.
struct alignas(64) TmapBlob {
  unsigned char bytes[128];
};
// Index of each map inside a matrix's block of kMapsPerMat maps.
// X-buffer maps come in triples (K-major 128-row box, K-major 256-row box,
// MN-major 64x64 box): X0 at 0, X1 at 3. A caller input buffer has its own
// triple per matrix in a separate table.
enum MapIdx : int {
  MAP_X0 = 0, MAP_X1 = 3,
  MAP_K128 = 0, MAP_K256 = 1, MAP_MN = 2,   // offsets inside a triple
  MAP_A_K128 = 6, MAP_A_K256 = 7,
  MAP_B_K128 = 8, MAP_B_K256 = 9,
  // 32 x 32 boxes with 64-byte swizzle for the epilogue's bulk stores
  MAP_X0_ST = 10, MAP_X1_ST = 11, MAP_A_ST = 12, MAP_B_ST = 13,
  // 64 x 64 boxes of A and B for M/N-major loads: the single-CTA kernel
  // writes only the upper 256-block triangle of a symmetric buffer and reads
  // the blocks below it transposed from there
  MAP_A_MN = 14, MAP_B_MN = 15,
  kMapsPerMat = 16,
  kInMapsPerMat = 3
};

// The parameter update p' = p (1 - lr wd) - lr scale O taken into the last
// combine's epilogue: O (rounded to bf16, as the separate apply pass reads
// it) is not stored; 32 x 32 blocks of p are bulk-loaded into shared memory,
// updated there and bulk-stored back through `p_maps` of the launch.
struct ApplyArgs {
  int on = 0;
  float lr = 0.0f, wd = 0.0f;
  int scale_mode = 0;
  float extra_scale = 1.0f;
};

struct NsLaunch {
  const MatPlan* plans = nullptr;     // device
  const MatBind* binds = nullptr;     // device
  const TmapBlob* maps = nullptr;     // device, kMapsPerMat per matrix (workspace)
  const TmapBlob* in_maps = nullptr;  // device, kInMapsPerMat per matrix (caller input) or NULL
  const int4* tiles = nullptr;        // device tile list of the phase
  int ntiles = 0;
  const double* sumsq = nullptr;      // device or NULL
  DevStatus* status = nullptr;        // device
  int grid = 0;                       // persistent CTAs
  unsigned long long timeout_ns = 0;
  const TmapBlob* gmaps = nullptr;   // device, kGramMapsPerMat per matrix (Gram form only)
  int tma_store = 0;                 // 1: the *_ST store maps are present, stage outputs
                                     //    in shared memory and write them with bulk stores
  const GramBufs* gbufs = nullptr;   // device, one per matrix (Gram form only)
  int max_s = 1 << 30;               // largest s = min(m, n) of the listed matrices, or an
                                     // upper bound (the polynomial's identity form needs < 2048)
  ApplyArgs apply;                   // COMB only: update p instead of storing O
  const TmapBlob* p_maps = nullptr;  // device, one fp32 32 x 32 map of p per matrix (apply only)
};

// Small-matrix path: one CTA per listed matrix runs every iteration on chip.
struct NsSmallLaunch {
  const MatPlan* plans;      // device
  const MatBind* binds;      // device
  const TmapBlob* maps;      // device, kMapsPerMat per matrix
  const TmapBlob* in_maps;   // device, kInMapsPerMat per matrix or NULL
  const int* mats;           // device list of matrix indices
  int nmats;
  const double* sumsq;       // device or NULL
  DevStatus* status;         // device
  unsigned long long timeout_ns;
  int max_l = 1 << 30;       // largest max(m, n) of the listed matrices (<= 128: compact kernel)
};

// abc: ns_steps rows of (a, b, c).
cudaError_t launch_ns_small(const NsSmallLaunch& L, int ns_steps, int src_sel, int final_sel, const float* abc,
                            cudaStream_t st);
int ns_small_smem_bytes();

cudaError_t launch_ns_phase_pair(const NsLaunch& L, int phase, int src_sel, int dst_sel, int first, float a,
                                 float b, float c, cudaStream_t st);
int ns_pair_smem_bytes();
int ns_pair_clusters_resident();

cudaError_t launch_ns_phase_bf16(const NsLaunch& L, int phase, int src_sel, int dst_sel, int first, float a,
                                 float b, float c, cudaStream_t st, const PhaseSpec& spec = PhaseSpec());

// fp32 debug Newton-Schulz: one launch per matrix and phase.
cudaError_t launch_ns_phase_fp32(const MatPlan& mp_host, int mat, int phase, const float* src, float* dst,
                                 const double* sumsq, int first, float a, float b, float c, cudaStream_t st);

int ns_bf16_smem_bytes();

// Sets the calling thread's muon_last_error text.
void record_last_error(const std::string& msg);

}  // namespace muon
