// Host-side plan builder: geometry, workspace layout, tile lists and the
// elementwise chunk prefix for a shape table. Pure C++ (no CUDA calls), so
// the integer tables can be produced and checked without a GPU.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include "common.cuh"

namespace muon {

constexpr int kTileM = 128;     // output rows per tile (single-CTA tiles)
constexpr int kTileMPair = 256; // output rows per tile (CTA-pair tiles)
constexpr int kTileN = 256;     // output columns per tile
constexpr int kRegionAlign = 1024;
constexpr int kMaxDim = 1 << 20;
constexpr int kSmallMaxS = 128;     // small path: min(m, n) <= 128 ...
constexpr int kSmallMaxL = 512;     // ... and max(m, n) <= 512

struct TileRec {
  int mat, ti, tj;
};

struct HostPlan {
  int count = 0;
  int prec = 0;                       // 0 bf16, 1 fp32
  std::vector<int> m, n;
  std::vector<MatPlan> mats;          // workspace pointers left null
  std::vector<int64_t> region_off;    // count * 4: X0, X1, A, B
  int64_t head_bytes = 0;             // sum-of-squares block
  int64_t ws_bytes = 0;
  std::vector<TileRec> tiles[3];      // Gram, polynomial, combine
  std::vector<int> small;             // matrices on the on-chip small path
  int tile_m = kTileM;                // 128 (single CTA) or 256 (CTA pair)
  std::vector<long long> prefix;      // count + 1
  // Matrix groups under a workspace cap: group g is matrices
  // [groups[g], groups[g + 1]); every group's regions start after the
  // sum-of-squares block, so groups share the workspace and run one after
  // another. Without a cap (or when everything fits) there is one group.
  std::vector<int> groups;
};

// Validates the shape table (m, n in [1, kMaxDim], flags in {0, 1}) and
// builds the plan. With small_path, matrices with s <= kSmallMaxS and
// l <= kSmallMaxL go to the on-chip small path instead of the tile lists.
// With pair_tiles the tiles are 256 x 256 (one per CTA pair), else
// 128 x 256. Returns false with a message on invalid input.
// With ws_cap > 0 and a workspace above it, consecutive matrices are packed
// into groups whose workspace fits (each group as large as the cap allows,
// in index order); a matrix that alone exceeds the cap is an error.
bool build_plan(const int32_t* shapes, int count, int prec, bool small_path, bool pair_tiles, HostPlan& out,
                std::string& why, int64_t ws_cap = 0);

}  // namespace muon
