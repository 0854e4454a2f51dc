// Plan builder. The rules (restated independently by the test oracle):
//  * orientation: m > n is tall, s = min(m, n), l = max(m, n) ("About Muon:
//    Why Not Adam", section "The whole thing, in about forty lines": the
//    iteration runs on the short side, square matrices are not transposed);
//  * storage: X buffers m x round_up(n, 8), A and B s x round_up(s, 8), so
//    every row starts on a 16-byte boundary as the bulk-tensor copy engine
//    requires; the workspace starts with one double per matrix (sum of
//    squares) padded to 1024 bytes, followed by all X0, all X1, all A and
//    all B regions, each aligned to 1024 bytes;
//  * tiles of BM x 256 (BM = 128 for single-CTA tiles, 256 for CTA pairs):
//    for the symmetric Gram and polynomial outputs only tiles whose
//    256-column block is on or right of the 256-block diagonal
//    (tj >= ti * BM / 256); for the combine every tile, column block outer for wide
//    matrices and row block outer for tall ones (each wave of CTAs then
//    shares the large X panel in L2); each phase's list is ordered by the
//    matrix's reduction length, longest first, ties by matrix index;
//  * small path (when enabled): matrices with s <= 128 and l <= 512 are left
//    out of the tile lists and listed, in index order, for the on-chip
//    kernel that runs the whole iteration in one CTA;
//  * elementwise: kElemChunk elements per block, prefix over matrices;
//  * workspace cap: when the layout above exceeds a cap, consecutive
//    matrices are packed into groups (each as large as fits, in index
//    order); each group's X0, X1, A and B regions are laid out as above
//    starting right after the sum-of-squares block, so the workspace is that
//    block plus the largest group.
#include "plan.h"

#include <algorithm>
#include <numeric>

namespace muon {

namespace {

int64_t round_up64(int64_t x, int64_t k) { return (x + k - 1) / k * k; }
int ceil_div_i(int x, int k) { return (x + k - 1) / k; }

void sym_tiles(int mat, int s, int bm, std::vector<TileRec>& out) {
  const int rt = ceil_div_i(s, bm), ct = ceil_div_i(s, kTileN);
  for (int ti = 0; ti < rt; ++ti)
    for (int tj = ti * bm / kTileN; tj < ct; ++tj) out.push_back({mat, ti, tj});
}

void comb_tiles(int mat, int m, int n, int bm, std::vector<TileRec>& out) {
  const int rt = ceil_div_i(m, bm), ct = ceil_div_i(n, kTileN);
  if (m <= n) {
    for (int tj = 0; tj < ct; ++tj)
      for (int ti = 0; ti < rt; ++ti) out.push_back({mat, ti, tj});
  } else {
    for (int ti = 0; ti < rt; ++ti)
      for (int tj = 0; tj < ct; ++tj) out.push_back({mat, ti, tj});
  }
}

}  // namespace

bool build_plan(const int32_t* shapes, int count, int prec, bool small_path, bool pair_tiles, HostPlan& P,
                std::string& why, int64_t ws_cap) {
  if (shapes == nullptr) { why = "shapes is NULL"; return false; }
  if (count < 1) { why = "count must be >= 1"; return false; }
  if (prec != 0 && prec != 1) { why = "ns_precision must be 0 (bf16) or 1 (fp32)"; return false; }
  P = HostPlan();
  P.count = count;
  P.prec = prec;
  P.tile_m = pair_tiles ? kTileMPair : kTileM;
  const int bm = P.tile_m;
  P.m.resize(count);
  P.n.resize(count);
  P.mats.resize(count);
  for (int i = 0; i < count; ++i) {
    const int m = shapes[3 * i], n = shapes[3 * i + 1], fl = shapes[3 * i + 2];
    if (m < 1 || n < 1 || m > kMaxDim || n > kMaxDim) {
      why = "matrix " + std::to_string(i) + ": m and n must be in [1, " + std::to_string(kMaxDim) + "], got " +
            std::to_string(m) + " x " + std::to_string(n);
      return false;
    }
    if (fl & ~1) { why = "matrix " + std::to_string(i) + ": unknown flag bits"; return false; }
    P.m[i] = m;
    P.n[i] = n;
    MatPlan& mp = P.mats[i];
    mp = MatPlan();
    mp.m = m;
    mp.n = n;
    mp.s = std::min(m, n);
    mp.l = std::max(m, n);
    mp.tall = m > n ? 1 : 0;
    mp.ldx = round_up_i(n, 8);
    mp.lds = round_up_i(mp.s, 8);
    mp.numel = (long long)m * (long long)n;
  }
  const int64_t elem = prec == 0 ? 2 : 4;
  P.head_bytes = round_up64(8 * (int64_t)count, kRegionAlign);
  auto region_bytes = [&](int i, int which) {
    const MatPlan& mp = P.mats[i];
    return round_up64((which < 2 ? (int64_t)mp.m * mp.ldx : (int64_t)mp.s * mp.lds) * elem, kRegionAlign);
  };
  auto matrix_bytes = [&](int i) {
    int64_t b = 0;
    for (int which = 0; which < 4; ++which) b += region_bytes(i, which);
    return b;
  };
  int64_t all = 0;
  for (int i = 0; i < count; ++i) all += matrix_bytes(i);
  P.groups.assign(1, 0);
  if (ws_cap > 0 && P.head_bytes + all > ws_cap) {
    int64_t in_group = 0;
    for (int i = 0; i < count; ++i) {
      const int64_t b = matrix_bytes(i);
      if (P.head_bytes + b > ws_cap) {
        why = "matrix " + std::to_string(i) + " alone needs " + std::to_string(P.head_bytes + b) +
              " bytes of workspace, above the cap of " + std::to_string(ws_cap);
        return false;
      }
      if (P.head_bytes + in_group + b > ws_cap) {
        P.groups.push_back(i);
        in_group = 0;
      }
      in_group += b;
    }
  }
  P.groups.push_back(count);
  P.region_off.assign((size_t)count * 4, 0);
  P.ws_bytes = P.head_bytes;
  for (size_t g = 0; g + 1 < P.groups.size(); ++g) {
    int64_t off = P.head_bytes;
    for (int which = 0; which < 4; ++which)
      for (int i = P.groups[g]; i < P.groups[g + 1]; ++i) {
        P.region_off[(size_t)i * 4 + which] = off;
        off += region_bytes(i, which);
      }
    P.ws_bytes = std::max(P.ws_bytes, off);
  }

  std::vector<char> is_small((size_t)count, 0);
  if (small_path)
    for (int i = 0; i < count; ++i)
      if (P.mats[i].s <= kSmallMaxS && P.mats[i].l <= kSmallMaxL) {
        is_small[i] = 1;
        P.small.push_back(i);
      }
  std::vector<int> order(count);
  auto sorted_by = [&](auto key) {
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return key(x) > key(y); });
    return order;
  };
  for (int i : sorted_by([&](int i) { return P.mats[i].l; }))
    if (!is_small[i]) sym_tiles(i, P.mats[i].s, bm, P.tiles[0]);
  for (int i : sorted_by([&](int i) { return P.mats[i].s; }))
    if (!is_small[i]) sym_tiles(i, P.mats[i].s, bm, P.tiles[1]);
  for (int i : sorted_by([&](int i) { return P.mats[i].s; }))
    if (!is_small[i]) comb_tiles(i, P.m[i], P.n[i], bm, P.tiles[2]);

  P.prefix.assign((size_t)count + 1, 0);
  for (int i = 0; i < count; ++i)
    P.prefix[i + 1] = P.prefix[i] + ceil_div_ll(P.mats[i].numel, kElemChunk);
  return true;
}

}  // namespace muon
