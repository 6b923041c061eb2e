// Host-side check of the fused QKV kernel's tile schedule. The kernel source
// is included whole so that its own schedule functions are the ones checked;
// nothing here runs on a GPU. For each shape: the runs that the CTA pairs take
// in turn cover every tile exactly once; a run is one column tile over the
// consecutive token tiles of one chunk; no pair gets more than the balance
// bound of tiles; and the partial workspace has one slot per (batch element,
// head group, chunk, CTA of the pair). Prints one line per shape and "ALL OK".
#include "la_qkv_tc.cu"

#include <algorithm>
#include <cstdio>
#include <vector>

static bool check(int B, int N, int H, int C) {
  const la::QkvSched s = la::make_sched(B, N, H, C);
  const int NT = (N + 255) / 256, G = (H + 3) / 4, QC = (H * 32 + 255) / 256;
  if (s.NT != NT || s.G != G || s.CT != G + QC || s.total != B * NT * (G + QC)) {
    std::printf("shape %d %d %d %d: tile counts\n", B, N, H, C);
    return false;
  }
  if (s.L < 1 || s.L > std::max(1, NT) || s.NK != (NT + s.L - 1) / s.L ||
      s.units != B * s.NK * s.CT || s.pairs != std::max(1, std::min(74, s.units))) {
    std::printf("shape %d %d %d %d: runs and pairs\n", B, N, H, C);
    return false;
  }
  std::vector<int> seen(static_cast<size_t>(s.total), 0);
  int most = 0;
  for (int pair = 0; pair < s.pairs; ++pair) {
    int tiles = 0;
    for (int u = pair; u < s.units; u += s.pairs) {
      int i0 = 0, i1 = 0;
      la::run_span(s, u, i0, i1);
      const int b = u / (s.NK * s.CT), rem = u - b * s.NK * s.CT;
      const int k = rem / s.CT, ct = rem - k * s.CT;
      const int len = std::min(s.L, NT - k * s.L);
      // tiles of batch element b, chunk k are [base, base + len * CT), column-major
      const int base = b * NT * s.CT + k * s.L * s.CT;
      if (i1 - i0 != len || i0 != base + ct * len) {
        std::printf("shape %d %d %d %d: run %d spans [%d, %d)\n", B, N, H, C, u, i0, i1);
        return false;
      }
      for (int i = i0; i < i1; ++i) {
        if (i < 0 || i >= s.total) return false;
        ++seen[static_cast<size_t>(i)];
        ++tiles;
      }
    }
    most = std::max(most, tiles);
  }
  for (int i = 0; i < s.total; ++i)
    if (seen[static_cast<size_t>(i)] != 1) {
      std::printf("shape %d %d %d %d: tile %d taken %d times\n", B, N, H, C, i, seen[i]);
      return false;
    }
  const int bound = (s.units + s.pairs - 1) / s.pairs * s.L;
  if (most > bound) {
    std::printf("shape %d %d %d %d: a pair has %d tiles > %d\n", B, N, H, C, most, bound);
    return false;
  }
  const size_t want = static_cast<size_t>(B) * G * s.NK * 2 * la::kPartFloats;
  if (la::qkv_workspace_floats(B, N, H, C) != want) {
    std::printf("shape %d %d %d %d: workspace\n", B, N, H, C);
    return false;
  }
  std::printf("shape B=%d N=%d H=%d C=%d: L=%d NK=%d runs=%d pairs=%d busiest pair %d tiles (%d total)\n",
              B, N, H, C, s.L, s.NK, s.units, s.pairs, most, s.total);
  return true;
}

int main() {
  const int shapes[][4] = {
      {4, 1024, 70, 2240}, {1, 16384, 70, 2240}, {1, 32760, 70, 2240}, {1, 1024, 36, 1152},
      {2, 300, 5, 160},    {3, 1, 1, 32},        {1, 5000, 9, 288},    {7, 777, 13, 416},
      {1, 65536, 70, 2240}, {16, 256, 4, 128},   {1, 256, 200, 6400},
  };
  bool ok = true;
  for (const auto& sh : shapes) ok = check(sh[0], sh[1], sh[2], sh[3]) && ok;
  std::printf(ok ? "ALL OK\n" : "FAILED\n");
  return ok ? 0 : 1;
}
