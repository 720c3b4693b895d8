// L2 prefetch of the weights the next GEMV of a decode step reads first.
#pragma once

#include "q4g_common.cuh"
#include "q4g_internal.h"

namespace q4g {

// Part `part` of `nparts` of the prefetch described by nx: the next GEMV's
// warps cw = part, part + nparts, ... each get the first nx.frac of their unit
// range prefetched (codes and scales of the rows of those units).
Q4G_DEV void prefetch_next(const NextGemv& nx, long long part, long long nparts) {
  if (nx.tw <= 0) return;
  const int kh = nx.k >> 1, nb = nx.k >> 5;
  for (long long cw = part; cw < nx.tw; cw += nparts) {
    const int ub = (int)(cw * nx.n_units / nx.tw), ue = (int)((cw + 1) * nx.n_units / nx.tw);
    const int cnt = (int)ceilf((float)(ue - ub) * nx.frac);
    if (cnt <= 0) continue;
    const int R = nx.unit_rows;
    if (nx.geglu) {
      const int h = R / 2;
      for (int s = 0; s < 2; ++s) {
        l2_prefetch(nx.seg[s].qs + (size_t)ub * h * kh, (uint64_t)cnt * h * kh);
        l2_prefetch(nx.seg[s].sc + (size_t)ub * h * nb, (uint64_t)cnt * h * nb * 2);
      }
    } else {
      const int r0 = R * ub, r1 = R * (ub + cnt);
      int base = 0;
      for (int s = 0; s < nx.nseg; ++s) {
        const int a = max(r0, base), b = min(r1, base + nx.seg[s].rows);
        if (a < b) {
          l2_prefetch(nx.seg[s].qs + (size_t)(a - base) * kh, (uint64_t)(b - a) * kh);
          l2_prefetch(nx.seg[s].sc + (size_t)(a - base) * nb, (uint64_t)(b - a) * nb * 2);
        }
        base += nx.seg[s].rows;
      }
    }
  }
}

}  // namespace q4g
