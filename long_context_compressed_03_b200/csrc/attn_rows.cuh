// attn_rows.cuh -- which keys one attention query row sees.
//
// Compressed part: the row's idx slots (CSA) or every visible entry
// s < min(floor((t+1)/m), n_entries) (HCA).  Window part: the raw rows whose
// positions lie in [max(0, t-W+1), t] and inside the cache's valid range
// [raw_pos0, raw_pos0 + raw_len).  ("百万上下文从「奢侈品」变「日用品」…" §4.3
// window bounds; "DS-V4 分析&学习" §1.4 HCA visibility.)
#pragma once
#include "common.cuh"
#include "kernels.h"

namespace csa {

struct RowKeys {
    int n_comp;      // compressed virtual keys (idx slots or visible entries)
    int win_lo;      // first raw row of the window
    int n_win;       // raw rows in the window
};

__device__ __forceinline__ RowKeys row_keys(const AttnArgs& a, int b, int t) {
    RowKeys k;
    if (a.dense) {
        const int ne = clampi(a.n_entries ? a.n_entries[b] : a.N_cap, 0, a.N_cap);
        k.n_comp = t < 0 ? 0 : min((t + 1) / a.m, ne);
    } else {
        k.n_comp = a.topk;
    }
    const int p0 = a.raw_pos0 ? a.raw_pos0[b] : a.raw_base;
    const int len = clampi(a.raw_len ? a.raw_len[b] : a.L_raw, 0, a.L_raw);
    // positions [max(0, t-W+1), t] ∩ [max(p0, 0), p0 + len - 1], as raw rows
    long lo = max((long)t - a.window + 1, 0L);
    lo = max(lo, (long)max(p0, 0));
    long hi = min((long)t, (long)p0 + len - 1);
    if (a.window <= 0 || hi < lo) {
        k.win_lo = 0;
        k.n_win = 0;
    } else {
        k.win_lo = (int)(lo - p0);
        k.n_win = (int)(hi - lo + 1);
    }
    return k;
}

}  // namespace csa
