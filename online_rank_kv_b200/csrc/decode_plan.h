// Host-side planning of the persistent decode grid (pure C++, no CUDA: the
// CPU test suite compiles it on its own).
#pragma once

#include <algorithm>
#include <cstdint>
#include <vector>

namespace iskv {

// Tile ranges of the persistent decode grid: contiguous runs of the flattened
// (head, tile) space, at most nmax of them, of equal cost, where a run costs
// its tiles plus kHeadSwitchTiles for every head it enters after its first
// (publishing a partial, and restarting the pipeline on the next head's basis
// and queries).  Smallest feasible cost by bisection, runs filled greedily.
// Returns the number of runs; start[0..n] holds their bounds.
constexpr int64_t kHeadSwitchTiles = 4;

inline int fill_decode_runs(int64_t total, int64_t tph, int nmax, int64_t cost, int64_t* start) {
    int k = 0;
    int64_t p = 0;
    while (p < total) {
        if (k == nmax) return nmax + 1;
        start[k++] = p;
        int64_t budget = cost, q = p;
        for (bool first = true; q < total; first = false) {
            if (!first) {
                budget -= kHeadSwitchTiles;
                if (budget < 1) break;
            }
            const int64_t seg_end = std::min((q / tph + 1) * tph, total);
            const int64_t take = std::min(seg_end - q, budget);
            q += take;
            budget -= take;
            if (q < seg_end) break;
        }
        p = q > p ? q : p + 1;
    }
    start[k] = total;
    return k;
}

inline int partition_decode_tiles(int64_t total, int64_t tph, int nmax, int64_t* start) {
    // hi: one run holds everything
    int64_t lo = 1, hi = total + kHeadSwitchTiles * ((total + tph - 1) / tph);
    while (lo < hi) {
        const int64_t mid = lo + (hi - lo) / 2;
        if (fill_decode_runs(total, tph, nmax, mid, start) <= nmax) hi = mid;
        else lo = mid + 1;
    }
    return fill_decode_runs(total, tph, nmax, lo, start);
}

// The most runs that share one head: each run publishes two partial slots
// (one per epilogue group) for every head it visits.  start[0..nruns] are the
// run bounds over heads x tph flattened tiles.
inline int max_runs_per_head(const int64_t* start, int nruns, int heads, int64_t tph) {
    int most = 1, c0 = 0;
    for (int hh = 0; hh < heads; ++hh) {
        const int64_t f_first = (int64_t)hh * tph, f_last = f_first + tph - 1;
        while (c0 + 1 < nruns && start[c0 + 1] <= f_first) ++c0;
        int c1 = c0;
        while (c1 + 1 < nruns && start[c1 + 1] <= f_last) ++c1;
        most = std::max(most, c1 - c0 + 1);
    }
    return most;
}

// The grid plan of one decode call: at most nmax runs, fewer when a head
// would span more than cap_slots partial slots (per_run per run: one per
// epilogue group).  Decode calls
// repeat the same shape for 32 or more tokens in a row, so the last plan is
// kept and reused while its inputs are unchanged.
struct DecodeGridPlan {
    int64_t total = -1, tph = 0;
    int heads = 0, nmax = 0, cap_slots = 0, per_run = 0;
    int nruns = 0, slots = 0;        // slots: the most runs sharing one head
    std::vector<int64_t> start;      // nruns + 1 bounds
};

// Fills *p (or keeps it when already planned for these inputs).  Returns
// false when no plan keeps per_run slots per run within cap_slots.
inline bool plan_decode_grid(int64_t total, int64_t tph, int heads, int nmax, int cap_slots,
                             int per_run, DecodeGridPlan* p) {
    if (p->total == total && p->tph == tph && p->heads == heads && p->nmax == nmax &&
        p->cap_slots == cap_slots && p->per_run == per_run)
        return per_run * p->slots <= cap_slots;
    p->total = total;
    p->tph = tph;
    p->heads = heads;
    p->nmax = nmax;
    p->cap_slots = cap_slots;
    p->per_run = per_run;
    p->start.assign((size_t)nmax + 1, 0);
    int n = nmax;
    for (;;) {
        p->nruns = partition_decode_tiles(total, tph, n, p->start.data());
        p->slots = max_runs_per_head(p->start.data(), p->nruns, heads, tph);
        if (per_run * p->slots <= cap_slots || n == 1) break;
        n = std::max(1, n * (cap_slots - per_run) / (per_run * p->slots));
    }
    return per_run * p->slots <= cap_slots;
}

}  // namespace iskv
