// rlb.cu -- run-time load balancing plan (FVAttn review, §1 Key Terms "RLB" and
// §3: once routing has fixed every head's amount of work, heads move between
// GPUs over P2P so that the critical path shortens).  Host code: the plan is a
// few dozen decisions over (batch, head) units, taken once per step.
//
// Rule: while the most loaded rank holds a unit whose work lies strictly between
// 0 and its gap to the least loaded rank, it hands the largest such unit (lowest
// home index among equal works) to that rank; ranks tie by lower index.  Each move
// lowers the sum of squared loads, so the plan ends.
#include <cstdint>
#include <set>
#include <utility>
#include <vector>

#include "fvattn.h"

extern "C" int fvattn_rlb_plan(const int64_t *work, int ranks, int units, int max_moves, int32_t *move_unit,
                               int32_t *move_src, int32_t *move_dst, int32_t *n_moves) {
    if (!work || !n_moves || ranks < 1 || units < 0 || max_moves < 0) return FVATTN_ERR_INVALID_ARG;
    if (max_moves > 0 && (!move_unit || !move_src || !move_dst)) return FVATTN_ERR_INVALID_ARG;
    const int64_t total = static_cast<int64_t>(ranks) * units;
    if (total >= (1LL << 31)) return FVATTN_ERR_UNSUPPORTED;
    for (int64_t u = 0; u < total; ++u)
        if (work[u] < 0) return FVATTN_ERR_INVALID_ARG;
    // per rank its movable units, ordered by (work ascending, home index descending):
    // the element just below (gap, lowest key) is the largest work under the gap,
    // and among equal works the lowest home index
    using Key = std::pair<int64_t, int32_t>;  // (work, -home index)
    std::vector<std::set<Key>> held(static_cast<size_t>(ranks));
    std::vector<int64_t> load(static_cast<size_t>(ranks), 0);
    for (int64_t u = 0; u < total; ++u) {
        const int r = static_cast<int>(u / (units > 0 ? units : 1));
        load[r] += work[u];
        if (work[u] > 0) held[r].insert(Key(work[u], -static_cast<int32_t>(u)));
    }
    int k = 0;
    for (;;) {
        int src = 0, dst = 0;
        for (int r = 1; r < ranks; ++r) {
            if (load[r] > load[src]) src = r;
            if (load[r] < load[dst]) dst = r;
        }
        const int64_t gap = load[src] - load[dst];
        auto it = held[src].lower_bound(Key(gap, INT32_MIN));
        if (it == held[src].begin()) break;  // no unit below the gap
        --it;
        const Key unit = *it;
        if (k == max_moves) {
            *n_moves = k;
            return FVATTN_ERR_CAPACITY;
        }
        held[src].erase(it);
        held[dst].insert(unit);
        load[src] -= unit.first;
        load[dst] += unit.first;
        move_unit[k] = -unit.second;
        move_src[k] = src;
        move_dst[k] = dst;
        ++k;
    }
    *n_moves = k;
    return FVATTN_OK;
}
