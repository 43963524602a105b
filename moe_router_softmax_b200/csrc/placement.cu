// placement.cu -- the expert residency pool's host logic (rlx_runtime
// expert_pool.rs): hit-ranked target selection, paired promote/demote on a
// cache-slot table, the refresh schedule and the VRAM budget formula.
// Pure host code; no CUDA.
#include <algorithm>
#include <vector>

#include "common.cuh"

using namespace moe;

extern "C" {

moe_status moe_refresh_target(const uint32_t *hits, int32_t E, int32_t budget, int32_t *target, int32_t *n_target) {
    if (!hits || !target || !n_target) return set_error(MOE_ERR_INVALID_ARG, "moe_refresh_target: NULL pointer");
    if (E < 1 || E > kMaxE || budget < 0) return set_error(MOE_ERR_INVALID_ARG, "moe_refresh_target: E=%d budget=%d", E, budget);
    // target_gpu_from_counts: count > 0, count descending, id ascending, first `budget`
    std::vector<int32_t> ranked;
    ranked.reserve(E);
    for (int32_t e = 0; e < E; ++e)
        if (hits[e] > 0) ranked.push_back(e);
    std::stable_sort(ranked.begin(), ranked.end(), [&](int32_t a, int32_t b) { return hits[a] > hits[b]; });
    const int32_t n = std::min<int32_t>(budget, (int32_t)ranked.size());
    for (int32_t i = 0; i < n; ++i) target[i] = ranked[i];
    *n_target = n;
    return MOE_OK;
}

moe_status moe_apply_placement(int32_t *slot_of, int32_t E, int32_t n_slots, const int32_t *target, int32_t n_target,
                               int32_t *promote, int32_t *demote, int32_t *n_promote, int32_t *n_demote) {
    if (!slot_of || (!target && n_target) || !promote || !demote || !n_promote || !n_demote)
        return set_error(MOE_ERR_INVALID_ARG, "moe_apply_placement: NULL pointer");
    if (E < 1 || E > kMaxE || n_slots < 0 || n_target < 0 || n_target > n_slots)
        return set_error(MOE_ERR_INVALID_ARG, "moe_apply_placement: E=%d n_slots=%d n_target=%d", E, n_slots, n_target);
    std::vector<char> in_target(E, 0), slot_used(n_slots, 0);
    for (int32_t i = 0; i < n_target; ++i) {
        if (target[i] < 0 || target[i] >= E) return set_error(MOE_ERR_INVALID_ARG, "target[%d]=%d outside [0,E)", i, target[i]);
        if (in_target[target[i]]) return set_error(MOE_ERR_INVALID_ARG, "expert %d twice in the target", target[i]);
        in_target[target[i]] = 1;
    }
    for (int32_t e = 0; e < E; ++e) {
        if (slot_of[e] >= n_slots) return set_error(MOE_ERR_INVALID_ARG, "slot_of[%d]=%d >= n_slots", e, slot_of[e]);
        if (slot_of[e] >= 0) {
            if (slot_used[slot_of[e]]) return set_error(MOE_ERR_INVALID_ARG, "slot %d held twice", slot_of[e]);
            slot_used[slot_of[e]] = 1;
        }
    }
    // paired promote / demote (apply_target_placement); demote candidates in id order
    int32_t np = 0, nd = 0;
    for (int32_t i = 0; i < n_target; ++i)
        if (slot_of[target[i]] < 0) promote[np++] = target[i];
    for (int32_t e = 0; e < E && nd < np; ++e)
        if (slot_of[e] >= 0 && !in_target[e]) demote[nd++] = e;
    int32_t free_cursor = 0;
    for (int32_t i = 0; i < np; ++i) {
        int32_t slot;
        if (i < nd) {
            slot = slot_of[demote[i]];
            slot_of[demote[i]] = -1;
        } else {
            while (free_cursor < n_slots && slot_used[free_cursor]) ++free_cursor;
            if (free_cursor >= n_slots) return set_error(MOE_ERR_INVALID_ARG, "no free slot for expert %d", promote[i]);
            slot = free_cursor;
            slot_used[slot] = 1;
        }
        slot_of[promote[i]] = slot;
    }
    *n_promote = np;
    *n_demote = nd;
    return MOE_OK;
}

moe_status moe_hits_window(const uint32_t *ring, int32_t W, int32_t E, uint32_t *sum) {
    if (!ring || !sum) return set_error(MOE_ERR_INVALID_ARG, "moe_hits_window: NULL pointer");
    if (E < 1 || E > kMaxE || W < 1) return set_error(MOE_ERR_INVALID_ARG, "moe_hits_window: E=%d W=%d", E, W);
    for (int32_t e = 0; e < E; ++e) {
        uint32_t acc = 0;
        for (int32_t s = 0; s < W; ++s) acc += ring[(size_t)s * E + e];
        sum[e] = acc;
    }
    return MOE_OK;
}

int32_t moe_should_refresh(int32_t offload_enabled, int32_t mode_refresh, int64_t step, int32_t is_prefill_block,
                           int64_t interval) {
    if (!offload_enabled) return 0;
    if (mode_refresh || is_prefill_block) return 1;
    const int64_t n = interval < 1 ? 1 : interval;
    return step % n == 0 ? 1 : 0;
}

int64_t moe_budget_from_vram(int64_t free_bytes, int64_t reserve_bytes, int64_t expert_bytes, int64_t layers,
                             int64_t max_per_layer, int64_t E) {
    const int64_t cap = std::min(max_per_layer, E);
    if (expert_bytes == 0 || layers == 0) return cap;
    const int64_t usable = free_bytes > reserve_bytes ? free_bytes - reserve_bytes : 0;
    return std::min(usable / (expert_bytes * layers), cap);
}

}  // extern "C"
