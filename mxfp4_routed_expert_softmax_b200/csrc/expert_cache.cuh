// Expert cache: S slots of device memory hold the most recently used routed
// experts, the rest stay in host memory and are copied in when a call
// selects them.  The kimi-k3-in-c pages' defining idea is that the routed
// experts are never all resident -- their CPU engine streams each selected
// expert from NVMe into an LRU of RAM slots -- and here the same policy runs
// one level up: host memory -> HBM by the copy engine.  The layer kernels
// need nothing new: they reach every expert through the device pointer
// table, which the cache rewrites after each fetch (slot address of each
// resident expert, NULL for the others, so a selection that was not fetched
// is reported as a device check instead of reading stale bytes).
//
// Host-side bookkeeping only (this file holds no device code): the policy is
// least recently used over slots, deterministic -- within one fetch the
// requested experts are all marked used first, so no requested expert is
// evicted by another; each missing expert takes the free or least recently
// used slot (lowest slot on ties), in the order of first appearance.
#pragma once

#include <cstdint>
#include <cstring>
#include <vector>

namespace k3 {

struct ExpertCache {
    int E = 0;
    int S = 0;
    size_t blob_bytes = 0;
    size_t slot_bytes = 0;          // blob bytes rounded up to 256
    uint8_t *slots = nullptr;       // device memory, S * slot_bytes (the caller's)
    std::vector<const void *> host;  // E host blobs
    std::vector<int> slot_of;       // expert -> slot or -1
    std::vector<int> expert_of;     // slot -> expert or -1
    std::vector<uint64_t> last;     // slot -> last use (0: never)
    std::vector<uint64_t> stamp;    // expert -> fetch number it was last requested in
    uint64_t clock = 0;
    uint64_t requests = 0, hits = 0, fills = 0, evictions = 0;

    // The bookkeeping of one fetch: which experts need a copy, into which
    // slot.  Returns false (nothing changed) when more distinct experts are
    // asked for than there are slots, or an id is out of range.
    bool plan(const int32_t *experts, int n, std::vector<int> &fill_expert, std::vector<int> &fill_slot) {
        fill_expert.clear();
        fill_slot.clear();
        const uint64_t now = ++clock;
        int distinct = 0;
        for (int i = 0; i < n; ++i) {
            const int e = experts[i];
            if (e < 0 || e >= E) return false;
            if (stamp[e] != now) {
                stamp[e] = now;
                ++distinct;
            }
        }
        if (distinct > S) {
            // undo the marks so a failed fetch leaves no trace
            for (int i = 0; i < n; ++i) stamp[experts[i]] = 0;
            return false;
        }
        // resident requested experts: used now (they cannot be evicted below)
        std::vector<char> seen(E, 0);
        for (int i = 0; i < n; ++i) {
            const int e = experts[i];
            if (seen[e]) continue;
            seen[e] = 1;
            ++requests;
            if (slot_of[e] >= 0) {
                ++hits;
                last[slot_of[e]] = now;
            }
        }
        std::fill(seen.begin(), seen.end(), 0);
        for (int i = 0; i < n; ++i) {
            const int e = experts[i];
            if (seen[e] || slot_of[e] >= 0) {
                seen[e] = 1;
                continue;
            }
            seen[e] = 1;
            int best = -1;
            for (int s = 0; s < S; ++s)
                if (last[s] != now && (best < 0 || last[s] < last[best])) best = s;
            // best >= 0: at most S distinct experts are marked `now`
            if (expert_of[best] >= 0) {
                slot_of[expert_of[best]] = -1;
                ++evictions;
            }
            expert_of[best] = e;
            slot_of[e] = best;
            last[best] = now;
            ++fills;
            fill_expert.push_back(e);
            fill_slot.push_back(best);
        }
        return true;
    }

    // The device pointer table after a fetch.
    void table(std::vector<uint64_t> &out) const {
        out.assign(E, 0);
        for (int e = 0; e < E; ++e)
            if (slot_of[e] >= 0) out[e] = reinterpret_cast<uint64_t>(slots + (size_t)slot_of[e] * slot_bytes);
    }
};

}  // namespace k3
