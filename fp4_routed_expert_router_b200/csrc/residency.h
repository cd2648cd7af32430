// residency.h -- which arena slot holds which expert when the arena is smaller
// than the set of experts: least-recently-used replacement.
//
// Prior art: the hot-expert arena of 10100.com article 151357339 (section
// "方案一"), where a fixed number of expert slots is filled on demand and the
// least recently used expert makes room.  Here a "request" is the set of
// distinct experts one forward of one layer needs; a key is layer * E + expert.
//
// Plain host C++ (no CUDA): the library calls it before issuing the copies,
// and a host-only test compiles it with g++ to check the policy.
#pragma once
#include <cstdint>

namespace moe {

// Plan one request of n distinct keys.
//   owner[slot]  key held by the slot or -1          (updated)
//   where[key]   slot holding the key or -1          (updated)
//   last[slot]   clock of the slot's last request    (updated)
//   clock        this request's clock, larger than every earlier one
// For each key: slot_out[i] = its slot, hit_out[i] = 1 if it was already
// resident, evicted_out[i] = the key it displaced or -1.  A missing key takes
// the lowest-numbered free slot, else the slot with the oldest `last` among
// the slots this request has not claimed (lowest number on equal clocks).
// Returns false (and changes nothing) if n exceeds the number of slots.
inline bool lru_plan(int64_t* owner, int32_t* where, uint64_t* last, int n_slots, uint64_t clock,
                     const int64_t* keys, int n, int32_t* slot_out, uint8_t* hit_out, int64_t* evicted_out) {
    if (n > n_slots) return false;
    for (int i = 0; i < n; ++i) {                 // hits first: they are not eviction candidates
        const int32_t s = where[keys[i]];
        hit_out[i] = s >= 0 ? 1 : 0;
        slot_out[i] = s;
        evicted_out[i] = -1;
        if (s >= 0) last[s] = clock;
    }
    for (int i = 0; i < n; ++i) {
        if (hit_out[i]) continue;
        int victim = -1;
        for (int s = 0; s < n_slots; ++s)
            if (owner[s] < 0) { victim = s; break; }
        if (victim < 0) {
            for (int s = 0; s < n_slots; ++s)
                if (last[s] < clock && (victim < 0 || last[s] < last[victim])) victim = s;
        }
        if (victim < 0) return false;             // unreachable when n <= n_slots
        if (owner[victim] >= 0) {
            evicted_out[i] = owner[victim];
            where[owner[victim]] = -1;
        }
        owner[victim] = keys[i];
        where[keys[i]] = victim;
        last[victim] = clock;
        slot_out[i] = victim;
    }
    return true;
}

}  // namespace moe
