// expert_cache.h -- placement of routed experts in a fixed number of HBM
// slots, for layers whose experts do not all stay resident.
//
// The Colibrì pages keep only part of a model's experts in fast memory and
// fetch the rest on demand: "Colibri: 2400 lines of pure C ..." (kechuai.cn),
// section 二 (a per-layer cache with least-recently-used eviction and a
// learned set of hot experts that is never evicted); the project page
// (gh.puless.com/p/colibri.html), section on placement tiers. Here HBM is the
// cache and pinned host memory the backing store. Host code only.
#pragma once

#include <cstdint>
#include <utility>
#include <vector>

namespace coli {

class ExpertCache {
public:
    void init(int n_experts, int n_slots) {
        E = n_experts;
        slots = n_slots;
        slot_of.assign(E, -1);
        expert_in.assign(slots, -1);
        last_use.assign(slots, 0);
        pinned.assign(E, 0);
        uses.assign(E, 0);
        batch_mark.assign(E, 0);
        for (int s = 0; s < slots && s < E; ++s) place(s, s);  // experts 0..slots-1 start resident
    }

    // The batch's distinct experts `ex` (n of them): every one becomes
    // resident. Appends the copies to make, (expert, slot) pairs, to
    // `copies`. A missing expert takes a free slot, else the slot whose
    // expert was used least recently among those neither pinned nor needed
    // by this batch. Returns false (and changes nothing) if no such slot is
    // left for some missing expert.
    bool admit(const int32_t* ex, int n, std::vector<std::pair<int, int>>* copies) {
        ++clock;
        for (int i = 0; i < n; ++i) batch_mark[ex[i]] = clock;
        std::vector<std::pair<int, int>> plan;
        for (int i = 0; i < n; ++i) {
            const int e = ex[i];
            if (slot_of[e] >= 0) continue;
            const int s = victim(plan);
            if (s < 0) return false;
            plan.emplace_back(e, s);
        }
        for (const auto& c : plan) place(c.first, c.second);
        for (int i = 0; i < n; ++i) {
            last_use[slot_of[ex[i]]] = clock;
            ++uses[ex[i]];
        }
        hits += n - (int64_t)plan.size();
        misses += (int64_t)plan.size();
        copies->insert(copies->end(), plan.begin(), plan.end());
        return true;
    }

    // Best effort, ahead of need: makes the distinct experts `ex` resident in
    // order while a slot is left by the same rule as admit() (the experts of
    // this call count as the batch), counts them as used now, and appends the
    // copies. Routing counts, hits and misses are not changed.
    void prefetch(const int32_t* ex, int n, std::vector<std::pair<int, int>>* copies) {
        ++clock;
        for (int i = 0; i < n; ++i) batch_mark[ex[i]] = clock;
        std::vector<std::pair<int, int>> plan;
        for (int i = 0; i < n; ++i) {
            const int e = ex[i];
            if (slot_of[e] >= 0) {
                last_use[slot_of[e]] = clock;
                continue;
            }
            const int s = victim(plan);
            if (s < 0) break;
            plan.emplace_back(e, s);
            place(e, s);
            last_use[s] = clock;
        }
        copies->insert(copies->end(), plan.begin(), plan.end());
    }

    // Marks experts as never evicted (the learned hot set). Fails when the
    // pinned experts would leave fewer than `reserve` slots for the others.
    bool pin(const int32_t* ex, int n, int reserve) {
        std::vector<char> p(E, 0);
        int count = 0;
        for (int i = 0; i < n; ++i) {
            if (ex[i] < 0 || ex[i] >= E) return false;
            count += !p[ex[i]];
            p[ex[i]] = 1;
        }
        if (count > slots - reserve) return false;
        pinned.swap(p);
        return true;
    }

    // The n experts routed to most often so far (ties: lower id), as a
    // learned hot set for pin().
    std::vector<int32_t> most_used(int n) const {
        std::vector<int32_t> out;
        std::vector<char> done(E, 0);
        for (int k = 0; k < n && k < E; ++k) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!done[e] && (best < 0 || uses[e] > uses[best])) best = e;
            done[best] = 1;
            out.push_back(best);
        }
        return out;
    }

    int slot(int e) const { return slot_of[e]; }
    bool is_pinned(int e) const { return pinned[e] != 0; }

    int E = 0, slots = 0;
    int64_t hits = 0, misses = 0;
    std::vector<int> slot_of;     // [E] slot of each expert, -1 when not resident
    std::vector<int> expert_in;   // [slots] expert in each slot, -1 when free
    std::vector<int64_t> uses;    // [E] batches that routed to each expert

private:
    // A slot for one more missing expert of the current batch: free, else
    // least recently used among those whose expert is neither pinned nor in
    // the batch; slots already given out in `plan` are skipped. -1: none.
    int victim(const std::vector<std::pair<int, int>>& plan) const {
        int best = -1;
        for (int s = 0; s < slots; ++s) {
            bool taken = false;
            for (const auto& c : plan) taken |= c.second == s;
            if (taken) continue;
            const int o = expert_in[s];
            if (o < 0) return s;
            if (pinned[o] || batch_mark[o] == clock) continue;
            if (best < 0 || last_use[s] < last_use[best]) best = s;
        }
        return best;
    }

    void place(int e, int s) {
        if (expert_in[s] >= 0) slot_of[expert_in[s]] = -1;
        expert_in[s] = e;
        slot_of[e] = s;
    }
    int64_t clock = 0;
    std::vector<int64_t> last_use;  // [slots]
    std::vector<char> pinned;       // [E]
    std::vector<int64_t> batch_mark;  // [E] batch that last needed each expert
};

}  // namespace coli
