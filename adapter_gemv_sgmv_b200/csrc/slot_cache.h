// Slot policy of the resident adapter pool ("Serving several LoRAs, ControlNet and
// IP-Adapter", section "Placement": adapters stay resident and are swapped in on
// demand).  Pure host C++, no CUDA: which slot each adapter of a batch occupies,
// and which adapters must be (re)loaded.
//
// A batch's keys all become resident at once.  A key already resident keeps its
// slot; a missing key takes a free slot, else the least recently used slot that no
// key of this batch occupies.  A batch with more distinct keys than slots is
// rejected before anything changes.
#pragma once

#include <algorithm>
#include <cstdint>
#include <unordered_map>
#include <unordered_set>
#include <vector>

namespace lora {

class SlotCache {
public:
    explicit SlotCache(int n_slots) : key_(n_slots, -1), last_(n_slots, 0) {}

    int n_slots() const { return (int)key_.size(); }

    // slot of `key`, or -1 when it is not resident
    int find(int64_t key) const
    {
        auto it = slot_of_.find(key);
        return it == slot_of_.end() ? -1 : it->second;
    }

    int64_t key_in(int slot) const { return key_[slot]; }

    // forget `key` (its slot becomes free); a no-op when it is not resident
    void drop(int64_t key)
    {
        const int s = find(key);
        if (s < 0)
            return;
        slot_of_.erase(key);
        key_[s] = -1;
        last_[s] = 0;
    }

    // Undo part of an assignment: the keys of loads[from..] were marked resident
    // by assign() but their copies never happened, so they become missing again
    // (their slots free) and the next batch that needs them loads them.
    void rollback(const std::vector<std::pair<int, int64_t>> &loads, size_t from)
    {
        for (size_t i = from; i < loads.size(); ++i)
            drop(loads[i].second);
    }

    // Assign slots to keys[0..n); slots[i] receives keys[i]'s slot.  `loads`
    // receives (slot, key) for every key that must be copied in (once per
    // distinct missing key).  Returns false (nothing changed) if the distinct
    // keys do not fit.
    bool assign(const int64_t *keys, int n, int *slots, std::vector<std::pair<int, int64_t>> *loads)
    {
        loads->clear();
        const uint64_t tick = ++clock_;
        // distinct keys of this batch, in order of first appearance
        std::unordered_map<int64_t, int> batch;
        std::vector<int64_t> order;
        for (int i = 0; i < n; ++i)
            if (batch.emplace(keys[i], -1).second)
                order.push_back(keys[i]);
        if ((int)order.size() > n_slots())
            return false;
        // resident ones keep their slot and are marked as used by this batch
        for (int64_t k : order) {
            const int s = find(k);
            if (s >= 0) {
                batch[k] = s;
                last_[s] = tick;
            }
        }
        // missing ones take a free slot, else the least recently used one not in this batch
        for (int64_t k : order) {
            if (batch[k] >= 0)
                continue;
            int victim = -1;
            for (int s = 0; s < n_slots(); ++s) {
                if (last_[s] == tick)
                    continue;                 // holds a key of this batch
                if (key_[s] < 0) {
                    victim = s;
                    break;
                }
                if (victim < 0 || last_[s] < last_[victim])
                    victim = s;
            }
            if (key_[victim] >= 0)
                slot_of_.erase(key_[victim]);
            key_[victim] = k;
            slot_of_[k] = victim;
            last_[victim] = tick;
            batch[k] = victim;
            loads->emplace_back(victim, k);
        }
        for (int i = 0; i < n; ++i)
            slots[i] = batch[keys[i]];
        return true;
    }

    // Bring keys[0..n) in ahead of need, after this tick's assign(): each one not
    // resident takes a free slot, else the least recently used slot that no key of
    // this tick holds (the batch's keys and earlier preloads are never evicted);
    // it stops when no such slot is left.  `loads` receives (slot, key) per key.
    void preload(const int64_t *keys, int n, std::vector<std::pair<int, int64_t>> *loads)
    {
        loads->clear();
        const uint64_t tick = clock_;
        for (int i = 0; i < n; ++i) {
            if (find(keys[i]) >= 0)
                continue;
            int victim = -1;
            for (int s = 0; s < n_slots(); ++s) {
                if (last_[s] == tick && key_[s] >= 0)
                    continue;
                if (key_[s] < 0) {
                    victim = s;
                    break;
                }
                if (victim < 0 || last_[s] < last_[victim])
                    victim = s;
            }
            if (victim < 0)
                return;
            if (key_[victim] >= 0)
                slot_of_.erase(key_[victim]);
            key_[victim] = keys[i];
            slot_of_[keys[i]] = victim;
            last_[victim] = tick;
            loads->emplace_back(victim, keys[i]);
        }
    }

private:
    std::vector<int64_t> key_;                // key held by each slot (-1: free)
    std::vector<uint64_t> last_;              // batch tick of each slot's last use
    std::unordered_map<int64_t, int> slot_of_;
    uint64_t clock_ = 0;
};

// Co-occurrence of adapters in requests ("Co-occurrence Patterns of LoRA Adapters in
// Production Diffusion Model Inference Services", abstract: requests that carry
// several adapters combine them in recurring patterns, and preloading each adapter's
// top-k co-occurring partners covers most of them).  Counts, for every pair of
// distinct keys, the requests that carried both; top() ranks a key's partners.
class CoOccurrence {
public:
    // one request's keys (duplicates count once)
    void observe(const int64_t *keys, int n)
    {
        std::vector<int64_t> d;
        for (int i = 0; i < n; ++i)
            if (std::find(d.begin(), d.end(), keys[i]) == d.end())
                d.push_back(keys[i]);
        for (size_t i = 0; i < d.size(); ++i)
            for (size_t j = 0; j < d.size(); ++j)
                if (i != j)
                    ++count_[d[i]][d[j]];
    }

    // up to k partners of `key`, most frequent first (ties: smaller key first)
    void top(int64_t key, int k, std::vector<int64_t> *out) const
    {
        out->clear();
        auto it = count_.find(key);
        if (it == count_.end() || k <= 0)
            return;
        std::vector<std::pair<uint64_t, int64_t>> v;
        v.reserve(it->second.size());
        for (const auto &e : it->second)
            v.emplace_back(e.second, e.first);
        const size_t m = std::min<size_t>((size_t)k, v.size());
        std::partial_sort(v.begin(), v.begin() + m, v.end(), [](const auto &a, const auto &b) {
            return a.first != b.first ? a.first > b.first : a.second < b.second;
        });
        for (size_t i = 0; i < m; ++i)
            out->push_back(v[i].second);
    }

    uint64_t pairs(int64_t a, int64_t b) const
    {
        auto it = count_.find(a);
        if (it == count_.end())
            return 0;
        auto jt = it->second.find(b);
        return jt == it->second.end() ? 0 : jt->second;
    }

private:
    std::unordered_map<int64_t, std::unordered_map<int64_t, uint64_t>> count_;
};

}  // namespace lora
