// Host-side directory of a device-resident expert cache.
//
// The pages stream each layer's K selected experts from the SSD on demand
// and leave the caching to the operating system's page cache, a least-
// recently-used cache that hits about 71 % of the time ([P1] "Técnicas
// innovadoras" §1, [P2] "SSD-Experten-Streaming", [P3] "Trust the OS").  On
// B200 the analogue keeps the experts in pinned host memory and a pool of
// device slots, one expert blob each, as the cache.  This directory decides,
// for one layer's selected experts, which are already in a slot (hits) and
// which slot each miss is copied into: the least recently used slot over all
// layers, after the never-used slots (lowest first).  It moves no data and
// makes no CUDA call.
#pragma once

#include <cstdint>
#include <list>
#include <unordered_map>
#include <utility>
#include <vector>

namespace fmoe {

class ExpertCache {
 public:
  explicit ExpertCache(int n_slots) : n_slots_(n_slots) {
    for (int s = n_slots - 1; s >= 0; --s) free_.push_back(s);  // back = lowest
  }

  int n_slots() const { return n_slots_; }

  // Slot of each of the K experts (layer, idx[k]); miss[k] = 1 where the blob
  // must be copied into its slot.  The entries this call touches become the
  // most recently used, in k order; an expert listed twice takes one slot.
  // Requires K <= n_slots, so a victim is never an entry of this call.
  void lookup(int layer, const int32_t* idx, int K, int32_t* slot, int32_t* miss) {
    for (int k = 0; k < K; ++k) {
      const uint64_t key = (static_cast<uint64_t>(static_cast<uint32_t>(layer)) << 32) |
                           static_cast<uint32_t>(idx[k]);
      auto it = where_.find(key);
      if (it != where_.end()) {
        lru_.splice(lru_.begin(), lru_, it->second);  // now the most recent
        slot[k] = it->second->second;
        miss[k] = 0;
        ++hits_;
        continue;
      }
      int s;
      if (!free_.empty()) {
        s = free_.back();
        free_.pop_back();
      } else {
        const auto& victim = lru_.back();
        s = victim.second;
        where_.erase(victim.first);
        lru_.pop_back();
        ++evictions_;
      }
      lru_.emplace_front(key, s);
      where_[key] = lru_.begin();
      slot[k] = s;
      miss[k] = 1;
      ++misses_;
    }
  }

  void stats(uint64_t* hits, uint64_t* misses, uint64_t* evictions) const {
    if (hits) *hits = hits_;
    if (misses) *misses = misses_;
    if (evictions) *evictions = evictions_;
  }

  void reset() {
    lru_.clear();
    where_.clear();
    free_.clear();
    for (int s = n_slots_ - 1; s >= 0; --s) free_.push_back(s);
    hits_ = misses_ = evictions_ = 0;
  }

 private:
  int n_slots_;
  std::vector<int> free_;                      // never-used slots, lowest at the back
  std::list<std::pair<uint64_t, int>> lru_;    // (key, slot), most recent first
  std::unordered_map<uint64_t, std::list<std::pair<uint64_t, int>>::iterator> where_;
  uint64_t hits_ = 0, misses_ = 0, evictions_ = 0;
};

}  // namespace fmoe
