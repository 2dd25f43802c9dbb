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
//
// Every table is sized when the directory is created (one list node per slot,
// an open-addressing index of twice the slot count), so a lookup never
// allocates and cannot fail part-way: it either completes or, for invalid
// arguments, is rejected by the caller before it starts.
#pragma once

#include <cstdint>
#include <vector>

namespace fmoe {

class ExpertCache {
 public:
  explicit ExpertCache(int n_slots)
      : n_slots_(n_slots), key_(n_slots), prev_(n_slots, -1), next_(n_slots, -1) {
    cap_ = 1;
    while (cap_ < 2 * n_slots) cap_ <<= 1;
    table_.assign(cap_, -1);
    reset();
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
      const int pos = find(key);
      if (table_[pos] >= 0) {
        const int s = table_[pos];
        unlink(s);
        push_front(s);  // now the most recent
        slot[k] = s;
        miss[k] = 0;
        ++hits_;
        continue;
      }
      int s;
      if (n_free_ > 0) {
        s = n_slots_ - n_free_;  // never-used slots in increasing order
        --n_free_;
      } else {
        s = tail_;  // the least recently used entry
        erase(key_[s]);
        unlink(s);
        ++evictions_;
      }
      key_[s] = key;
      table_[find(key)] = s;
      push_front(s);
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
    for (int& t : table_) t = -1;
    head_ = tail_ = -1;
    n_free_ = n_slots_;
    hits_ = misses_ = evictions_ = 0;
  }

 private:
  static uint64_t mix(uint64_t k) {  // a 64-bit finaliser to spread (layer, expert) keys
    k ^= k >> 33;
    k *= 0xff51afd7ed558ccdull;
    k ^= k >> 33;
    return k;
  }
  // Index position holding `key`, or the empty position where it would go
  // (linear probing; the table is never more than half full).
  int find(uint64_t key) const {
    int p = static_cast<int>(mix(key) & (cap_ - 1));
    while (table_[p] >= 0 && key_[table_[p]] != key) p = (p + 1) & (cap_ - 1);
    return p;
  }
  // Remove `key` (present) from the index, shifting later entries of its
  // probe run back so that no lookup stops early.
  void erase(uint64_t key) {
    int p = find(key);
    table_[p] = -1;
    for (int q = (p + 1) & (cap_ - 1); table_[q] >= 0; q = (q + 1) & (cap_ - 1)) {
      const int home = static_cast<int>(mix(key_[table_[q]]) & (cap_ - 1));
      // move the entry at q into the hole at p when its home is not in (p, q]
      const bool stays = (p <= q) ? (home > p && home <= q) : (home > p || home <= q);
      if (!stays) {
        table_[p] = table_[q];
        table_[q] = -1;
        p = q;
      }
    }
  }
  void unlink(int s) {
    if (prev_[s] >= 0) next_[prev_[s]] = next_[s]; else head_ = next_[s];
    if (next_[s] >= 0) prev_[next_[s]] = prev_[s]; else tail_ = prev_[s];
    prev_[s] = next_[s] = -1;
  }
  void push_front(int s) {
    prev_[s] = -1;
    next_[s] = head_;
    if (head_ >= 0) prev_[head_] = s; else tail_ = s;
    head_ = s;
  }

  int n_slots_;
  int cap_ = 1;
  int n_free_ = 0;                 // slots n_slots - n_free .. n_slots - 1 were never used
  std::vector<uint64_t> key_;      // (layer, expert) held by each used slot
  std::vector<int> prev_, next_;   // recency list over the used slots, most recent at head_
  std::vector<int> table_;         // open-addressing index: key -> slot (-1 = empty)
  int head_ = -1, tail_ = -1;
  uint64_t hits_ = 0, misses_ = 0, evictions_ = 0;
};

}  // namespace fmoe
