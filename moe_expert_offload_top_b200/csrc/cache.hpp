// Host-side shared LRU slot table for routed experts.
//
// Method: one LRU over the GPU expert slots, shared by every MoE layer, so
// recently chosen experts stay for later tokens; a miss copies the expert from
// host memory into a slot and keeps it ("FreeToken linux", "FreeToken's MoE
// memory handling"; "FreeToken gguf", the `offload` backend).  Resizing at a
// safe point changes capacity, not results ("FreeToken RTX 5090", dynamic
// reconfiguration).
//
// Order inside one access set (the pages give none; this library's rule):
// the resident experts of the set, ascending, become most recently used; then
// the missing ones, ascending, each take the lowest free slot or evict the
// least recently used entry, and become most recently used.
//
// Representation: key = layer * E + expert; slot_of[key] (dense, -1 if absent),
// key_of[slot]; a doubly linked recency list threaded through the slots
// (head = least recently used); a min-heap of free slots.
#pragma once
#include <algorithm>
#include <functional>
#include <queue>
#include <utility>
#include <vector>

namespace ftc {

struct Access {
  int call, layer, expert, kind, hit, slot, ev_layer, ev_expert;
};

class SlotLru {
 public:
  void reset(int num_keys, int capacity) {
    cap_ = capacity;
    slot_of_.assign(num_keys, -1);
    key_of_.assign(capacity, -1);
    prev_.assign(capacity, -1);
    next_.assign(capacity, -1);
    head_ = tail_ = -1;
    size_ = 0;
    free_ = decltype(free_)();
    for (int s = 0; s < capacity; ++s) free_.push(s);
  }
  int capacity() const { return cap_; }
  int size() const { return size_; }
  int slot_of(int key) const { return key >= 0 && key < (int)slot_of_.size() ? slot_of_[key] : -1; }
  int key_of(int slot) const { return slot >= 0 && slot < cap_ ? key_of_[slot] : -1; }

  // Accesses the sorted distinct keys `keys` (all of one layer).  Appends one
  // record per key to `out` (hits first, then misses) and returns false,
  // changing nothing, if keys.size() > capacity.
  bool access_set(const std::vector<int>& keys, int E, int call, int kind, std::vector<Access>& out) {
    if ((int)keys.size() > cap_) return false;
    for (int key : keys) {
      int s = slot_of_[key];
      if (s >= 0) {
        unlink(s);
        push_mru(s);
        out.push_back({call, key / E, key % E, kind, 1, s, -1, -1});
      }
    }
    for (int key : keys) {
      if (slot_of_[key] >= 0) continue;
      int s, evl = -1, eve = -1;
      if (!free_.empty()) {
        s = free_.top();
        free_.pop();
      } else {
        s = head_;
        int victim = key_of_[s];
        unlink(s);
        slot_of_[victim] = -1;
        --size_;
        evl = victim / E;
        eve = victim % E;
      }
      key_of_[s] = key;
      slot_of_[key] = s;
      push_mru(s);
      ++size_;
      out.push_back({call, key / E, key % E, kind, 0, s, evl, eve});
    }
    return true;
  }

  // Removes the entry in `slot` (used to roll back a failed fill).
  void drop(int slot) {
    int key = key_of_[slot];
    if (key < 0) return;
    unlink(slot);
    slot_of_[key] = -1;
    key_of_[slot] = -1;
    --size_;
    free_.push(slot);
  }

  // Changes capacity.  Returns evicted keys and (old_slot, new_slot) moves.
  void resize(int new_cap, std::vector<int>& evicted, std::vector<std::pair<int, int>>& moves) {
    if (new_cap >= cap_) {
      key_of_.resize(new_cap, -1);
      prev_.resize(new_cap, -1);
      next_.resize(new_cap, -1);
      for (int s = cap_; s < new_cap; ++s) free_.push(s);
      cap_ = new_cap;
      return;
    }
    while (size_ > new_cap) {
      int s = head_;
      int key = key_of_[s];
      unlink(s);
      slot_of_[key] = -1;
      key_of_[s] = -1;
      --size_;
      evicted.push_back(key);
    }
    // recency order, MRU first
    std::vector<int> order;
    for (int s = tail_; s >= 0; s = prev_[s]) order.push_back(s);
    std::vector<char> used(new_cap, 0);
    for (int s : order)
      if (s < new_cap) used[s] = 1;
    int low = 0;
    std::vector<int> new_slot_of_old(cap_, -1);
    for (int s : order) {
      if (s < new_cap) { new_slot_of_old[s] = s; continue; }
      while (used[low]) ++low;
      used[low] = 1;
      moves.push_back({s, low});
      new_slot_of_old[s] = low;
    }
    // rebuild arrays with the new numbering, keeping recency (order is MRU first)
    std::vector<int> keys_lru_first;
    for (auto it = order.rbegin(); it != order.rend(); ++it) keys_lru_first.push_back(key_of_[*it]);
    std::vector<int> slots_lru_first;
    for (auto it = order.rbegin(); it != order.rend(); ++it) slots_lru_first.push_back(new_slot_of_old[*it]);
    cap_ = new_cap;
    key_of_.assign(new_cap, -1);
    prev_.assign(new_cap, -1);
    next_.assign(new_cap, -1);
    head_ = tail_ = -1;
    size_ = 0;
    for (size_t i = 0; i < keys_lru_first.size(); ++i) {
      int s = slots_lru_first[i], key = keys_lru_first[i];
      key_of_[s] = key;
      slot_of_[key] = s;
      push_mru(s);
      ++size_;
    }
    free_ = decltype(free_)();
    for (int s = 0; s < new_cap; ++s)
      if (key_of_[s] < 0) free_.push(s);
  }

 private:
  void unlink(int s) {
    int p = prev_[s], n = next_[s];
    if (p >= 0) next_[p] = n; else head_ = n;
    if (n >= 0) prev_[n] = p; else tail_ = p;
    prev_[s] = next_[s] = -1;
  }
  void push_mru(int s) {
    prev_[s] = tail_;
    next_[s] = -1;
    if (tail_ >= 0) next_[tail_] = s; else head_ = s;
    tail_ = s;
  }

  int cap_ = 0, head_ = -1, tail_ = -1, size_ = 0;
  std::vector<int> slot_of_, key_of_, prev_, next_;
  std::priority_queue<int, std::vector<int>, std::greater<int>> free_;
};

}  // namespace ftc
