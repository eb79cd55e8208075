// Host block allocator of the paged KV cache: fixed-size blocks, per-sequence
// block tables, blocks handed out on demand, reference counts and
// copy-on-write for shared prompt blocks (vLLM launch blog, "PagedAttention"
// section, as summarised on the CSDN discovery note, item 2; agientry.com
// overview, opening section).  The exact orders (LIFO free stack seeded from
// the caller's order, copy-on-write trigger, free in table order) are stated
// in include/pa.h.
//
// Plain host code: O(1) per token, no CUDA.  Every request checks its
// arguments and its block needs before changing anything, so a failed call
// leaves the state untouched.

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <list>
#include <memory>
#include <set>
#include <unordered_map>
#include <vector>

#include "../../include/pa.h"

namespace {

struct Seq {
  std::vector<int32_t> table;
  int32_t len = 0;
  bool tracked = true;          // token ids of every position are known
  std::vector<int64_t> tokens;  // (prefix caching) ids of positions 0..len-1
  bool swapped = false;         // swapped out: table is empty, host holds the blocks
  std::vector<int32_t> host;    // host blocks of a swapped-out sequence, in table order
};

// Prefix-cache key of a full block: its parent block (-1 for a sequence's
// first block) and its token ids.  Exact comparison: a match never relies on
// a hash alone.
struct Key {
  int32_t parent;
  std::vector<int64_t> toks;
  bool operator==(const Key& o) const { return parent == o.parent && toks == o.toks; }
};

struct KeyHash {
  size_t operator()(const Key& k) const {
    uint64_t h = 0x9E3779B97F4A7C15ull ^ static_cast<uint64_t>(static_cast<uint32_t>(k.parent));
    for (int64_t t : k.toks) {
      h ^= static_cast<uint64_t>(t) + 0x9E3779B97F4A7C15ull + (h << 6) + (h >> 2);
    }
    return static_cast<size_t>(h);
  }
};

// Runs the body of a C entry point: no C++ exception may cross the C ABI,
// and the only ones this code can raise come from host allocation
// (std::bad_alloc, or std::length_error for an impossible size).
template <typename F>
pa_status no_throw(F&& body) {
  try {
    return body();
  } catch (...) {
    return PA_ERR_HOST_ALLOC;
  }
}

}  // namespace

struct pa_allocator {
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  std::vector<int32_t> free_stack;  // top = back()
  std::vector<int32_t> ref;
  std::unordered_map<int64_t, Seq> seqs;

  // Prefix caching: registered full blocks, their children, and the
  // registered blocks nobody holds (evictable, least recently freed first).
  std::unordered_map<Key, int32_t, KeyHash> cache;
  std::vector<uint8_t> reg;
  std::vector<Key> key_of;
  std::vector<std::set<int32_t>> children;
  std::list<int32_t> lru;
  std::vector<std::list<int32_t>::iterator> lru_pos;
  std::vector<uint8_t> in_lru;

  // Swapping: a pool of host blocks with its own LIFO free stack.
  int32_t num_host_blocks = 0;
  std::vector<int32_t> host_free;

  void init_cache_state() {
    reg.assign(num_blocks, 0);
    key_of.assign(num_blocks, Key{-1, {}});
    children.assign(num_blocks, {});
    lru_pos.assign(num_blocks, lru.end());
    in_lru.assign(num_blocks, 0);
  }

  int64_t available() const { return static_cast<int64_t>(free_stack.size()) + static_cast<int64_t>(lru.size()); }

  // Unregister block `root` and, below it, every registered descendant in
  // increasing block order, depth first.  A descendant that nobody holds
  // loses its key and goes back on the free stack once its own subtree is
  // done.  Iterative: a registered chain is as deep as its sequence is long
  // in blocks, far beyond what recursion on a thread's stack can take.
  void unregister(int32_t root) {
    struct Frame {
      int32_t b;
      std::vector<int32_t> kids;  // b's registered children, increasing
      size_t next;
    };
    std::vector<Frame> stack;
    auto enter = [&](int32_t b) {
      cache.erase(key_of[b]);
      reg[b] = 0;
      const int32_t parent = key_of[b].parent;
      if (parent >= 0) children[parent].erase(b);
      Frame f{b, std::vector<int32_t>(children[b].begin(), children[b].end()), 0};
      children[b].clear();
      stack.push_back(std::move(f));
    };
    enter(root);
    while (!stack.empty()) {
      Frame& top = stack.back();
      if (top.next < top.kids.size()) {
        const int32_t c = top.kids[top.next++];
        enter(c);  // may reallocate `stack`: `top` is not used after this
        continue;
      }
      const int32_t c = top.b;
      stack.pop_back();
      if (!stack.empty() && in_lru[c]) {  // a descendant, not the root
        lru.erase(lru_pos[c]);
        in_lru[c] = 0;
        free_stack.push_back(c);
      }
    }
  }

  int32_t take_block() {
    if (!free_stack.empty()) {
      const int32_t b = free_stack.back();
      free_stack.pop_back();
      return b;
    }
    const int32_t b = lru.front();
    lru.pop_front();
    in_lru[b] = 0;
    unregister(b);
    return b;
  }

  void register_block(int32_t b, int32_t parent, const int64_t* toks) {
    if (parent >= 0 && !reg[parent]) return;
    Key k{parent, std::vector<int64_t>(toks, toks + block_size)};
    if (reg[b] || cache.count(k)) return;
    key_of[b] = k;
    cache.emplace(std::move(k), b);
    reg[b] = 1;
    if (parent >= 0) children[parent].insert(b);
  }

  void release(int32_t b) {
    ref[b] -= 1;
    if (ref[b] == 0) {
      if (reg[b]) {
        lru.push_back(b);
        lru_pos[b] = std::prev(lru.end());
        in_lru[b] = 1;
      } else {
        free_stack.push_back(b);
      }
    }
  }

  // Blocks an append of n tokens to s needs (copy-on-write + fresh blocks).
  int64_t blocks_needed(const Seq& s, int64_t n) const {
    const int64_t bs = block_size;
    const int64_t pos = s.len;
    int64_t need = 0;
    if (n > 0 && pos % bs != 0 && ref[s.table.back()] > 1) need += 1;
    const int64_t first = (pos + bs - 1) / bs * bs;  // first position >= pos opening a block
    if (first < pos + n) need += (pos + n - 1 - first) / bs + 1;
    return need;
  }

  // ids: token ids of the n tokens (prefix caching), or null (unknown ids).
  pa_status append(int64_t seq_id, int32_t n, const int64_t* ids, int64_t* slots, int64_t* cow_pair,
                   int32_t* n_cow) {
    auto it = seqs.find(seq_id);
    if (it == seqs.end() || n < 0 || it->second.swapped) return PA_ERR_INVALID_ARG;
    if (n > 0 && slots == nullptr) return PA_ERR_INVALID_ARG;
    Seq& s = it->second;
    if (ids != nullptr && !s.tracked) return PA_ERR_INVALID_ARG;
    if (static_cast<int64_t>(s.len) + n > INT32_MAX) return PA_ERR_INVALID_ARG;
    if (blocks_needed(s, n) > available()) return PA_ERR_OUT_OF_BLOCKS;
    if (ids == nullptr) {
      s.tracked = false;
      s.tokens.clear();
      s.tokens.shrink_to_fit();
    }
    const int32_t bs = block_size;
    int32_t cows = 0;
    for (int32_t k = 0; k < n; ++k) {
      const int32_t pos = s.len;
      if (pos % bs == 0) {
        const int32_t b = take_block();
        ref[b] = 1;
        s.table.push_back(b);
      } else {
        const int32_t last = s.table.back();
        if (ref[last] > 1) {
          const int32_t b = take_block();
          ref[b] = 1;
          ref[last] -= 1;
          s.table.back() = b;
          if (cow_pair != nullptr) {
            cow_pair[0] = last;
            cow_pair[1] = b;
          }
          ++cows;
        }
      }
      slots[k] = static_cast<int64_t>(s.table[pos / bs]) * bs + pos % bs;
      s.len = pos + 1;
      if (s.tracked) {
        s.tokens.push_back(ids[k]);
        if ((pos + 1) % bs == 0) {
          const int32_t j = pos / bs;
          register_block(s.table[j], j ? s.table[j - 1] : -1, s.tokens.data() + static_cast<int64_t>(j) * bs);
        }
      }
    }
    if (n_cow != nullptr) *n_cow = cows;
    return PA_OK;
  }
};

extern "C" {

pa_status pa_alloc_create(int32_t num_blocks, int32_t block_size, const int32_t* free_order, pa_allocator** out) {
  if (out == nullptr || num_blocks <= 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
  *out = nullptr;
  return no_throw([&]() -> pa_status {
    std::unique_ptr<pa_allocator> a(new pa_allocator());
    a->num_blocks = num_blocks;
    a->block_size = block_size;
    a->ref.assign(num_blocks, 0);
    a->init_cache_state();
    a->free_stack.resize(num_blocks);
    if (free_order != nullptr) {
      std::vector<uint8_t> seen(num_blocks, 0);
      for (int32_t k = 0; k < num_blocks; ++k) {
        const int32_t b = free_order[k];
        if (b < 0 || b >= num_blocks || seen[b]) return PA_ERR_INVALID_ARG;
        seen[b] = 1;
        a->free_stack[num_blocks - 1 - k] = b;
      }
    } else {
      for (int32_t k = 0; k < num_blocks; ++k) a->free_stack[num_blocks - 1 - k] = k;
    }
    *out = a.release();
    return PA_OK;
  });
}

void pa_alloc_destroy(pa_allocator* a) { delete a; }

pa_status pa_seq_add(pa_allocator* a, int64_t seq_id) {
  return no_throw([&]() -> pa_status {
    if (a == nullptr) return PA_ERR_INVALID_ARG;
    if (a->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
    a->seqs.emplace(seq_id, Seq());
    return PA_OK;
  });
}

pa_status pa_seq_append(pa_allocator* a, int64_t seq_id, int32_t n_tokens, int64_t* slots_out,
                        int64_t* cow_pair_out, int32_t* n_cow_out) {
  return no_throw([&]() -> pa_status {
    if (a == nullptr) return PA_ERR_INVALID_ARG;
    return a->append(seq_id, n_tokens, nullptr, slots_out, cow_pair_out, n_cow_out);
  });
}

pa_status pa_seq_add_prefix(pa_allocator* a, int64_t seq_id, const int64_t* tokens, int32_t n_tokens,
                            int32_t* n_cached_out) {
  return no_throw([&]() -> pa_status {
    if (a == nullptr || n_tokens < 0 || (n_tokens > 0 && tokens == nullptr)) return PA_ERR_INVALID_ARG;
    if (a->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
    const int32_t bs = a->block_size;
    std::vector<int32_t> hits;
    int32_t parent = -1;
    Key k{-1, std::vector<int64_t>(bs)};
    for (int32_t j = 0; j < (n_tokens > 0 ? (n_tokens - 1) / bs : 0); ++j) {
      k.parent = parent;
      std::copy(tokens + static_cast<int64_t>(j) * bs, tokens + static_cast<int64_t>(j + 1) * bs, k.toks.begin());
      auto it = a->cache.find(k);
      if (it == a->cache.end()) break;
      hits.push_back(it->second);
      parent = it->second;
    }
    for (int32_t b : hits) {
      if (a->ref[b] == 0 && a->in_lru[b]) {
        a->lru.erase(a->lru_pos[b]);
        a->in_lru[b] = 0;
      }
      a->ref[b] += 1;
    }
    Seq s;
    s.table = hits;
    s.len = static_cast<int32_t>(hits.size()) * bs;
    s.tokens.assign(tokens, tokens + s.len);
    a->seqs.emplace(seq_id, std::move(s));
    if (n_cached_out != nullptr) *n_cached_out = static_cast<int32_t>(hits.size()) * bs;
    return PA_OK;
  });
}

pa_status pa_seq_append_tokens(pa_allocator* a, int64_t seq_id, const int64_t* tokens, int32_t n_tokens,
                               int64_t* slots_out, int64_t* cow_pair_out, int32_t* n_cow_out) {
  return no_throw([&]() -> pa_status {
    if (a == nullptr || (n_tokens > 0 && tokens == nullptr)) return PA_ERR_INVALID_ARG;
    static const int64_t kNone = 0;
    return a->append(seq_id, n_tokens, n_tokens > 0 ? tokens : &kNone, slots_out, cow_pair_out, n_cow_out);
  });
}

pa_status pa_alloc_set_host_pool(pa_allocator* a, int32_t num_host_blocks, const int32_t* host_free_order) {
  return no_throw([&]() -> pa_status {
    if (a == nullptr || num_host_blocks < 0) return PA_ERR_INVALID_ARG;
    for (const auto& kv : a->seqs)
      if (kv.second.swapped) return PA_ERR_INVALID_ARG;
    std::vector<int32_t> st(num_host_blocks);
    std::vector<uint8_t> seen(num_host_blocks, 0);
    for (int32_t k = 0; k < num_host_blocks; ++k) {
      const int32_t h = host_free_order ? host_free_order[k] : k;
      if (h < 0 || h >= num_host_blocks || seen[h]) return PA_ERR_INVALID_ARG;
      seen[h] = 1;
      st[num_host_blocks - 1 - k] = h;
    }
    a->num_host_blocks = num_host_blocks;
    a->host_free.swap(st);
    return PA_OK;
  });
}

pa_status pa_seq_swap_out(pa_allocator* a, int64_t seq_id, int64_t* pairs_out, int32_t cap, int32_t* n_out) {
  return no_throw([&]() -> pa_status {
    if (a == nullptr || n_out == nullptr) return PA_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end() || it->second.swapped) return PA_ERR_INVALID_ARG;
    Seq& s = it->second;
    const int32_t n = static_cast<int32_t>(s.table.size());
    *n_out = n;
    if (n > cap || (n > 0 && pairs_out == nullptr)) return PA_ERR_INVALID_ARG;
    if (n > static_cast<int32_t>(a->host_free.size())) return PA_ERR_OUT_OF_BLOCKS;
    s.host.resize(n);
    for (int32_t k = 0; k < n; ++k) {
      const int32_t h = a->host_free.back();
      a->host_free.pop_back();
      s.host[k] = h;
      pairs_out[2 * k] = s.table[k];
      pairs_out[2 * k + 1] = h;
    }
    for (int32_t b : s.table) a->release(b);
    s.table.clear();
    s.swapped = true;
    return PA_OK;
  });
}

pa_status pa_seq_swap_in(pa_allocator* a, int64_t seq_id, int64_t* pairs_out, int32_t cap, int32_t* n_out) {
  return no_throw([&]() -> pa_status {
    if (a == nullptr || n_out == nullptr) return PA_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end() || !it->second.swapped) return PA_ERR_INVALID_ARG;
    Seq& s = it->second;
    const int32_t n = static_cast<int32_t>(s.host.size());
    *n_out = n;
    if (n > cap || (n > 0 && pairs_out == nullptr)) return PA_ERR_INVALID_ARG;
    if (n > a->available()) return PA_ERR_OUT_OF_BLOCKS;
    s.table.resize(n);
    for (int32_t k = 0; k < n; ++k) {
      const int32_t b = a->take_block();
      a->ref[b] = 1;
      s.table[k] = b;
      pairs_out[2 * k] = s.host[k];
      pairs_out[2 * k + 1] = b;
    }
    for (int32_t h : s.host) a->host_free.push_back(h);
    s.host.clear();
    s.swapped = false;
    if (s.tracked) {
      const int32_t bs = a->block_size;
      for (int32_t j = 0; j < s.len / bs; ++j)
        a->register_block(s.table[j], j ? s.table[j - 1] : -1, s.tokens.data() + static_cast<int64_t>(j) * bs);
    }
    return PA_OK;
  });
}

int32_t pa_alloc_num_host_free(const pa_allocator* a) {
  return a == nullptr ? -1 : static_cast<int32_t>(a->host_free.size());
}

pa_status pa_seq_host_table(const pa_allocator* a, int64_t seq_id, int32_t* out, int32_t cap, int32_t* n_out) {
  if (a == nullptr || n_out == nullptr) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end() || !it->second.swapped) return PA_ERR_INVALID_ARG;
  const auto& h = it->second.host;
  *n_out = static_cast<int32_t>(h.size());
  if (static_cast<int64_t>(h.size()) > cap || (!h.empty() && out == nullptr)) return PA_ERR_INVALID_ARG;
  if (!h.empty()) std::memcpy(out, h.data(), h.size() * sizeof(int32_t));
  return PA_OK;
}

pa_status pa_alloc_evictable(const pa_allocator* a, int32_t* out, int32_t cap, int32_t* n_out) {
  if (a == nullptr || n_out == nullptr) return PA_ERR_INVALID_ARG;
  *n_out = static_cast<int32_t>(a->lru.size());
  if (static_cast<int64_t>(a->lru.size()) > cap || (!a->lru.empty() && out == nullptr)) return PA_ERR_INVALID_ARG;
  int32_t k = 0;
  for (int32_t b : a->lru) out[k++] = b;
  return PA_OK;
}

pa_status pa_seq_append_batch(pa_allocator* a, const int64_t* seq_ids, const int32_t* n_tokens, int32_t n,
                              int64_t* slots_out, int64_t* cow_pairs_out, int32_t* n_cow_out, int32_t* n_done_out) {
  return no_throw([&]() -> pa_status {
    if (a == nullptr || n < 0 || (n > 0 && (seq_ids == nullptr || n_tokens == nullptr))) return PA_ERR_INVALID_ARG;
    int64_t off = 0;
    int32_t cows = 0;
    pa_status st = PA_OK;
    int32_t k = 0;
    for (; k < n; ++k) {
      int32_t c = 0;
      int64_t pair[2] = {-1, -1};
      st = a->append(seq_ids[k], n_tokens[k], nullptr, slots_out == nullptr ? nullptr : slots_out + off, pair, &c);
      if (st != PA_OK) break;
      off += n_tokens[k];
      if (c) {
        if (cow_pairs_out != nullptr) {
          cow_pairs_out[2 * cows] = pair[0];
          cow_pairs_out[2 * cows + 1] = pair[1];
        }
        ++cows;
      }
    }
    if (n_cow_out != nullptr) *n_cow_out = cows;
    if (n_done_out != nullptr) *n_done_out = k;
    return st;
  });
}

pa_status pa_seq_fork(pa_allocator* a, int64_t parent, int64_t child) {
  return no_throw([&]() -> pa_status {
    if (a == nullptr) return PA_ERR_INVALID_ARG;
    auto it = a->seqs.find(parent);
    if (it == a->seqs.end() || it->second.swapped || a->seqs.count(child)) return PA_ERR_INVALID_ARG;
    Seq c = it->second;  // copy before emplace may rehash
    for (int32_t b : c.table) a->ref[b] += 1;
    a->seqs.emplace(child, std::move(c));
    return PA_OK;
  });
}

pa_status pa_seq_free(pa_allocator* a, int64_t seq_id) {
  return no_throw([&]() -> pa_status {
    if (a == nullptr) return PA_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PA_ERR_INVALID_ARG;
    for (int32_t b : it->second.table) a->release(b);
    for (int32_t h : it->second.host) a->host_free.push_back(h);
    a->seqs.erase(it);
    return PA_OK;
  });
}

pa_status pa_seq_len(const pa_allocator* a, int64_t seq_id, int32_t* len_out) {
  if (a == nullptr || len_out == nullptr) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PA_ERR_INVALID_ARG;
  *len_out = it->second.len;
  return PA_OK;
}

pa_status pa_seq_block_table(const pa_allocator* a, int64_t seq_id, int32_t* out, int32_t cap, int32_t* n_out) {
  if (a == nullptr || n_out == nullptr) return PA_ERR_INVALID_ARG;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PA_ERR_INVALID_ARG;
  const auto& t = it->second.table;
  *n_out = static_cast<int32_t>(t.size());
  if (static_cast<int64_t>(t.size()) > cap || (!t.empty() && out == nullptr)) return PA_ERR_INVALID_ARG;
  if (!t.empty()) std::memcpy(out, t.data(), t.size() * sizeof(int32_t));
  return PA_OK;
}

pa_status pa_alloc_block_tables(const pa_allocator* a, const int64_t* seq_ids, int32_t n, int32_t* out,
                                int32_t max_blocks, int32_t* context_lens_out) {
  if (a == nullptr || n < 0 || max_blocks < 0) return PA_ERR_INVALID_ARG;
  if (n > 0 && (seq_ids == nullptr || (out == nullptr && max_blocks > 0))) return PA_ERR_INVALID_ARG;
  for (int32_t r = 0; r < n; ++r) {
    auto it = a->seqs.find(seq_ids[r]);
    if (it == a->seqs.end() || static_cast<int64_t>(it->second.table.size()) > max_blocks) return PA_ERR_INVALID_ARG;
  }
  for (int32_t r = 0; r < n; ++r) {
    const Seq& s = a->seqs.find(seq_ids[r])->second;
    int32_t* row = out + static_cast<int64_t>(r) * max_blocks;
    const int32_t nt = static_cast<int32_t>(s.table.size());
    for (int32_t k = 0; k < max_blocks; ++k) row[k] = k < nt ? s.table[k] : -1;
    if (context_lens_out != nullptr) context_lens_out[r] = s.len;
  }
  return PA_OK;
}

pa_status pa_alloc_prefix_groups(const pa_allocator* a, const int64_t* seq_ids, int32_t n, int32_t max_group_size,
                                 int32_t* group_start_out, int32_t* group_blocks_out, int32_t* n_groups_out) {
  if (a == nullptr || n < 0 || max_group_size < 1 || group_start_out == nullptr || n_groups_out == nullptr ||
      (n > 0 && (seq_ids == nullptr || group_blocks_out == nullptr)))
    return PA_ERR_INVALID_ARG;
  std::vector<const Seq*> ss(static_cast<size_t>(n));
  for (int32_t r = 0; r < n; ++r) {
    auto it = a->seqs.find(seq_ids[r]);
    if (it == a->seqs.end() || it->second.swapped) return PA_ERR_INVALID_ARG;
    ss[r] = &it->second;
  }
  const int32_t bs = a->block_size;
  int32_t g = 0, k = 0;
  while (k < n) {
    const int32_t start = k;
    const Seq& lead = *ss[k];
    int32_t common = lead.len / bs;  // the leader's full blocks
    ++k;
    while (k < n && k - start < max_group_size) {
      const Seq& s = *ss[k];
      const int32_t cap = std::min(common, s.len / bs);
      int32_t c = 0;
      while (c < cap && s.table[c] == lead.table[c]) ++c;
      if (c == 0 || 2 * c < common) break;  // joining would give up more than half the shared blocks
      common = c;
      ++k;
    }
    group_start_out[g] = start;
    group_blocks_out[g] = (k - start > 1) ? common : 0;
    ++g;
  }
  group_start_out[g] = n;
  *n_groups_out = g;
  return PA_OK;
}

int32_t pa_alloc_num_free(const pa_allocator* a) { return a == nullptr ? -1 : static_cast<int32_t>(a->available()); }

int32_t pa_block_refcount(const pa_allocator* a, int32_t block) {
  if (a == nullptr || block < 0 || block >= a->num_blocks) return -1;
  return a->ref[block];
}

pa_status pa_alloc_get_stats(const pa_allocator* a, pa_alloc_stats* out) {
  return no_throw([&]() -> pa_status {
    if (a == nullptr || out == nullptr) return PA_ERR_INVALID_ARG;
    const int32_t bs = a->block_size;
    std::vector<int32_t> filled(a->num_blocks, 0);
    int64_t tokens = 0;
    for (const auto& kv : a->seqs) {
      const Seq& s = kv.second;
      tokens += s.len;
      for (size_t k = 0; k < s.table.size(); ++k) {
        const int64_t f = std::min<int64_t>(bs, s.len - static_cast<int64_t>(k) * bs);
        int32_t& slot = filled[s.table[k]];
        if (f > slot) slot = static_cast<int32_t>(f);
      }
    }
    int64_t waste = 0;
    for (int32_t b = 0; b < a->num_blocks; ++b)
      if (a->ref[b] > 0) waste += bs - filled[b];
    out->num_blocks = a->num_blocks;
    out->num_free = static_cast<int32_t>(a->available());
    out->num_cached = static_cast<int32_t>(a->cache.size());
    out->num_evictable = static_cast<int32_t>(a->lru.size());
    out->num_seqs = static_cast<int32_t>(a->seqs.size());
    out->block_size = bs;
    out->num_tokens = tokens;
    out->waste_slots = waste;
    return PA_OK;
  });
}

}  // extern "C"
