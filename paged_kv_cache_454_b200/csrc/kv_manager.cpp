// Host-side KV-cache block manager (the pa_kvm_* calls of pa_kv_manager.h).
//
// Per physical block: a reference count (tables holding it), and for cached
// full blocks the chain hash of its prefix, the hash of the prefix before it,
// its own tokens (checked on every lookup, so a hash collision is a miss, not
// a wrong hit) and the cached blocks registered under it.  Free blocks that
// never held a cached block sit in a two-level bitmap (lowest id in O(1)
// words); unreferenced cached blocks sit in an intrusive LRU list, oldest at
// the head.  A sequence keeps its table, length, tokens and the chain hash of
// each full block.
//
// Chain hash of full block i of a sequence: h_i = FNV-1a-64 over the 8 bytes
// of h_{i-1} (a fixed root value for i = 0) followed by the 4 bytes of each of
// its tokens, least significant byte first.  Two blocks are the same cache
// entry when their prefixes are token for token equal, which the stored
// (parent hash, tokens) pair checks block by block.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pa_kv_manager.h"

namespace {

constexpr uint64_t kFnvOffset = 0xcbf29ce484222325ull;  // FNV-1a 64-bit offset basis
constexpr uint64_t kFnvPrime = 0x100000001b3ull;        // FNV 64-bit prime
constexpr uint64_t kRoot = 0x9e3779b97f4a7c15ull;       // parent hash of a first block

uint64_t chain_hash(uint64_t parent, const int32_t* tok, int n) {
  uint64_t h = kFnvOffset;
  for (int i = 0; i < 8; ++i) {
    h ^= (parent >> (8 * i)) & 0xffu;
    h *= kFnvPrime;
  }
  for (int t = 0; t < n; ++t) {
    const uint32_t v = static_cast<uint32_t>(tok[t]);
    for (int i = 0; i < 4; ++i) {
      h ^= (v >> (8 * i)) & 0xffu;
      h *= kFnvPrime;
    }
  }
  return h;
}

// Set of block ids with "lowest member" in a few word scans.
class IdSet {
 public:
  explicit IdSet(int32_t n) : n_(n), lo_((n + 63) / 64, 0), hi_(((n + 63) / 64 + 63) / 64, 0) {}
  void insert(int32_t b) {
    const int32_t w = b >> 6;
    if (!(lo_[w] >> (b & 63) & 1)) {
      lo_[w] |= 1ull << (b & 63);
      hi_[w >> 6] |= 1ull << (w & 63);
      ++count_;
    }
  }
  void erase(int32_t b) {
    const int32_t w = b >> 6;
    if (lo_[w] >> (b & 63) & 1) {
      lo_[w] &= ~(1ull << (b & 63));
      if (!lo_[w]) hi_[w >> 6] &= ~(1ull << (w & 63));
      --count_;
    }
  }
  bool contains(int32_t b) const { return lo_[b >> 6] >> (b & 63) & 1; }
  int32_t lowest() const {
    for (size_t i = 0; i < hi_.size(); ++i)
      if (hi_[i]) {
        const int32_t w = static_cast<int32_t>(i * 64 + __builtin_ctzll(hi_[i]));
        return w * 64 + __builtin_ctzll(lo_[w]);
      }
    return -1;
  }
  int32_t size() const { return count_; }

 private:
  int32_t n_;
  int32_t count_ = 0;
  std::vector<uint64_t> lo_, hi_;
};

struct Seq {
  std::vector<int32_t> table;
  int32_t len = 0;
  uint64_t stamp = 0;           // last batch call that listed this sequence
  bool swapped = false;         // table lists host swap-space blocks
  std::vector<int32_t> tokens;  // kept only with prefix caching
  std::vector<uint64_t> hash;   // chain hash of each full block (prefix caching)
};

}  // namespace

struct pa_kvm {
  int32_t nb, bs;
  bool pc;
  std::vector<int32_t> ref;
  IdSet free_set;
  IdSet host_free;  // host swap-space blocks
  // LRU of unreferenced cached blocks
  std::vector<int32_t> prev, next;
  std::vector<uint8_t> in_lru;
  int32_t head = -1, tail = -1, n_lru = 0;
  // prefix cache
  std::unordered_map<uint64_t, int32_t> cache;  // chain hash -> block
  std::vector<uint8_t> cached;
  std::vector<uint64_t> bhash, bparent;
  std::vector<std::vector<int32_t>> btokens, children;
  std::unordered_map<int64_t, Seq> seqs;
  uint64_t calls = 0;  // batch-call counter (duplicate detection)

  pa_kvm(int32_t n, int32_t b, bool p, int32_t nh)
      : nb(n), bs(b), pc(p), ref(n, 0), free_set(n), host_free(nh > 0 ? nh : 1), prev(n, -1),
        next(n, -1), in_lru(n, 0), cached(n, 0), bhash(n, 0), bparent(n, 0),
        btokens(p ? n : 0), children(p ? n : 0) {
    for (int32_t i = 0; i < n; ++i) free_set.insert(i);
    for (int32_t i = 0; i < nh; ++i) host_free.insert(i);
  }

  // A sequence that is present and resident on the device, or NULL.
  Seq* resident(int64_t id) {
    auto it = seqs.find(id);
    return it == seqs.end() || it->second.swapped ? nullptr : &it->second;
  }

  int32_t num_free() const { return free_set.size() + n_lru; }

  // ---- LRU ----
  void lru_push(int32_t b) {
    prev[b] = tail;
    next[b] = -1;
    if (tail >= 0) next[tail] = b; else head = b;
    tail = b;
    in_lru[b] = 1;
    ++n_lru;
  }
  void lru_remove(int32_t b) {
    if (prev[b] >= 0) next[prev[b]] = next[b]; else head = next[b];
    if (next[b] >= 0) prev[next[b]] = prev[b]; else tail = prev[b];
    prev[b] = next[b] = -1;
    in_lru[b] = 0;
    --n_lru;
  }

  // ---- cache ----
  // The cached block of prefix hash h whose parent hash and tokens match, or -1.
  int32_t find(uint64_t h, uint64_t parent, const int32_t* tok) const {
    auto it = cache.find(h);
    if (it == cache.end()) return -1;
    const int32_t b = it->second;
    if (bparent[b] != parent || std::memcmp(btokens[b].data(), tok, sizeof(int32_t) * bs) != 0)
      return -1;
    return b;
  }

  // Drop block b's entry and every entry registered under it (transitively);
  // unreferenced blocks among them leave the LRU for the free set.
  void uncache(int32_t b) {
    std::vector<int32_t> stack{b};
    while (!stack.empty()) {
      const int32_t x = stack.back();
      stack.pop_back();
      if (!cached[x]) continue;
      cache.erase(bhash[x]);
      cached[x] = 0;
      if (ref[x] == 0 && in_lru[x]) {
        lru_remove(x);
        free_set.insert(x);
      }
      for (int32_t c : children[x])
        if (cached[c] && bparent[c] == bhash[x]) stack.push_back(c);
      children[x].clear();
    }
  }

  // Register full block b (logical index i) with prefix hash h and parent hash
  // `parent`, if its prefix is cached and it is not.
  void reg(int32_t b, int32_t i, uint64_t h, uint64_t parent, const int32_t* tok) {
    if (!pc || cache.count(h)) return;
    int32_t pb = -1;
    if (i > 0) {
      auto it = cache.find(parent);
      if (it == cache.end()) return;
      pb = it->second;
    }
    cache.emplace(h, b);
    cached[b] = 1;
    bhash[b] = h;
    bparent[b] = parent;
    btokens[b].assign(tok, tok + bs);
    if (pb >= 0) children[pb].push_back(b);
  }

  // ---- references ----
  int32_t alloc() {
    int32_t b = free_set.lowest();
    if (b >= 0) {
      free_set.erase(b);
    } else if (head >= 0) {
      b = head;
      lru_remove(b);
      uncache(b);
    } else {
      return -1;
    }
    ref[b] = 1;
    return b;
  }
  void release(int32_t b) {
    if (--ref[b] == 0) {
      if (cached[b]) lru_push(b); else free_set.insert(b);
    }
  }
  void retain(int32_t b) {
    if (ref[b] == 0 && in_lru[b]) lru_remove(b);
    ++ref[b];
  }

  uint64_t parent_hash(const Seq& s, int32_t i) const { return i == 0 ? kRoot : s.hash[i - 1]; }

  // Blocks appending n tokens to s takes from the pool (a copy of a shared
  // partial last block, then fresh blocks).
  int32_t blocks_needed(const Seq& s, int32_t n, bool* cow) const {
    *cow = n > 0 && s.len % bs != 0 && ref[s.table.back()] > 1;
    return (s.len + n + bs - 1) / bs - (s.len + bs - 1) / bs + (*cow ? 1 : 0);
  }

  // Append n tokens to s; the caller has checked the pool can supply the blocks.
  void append(Seq& s, const int32_t* tokens, int32_t n, bool cow, int64_t* slots,
              int64_t* pair, int32_t* num_pairs) {
    int32_t L = s.len;
    if (cow) {
      const int32_t old = s.table.back();
      const int32_t fresh = alloc();
      release(old);
      s.table.back() = fresh;
      pair[0] = old;
      pair[1] = fresh;
      ++*num_pairs;
    }
    for (int32_t t = 0; t < n; ++t) {
      if (L % bs == 0) s.table.push_back(alloc());
      slots[t] = static_cast<int64_t>(s.table[L / bs]) * bs + L % bs;
      if (pc) s.tokens.push_back(tokens[t]);
      ++L;
      if (pc && L % bs == 0) {
        const int32_t k = L / bs - 1;
        const uint64_t parent = parent_hash(s, k);
        const uint64_t h = chain_hash(parent, s.tokens.data() + k * bs, bs);
        s.hash.push_back(h);
        reg(s.table[k], k, h, parent, s.tokens.data() + k * bs);
      }
    }
    s.len = L;
  }

  // Chain hashes of s's full blocks from block `from` on (after its tokens changed).
  void rehash(Seq& s, int32_t from) {
    if (!pc) return;
    const int32_t full = s.len / bs;
    s.hash.resize(full);
    for (int32_t i = from; i < full; ++i)
      s.hash[i] = chain_hash(parent_hash(s, i), s.tokens.data() + i * bs, bs);
  }
};

using namespace std;

extern "C" {

PA_API pa_kvm* pa_kvm_create(int32_t num_blocks, int32_t block_size, int32_t prefix_caching,
                             int32_t num_host_blocks) {
  if (num_blocks <= 0 || block_size <= 0 || num_host_blocks < 0) return nullptr;
  return new (std::nothrow) pa_kvm(num_blocks, block_size, prefix_caching != 0, num_host_blocks);
}

PA_API void pa_kvm_destroy(pa_kvm* m) { delete m; }

PA_API int32_t pa_kvm_num_free_blocks(const pa_kvm* m) { return m ? m->num_free() : 0; }

PA_API int pa_kvm_add_sequence(pa_kvm* m, int64_t seq_id, const int32_t* tokens, int32_t n,
                               int64_t* slots, int32_t* cached_tokens) {
  if (!m || n < 0 || (n > 0 && !slots) || (m->pc && n > 0 && !tokens)) return PA_ERR_ARG;
  if (m->seqs.count(seq_id)) return PA_ERR_ARG;
  const int32_t bs = m->bs;
  const int32_t nblk = (n + bs - 1) / bs;
  vector<int32_t> hits;
  vector<uint64_t> hashes;
  if (m->pc) {
    uint64_t parent = kRoot;
    for (int32_t i = 0; i < n / bs; ++i) {
      const uint64_t h = chain_hash(parent, tokens + i * bs, bs);
      hashes.push_back(h);
      if (static_cast<int32_t>(hits.size()) == i) {
        const int32_t b = m->find(h, parent, tokens + i * bs);
        if (b >= 0) hits.push_back(b);
      }
      parent = h;
    }
  }
  int32_t revived = 0;
  for (int32_t b : hits) revived += m->ref[b] == 0;
  if (nblk - static_cast<int32_t>(hits.size()) > m->num_free() - revived) return PA_ERR_NO_BLOCKS;
  Seq s;
  s.table.reserve(nblk);
  for (int32_t b : hits) {
    m->retain(b);
    s.table.push_back(b);
  }
  for (int32_t i = static_cast<int32_t>(hits.size()); i < nblk; ++i) {
    const int32_t b = m->alloc();
    s.table.push_back(b);
    if (m->pc && (i + 1) * bs <= n)
      m->reg(b, i, hashes[i], i == 0 ? kRoot : hashes[i - 1], tokens + i * bs);
  }
  const int32_t cached = static_cast<int32_t>(hits.size()) * bs;
  for (int32_t t = 0; t < n; ++t)
    slots[t] = t < cached ? -1 : static_cast<int64_t>(s.table[t / bs]) * bs + t % bs;
  s.len = n;
  if (m->pc) {
    s.tokens.assign(tokens, tokens + n);
    s.hash = std::move(hashes);
  }
  m->seqs.emplace(seq_id, std::move(s));
  if (cached_tokens) *cached_tokens = cached;
  return PA_OK;
}

PA_API int pa_kvm_append_tokens(pa_kvm* m, int64_t seq_id, const int32_t* tokens, int32_t n,
                                int64_t* slots, int64_t* copy_pair, int32_t* num_pairs) {
  if (!m || n < 0 || (n > 0 && !slots) || (m->pc && n > 0 && !tokens) || !num_pairs)
    return PA_ERR_ARG;
  Seq* sp = m->resident(seq_id);
  if (!sp) return PA_ERR_ARG;
  Seq& s = *sp;
  *num_pairs = 0;
  if (n == 0) return PA_OK;
  bool cow = false;
  const int32_t need = m->blocks_needed(s, n, &cow);
  if (cow && !copy_pair) return PA_ERR_ARG;
  if (need > m->num_free()) return PA_ERR_NO_BLOCKS;
  m->append(s, tokens, n, cow, slots, copy_pair, num_pairs);
  return PA_OK;
}

PA_API int pa_kvm_decode_step(pa_kvm* m, const int64_t* seq_ids, int32_t num_seqs,
                              const int32_t* tokens, int64_t* slots, int64_t* copy_pairs,
                              int32_t* num_pairs) {
  if (!m || num_seqs < 0 || !num_pairs ||
      (num_seqs > 0 && (!seq_ids || !slots || !copy_pairs || (m->pc && !tokens))))
    return PA_ERR_ARG;
  *num_pairs = 0;
  std::vector<Seq*> ss(num_seqs);
  std::unordered_map<int32_t, int32_t> drops;  // references an earlier copy in the batch drops
  const uint64_t stamp = ++m->calls;
  int32_t need = 0;
  for (int32_t i = 0; i < num_seqs; ++i) {
    auto it = m->seqs.find(seq_ids[i]);
    if (it == m->seqs.end() || it->second.swapped || it->second.stamp == stamp) return PA_ERR_ARG;
    Seq& s = it->second;
    s.stamp = stamp;
    ss[i] = &s;
    if (s.len % m->bs == 0) {
      ++need;
    } else {
      const int32_t b = s.table.back();
      if (m->ref[b] > 1) {  // shared: copied unless earlier copies left one holder
        int32_t& d = drops[b];
        if (m->ref[b] - d > 1) {
          ++need;
          ++d;
        }
      }
    }
  }
  if (need > m->num_free()) return PA_ERR_NO_BLOCKS;
  for (int32_t i = 0; i < num_seqs; ++i) {
    bool cow = false;
    m->blocks_needed(*ss[i], 1, &cow);
    m->append(*ss[i], tokens ? tokens + i : nullptr, 1, cow, slots + i,
              copy_pairs + 2 * *num_pairs, num_pairs);
  }
  return PA_OK;
}

PA_API int pa_kvm_fork(pa_kvm* m, int64_t parent, int64_t child) {
  if (!m) return PA_ERR_ARG;
  Seq* p = m->resident(parent);
  if (!p || m->seqs.count(child)) return PA_ERR_ARG;
  Seq c = *p;
  for (int32_t b : c.table) m->retain(b);
  m->seqs.emplace(child, std::move(c));
  return PA_OK;
}

PA_API int pa_kvm_share_prefix(pa_kvm* m, int64_t src, int64_t dst, int32_t n_blocks) {
  if (!m) return PA_ERR_ARG;
  const Seq* sp = m->resident(src);
  if (!sp || m->seqs.count(dst)) return PA_ERR_ARG;
  const Seq& s = *sp;
  if (n_blocks < 0 || n_blocks > static_cast<int32_t>(s.table.size())) return PA_ERR_ARG;
  Seq d;
  d.len = std::min(s.len, n_blocks * m->bs);
  d.table.assign(s.table.begin(), s.table.begin() + n_blocks);
  if (m->pc) {
    d.tokens.assign(s.tokens.begin(), s.tokens.begin() + d.len);
    d.hash.assign(s.hash.begin(), s.hash.begin() + d.len / m->bs);
  }
  for (int32_t b : d.table) m->retain(b);
  m->seqs.emplace(dst, std::move(d));
  return PA_OK;
}

PA_API int pa_kvm_share_blocks(pa_kvm* m, int64_t src, int64_t dst, const int32_t* idx, int32_t n) {
  if (!m || n < 0 || (n > 0 && !idx)) return PA_ERR_ARG;
  Seq* sp = m->resident(src);
  Seq* dp = m->resident(dst);
  if (!sp || !dp) return PA_ERR_ARG;
  Seq& s = *sp;
  Seq& d = *dp;
  const int32_t bs = m->bs;
  for (int32_t k = 0; k < n; ++k) {
    const int32_t i = idx[k];
    if (i < 0 || (i + 1) * bs > s.len || i >= static_cast<int32_t>(d.table.size()))
      return PA_ERR_ARG;
  }
  int32_t first = INT32_MAX;
  for (int32_t k = 0; k < n; ++k) {
    const int32_t i = idx[k];
    const int32_t b = s.table[i];
    m->retain(b);
    m->release(d.table[i]);
    d.table[i] = b;
    if (m->pc) {
      const int32_t end = std::min(std::min((i + 1) * bs, d.len), s.len);
      for (int32_t t = i * bs; t < end; ++t) d.tokens[t] = s.tokens[t];
    }
    first = std::min(first, i);
  }
  if (n > 0) m->rehash(d, first);
  return PA_OK;
}

PA_API int pa_kvm_free_sequence(pa_kvm* m, int64_t seq_id) {
  if (!m) return PA_ERR_ARG;
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PA_ERR_ARG;
  const vector<int32_t>& t = it->second.table;
  if (it->second.swapped) {
    for (int32_t h : t) m->host_free.insert(h);
  } else {
    for (auto b = t.rbegin(); b != t.rend(); ++b) m->release(*b);
  }
  m->seqs.erase(it);
  return PA_OK;
}

PA_API int pa_kvm_sequence_info(const pa_kvm* m, int64_t seq_id, int32_t* context_len,
                                int32_t* num_blocks) {
  if (!m) return PA_ERR_ARG;
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PA_ERR_ARG;
  if (context_len) *context_len = it->second.len;
  if (num_blocks) *num_blocks = static_cast<int32_t>(it->second.table.size());
  return PA_OK;
}

PA_API int pa_kvm_block_table(const pa_kvm* m, int64_t seq_id, int32_t* table, int32_t capacity) {
  if (!m || capacity < 0 || (capacity > 0 && !table)) return PA_ERR_ARG;
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PA_ERR_ARG;
  const vector<int32_t>& t = it->second.table;
  if (static_cast<int32_t>(t.size()) > capacity) return PA_ERR_SHAPE;
  std::copy(t.begin(), t.end(), table);
  return PA_OK;
}

PA_API int pa_kvm_batch(const pa_kvm* m, const int64_t* seq_ids, int32_t num_seqs,
                        int32_t max_blocks, int32_t* block_tables, int32_t* context_lens) {
  if (!m || num_seqs < 0 || max_blocks < 0 ||
      (num_seqs > 0 && (!seq_ids || !context_lens || (max_blocks > 0 && !block_tables))))
    return PA_ERR_ARG;
  for (int32_t i = 0; i < num_seqs; ++i) {
    auto it = m->seqs.find(seq_ids[i]);
    if (it == m->seqs.end() || it->second.swapped) return PA_ERR_ARG;
    if (static_cast<int32_t>(it->second.table.size()) > max_blocks) return PA_ERR_SHAPE;
  }
  for (int32_t i = 0; i < num_seqs; ++i) {
    const Seq& s = m->seqs.find(seq_ids[i])->second;
    int32_t* row = block_tables + static_cast<int64_t>(i) * max_blocks;
    const int32_t nt = static_cast<int32_t>(s.table.size());
    std::copy(s.table.begin(), s.table.end(), row);
    for (int32_t j = nt; j < max_blocks; ++j) row[j] = -1;
    context_lens[i] = s.len;
  }
  return PA_OK;
}

PA_API int pa_kvm_batch_update(const pa_kvm* m, const int64_t* seq_ids, int32_t num_seqs,
                               int32_t max_blocks, int32_t* block_tables, int32_t* context_lens) {
  if (!m || num_seqs < 0 || max_blocks < 0 ||
      (num_seqs > 0 && (!seq_ids || !context_lens || (max_blocks > 0 && !block_tables))))
    return PA_ERR_ARG;
  for (int32_t i = 0; i < num_seqs; ++i) {
    auto it = m->seqs.find(seq_ids[i]);
    if (it == m->seqs.end() || it->second.swapped) return PA_ERR_ARG;
    const Seq& s = it->second;
    const int32_t nt = static_cast<int32_t>(s.table.size());
    if (nt > max_blocks) return PA_ERR_SHAPE;
    if (nt > 0) block_tables[static_cast<int64_t>(i) * max_blocks + nt - 1] = s.table.back();
    context_lens[i] = s.len;
  }
  return PA_OK;
}

PA_API int pa_kvm_swap_out(pa_kvm* m, int64_t seq_id, int64_t* pairs, int32_t capacity,
                           int32_t* num_pairs) {
  if (!m || capacity < 0 || !num_pairs || (capacity > 0 && !pairs)) return PA_ERR_ARG;
  Seq* sp = m->resident(seq_id);
  if (!sp) return PA_ERR_ARG;
  Seq& s = *sp;
  const int32_t n = static_cast<int32_t>(s.table.size());
  for (int32_t b : s.table)
    if (m->ref[b] != 1) return PA_ERR_ARG;  // shared with another table
  if (n > capacity) return PA_ERR_SHAPE;
  if (n > m->host_free.size()) return PA_ERR_NO_BLOCKS;
  vector<int32_t> host(n);
  for (int32_t i = 0; i < n; ++i) {
    host[i] = m->host_free.lowest();
    m->host_free.erase(host[i]);
    pairs[2 * i] = s.table[i];
    pairs[2 * i + 1] = host[i];
  }
  for (auto b = s.table.rbegin(); b != s.table.rend(); ++b) m->release(*b);
  s.table = std::move(host);
  s.swapped = true;
  *num_pairs = n;
  return PA_OK;
}

PA_API int pa_kvm_swap_in(pa_kvm* m, int64_t seq_id, int64_t* pairs, int32_t capacity,
                          int32_t* num_pairs) {
  if (!m || capacity < 0 || !num_pairs || (capacity > 0 && !pairs)) return PA_ERR_ARG;
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end() || !it->second.swapped) return PA_ERR_ARG;
  Seq& s = it->second;
  const int32_t n = static_cast<int32_t>(s.table.size());
  if (n > capacity) return PA_ERR_SHAPE;
  if (n > m->num_free()) return PA_ERR_NO_BLOCKS;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t b = m->alloc();
    pairs[2 * i] = s.table[i];
    pairs[2 * i + 1] = b;
  }
  for (int32_t i = 0; i < n; ++i) {
    m->host_free.insert(s.table[i]);
    s.table[i] = static_cast<int32_t>(pairs[2 * i + 1]);
  }
  s.swapped = false;
  *num_pairs = n;
  return PA_OK;
}

PA_API int32_t pa_kvm_num_free_host_blocks(const pa_kvm* m) {
  return m ? m->host_free.size() : 0;
}

PA_API int32_t pa_kvm_ref_count(const pa_kvm* m, int32_t block) {
  if (!m || block < 0 || block >= m->nb) return -1;
  return m->ref[block];
}

}  // extern "C"
