// Host block allocator of the paged KV cache: FIFO free list, per-block
// reference counts, per-sequence block tables, fork and copy-on-write.
//
// Blocks are taken on demand and returned when a request ends ("vLLM +
// PagedAttention：打造高并发LLM推理引擎", "它是怎么工作的"); shared blocks are
// reference counted and copied only when a sharer writes into them
// ("PagedAttention 与 vLLM 推理加速" §3.2(3); "LLM Systems 24: Efficient LLM
// Inference with PagedAttention and vLLM" §3).  The policy for the parts the
// pages leave open is stated in pkv.h.  Every call validates first and
// mutates only once it cannot fail, so a failed call changes nothing.
//
// Preemption by swapping ("LLM Systems 24 ..." §3, conclusion): a second,
// host-side pool with its own FIFO free list and counts; swap-out moves the
// listed sequences' blocks there, swap-in brings them back, both returning
// the block pairs for the caller to copy.

#include <climits>
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "pkv.h"

namespace {

constexpr int kBlock = PKV_BLOCK_SIZE;

// FIFO of block ids over a fixed ring (never holds more than num_blocks).
class FreeRing {
 public:
  explicit FreeRing(int cap) : buf_(static_cast<size_t>(cap)), head_(0), size_(0) {}
  int size() const { return size_; }
  int32_t pop_front() {
    int32_t v = buf_[head_];
    head_ = (head_ + 1) % static_cast<int>(buf_.size());
    --size_;
    return v;
  }
  void push_back(int32_t v) {
    buf_[(head_ + size_) % static_cast<int>(buf_.size())] = v;
    ++size_;
  }
  int32_t at(int i) const { return buf_[(head_ + i) % static_cast<int>(buf_.size())]; }

 private:
  std::vector<int32_t> buf_;
  int head_;
  int size_;
};

struct Seq {
  std::vector<int32_t> table;
  int64_t len = 0;
};

}  // namespace

struct pkv_alloc {
  int num_blocks;
  FreeRing free_list;
  std::vector<int32_t> refcount;
  std::unordered_map<int64_t, Seq> seqs;
  // host-side swap pool
  int num_host_blocks = 0;
  FreeRing host_free{0};
  std::vector<int32_t> host_refcount;
  std::unordered_map<int64_t, Seq> swapped;  // tables hold host block ids

  explicit pkv_alloc(int nb) : num_blocks(nb), free_list(nb), refcount(static_cast<size_t>(nb), 0) {}

  bool known(int64_t id) const { return seqs.count(id) != 0 || swapped.count(id) != 0; }

  // Does appending to s take a block?  `count` gives the (possibly
  // adjusted) reference count of a block.
  template <typename CountFn>
  static bool needs_block(const Seq& s, CountFn count) {
    if (s.len % kBlock == 0) return true;
    return count(s.table.back()) > 1;
  }

  // Append one token; the caller has made sure a block is free if needed.
  int64_t append_unchecked(Seq& s, int32_t* cow_src, int32_t* cow_dst) {
    const int64_t pos = s.len;
    const int64_t page = pos / kBlock;
    const int off = static_cast<int>(pos % kBlock);
    *cow_src = -1;
    *cow_dst = -1;
    if (off == 0) {
      const int32_t blk = free_list.pop_front();
      refcount[blk] = 1;
      s.table.push_back(blk);
    } else if (refcount[s.table.back()] > 1) {
      const int32_t src = s.table.back();
      const int32_t dst = free_list.pop_front();
      refcount[dst] = 1;
      refcount[src] -= 1;
      s.table.back() = dst;
      *cow_src = src;
      *cow_dst = dst;
    }
    s.len = pos + 1;
    return static_cast<int64_t>(s.table[static_cast<size_t>(page)]) * kBlock + off;
  }
};

extern "C" {

pkv_status pkv_alloc_create(int num_blocks, const int32_t* initial_free_order, pkv_alloc** out) {
  if (out == nullptr || num_blocks <= 0) return PKV_EINVAL;
  *out = nullptr;
  if (initial_free_order != nullptr) {
    std::vector<char> seen(static_cast<size_t>(num_blocks), 0);
    for (int i = 0; i < num_blocks; ++i) {
      const int32_t b = initial_free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) return PKV_EINVAL;
      seen[b] = 1;
    }
  }
  pkv_alloc* a = new (std::nothrow) pkv_alloc(num_blocks);
  if (a == nullptr) return PKV_ENOMEM;
  for (int i = 0; i < num_blocks; ++i)
    a->free_list.push_back(initial_free_order ? initial_free_order[i] : i);
  *out = a;
  return PKV_OK;
}

void pkv_alloc_destroy(pkv_alloc* a) { delete a; }

pkv_status pkv_alloc_add_seq(pkv_alloc* a, int64_t seq_id) {
  if (a == nullptr || a->known(seq_id)) return PKV_EINVAL;
  a->seqs.emplace(seq_id, Seq{});
  return PKV_OK;
}

pkv_status pkv_alloc_fork(pkv_alloc* a, int64_t parent, int64_t child) {
  if (a == nullptr) return PKV_EINVAL;
  auto it = a->seqs.find(parent);
  if (it == a->seqs.end() || a->known(child)) return PKV_EINVAL;
  Seq copy = it->second;
  for (int32_t blk : copy.table) a->refcount[blk] += 1;
  a->seqs.emplace(child, std::move(copy));
  return PKV_OK;
}

pkv_status pkv_alloc_free_seq(pkv_alloc* a, int64_t seq_id) {
  if (a == nullptr) return PKV_EINVAL;
  auto sw = a->swapped.find(seq_id);
  if (sw != a->swapped.end()) {
    for (int32_t blk : sw->second.table) {
      if (--a->host_refcount[blk] == 0) a->host_free.push_back(blk);
    }
    a->swapped.erase(sw);
    return PKV_OK;
  }
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PKV_EINVAL;
  for (int32_t blk : it->second.table) {
    if (--a->refcount[blk] == 0) a->free_list.push_back(blk);
  }
  a->seqs.erase(it);
  return PKV_OK;
}

pkv_status pkv_alloc_append_slot(pkv_alloc* a, int64_t seq_id, int64_t* slot, int32_t* cow_src,
                                 int32_t* cow_dst) {
  if (a == nullptr || slot == nullptr || cow_src == nullptr || cow_dst == nullptr) return PKV_EINVAL;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PKV_EINVAL;
  Seq& s = it->second;
  if (pkv_alloc::needs_block(s, [&](int32_t b) { return a->refcount[b]; }) && a->free_list.size() == 0)
    return PKV_ENOMEM;
  *slot = a->append_unchecked(s, cow_src, cow_dst);
  return PKV_OK;
}

pkv_status pkv_alloc_append_tokens(pkv_alloc* a, int64_t seq_id, int n, int64_t* slots,
                                   int32_t* cow_pairs, int* n_cow) {
  if (a == nullptr || n < 0 || n_cow == nullptr || (n > 0 && (slots == nullptr || cow_pairs == nullptr)))
    return PKV_EINVAL;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PKV_EINVAL;
  Seq& s = it->second;
  // blocks needed: one per page boundary crossed, plus one copy if the
  // first token lands in a shared partial block
  int64_t need = 0;
  const int64_t pos = s.len;
  if (n > 0) {
    if (pos % kBlock != 0 && a->refcount[s.table.back()] > 1) need += 1;
    const int64_t first_new_page = (pos + kBlock - 1) / kBlock;   // first page index starting at/after pos
    const int64_t last_page = (pos + n - 1) / kBlock;
    if (last_page >= first_new_page) need += last_page - first_new_page + 1;
  }
  if (need > a->free_list.size()) return PKV_ENOMEM;
  *n_cow = 0;
  for (int i = 0; i < n; ++i) {
    int32_t src, dst;
    slots[i] = a->append_unchecked(s, &src, &dst);
    if (src >= 0) {
      cow_pairs[0] = src;
      cow_pairs[1] = dst;
      *n_cow = 1;
    }
  }
  return PKV_OK;
}

pkv_status pkv_alloc_step(pkv_alloc* a, const int64_t* seq_ids, int n, int64_t* slots,
                          int32_t* cow_pairs, int* n_cow) {
  if (a == nullptr || n < 0 || n_cow == nullptr ||
      (n > 0 && (seq_ids == nullptr || slots == nullptr || cow_pairs == nullptr)))
    return PKV_EINVAL;
  std::vector<Seq*> seqs(static_cast<size_t>(n));
  {
    std::unordered_set<int64_t> seen;
    seen.reserve(static_cast<size_t>(n) * 2);
    for (int i = 0; i < n; ++i) {
      auto it = a->seqs.find(seq_ids[i]);
      if (it == a->seqs.end() || !seen.insert(seq_ids[i]).second) return PKV_EINVAL;
      seqs[i] = &it->second;
    }
  }
  // Dry run: count the blocks the step takes.  A copy drops one reference
  // from the shared block, which a later sibling in the same step may then
  // hold alone and write into without copying.
  std::unordered_map<int32_t, int32_t> drops;
  int64_t need = 0;
  for (int i = 0; i < n; ++i) {
    const Seq& s = *seqs[i];
    auto count = [&](int32_t b) {
      auto d = drops.find(b);
      return a->refcount[b] - (d == drops.end() ? 0 : d->second);
    };
    if (pkv_alloc::needs_block(s, count)) {
      need += 1;
      if (s.len % kBlock != 0) drops[s.table.back()] += 1;
    }
  }
  if (need > a->free_list.size()) return PKV_ENOMEM;
  int nc = 0;
  for (int i = 0; i < n; ++i) {
    int32_t src, dst;
    slots[i] = a->append_unchecked(*seqs[i], &src, &dst);
    if (src >= 0) {
      cow_pairs[2 * nc] = src;
      cow_pairs[2 * nc + 1] = dst;
      ++nc;
    }
  }
  *n_cow = nc;
  return PKV_OK;
}

pkv_status pkv_alloc_block_table(const pkv_alloc* a, int64_t seq_id, int32_t* out, int cap,
                                 int* n_blocks, int64_t* context_len) {
  if (a == nullptr || cap < 0 || (cap > 0 && out == nullptr)) return PKV_EINVAL;
  auto it = a->seqs.find(seq_id);
  if (it == a->seqs.end()) return PKV_EINVAL;
  const Seq& s = it->second;
  const int nb = static_cast<int>(s.table.size());
  if (n_blocks) *n_blocks = nb;
  if (context_len) *context_len = s.len;
  const int m = nb < cap ? nb : cap;
  if (m > 0) std::memcpy(out, s.table.data(), sizeof(int32_t) * static_cast<size_t>(m));
  return PKV_OK;
}

pkv_status pkv_alloc_block_tables(const pkv_alloc* a, const int64_t* seq_ids, int n, int32_t* tables,
                                  int width, int32_t pad, int32_t* context_lens) {
  if (a == nullptr || n < 0 || width < 0) return PKV_EINVAL;
  if (n > 0 && (seq_ids == nullptr || tables == nullptr || context_lens == nullptr)) return PKV_EINVAL;
  std::vector<const Seq*> seqs(static_cast<size_t>(n));
  for (int i = 0; i < n; ++i) {
    auto it = a->seqs.find(seq_ids[i]);
    if (it == a->seqs.end()) return PKV_EINVAL;
    if (static_cast<int64_t>(it->second.table.size()) > width || it->second.len > INT32_MAX) return PKV_EINVAL;
    seqs[i] = &it->second;
  }
  for (int i = 0; i < n; ++i) {
    int32_t* row = tables + static_cast<size_t>(i) * static_cast<size_t>(width);
    const auto& t = seqs[i]->table;
    for (int j = 0; j < width; ++j) row[j] = j < static_cast<int>(t.size()) ? t[j] : pad;
    context_lens[i] = static_cast<int32_t>(seqs[i]->len);
  }
  return PKV_OK;
}

pkv_status pkv_alloc_state(const pkv_alloc* a, int32_t* free_list, int* n_free, int32_t* refcounts) {
  if (a == nullptr) return PKV_EINVAL;
  const int nf = a->free_list.size();
  if (n_free) *n_free = nf;
  if (free_list)
    for (int i = 0; i < nf; ++i) free_list[i] = a->free_list.at(i);
  if (refcounts) std::memcpy(refcounts, a->refcount.data(), sizeof(int32_t) * a->refcount.size());
  return PKV_OK;
}

int pkv_alloc_num_free(const pkv_alloc* a) { return a ? a->free_list.size() : -1; }
int pkv_alloc_num_blocks(const pkv_alloc* a) { return a ? a->num_blocks : -1; }
int pkv_alloc_num_seqs(const pkv_alloc* a) { return a ? static_cast<int>(a->seqs.size()) : -1; }

}  // extern "C"

// ---- preemption by swapping -------------------------------------------------

extern "C" pkv_status pkv_alloc_set_host_pool(pkv_alloc* a, int num_host_blocks) {
  if (a == nullptr || num_host_blocks < 0 || !a->swapped.empty()) return PKV_EINVAL;
  FreeRing ring(num_host_blocks);
  for (int i = 0; i < num_host_blocks; ++i) ring.push_back(i);
  a->host_free = std::move(ring);
  a->host_refcount.assign(static_cast<size_t>(num_host_blocks), 0);
  a->num_host_blocks = num_host_blocks;
  return PKV_OK;
}

namespace {

// Move the listed sequences from `from` (tables over the source pool) to
// `to` (tables over the destination pool): every distinct source block, in
// id order then table order, gets one block popped from `dst_free`; every
// holder drops one source reference (a block reaching zero goes to the back
// of `src_free`) and adds one destination reference.  Validates first: ids
// distinct and in `from`, the destination pool and `cap` large enough.
pkv_status move_seqs(std::unordered_map<int64_t, Seq>& from, std::unordered_map<int64_t, Seq>& to,
                     std::vector<int32_t>& src_ref, FreeRing& src_free, std::vector<int32_t>& dst_ref,
                     FreeRing& dst_free, const int64_t* seq_ids, int n, int32_t* pairs, int cap, int* n_pairs) {
  if (n < 0 || n_pairs == nullptr || cap < 0 || (n > 0 && seq_ids == nullptr) || (cap > 0 && pairs == nullptr))
    return PKV_EINVAL;
  std::vector<Seq*> list(static_cast<size_t>(n));
  std::unordered_set<int64_t> seen;
  std::unordered_set<int32_t> distinct;
  for (int i = 0; i < n; ++i) {
    auto it = from.find(seq_ids[i]);
    if (it == from.end() || !seen.insert(seq_ids[i]).second) return PKV_EINVAL;
    list[i] = &it->second;
    for (int32_t b : it->second.table) distinct.insert(b);
  }
  const int64_t need = static_cast<int64_t>(distinct.size());
  if (need > cap) return PKV_EINVAL;
  if (need > dst_free.size()) return PKV_ENOMEM;
  std::unordered_map<int32_t, int32_t> map;
  map.reserve(distinct.size() * 2);
  int np = 0;
  std::vector<Seq> moved(static_cast<size_t>(n));
  for (int i = 0; i < n; ++i) {
    moved[i].len = list[i]->len;
    moved[i].table.reserve(list[i]->table.size());
    for (int32_t b : list[i]->table) {
      auto m = map.find(b);
      int32_t nb;
      if (m == map.end()) {
        nb = dst_free.pop_front();
        map.emplace(b, nb);
        pairs[2 * np] = b;
        pairs[2 * np + 1] = nb;
        ++np;
      } else {
        nb = m->second;
      }
      moved[i].table.push_back(nb);
    }
  }
  for (int i = 0; i < n; ++i) {
    for (size_t j = 0; j < list[i]->table.size(); ++j) {
      dst_ref[moved[i].table[j]] += 1;
      const int32_t b = list[i]->table[j];
      if (--src_ref[b] == 0) src_free.push_back(b);
    }
  }
  for (int i = 0; i < n; ++i) {
    from.erase(seq_ids[i]);
    to.emplace(seq_ids[i], std::move(moved[i]));
  }
  *n_pairs = np;
  return PKV_OK;
}

}  // namespace

extern "C" {

pkv_status pkv_alloc_swap_out(pkv_alloc* a, const int64_t* seq_ids, int n, int32_t* pairs, int cap, int* n_pairs) {
  if (a == nullptr) return PKV_EINVAL;
  return move_seqs(a->seqs, a->swapped, a->refcount, a->free_list, a->host_refcount, a->host_free, seq_ids, n,
                   pairs, cap, n_pairs);
}

pkv_status pkv_alloc_swap_in(pkv_alloc* a, const int64_t* seq_ids, int n, int32_t* pairs, int cap, int* n_pairs) {
  if (a == nullptr) return PKV_EINVAL;
  return move_seqs(a->swapped, a->seqs, a->host_refcount, a->host_free, a->refcount, a->free_list, seq_ids, n,
                   pairs, cap, n_pairs);
}

pkv_status pkv_alloc_host_state(const pkv_alloc* a, int32_t* free_list, int* n_free, int32_t* refcounts) {
  if (a == nullptr) return PKV_EINVAL;
  const int nf = a->host_free.size();
  if (n_free) *n_free = nf;
  if (free_list)
    for (int i = 0; i < nf; ++i) free_list[i] = a->host_free.at(i);
  if (refcounts && !a->host_refcount.empty())
    std::memcpy(refcounts, a->host_refcount.data(), sizeof(int32_t) * a->host_refcount.size());
  return PKV_OK;
}

pkv_status pkv_alloc_swapped_table(const pkv_alloc* a, int64_t seq_id, int32_t* out, int cap, int* n_blocks,
                                   int64_t* context_len) {
  if (a == nullptr || cap < 0 || (cap > 0 && out == nullptr)) return PKV_EINVAL;
  auto it = a->swapped.find(seq_id);
  if (it == a->swapped.end()) return PKV_EINVAL;
  const Seq& s = it->second;
  const int nb = static_cast<int>(s.table.size());
  if (n_blocks) *n_blocks = nb;
  if (context_len) *context_len = s.len;
  const int m = nb < cap ? nb : cap;
  if (m > 0) std::memcpy(out, s.table.data(), sizeof(int32_t) * static_cast<size_t>(m));
  return PKV_OK;
}

int pkv_alloc_num_swapped(const pkv_alloc* a) { return a ? static_cast<int>(a->swapped.size()) : -1; }

}  // extern "C"
