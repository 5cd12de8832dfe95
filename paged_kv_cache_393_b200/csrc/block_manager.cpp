// Host block manager of the paged KV cache: free list, reference counts,
// on-demand growth, fork, copy-on-write and release.  Contract: include/pagedkv.h.
//
// Sources of the rules (all restated, none copied):
//  * a free list from which allocation takes the LAST entry, refcount 1 on
//    allocation, growth by one block when the sequence has none or its last
//    block is full, failure on an empty pool: the PagedKVManager concept model
//    (n1n.ai "PagedAttention 对比传统 KV 缓存", section "实现逻辑代码示例") and
//    lpnh.cn/news/2758356 §3.1-§3.2;
//  * release decrements every block and returns those at 0 (lpnh.cn/news/2758356
//    §3.2; lpnh.cn/news/1824136 §3.2 step 6);
//  * sharing on fork and copy-on-write of a shared, not yet full block, with a
//    shared full block needing no copy (lpnh.cn/news/2758356 §4.2);
//  * counts updated under a lock (lpnh.cn/news/2758356 §4.3 warns that
//    unsynchronised counts free shared blocks early);
//  * a queued copy has not happened yet: the pages copy a shared block first
//    and only then drop its count (§4.2), and a block reclaimed early is handed
//    out again and overwritten (§4.3).  Both ends of a queued (src, dst) pair
//    therefore stay off the free list until bm_take_copies hands the pair out,
//    and a write into a block that is still waiting for its own copy is copied
//    from that block's source, so one batch of pairs is free of overlaps.
#include "../../include/pagedkv.h"

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <utility>
#include <vector>

struct pagedkv_block_manager {
  struct Seq {
    std::vector<int32_t> table;
    int64_t len = 0;
    bool alive = false;
  };
  int num_blocks = 0;
  int block_size = 0;
  std::vector<int32_t> free_list;   // allocation pops the back
  std::vector<int32_t> refcount;    // per physical block
  std::vector<int32_t> pinned;      // per physical block: queued copy pairs naming it
  std::vector<int32_t> copy_source; // per physical block: source of its queued copy, -1 = none
  // The id indexes this vector directly.  A released sequence leaves an empty,
  // dead entry whose id goes on free_ids; new sequences take the most recently
  // released id first, so the vector never outgrows the most sequences alive
  // at once.
  std::vector<Seq> seqs;
  std::vector<int32_t> free_ids;
  int64_t live = 0;
  std::vector<std::pair<int64_t, int64_t>> copies;  // queued (src, dst)
  std::mutex mu;
};

namespace {

thread_local std::string g_bm_error;

int bm_fail(int code, const char* msg, long long a = 0) {
  char buf[256];
  snprintf(buf, sizeof(buf), msg, a);
  g_bm_error = buf;
  return code;
}

// The live sequence with this id, or NULL.
pagedkv_block_manager::Seq* find_seq(pagedkv_block_manager* m, long long id) {
  if (id < 0 || id >= (long long)m->seqs.size() || !m->seqs[id].alive) return nullptr;
  return &m->seqs[id];
}

int add_live(pagedkv_block_manager* m, pagedkv_block_manager::Seq&& s) {
  s.alive = true;
  m->live += 1;
  if (!m->free_ids.empty()) {
    const int id = m->free_ids.back();
    m->free_ids.pop_back();
    m->seqs[id] = std::move(s);
    return id;
  }
  m->seqs.push_back(std::move(s));
  return (int)m->seqs.size() - 1;
}

// Returns blk to the free list once no table references it and no queued copy names it.
void release_if_unused(pagedkv_block_manager* m, int32_t blk) {
  if (m->refcount[blk] == 0 && m->pinned[blk] == 0) m->free_list.push_back(blk);
}

int32_t pop_free(pagedkv_block_manager* m) {
  const int32_t blk = m->free_list.back();
  m->free_list.pop_back();
  m->refcount[blk] = 1;
  return blk;
}

// Append one token to s; on success *slot holds its flat slot.  Changes nothing
// when the pool is empty.
int append_one(pagedkv_block_manager* m, pagedkv_block_manager::Seq& s, int64_t* slot) {
  const int bs = m->block_size;
  const int64_t pos = s.len;
  if (pos % bs == 0) {
    // no block yet, or the last block is full: a fresh block (no copy needed,
    // even when the full last block is shared)
    if (m->free_list.empty()) return bm_fail(PAGEDKV_ENOMEM, "block pool exhausted");
    s.table.push_back(pop_free(m));
  } else {
    const int32_t last = s.table.back();
    if (m->refcount[last] > 1) {
      // shared and not full: copy on write
      if (m->free_list.empty()) return bm_fail(PAGEDKV_ENOMEM, "block pool exhausted (copy on write)");
      const int32_t fresh = pop_free(m);
      // a block still waiting for its own copy holds its source's contents
      const int32_t src = m->copy_source[last] >= 0 ? m->copy_source[last] : last;
      m->copies.emplace_back(src, fresh);
      m->copy_source[fresh] = src;
      m->pinned[src] += 1;
      m->pinned[fresh] += 1;
      m->refcount[last] -= 1;
      s.table.back() = fresh;
    }
  }
  *slot = (int64_t)s.table[pos / bs] * bs + pos % bs;
  s.len = pos + 1;
  return PAGEDKV_OK;
}

}  // namespace

extern "C" {

pagedkv_block_manager* bm_create(int num_blocks, int block_size, const int32_t* free_order) {
  if (num_blocks <= 0 || block_size <= 0) return nullptr;
  pagedkv_block_manager* m = new (std::nothrow) pagedkv_block_manager();
  if (!m) return nullptr;
  m->num_blocks = num_blocks;
  m->block_size = block_size;
  m->refcount.assign(num_blocks, 0);
  m->pinned.assign(num_blocks, 0);
  m->copy_source.assign(num_blocks, -1);
  m->free_list.resize(num_blocks);
  if (free_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      const int32_t b = free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete m;
        return nullptr;  // not a permutation
      }
      seen[b] = 1;
      m->free_list[i] = b;
    }
  } else {
    for (int i = 0; i < num_blocks; ++i) m->free_list[i] = i;
  }
  return m;
}

void bm_destroy(pagedkv_block_manager* m) { delete m; }

int bm_add_seq(pagedkv_block_manager* m, int num_tokens) {
  if (!m) return bm_fail(PAGEDKV_EINVAL, "NULL manager");
  if (num_tokens < 0) return bm_fail(PAGEDKV_EINVAL, "num_tokens %lld < 0", num_tokens);
  std::lock_guard<std::mutex> lock(m->mu);
  const int64_t need = ((int64_t)num_tokens + m->block_size - 1) / m->block_size;
  if (need > (int64_t)m->free_list.size())
    return bm_fail(PAGEDKV_ENOMEM, "pool cannot hold %lld more blocks", need);
  pagedkv_block_manager::Seq s;
  s.table.reserve(need);
  for (int64_t i = 0; i < need; ++i) s.table.push_back(pop_free(m));
  s.len = num_tokens;
  return add_live(m, std::move(s));
}

int bm_append_token(pagedkv_block_manager* m, int seq, int64_t* slot_out) {
  if (!m || !slot_out) return bm_fail(PAGEDKV_EINVAL, "NULL argument");
  std::lock_guard<std::mutex> lock(m->mu);
  pagedkv_block_manager::Seq* s = find_seq(m, seq);
  if (!s) return bm_fail(PAGEDKV_ENOENT, "unknown sequence %lld", seq);
  return append_one(m, *s, slot_out);
}

int bm_append_tokens(pagedkv_block_manager* m, const int32_t* seqs, int n, int64_t* slots_out) {
  if (!m || (n > 0 && (!seqs || !slots_out)) || n < 0) return bm_fail(PAGEDKV_EINVAL, "bad arguments");
  std::lock_guard<std::mutex> lock(m->mu);
  for (int i = 0; i < n; ++i) {
    pagedkv_block_manager::Seq* s = find_seq(m, seqs[i]);
    if (!s) {
      bm_fail(PAGEDKV_ENOENT, "unknown sequence %lld", seqs[i]);
      return i;
    }
    if (append_one(m, *s, &slots_out[i]) != PAGEDKV_OK) return i;
  }
  return n;
}

int bm_fork(pagedkv_block_manager* m, int seq, int n, int32_t* ids_out) {
  if (!m || n < 0 || (n > 0 && !ids_out)) return bm_fail(PAGEDKV_EINVAL, "bad arguments");
  std::lock_guard<std::mutex> lock(m->mu);
  const pagedkv_block_manager::Seq* p = find_seq(m, seq);
  if (!p) return bm_fail(PAGEDKV_ENOENT, "unknown sequence %lld", seq);
  const pagedkv_block_manager::Seq parent = *p;  // the vector may grow below
  if (m->seqs.size() - m->free_ids.size() + (size_t)n > (size_t)INT32_MAX)
    return bm_fail(PAGEDKV_EINVAL, "too many sequences");
  for (int c = 0; c < n; ++c) {
    for (int32_t b : parent.table) m->refcount[b] += 1;
    pagedkv_block_manager::Seq child = parent;
    ids_out[c] = add_live(m, std::move(child));
  }
  return PAGEDKV_OK;
}

int bm_free_seq(pagedkv_block_manager* m, int seq) {
  if (!m) return bm_fail(PAGEDKV_EINVAL, "NULL manager");
  std::lock_guard<std::mutex> lock(m->mu);
  pagedkv_block_manager::Seq* s = find_seq(m, seq);
  if (!s) return bm_fail(PAGEDKV_ENOENT, "unknown sequence %lld", seq);
  for (int32_t b : s->table) {
    --m->refcount[b];
    release_if_unused(m, b);
  }
  std::vector<int32_t>().swap(s->table);  // release its memory
  s->len = 0;
  s->alive = false;
  m->live -= 1;
  m->free_ids.push_back(seq);
  return PAGEDKV_OK;
}

int bm_block_table(pagedkv_block_manager* m, int seq, int32_t* out, int cap) {
  if (!m) return bm_fail(PAGEDKV_EINVAL, "NULL manager");
  std::lock_guard<std::mutex> lock(m->mu);
  const pagedkv_block_manager::Seq* s = find_seq(m, seq);
  if (!s) return bm_fail(PAGEDKV_ENOENT, "unknown sequence %lld", seq);
  const int n = (int)s->table.size();
  if (!out) return n;
  if (cap < n) return bm_fail(PAGEDKV_ERANGE, "table of %lld entries does not fit", n);
  if (n) memcpy(out, s->table.data(), n * sizeof(int32_t));
  return n;
}

int bm_seq_len(pagedkv_block_manager* m, int seq) {
  if (!m) return bm_fail(PAGEDKV_EINVAL, "NULL manager");
  std::lock_guard<std::mutex> lock(m->mu);
  const pagedkv_block_manager::Seq* s = find_seq(m, seq);
  if (!s) return bm_fail(PAGEDKV_ENOENT, "unknown sequence %lld", seq);
  return (int)s->len;
}

int bm_seq_slots(pagedkv_block_manager* m, int seq, int first, int count, int64_t* slots_out) {
  if (!m || first < 0 || count < 0 || (count > 0 && !slots_out))
    return bm_fail(PAGEDKV_EINVAL, "bad arguments");
  std::lock_guard<std::mutex> lock(m->mu);
  const pagedkv_block_manager::Seq* s = find_seq(m, seq);
  if (!s) return bm_fail(PAGEDKV_ENOENT, "unknown sequence %lld", seq);
  if ((int64_t)first + count > s->len)
    return bm_fail(PAGEDKV_ERANGE, "tokens beyond the sequence's %lld", s->len);
  const int bs = m->block_size;
  for (int i = 0; i < count; ++i) {
    const int64_t pos = (int64_t)first + i;
    slots_out[i] = (int64_t)s->table[pos / bs] * bs + pos % bs;
  }
  return count;
}

int bm_build_batch(pagedkv_block_manager* m, const int32_t* seqs, int n, int32_t* block_tables,
                   int max_blocks, int32_t* context_lens) {
  if (!m || n < 0 || max_blocks <= 0 || (n > 0 && (!seqs || !block_tables || !context_lens)))
    return bm_fail(PAGEDKV_EINVAL, "bad arguments");
  std::lock_guard<std::mutex> lock(m->mu);
  for (int i = 0; i < n; ++i) {
    const pagedkv_block_manager::Seq* s = find_seq(m, seqs[i]);
    if (!s) return bm_fail(PAGEDKV_ENOENT, "unknown sequence %lld", seqs[i]);
    if ((int)s->table.size() > max_blocks)
      return bm_fail(PAGEDKV_ERANGE, "sequence %lld has more blocks than max_blocks", seqs[i]);
  }
  for (int i = 0; i < n; ++i) {
    const auto& s = *find_seq(m, seqs[i]);
    int32_t* row = block_tables + (size_t)i * max_blocks;
    const int nb = (int)s.table.size();
    for (int j = 0; j < nb; ++j) row[j] = s.table[j];
    for (int j = nb; j < max_blocks; ++j) row[j] = -1;
    context_lens[i] = (int32_t)s.len;
  }
  return PAGEDKV_OK;
}

int bm_take_copies(pagedkv_block_manager* m, int64_t* pairs, int cap) {
  if (!m) return bm_fail(PAGEDKV_EINVAL, "NULL manager");
  std::lock_guard<std::mutex> lock(m->mu);
  const int n = (int)m->copies.size();
  if (!pairs) return n;
  if (cap < n) return bm_fail(PAGEDKV_ERANGE, "%lld pairs do not fit", n);
  for (int i = 0; i < n; ++i) {
    pairs[2 * i] = m->copies[i].first;
    pairs[2 * i + 1] = m->copies[i].second;
  }
  // the pairs are handed out: their blocks leave the queue, in pair order
  for (const auto& pr : m->copies) {
    for (const int64_t blk : {pr.first, pr.second}) {
      m->pinned[blk] -= 1;
      release_if_unused(m, (int32_t)blk);
    }
    m->copy_source[pr.second] = -1;
  }
  m->copies.clear();
  return n;
}

int bm_refcount(pagedkv_block_manager* m, int block) {
  if (!m) return bm_fail(PAGEDKV_EINVAL, "NULL manager");
  std::lock_guard<std::mutex> lock(m->mu);
  if (block < 0 || block >= m->num_blocks) return bm_fail(PAGEDKV_EINVAL, "block %lld out of range", block);
  return m->refcount[block];
}

int bm_num_free(pagedkv_block_manager* m) {
  if (!m) return bm_fail(PAGEDKV_EINVAL, "NULL manager");
  std::lock_guard<std::mutex> lock(m->mu);
  return (int)m->free_list.size();
}

int bm_free_list(pagedkv_block_manager* m, int32_t* out, int cap) {
  if (!m) return bm_fail(PAGEDKV_EINVAL, "NULL manager");
  std::lock_guard<std::mutex> lock(m->mu);
  const int n = (int)m->free_list.size();
  if (!out) return n;
  if (cap < n) return bm_fail(PAGEDKV_ERANGE, "free list of %lld does not fit", n);
  if (n) memcpy(out, m->free_list.data(), n * sizeof(int32_t));
  return n;
}

int bm_stats(pagedkv_block_manager* m, pagedkv_bm_stats* out) {
  if (!m || !out) return bm_fail(PAGEDKV_EINVAL, "NULL argument");
  std::lock_guard<std::mutex> lock(m->mu);
  std::vector<int32_t> fill(m->num_blocks, 0);
  int64_t logical = 0, entries = 0;
  for (const auto& s : m->seqs) {
    if (!s.alive) continue;
    logical += s.len;
    entries += (int64_t)s.table.size();
    for (size_t j = 0; j < s.table.size(); ++j) {
      const int64_t in_block = std::min<int64_t>(m->block_size, s.len - (int64_t)j * m->block_size);
      int32_t& f = fill[s.table[j]];
      if (in_block > f) f = (int32_t)in_block;
    }
  }
  int64_t used = 0, filled = 0, held = 0;
  for (int b = 0; b < m->num_blocks; ++b) {
    if (m->refcount[b] > 0) ++used;
    else if (m->pinned[b] > 0) ++held;
    filled += fill[b];
  }
  out->num_blocks = m->num_blocks;
  out->free_blocks = (int64_t)m->free_list.size();
  out->used_blocks = used;
  out->num_seqs = m->live;
  out->logical_tokens = logical;
  out->filled_slots = filled;
  out->allocated_slots = used * m->block_size;
  out->table_entries = entries;
  out->held_blocks = held;
  return PAGEDKV_OK;
}

// Message of the calling thread's last failed bm_* call.
const char* bm_last_error(void) { return g_bm_error.c_str(); }

}  // extern "C"
