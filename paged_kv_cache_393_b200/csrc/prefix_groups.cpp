// Host grouping of a decode batch by shared table prefixes, for the
// shared-prefix decode.  Contract: include/pagedkv.h (pagedkv_prefix_groups).
//
// Sequences forked from one prompt (parallel sampling, beam search) or served
// from one cached prefix reference the same physical blocks at the start of
// their tables (lpnh.cn/news/2758356 §4.1-§4.2; n1n.ai "前缀缓存").  The
// grouping only looks at the tables: sequences whose first entries are equal
// physical blocks hold the same tokens there, so one read of those blocks can
// serve all of them.
//
//  1. A sequence can share at most its whole blocks before the block holding
//     its last token: (L - 1) / block_size blocks.
//  2. Sequences are bucketed by their first block id and, inside a bucket,
//     sorted by their shareable table prefix, so that sequences with longer
//     common prefixes sit next to each other.
//  3. Each bucket is cut, in that order, into runs of at most max_members
//     sequences; a run of two or more whose common prefix is at least one
//     block becomes a group of that many blocks.
#include "../../include/pagedkv.h"

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <unordered_map>
#include <vector>

namespace pkv {
int record_error(int code, const char* message);  // pagedkv_last_error() reports it
}

namespace {

int fail(int code, const char* msg) { return pkv::record_error(code, msg); }

}  // namespace

extern "C" {

int pagedkv_prefix_groups(const int32_t* block_tables, const int32_t* context_lens,
                          int num_seqs, int max_blocks_per_seq, int block_size, int max_members,
                          int32_t* seq_prefix_tokens, int32_t* groups, int groups_capacity) {
  if (num_seqs < 0) return fail(PAGEDKV_EINVAL, "num_seqs must be >= 0");
  if (num_seqs == 0) return 0;
  if (!block_tables || !context_lens || !seq_prefix_tokens)
    return fail(PAGEDKV_EINVAL, "a required pointer is NULL");
  if (max_blocks_per_seq <= 0 || block_size <= 0)
    return fail(PAGEDKV_EINVAL, "max_blocks_per_seq and block_size must be positive");
  if (max_members < 1 || max_members > PAGEDKV_GROUP_MAX_MEMBERS)
    return fail(PAGEDKV_EINVAL, "max_members must be in [1, 8]");
  if (groups_capacity < 0 || (groups_capacity > 0 && !groups))
    return fail(PAGEDKV_EINVAL, "bad groups buffer");

  const auto row = [&](int b) { return block_tables + (size_t)b * max_blocks_per_seq; };
  std::vector<int> shareable(num_seqs, 0);
  std::unordered_map<int32_t, std::vector<int>> buckets;
  std::vector<int32_t> keys;  // first appearance order
  for (int b = 0; b < num_seqs; ++b) {
    seq_prefix_tokens[b] = 0;
    const int L = context_lens[b];
    int n = L >= 1 ? (L - 1) / block_size : 0;
    if (n > max_blocks_per_seq) n = max_blocks_per_seq;
    int valid = 0;  // entries that are block ids
    while (valid < n && row(b)[valid] >= 0) ++valid;
    shareable[b] = valid;
    if (valid == 0 || max_members < 2) continue;
    auto it = buckets.find(row(b)[0]);
    if (it == buckets.end()) {
      keys.push_back(row(b)[0]);
      buckets.emplace(row(b)[0], std::vector<int>{b});
    } else {
      it->second.push_back(b);
    }
  }

  int count = 0;
  for (int32_t key : keys) {
    std::vector<int>& seqs = buckets[key];
    if (seqs.size() < 2) continue;
    std::stable_sort(seqs.begin(), seqs.end(), [&](int a, int b) {
      return std::lexicographical_compare(row(a), row(a) + shareable[a], row(b),
                                          row(b) + shareable[b]);
    });
    for (size_t i0 = 0; i0 < seqs.size(); i0 += (size_t)max_members) {
      const size_t i1 = std::min(seqs.size(), i0 + (size_t)max_members);
      if (i1 - i0 < 2) continue;
      const int first = seqs[i0];
      int common = shareable[first];
      for (size_t i = i0 + 1; i < i1; ++i) {
        const int m = seqs[i];
        int k = 0;
        const int lim = std::min(common, shareable[m]);
        while (k < lim && row(m)[k] == row(first)[k]) ++k;
        common = k;
      }
      if (common < 1) continue;
      if (count >= groups_capacity) {
        for (int b = 0; b < num_seqs; ++b) seq_prefix_tokens[b] = 0;
        return fail(PAGEDKV_ERANGE, "more groups than groups_capacity");
      }
      int32_t* g = groups + (size_t)count * PAGEDKV_GROUP_WIDTH;
      g[0] = common;
      for (int j = 0; j < PAGEDKV_GROUP_MAX_MEMBERS; ++j)
        g[1 + j] = (size_t)j < i1 - i0 ? seqs[i0 + j] : -1;
      for (size_t i = i0; i < i1; ++i) seq_prefix_tokens[seqs[i]] = common * block_size;
      ++count;
    }
  }
  return count;
}

}  // extern "C"
