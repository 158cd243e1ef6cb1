// Host block manager of libpagedkv (see include/pagedkv.h for the contract).
//
// Rules, by source page:
//  * "What is PagedAttention?" (qubittool glossary), How It Works / Map
//    Logical to Physical Blocks: per-sequence block tables map logical block
//    indices to physical block ids; prefill reserves enough blocks for the
//    input; decode appends into the partly filled tail and takes a new block
//    only when the tail is full; a failed allocation is reported explicitly
//    and corrupts no sequence's state.
//  * "PagedAttention: Optimizing KV Cache in vLLM" (grasp.study), section 4:
//    sharing points tables at the same blocks and raises reference counts; a
//    writer into a shared block gets a new block with a copy of the contents,
//    only its own table changes; counts govern reclamation.
// Open points, read plainly: FIFO free queue; reclaimed blocks go to the back
// in ascending id order; a batched step processes sequences in the order given
// and is all-or-nothing.
#include <algorithm>
#include <climits>
#include <cstdint>
#include <deque>
#include <new>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "pa_internal.h"

using pagedkv::fail;
using pagedkv::ok;

struct pa_bm {
  struct Seq {
    std::vector<int32_t> table;
    int64_t ctx = 0;
    bool swapped = false;
    std::vector<int32_t> swapped_table;  // table at swap-out time
  };
  int num_blocks = 0;
  int block_size = 0;
  int max_blocks_per_seq = 0;
  std::deque<int32_t> free_queue;
  std::vector<int32_t> refcount;
  std::unordered_map<int64_t, Seq> seqs;
  int64_t cow_copies = 0;
};

namespace {

bool find_seq(pa_bm* bm, int64_t id, pa_bm::Seq** out) {
  auto it = bm->seqs.find(id);
  if (it == bm->seqs.end()) return false;
  *out = &it->second;
  return true;
}

// Blocks one append of `seq` needs given the (possibly overlaid) count of its
// tail; -1 when the table is full and the tail is full (capacity error).
int need_for_append(const pa_bm* bm, const pa_bm::Seq& s, int tail_count) {
  if (s.ctx % bm->block_size == 0) {
    if (static_cast<int>(s.table.size()) >= bm->max_blocks_per_seq) return -1;
    return 1;
  }
  return tail_count > 1 ? 1 : 0;
}

// Dry run of a batched step: validates ids and capacity and counts the blocks
// needed, with earlier copies lowering the counts later writers see.
pa_status_t plan_step(pa_bm* bm, const int64_t* ids, int n, int64_t* need_out) {
  if (n < 0 || (n > 0 && ids == nullptr)) return fail(PA_ERR_INVALID_ARG, "bad seq_ids/n");
  std::unordered_set<int64_t> seen;
  std::unordered_map<int32_t, int32_t> overlay;
  int64_t need = 0;
  for (int i = 0; i < n; ++i) {
    pa_bm::Seq* s = nullptr;
    if (!find_seq(bm, ids[i], &s))
      return fail(PA_ERR_INVALID_ARG, "unknown sequence %lld", (long long)ids[i]);
    if (!seen.insert(ids[i]).second)
      return fail(PA_ERR_INVALID_ARG, "sequence %lld appears twice in one step", (long long)ids[i]);
    if (s->swapped) return fail(PA_ERR_INVALID_ARG, "sequence %lld is swapped out", (long long)ids[i]);
    int tail_count = 0;
    int32_t tail = -1;
    if (s->ctx % bm->block_size != 0) {
      tail = s->table.back();
      auto it = overlay.find(tail);
      tail_count = it != overlay.end() ? it->second : bm->refcount[tail];
    }
    int k = need_for_append(bm, *s, tail_count);
    if (k < 0)
      return fail(PA_ERR_INVALID_ARG, "sequence %lld is at max_blocks_per_seq", (long long)ids[i]);
    if (k == 1 && tail >= 0) overlay[tail] = tail_count - 1;
    need += k;
  }
  *need_out = need;
  return PA_OK;
}

void append_one(pa_bm* bm, pa_bm::Seq& s, int64_t* slot, int64_t* cow_src, int64_t* cow_dst) {
  const int64_t offset = s.ctx % bm->block_size;
  int32_t block;
  *cow_src = -1;
  *cow_dst = -1;
  if (offset == 0) {
    block = bm->free_queue.front();
    bm->free_queue.pop_front();
    bm->refcount[block] = 1;
    s.table.push_back(block);
  } else {
    block = s.table.back();
    if (bm->refcount[block] > 1) {
      const int32_t fresh = bm->free_queue.front();
      bm->free_queue.pop_front();
      bm->refcount[fresh] = 1;
      bm->refcount[block] -= 1;
      s.table.back() = fresh;
      *cow_src = block;
      *cow_dst = fresh;
      bm->cow_copies += 1;
      block = fresh;
    }
  }
  *slot = static_cast<int64_t>(block) * bm->block_size + offset;
  s.ctx += 1;
}

}  // namespace

extern "C" {

pa_status_t pa_bm_create(int num_blocks, int block_size, int max_blocks_per_seq,
                         const int32_t* initial_free_order, pa_bm_t* out) {
  if (out == nullptr) return fail(PA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (num_blocks <= 0 || block_size <= 0 || max_blocks_per_seq <= 0)
    return fail(PA_ERR_INVALID_ARG, "sizes must be positive");
  pa_bm* bm = new (std::nothrow) pa_bm();
  if (bm == nullptr) return fail(PA_ERR_INVALID_ARG, "out of host memory");
  bm->num_blocks = num_blocks;
  bm->block_size = block_size;
  bm->max_blocks_per_seq = max_blocks_per_seq;
  bm->refcount.assign(num_blocks, 0);
  if (initial_free_order != nullptr) {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      const int32_t b = initial_free_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete bm;
        return fail(PA_ERR_INVALID_ARG, "initial_free_order is not a permutation of 0..%d",
                    num_blocks - 1);
      }
      seen[b] = 1;
      bm->free_queue.push_back(b);
    }
  } else {
    for (int i = 0; i < num_blocks; ++i) bm->free_queue.push_back(i);
  }
  *out = bm;
  return ok();
}

pa_status_t pa_bm_destroy(pa_bm_t bm) {
  delete bm;
  return ok();
}

pa_status_t pa_bm_allocate(pa_bm_t bm, int64_t seq_id, int64_t num_tokens) {
  if (bm == nullptr) return fail(PA_ERR_INVALID_ARG, "bm is NULL");
  if (bm->seqs.count(seq_id)) return fail(PA_ERR_INVALID_ARG, "sequence %lld exists", (long long)seq_id);
  if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "num_tokens < 0");
  const int64_t need = (num_tokens + bm->block_size - 1) / bm->block_size;
  if (need > bm->max_blocks_per_seq)
    return fail(PA_ERR_INVALID_ARG, "%lld tokens exceed max_blocks_per_seq", (long long)num_tokens);
  if (need > static_cast<int64_t>(bm->free_queue.size()))
    return fail(PA_ERR_NO_FREE_BLOCKS, "need %lld blocks, %zu free", (long long)need,
                bm->free_queue.size());
  pa_bm::Seq s;
  s.table.reserve(need);
  for (int64_t i = 0; i < need; ++i) {
    const int32_t b = bm->free_queue.front();
    bm->free_queue.pop_front();
    bm->refcount[b] = 1;
    s.table.push_back(b);
  }
  s.ctx = num_tokens;
  bm->seqs.emplace(seq_id, std::move(s));
  return ok();
}

pa_status_t pa_bm_fork(pa_bm_t bm, int64_t parent_id, int64_t child_id) {
  if (bm == nullptr) return fail(PA_ERR_INVALID_ARG, "bm is NULL");
  pa_bm::Seq* p = nullptr;
  if (!find_seq(bm, parent_id, &p)) return fail(PA_ERR_INVALID_ARG, "unknown parent %lld", (long long)parent_id);
  if (bm->seqs.count(child_id)) return fail(PA_ERR_INVALID_ARG, "sequence %lld exists", (long long)child_id);
  if (p->swapped) return fail(PA_ERR_INVALID_ARG, "sequence %lld is swapped out", (long long)parent_id);
  pa_bm::Seq c = *p;  // copy before emplace may rehash
  for (int32_t b : c.table)
    if (b >= 0) bm->refcount[b] += 1;  // released entries (-1) hold nothing
  bm->seqs.emplace(child_id, std::move(c));
  return ok();
}

pa_status_t pa_bm_append_slots(pa_bm_t bm, const int64_t* seq_ids, int n, int64_t* slots,
                               int64_t* cow_pairs, int* num_cow) {
  if (bm == nullptr) return fail(PA_ERR_INVALID_ARG, "bm is NULL");
  if (n > 0 && (slots == nullptr || cow_pairs == nullptr))
    return fail(PA_ERR_INVALID_ARG, "slots/cow_pairs is NULL");
  int64_t need = 0;
  pa_status_t st = plan_step(bm, seq_ids, n, &need);
  if (st != PA_OK) return st;
  if (need > static_cast<int64_t>(bm->free_queue.size()))
    return fail(PA_ERR_NO_FREE_BLOCKS, "step needs %lld blocks, %zu free", (long long)need,
                bm->free_queue.size());
  int cows = 0;
  for (int i = 0; i < n; ++i) {
    pa_bm::Seq& s = bm->seqs.find(seq_ids[i])->second;
    int64_t src, dst;
    append_one(bm, s, &slots[i], &src, &dst);
    if (src >= 0) {
      cow_pairs[2 * cows] = src;
      cow_pairs[2 * cows + 1] = dst;
      ++cows;
    }
  }
  if (num_cow) *num_cow = cows;
  return ok();
}

pa_status_t pa_bm_append_slot(pa_bm_t bm, int64_t seq_id, int64_t* slot, int64_t* cow_src,
                              int64_t* cow_dst) {
  if (slot == nullptr || cow_src == nullptr || cow_dst == nullptr)
    return fail(PA_ERR_INVALID_ARG, "NULL output");
  int64_t pair[2] = {-1, -1};
  int cows = 0;
  pa_status_t st = pa_bm_append_slots(bm, &seq_id, 1, slot, pair, &cows);
  if (st != PA_OK) return st;
  *cow_src = cows ? pair[0] : -1;
  *cow_dst = cows ? pair[1] : -1;
  return PA_OK;
}

pa_status_t pa_bm_can_append(pa_bm_t bm, const int64_t* seq_ids, int n, int* ok_out) {
  if (bm == nullptr || ok_out == nullptr) return fail(PA_ERR_INVALID_ARG, "NULL argument");
  int64_t need = 0;
  pa_status_t st = plan_step(bm, seq_ids, n, &need);
  if (st != PA_OK) return st;
  *ok_out = need <= static_cast<int64_t>(bm->free_queue.size()) ? 1 : 0;
  return ok();
}

pa_status_t pa_bm_free(pa_bm_t bm, int64_t seq_id) {
  if (bm == nullptr) return fail(PA_ERR_INVALID_ARG, "bm is NULL");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return fail(PA_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq_id);
  std::vector<int32_t> reclaimed;
  for (int32_t b : it->second.table) {
    if (b < 0) continue;
    bm->refcount[b] -= 1;
    if (bm->refcount[b] == 0) reclaimed.push_back(b);
  }
  std::sort(reclaimed.begin(), reclaimed.end());
  for (int32_t b : reclaimed) bm->free_queue.push_back(b);
  bm->seqs.erase(it);
  return ok();
}

pa_status_t pa_bm_release_before(pa_bm_t bm, int64_t seq_id, int64_t first_token, int* num_reclaimed) {
  if (bm == nullptr) return fail(PA_ERR_INVALID_ARG, "bm is NULL");
  if (first_token < 0) return fail(PA_ERR_INVALID_ARG, "first_token < 0");
  pa_bm::Seq* s = nullptr;
  if (!find_seq(bm, seq_id, &s)) return fail(PA_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq_id);
  if (s->swapped) return fail(PA_ERR_INVALID_ARG, "sequence %lld is swapped out", (long long)seq_id);
  const int64_t n_out = std::min<int64_t>(first_token / bm->block_size,
                                          static_cast<int64_t>(s->table.size()));
  std::vector<int32_t> reclaimed;
  for (int64_t i = 0; i < n_out; ++i) {
    const int32_t b = s->table[i];
    if (b < 0) continue;
    bm->refcount[b] -= 1;
    if (bm->refcount[b] == 0) reclaimed.push_back(b);
    s->table[i] = -1;
  }
  std::sort(reclaimed.begin(), reclaimed.end());
  for (int32_t b : reclaimed) bm->free_queue.push_back(b);
  if (num_reclaimed) *num_reclaimed = static_cast<int>(reclaimed.size());
  return ok();
}

pa_status_t pa_bm_swap_out(pa_bm_t bm, int64_t seq_id, int32_t* blocks, int capacity, int* n) {
  if (bm == nullptr || n == nullptr) return fail(PA_ERR_INVALID_ARG, "NULL argument");
  pa_bm::Seq* s = nullptr;
  if (!find_seq(bm, seq_id, &s)) return fail(PA_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq_id);
  if (s->swapped) return fail(PA_ERR_INVALID_ARG, "sequence %lld is already swapped out", (long long)seq_id);
  const int len = static_cast<int>(s->table.size());
  if (len > capacity || (len > 0 && blocks == nullptr))
    return fail(PA_ERR_INVALID_ARG, "capacity %d < %d blocks", capacity, len);
  std::vector<int32_t> reclaimed;
  for (int32_t b : s->table) {
    if (b < 0) continue;
    bm->refcount[b] -= 1;
    if (bm->refcount[b] == 0) reclaimed.push_back(b);
  }
  std::sort(reclaimed.begin(), reclaimed.end());
  for (int32_t b : reclaimed) bm->free_queue.push_back(b);
  std::copy(s->table.begin(), s->table.end(), blocks);
  s->swapped_table = s->table;
  for (int32_t& b : s->table) b = -1;
  s->swapped = true;
  *n = len;
  return ok();
}

pa_status_t pa_bm_swap_in(pa_bm_t bm, int64_t seq_id, int32_t* blocks, int capacity, int* n) {
  if (bm == nullptr || n == nullptr) return fail(PA_ERR_INVALID_ARG, "NULL argument");
  pa_bm::Seq* s = nullptr;
  if (!find_seq(bm, seq_id, &s)) return fail(PA_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq_id);
  if (!s->swapped) return fail(PA_ERR_INVALID_ARG, "sequence %lld is not swapped out", (long long)seq_id);
  const int len = static_cast<int>(s->swapped_table.size());
  if (len > capacity || (len > 0 && blocks == nullptr))
    return fail(PA_ERR_INVALID_ARG, "capacity %d < %d blocks", capacity, len);
  int64_t need = 0;
  for (int32_t b : s->swapped_table) need += b >= 0;
  if (need > static_cast<int64_t>(bm->free_queue.size()))
    return fail(PA_ERR_NO_FREE_BLOCKS, "swap-in needs %lld blocks, %zu free", (long long)need,
                bm->free_queue.size());
  for (int i = 0; i < len; ++i) {
    if (s->swapped_table[i] < 0) {
      s->table[i] = s->swapped_table[i];
      continue;
    }
    const int32_t b = bm->free_queue.front();
    bm->free_queue.pop_front();
    bm->refcount[b] = 1;
    s->table[i] = b;
  }
  std::copy(s->table.begin(), s->table.end(), blocks);
  s->swapped = false;
  s->swapped_table.clear();
  *n = len;
  return ok();
}

pa_status_t pa_bm_block_table(pa_bm_t bm, int64_t seq_id, int32_t* row, int row_capacity,
                              int* n_blocks) {
  if (bm == nullptr || n_blocks == nullptr) return fail(PA_ERR_INVALID_ARG, "NULL argument");
  pa_bm::Seq* s = nullptr;
  if (!find_seq(bm, seq_id, &s)) return fail(PA_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq_id);
  const int n = static_cast<int>(s->table.size());
  if (n > row_capacity || (n > 0 && row == nullptr))
    return fail(PA_ERR_INVALID_ARG, "row_capacity %d < %d blocks", row_capacity, n);
  std::copy(s->table.begin(), s->table.end(), row);
  *n_blocks = n;
  return ok();
}

pa_status_t pa_bm_context_len(pa_bm_t bm, int64_t seq_id, int64_t* context_len) {
  if (bm == nullptr || context_len == nullptr) return fail(PA_ERR_INVALID_ARG, "NULL argument");
  pa_bm::Seq* s = nullptr;
  if (!find_seq(bm, seq_id, &s)) return fail(PA_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq_id);
  *context_len = s->ctx;
  return ok();
}

pa_status_t pa_bm_export(pa_bm_t bm, const int64_t* seq_ids, int n, int32_t* tables,
                         int32_t* context_lens, int32_t pad_value) {
  if (bm == nullptr || n < 0 || (n > 0 && (seq_ids == nullptr || tables == nullptr ||
                                           context_lens == nullptr)))
    return fail(PA_ERR_INVALID_ARG, "NULL argument");
  const int mbs = bm->max_blocks_per_seq;
  for (int i = 0; i < n; ++i) {
    pa_bm::Seq* s = nullptr;
    if (!find_seq(bm, seq_ids[i], &s))
      return fail(PA_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq_ids[i]);
  }
  for (int i = 0; i < n; ++i) {
    const pa_bm::Seq& s = bm->seqs.find(seq_ids[i])->second;
    int32_t* row = tables + static_cast<int64_t>(i) * mbs;
    const int nb = static_cast<int>(s.table.size());
    std::copy(s.table.begin(), s.table.end(), row);
    std::fill(row + nb, row + mbs, pad_value);
    context_lens[i] = static_cast<int32_t>(s.ctx);
  }
  return ok();
}

pa_status_t pa_bm_prefix_groups(pa_bm_t bm, const int64_t* seq_ids, int n, int min_shared_blocks,
                                int32_t* group_offsets, int32_t* group_members,
                                int32_t* group_blocks, int* num_groups) {
  if (bm == nullptr || num_groups == nullptr || n < 0 ||
      (n > 0 && (seq_ids == nullptr || group_offsets == nullptr || group_members == nullptr ||
                 group_blocks == nullptr)))
    return fail(PA_ERR_INVALID_ARG, "NULL argument");
  std::vector<const pa_bm::Seq*> seqs(n);
  for (int i = 0; i < n; ++i) {
    pa_bm::Seq* s = nullptr;
    if (!find_seq(bm, seq_ids[i], &s))
      return fail(PA_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq_ids[i]);
    seqs[i] = s;
  }
  // Bucket by first physical block, keeping batch order inside a bucket.
  std::unordered_map<int32_t, std::vector<int32_t>> buckets;
  std::vector<int32_t> first_seen;
  for (int i = 0; i < n; ++i) {
    if (seqs[i]->table.empty() || seqs[i]->table[0] < 0) continue;  // none, or released
    const int32_t b0 = seqs[i]->table[0];
    auto it = buckets.find(b0);
    if (it == buckets.end()) {
      buckets.emplace(b0, std::vector<int32_t>{i});
      first_seen.push_back(b0);
    } else {
      it->second.push_back(i);
    }
  }
  int groups = 0, written = 0;
  group_offsets[0] = 0;
  for (int32_t b0 : first_seen) {
    const std::vector<int32_t>& mem = buckets[b0];
    if (mem.size() < 2) continue;
    // shared = longest common table prefix, limited to blocks full for all
    int64_t shared = INT64_MAX;
    for (int32_t i : mem) shared = std::min<int64_t>(shared, seqs[i]->ctx / bm->block_size);
    const std::vector<int32_t>& t0 = seqs[mem[0]]->table;
    for (int32_t i : mem) {
      const std::vector<int32_t>& t = seqs[i]->table;
      int64_t k = 0;
      while (k < shared && t[k] == t0[k]) ++k;
      shared = k;
    }
    if (shared < std::max(1, min_shared_blocks)) continue;
    for (int32_t i : mem) group_members[written++] = i;
    group_blocks[groups] = static_cast<int32_t>(shared);
    group_offsets[++groups] = written;
  }
  *num_groups = groups;
  return ok();
}

pa_status_t pa_bm_refcount(pa_bm_t bm, int block_id, int* refcount) {
  if (bm == nullptr || refcount == nullptr) return fail(PA_ERR_INVALID_ARG, "NULL argument");
  if (block_id < 0 || block_id >= bm->num_blocks) return fail(PA_ERR_INVALID_ARG, "block %d out of range", block_id);
  *refcount = bm->refcount[block_id];
  return ok();
}

pa_status_t pa_bm_free_queue(pa_bm_t bm, int32_t* out, int capacity, int* n) {
  if (bm == nullptr || n == nullptr) return fail(PA_ERR_INVALID_ARG, "NULL argument");
  const int len = static_cast<int>(bm->free_queue.size());
  if (len > capacity || (len > 0 && out == nullptr))
    return fail(PA_ERR_INVALID_ARG, "capacity %d < %d", capacity, len);
  std::copy(bm->free_queue.begin(), bm->free_queue.end(), out);
  *n = len;
  return ok();
}

pa_status_t pa_bm_stats(pa_bm_t bm, pa_bm_stats_t* st) {
  if (bm == nullptr || st == nullptr) return fail(PA_ERR_INVALID_ARG, "NULL argument");
  pa_bm_stats_t r{};
  r.num_blocks = bm->num_blocks;
  r.free_blocks = static_cast<int64_t>(bm->free_queue.size());
  for (int32_t c : bm->refcount) {
    r.used_blocks += c > 0;
    r.shared_blocks += c > 1;
  }
  r.num_seqs = static_cast<int64_t>(bm->seqs.size());
  for (const auto& kv : bm->seqs) {  // resident blocks and tokens only
    int64_t resident = 0;
    for (int32_t b : kv.second.table) resident += b >= 0;
    const int64_t released = static_cast<int64_t>(kv.second.table.size()) - resident;
    if (!kv.second.swapped) r.logical_tokens += kv.second.ctx - released * bm->block_size;
    r.logical_slots += resident * bm->block_size;
  }
  r.tail_waste_slots = r.logical_slots - r.logical_tokens;
  r.cow_copies = bm->cow_copies;
  *st = r;
  return ok();
}

}  // extern "C"
