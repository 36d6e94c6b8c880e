// block_manager.cpp -- host-side block manager of a paged KV cache (declared in
// include/pagedkv.h, pa_bm_*): a pool of fixed-size physical blocks, one block table per
// sequence, reference counts, on-demand allocation, copy-on-write on divergence, and
// release back to the pool.
//
// Follows "PagedAttention in Production: Boosting LLM Serving Throughput with Paged KV
// Cache", section "Core Principle" (logical blocks map to physical blocks through a
// per-request block table; blocks are allocated on demand and returned to the pool when
// the request finishes); "Paged Attention and Memory Efficiency in Production LLM
// Serving", section "How PagedAttention borrows OS paging" (requests with an identical
// prefix point at the same physical blocks and a new block is allocated only when a
// sequence diverges, as in copy-on-write); "PagedAttention -- The KV Cache Problem",
// sections "How It Works" (fixed-size blocks, allocate on demand, free immediately) and
// "Why This Matters for Production" (parallel sampling and beam search share blocks
// copy-on-write).
//
// It produces what the CUDA calls consume: int32 block tables, int32 context lengths,
// int64 slot mappings and int32 (src, dst) copy pairs.  Not thread-safe: a caller
// serialises calls on one manager.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <deque>
#include <new>
#include <unordered_map>
#include <vector>

#include "pagedkv.h"

struct pa_block_manager {
  struct Seq {
    std::vector<int32_t> table;  // logical block i -> physical block
    int64_t len = 0;             // cached tokens
    bool swapped = false;        // preempted: holds no block, keeps its length
  };
  int32_t num_blocks = 0, block_size = 0;
  std::vector<int32_t> ref;      // reference count per physical block
  std::deque<int32_t> free;      // free blocks, handed out from the front
  std::unordered_map<int32_t, Seq> seqs;
  int32_t next_id = 0;

  int32_t take() {               // caller has checked that a block is free
    const int32_t b = free.front();
    free.pop_front();
    ref[b] = 1;
    return b;
  }
  Seq* find(int32_t id) {
    auto it = seqs.find(id);
    return it == seqs.end() ? nullptr : &it->second;
  }
  const Seq* find(int32_t id) const {
    auto it = seqs.find(id);
    return it == seqs.end() ? nullptr : &it->second;
  }
  // a sequence that holds its blocks (known and not swapped out)
  const Seq* resident(int32_t id) const {
    const Seq* s = find(id);
    return s && !s->swapped ? s : nullptr;
  }
  void drop(int32_t b) {         // one reference less; a block nobody holds is free again
    if (--ref[(size_t)b] == 0) free.push_back(b);
  }
  int64_t blocks_for(int64_t tokens) const { return (tokens + block_size - 1) / block_size; }
};

extern "C" {

pa_status pa_bm_create(int num_blocks, int block_size, const int32_t* free_order,
                       pa_block_manager** out) {
  if (!out) return PA_ERR_INVALID;
  *out = nullptr;
  if (num_blocks <= 0 || block_size <= 0) return PA_ERR_INVALID;
  pa_block_manager* bm = new (std::nothrow) pa_block_manager();
  if (!bm) return PA_ERR_NO_MEMORY;
  bm->num_blocks = num_blocks;
  bm->block_size = block_size;
  bm->ref.assign((size_t)num_blocks, 0);
  if (free_order) {
    std::vector<uint8_t> seen((size_t)num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      const int32_t b = free_order[i];
      if (b < 0 || b >= num_blocks || seen[(size_t)b]) {
        delete bm;
        return PA_ERR_INVALID;   // not a permutation of the pool
      }
      seen[(size_t)b] = 1;
      bm->free.push_back(b);
    }
  } else {
    for (int i = 0; i < num_blocks; ++i) bm->free.push_back(i);
  }
  *out = bm;
  return PA_OK;
}

void pa_bm_destroy(pa_block_manager* bm) { delete bm; }

int pa_bm_free_blocks(const pa_block_manager* bm) { return bm ? (int)bm->free.size() : -1; }

int pa_bm_refcount(const pa_block_manager* bm, int block) {
  if (!bm || block < 0 || block >= bm->num_blocks) return -1;
  return bm->ref[(size_t)block];
}

pa_status pa_bm_allocate(pa_block_manager* bm, int num_tokens, int32_t* seq_id) {
  if (!bm || !seq_id || num_tokens < 0) return PA_ERR_INVALID;
  const int64_t need = bm->blocks_for(num_tokens);
  if (need > (int64_t)bm->free.size()) return PA_ERR_NO_BLOCKS;
  pa_block_manager::Seq s;
  s.table.reserve((size_t)need);
  for (int64_t i = 0; i < need; ++i) s.table.push_back(bm->take());
  s.len = num_tokens;
  const int32_t id = bm->next_id++;
  bm->seqs.emplace(id, std::move(s));
  *seq_id = id;
  return PA_OK;
}

pa_status pa_bm_fork(pa_block_manager* bm, int32_t seq, int32_t* child) {
  if (!bm || !child) return PA_ERR_INVALID;
  const pa_block_manager::Seq* p = bm->resident(seq);
  if (!p) return PA_ERR_INVALID;
  pa_block_manager::Seq c = *p;                  // shares every block of the parent
  for (int32_t b : c.table) ++bm->ref[(size_t)b];
  const int32_t id = bm->next_id++;
  bm->seqs.emplace(id, std::move(c));
  *child = id;
  return PA_OK;
}

pa_status pa_bm_append_tokens(pa_block_manager* bm, const int32_t* seqs, int n, int64_t* slots,
                              int32_t* cow_pairs, int* num_cow) {
  if (!bm || n < 0 || (n && (!seqs || !slots || !cow_pairs || !num_cow))) return PA_ERR_INVALID;
  if (num_cow) *num_cow = 0;
  if (n == 0) return PA_OK;
  // Dry run on copies of the touched state: how many fresh blocks the whole batch needs
  // (a new logical block, or a private copy of a shared partial block), so that a batch
  // the pool cannot serve changes nothing.
  struct Sim {
    int64_t len, nblk;
    std::vector<int64_t> priv;   // logical blocks made private earlier in this batch
  };
  std::unordered_map<int32_t, Sim> sim;
  std::unordered_map<int32_t, int32_t> ref;
  int64_t need = 0;
  for (int i = 0; i < n; ++i) {
    const pa_block_manager::Seq* s = bm->resident(seqs[i]);
    if (!s) return PA_ERR_INVALID;
    Sim& m = sim.try_emplace(seqs[i], Sim{s->len, (int64_t)s->table.size(), {}}).first->second;
    const int64_t lb = m.len / bm->block_size;
    if (lb == m.nblk) {
      ++need;
      ++m.nblk;
      m.priv.push_back(lb);
    } else {
      bool priv = false;
      for (int64_t x : m.priv) priv |= x == lb;
      if (!priv) {
        const int32_t b = s->table[(size_t)lb];
        auto ri = ref.find(b);
        const int32_t r = ri == ref.end() ? bm->ref[(size_t)b] : ri->second;
        if (r > 1) {
          ++need;
          ref[b] = r - 1;
          m.priv.push_back(lb);
        }
      }
    }
    ++m.len;
  }
  if (need > (int64_t)bm->free.size()) return PA_ERR_NO_BLOCKS;
  int nc = 0;
  for (int i = 0; i < n; ++i) {
    pa_block_manager::Seq& s = *bm->find(seqs[i]);
    const int64_t pos = s.len;
    const int64_t lb = pos / bm->block_size, off = pos % bm->block_size;
    if (lb == (int64_t)s.table.size()) {
      s.table.push_back(bm->take());
    } else if (bm->ref[(size_t)s.table[(size_t)lb]] > 1) {
      const int32_t src = s.table[(size_t)lb];
      const int32_t dst = bm->take();
      --bm->ref[(size_t)src];
      s.table[(size_t)lb] = dst;
      cow_pairs[2 * nc] = src;
      cow_pairs[2 * nc + 1] = dst;
      ++nc;
    }
    s.len = pos + 1;
    slots[i] = (int64_t)s.table[(size_t)lb] * bm->block_size + off;
  }
  *num_cow = nc;
  return PA_OK;
}

pa_status pa_bm_release(pa_block_manager* bm, int32_t seq) {
  if (!bm) return PA_ERR_INVALID;
  auto it = bm->seqs.find(seq);
  if (it == bm->seqs.end()) return PA_ERR_INVALID;
  for (int32_t b : it->second.table) bm->drop(b);
  bm->seqs.erase(it);
  return PA_OK;
}

int64_t pa_bm_context_len(const pa_block_manager* bm, int32_t seq) {
  const pa_block_manager::Seq* s = bm ? bm->find(seq) : nullptr;
  return s ? s->len : -1;
}

int pa_bm_num_blocks_of(const pa_block_manager* bm, int32_t seq) {
  const pa_block_manager::Seq* s = bm ? bm->find(seq) : nullptr;
  return s ? (int)s->table.size() : -1;
}

int pa_bm_max_blocks(const pa_block_manager* bm, const int32_t* seqs, int n) {
  if (!bm || n < 0 || (n && !seqs)) return -1;
  int mx = 0;
  for (int i = 0; i < n; ++i) {
    const pa_block_manager::Seq* s = bm->find(seqs[i]);
    if (!s) return -1;
    if ((int)s->table.size() > mx) mx = (int)s->table.size();
  }
  return mx;
}

pa_status pa_bm_block_tables(const pa_block_manager* bm, const int32_t* seqs, int n, int width,
                             int32_t fill, int32_t* tables, int32_t* context_lens) {
  if (!bm || n < 0 || width <= 0 || (n && (!seqs || !tables))) return PA_ERR_INVALID;
  for (int i = 0; i < n; ++i) {
    const pa_block_manager::Seq* s = bm->resident(seqs[i]);
    if (!s || (int64_t)s->table.size() > width || s->len > INT32_MAX) return PA_ERR_INVALID;
  }
  for (int i = 0; i < n; ++i) {
    const pa_block_manager::Seq* s = bm->find(seqs[i]);
    int32_t* row = tables + (int64_t)i * width;
    const size_t k = s->table.size();
    if (k) std::memcpy(row, s->table.data(), k * sizeof(int32_t));
    for (int j = (int)k; j < width; ++j) row[j] = fill;
    if (context_lens) context_lens[i] = (int32_t)s->len;
  }
  return PA_OK;
}

pa_status pa_bm_slot_of(const pa_block_manager* bm, int32_t seq, int64_t pos, int64_t* slot) {
  const pa_block_manager::Seq* s = bm ? bm->resident(seq) : nullptr;
  if (!s || !slot || pos < 0 || pos >= s->len) return PA_ERR_INVALID;
  *slot = (int64_t)s->table[(size_t)(pos / bm->block_size)] * bm->block_size + pos % bm->block_size;
  return PA_OK;
}

// Preemption ("Paged Attention and Memory Efficiency in Production LLM Serving", section
// "Why KV cache memory was the bottleneck": in-flight requests are preempted when the
// cache runs out): the sequence's blocks go back to the pool as on release, after the
// caller has saved their contents; it keeps its id and length and later takes fresh
// blocks for the saved contents.
pa_status pa_bm_swap_out(pa_block_manager* bm, int32_t seq, int32_t* blocks, int* num_blocks) {
  if (!bm || !num_blocks) return PA_ERR_INVALID;
  pa_block_manager::Seq* s = bm->find(seq);
  if (!s || s->swapped || (!s->table.empty() && !blocks)) return PA_ERR_INVALID;
  const size_t n = s->table.size();
  if (n) std::memcpy(blocks, s->table.data(), n * sizeof(int32_t));
  for (int32_t b : s->table) bm->drop(b);
  s->table.clear();
  s->swapped = true;
  *num_blocks = (int)n;
  return PA_OK;
}

pa_status pa_bm_swap_in(pa_block_manager* bm, int32_t seq, int32_t* blocks, int* num_blocks) {
  if (!bm || !num_blocks) return PA_ERR_INVALID;
  pa_block_manager::Seq* s = bm->find(seq);
  if (!s || !s->swapped) return PA_ERR_INVALID;
  const int64_t need = bm->blocks_for(s->len);
  if (need && !blocks) return PA_ERR_INVALID;
  if (need > (int64_t)bm->free.size()) return PA_ERR_NO_BLOCKS;
  s->table.resize((size_t)need);
  for (int64_t i = 0; i < need; ++i) s->table[(size_t)i] = blocks[i] = bm->take();
  s->swapped = false;
  *num_blocks = (int)need;
  return PA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Cascade planning: which sequences of a batch read the same physical blocks at the start
// of their tables ("How PagedAttention borrows OS paging": requests with an identical
// prefix point their block tables at the same physical blocks), grouped into chunks whose
// members' query rows pa_decode_cascade decodes together over the shared prefix.
// ---------------------------------------------------------------------------------------
namespace {

constexpr int kCascadeMaxRows = 64;     // query rows a prefix chunk holds (group x members)

// Rows of one batch: table row i (entries row(i)[0..nblk(i))) and its length.
template <typename RowFn, typename LenFn>
pa_status plan_rows(int n, int block_size, int group, int chunk_width, RowFn row, LenFn len,
                    int32_t* prefix_lens, int32_t* chunk_members, int32_t* chunk_prefix_lens,
                    int* num_chunks, int* width_out) {
  if (n < 0 || block_size <= 0 || group <= 0 || !num_chunks ||
      (n && (!prefix_lens || !chunk_members || !chunk_prefix_lens)))
    return PA_ERR_INVALID;
  const int wmax = std::max(1, kCascadeMaxRows / group);
  if (chunk_width > 0 && (int64_t)group * chunk_width > kCascadeMaxRows) return PA_ERR_UNSUPPORTED;
  *num_chunks = 0;
  // sharing groups: rows with a non-empty context whose first physical block is the same,
  // in order of first appearance, members in batch order
  std::unordered_map<int32_t, int> by_first;
  std::vector<std::vector<int>> groups;
  for (int i = 0; i < n; ++i) {
    prefix_lens[i] = 0;
    if (len(i) <= 0) continue;
    const int32_t b0 = row(i)[0];
    auto it = by_first.find(b0);
    if (it == by_first.end()) {
      by_first.emplace(b0, (int)groups.size());
      groups.push_back({i});
    } else {
      groups[(size_t)it->second].push_back(i);
    }
  }
  // each sharing group's prefix: the leading table entries common to every member,
  // capped at the shortest member (0: the group shares nothing)
  std::vector<int64_t> plens(groups.size(), 0);
  int fit = 0;      // the default width: the widest group's members spread evenly over the
                    // fewest chunks of at most wmax members
  for (size_t gi = 0; gi < groups.size(); ++gi) {
    const std::vector<int>& mem = groups[gi];
    if (mem.size() < 2) continue;
    int64_t minlen = INT64_MAX;
    for (int i : mem) minlen = std::min<int64_t>(minlen, len(i));
    const int64_t nb = (minlen + block_size - 1) / block_size;
    int64_t common = 0;
    const int32_t* r0 = row(mem[0]);
    while (common < nb) {
      bool same = true;
      for (int i : mem) same = same && row(i)[common] == r0[common];
      if (!same) break;
      ++common;
    }
    plens[gi] = std::min<int64_t>(common * block_size, minlen);
    if (plens[gi] == 0) continue;
    const int m = (int)mem.size(), k = (m + wmax - 1) / wmax;
    fit = std::max(fit, (m + k - 1) / k);
  }
  const int width = chunk_width > 0 ? chunk_width : (fit > 0 ? fit : wmax);
  if (width_out) *width_out = width;
  int nc = 0;
  for (size_t gi = 0; gi < groups.size(); ++gi) {
    const std::vector<int>& mem = groups[gi];
    const int64_t plen = plens[gi];
    if (mem.size() < 2 || plen == 0) continue;
    for (size_t k = 0; k < mem.size(); k += (size_t)width) {
      int32_t* out = chunk_members + (int64_t)nc * width;
      for (int j = 0; j < width; ++j) {
        const size_t m = k + (size_t)j;
        out[j] = m < mem.size() ? mem[m] : -1;
        if (m < mem.size()) prefix_lens[mem[m]] = (int32_t)plen;
      }
      chunk_prefix_lens[nc] = (int32_t)plen;
      ++nc;
    }
  }
  *num_chunks = nc;
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_plan_cascade(const int32_t* block_tables, int max_blocks_per_seq,
                          const int32_t* context_lens, int num_seqs, int block_size, int group,
                          int chunk_width, int32_t* prefix_lens, int32_t* chunk_members,
                          int32_t* chunk_prefix_lens, int* num_chunks, int* chunk_width_out) {
  if (block_size <= 0 || (num_seqs > 0 && (!block_tables || !context_lens || max_blocks_per_seq <= 0)))
    return PA_ERR_INVALID;
  for (int i = 0; i < num_seqs; ++i) {     // every table must hold its sequence's blocks
    const int64_t c = context_lens[i];
    if (c < 0 || (c + block_size - 1) / block_size > max_blocks_per_seq) return PA_ERR_INVALID;
  }
  return plan_rows(
      num_seqs, block_size, group, chunk_width,
      [&](int i) { return block_tables + (int64_t)i * max_blocks_per_seq; },
      [&](int i) { return (int64_t)context_lens[i]; }, prefix_lens, chunk_members,
      chunk_prefix_lens, num_chunks, chunk_width_out);
}

pa_status pa_bm_plan_cascade(const pa_block_manager* bm, const int32_t* seqs, int n, int group,
                             int chunk_width, int32_t* prefix_lens, int32_t* chunk_members,
                             int32_t* chunk_prefix_lens, int* num_chunks, int* chunk_width_out) {
  if (!bm || n < 0 || (n && !seqs)) return PA_ERR_INVALID;
  std::vector<const pa_block_manager::Seq*> rows((size_t)n);
  for (int i = 0; i < n; ++i) {
    rows[(size_t)i] = bm->resident(seqs[i]);
    if (!rows[(size_t)i]) return PA_ERR_INVALID;
  }
  return plan_rows(
      n, bm->block_size, group, chunk_width,
      [&](int i) { return rows[(size_t)i]->table.data(); },
      [&](int i) { return rows[(size_t)i]->len; }, prefix_lens, chunk_members, chunk_prefix_lens,
      num_chunks, chunk_width_out);
}

}  // extern "C"
