// Host-side block manager for the paged KV cache (C ABI in include/pkv.h).
//
// What the pages describe ("LLM推理显存优化KV Cache管理3大策略" §2: fixed-size
// blocks, a block table mapping logical to physical blocks, Block.ref_count;
// "大模型推理加速实战：KV Cache内存优化与PagedAttention分页管理方案", PagedAttention
// section: blocks are allocated on demand and reclaimed as soon as a sequence
// ends; vLLM's swap_space lets inactive KV move to CPU memory):
//   * a pool of num_blocks physical blocks of block_size token slots;
//   * per sequence, its block list (the block table) and its length;
//   * reserving the slot of a new token allocates a block when the sequence
//     crosses a block boundary;
//   * fork() makes a child share all of its parent's blocks (ref_count + 1),
//     e.g. sequences that start from a cached prompt prefix;
//   * a token appended to a shared, partially filled last block first gets a
//     private copy of that block (copy-on-write): the manager allocates the
//     new block and returns the (source, destination) pair; the caller copies
//     the rows with pkv_copy_blocks before writing the token;
//   * free() drops a sequence's references and returns blocks that reach zero;
//   * swap_out()/swap_in() move a sequence's blocks between this pool and a
//     second manager's pool (host memory), returning the block pairs to copy.
// Operations are atomic: when the pool cannot supply every block an operation
// needs, nothing changes and PKV_ERR_NO_BLOCKS is returned.  One mutex per
// manager serialises calls.
#include <stdint.h>

#include <mutex>
#include <new>
#include <unordered_map>
#include <vector>

#include "pkv.h"

struct pkv_block_manager {
  int num_blocks;
  int block_size;
  std::vector<int32_t> free_list;  // LIFO stack of free block ids
  std::vector<int32_t> ref;        // references per block
  struct Seq {
    std::vector<int32_t> blocks;
    int64_t len = 0;
  };
  std::unordered_map<int64_t, Seq> seqs;
  std::mutex mu;

  int32_t take() {
    const int32_t b = free_list.back();
    free_list.pop_back();
    ref[b] = 1;
    return b;
  }
  void drop(int32_t b) {
    if (--ref[b] == 0) free_list.push_back(b);
  }
  // blocks a sequence needs to grow by n tokens (including a copy-on-write)
  int64_t needed(const Seq& s, int64_t n) const {
    if (n <= 0) return 0;
    const int64_t bs = block_size;
    const int64_t have = (int64_t)s.blocks.size() * bs;
    int64_t fresh = (s.len + n > have) ? (s.len + n - have + bs - 1) / bs : 0;
    const bool cow = (s.len % bs) != 0 && !s.blocks.empty() && ref[s.blocks.back()] > 1;
    return fresh + (cow ? 1 : 0);
  }
};

extern "C" {

int pkv_bm_create(int num_blocks, int block_size, pkv_block_manager** out) {
  if (!out || num_blocks <= 0 || block_size <= 0) return PKV_ERR_ARG;
  pkv_block_manager* m = new (std::nothrow) pkv_block_manager();
  if (!m) return PKV_ERR_ARG;
  m->num_blocks = num_blocks;
  m->block_size = block_size;
  m->ref.assign(num_blocks, 0);
  m->free_list.reserve(num_blocks);
  for (int b = num_blocks - 1; b >= 0; --b) m->free_list.push_back(b);  // block 0 first
  *out = m;
  return PKV_OK;
}

void pkv_bm_destroy(pkv_block_manager* m) { delete m; }

int pkv_bm_num_free(pkv_block_manager* m) {
  if (!m) return PKV_ERR_ARG;
  std::lock_guard<std::mutex> lock(m->mu);
  return (int)m->free_list.size();
}

int pkv_bm_ref_count(pkv_block_manager* m, int32_t block) {
  if (!m || block < 0 || block >= m->num_blocks) return PKV_ERR_ARG;
  std::lock_guard<std::mutex> lock(m->mu);
  return m->ref[block];
}

int pkv_bm_add_sequence(pkv_block_manager* m, int64_t seq_id) {
  if (!m) return PKV_ERR_ARG;
  std::lock_guard<std::mutex> lock(m->mu);
  if (m->seqs.count(seq_id)) return PKV_ERR_ARG;
  m->seqs.emplace(seq_id, pkv_block_manager::Seq());
  return PKV_OK;
}

int pkv_bm_fork(pkv_block_manager* m, int64_t parent, int64_t child) {
  if (!m) return PKV_ERR_ARG;
  std::lock_guard<std::mutex> lock(m->mu);
  auto it = m->seqs.find(parent);
  if (it == m->seqs.end() || m->seqs.count(child)) return PKV_ERR_ARG;
  pkv_block_manager::Seq s = it->second;
  for (int32_t b : s.blocks) ++m->ref[b];
  m->seqs.emplace(child, std::move(s));
  return PKV_OK;
}

int pkv_bm_blocks_needed(pkv_block_manager* m, int64_t seq_id, int num_tokens) {
  if (!m || num_tokens < 0) return PKV_ERR_ARG;
  std::lock_guard<std::mutex> lock(m->mu);
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PKV_ERR_ARG;
  return (int)m->needed(it->second, num_tokens);
}

int pkv_bm_reserve(pkv_block_manager* m, int64_t seq_id, int num_tokens, int64_t* slots_out,
                   int32_t* cow_pairs_out, int* num_cow) {
  if (!m || num_tokens < 0 || (num_tokens > 0 && !slots_out) || !num_cow) return PKV_ERR_ARG;
  std::lock_guard<std::mutex> lock(m->mu);
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PKV_ERR_ARG;
  pkv_block_manager::Seq& s = it->second;
  *num_cow = 0;
  if (num_tokens == 0) return PKV_OK;
  if ((int64_t)m->free_list.size() < m->needed(s, num_tokens)) return PKV_ERR_NO_BLOCKS;
  const int bs = m->block_size;
  if (s.len % bs != 0 && m->ref[s.blocks.back()] > 1) {
    if (!cow_pairs_out) return PKV_ERR_ARG;
    const int32_t old = s.blocks.back();
    const int32_t fresh = m->take();
    m->drop(old);
    s.blocks.back() = fresh;
    cow_pairs_out[0] = old;
    cow_pairs_out[1] = fresh;
    *num_cow = 1;
  }
  for (int i = 0; i < num_tokens; ++i) {
    if (s.len == (int64_t)s.blocks.size() * bs) s.blocks.push_back(m->take());
    slots_out[i] = (int64_t)s.blocks.back() * bs + s.len % bs;
    ++s.len;
  }
  return PKV_OK;
}

int pkv_bm_free(pkv_block_manager* m, int64_t seq_id) {
  if (!m) return PKV_ERR_ARG;
  std::lock_guard<std::mutex> lock(m->mu);
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PKV_ERR_ARG;
  for (int32_t b : it->second.blocks) m->drop(b);
  m->seqs.erase(it);
  return PKV_OK;
}

int pkv_bm_seq_len(pkv_block_manager* m, int64_t seq_id, int64_t* len_out, int* num_blocks_out) {
  if (!m || !len_out) return PKV_ERR_ARG;
  std::lock_guard<std::mutex> lock(m->mu);
  auto it = m->seqs.find(seq_id);
  if (it == m->seqs.end()) return PKV_ERR_ARG;
  *len_out = it->second.len;
  if (num_blocks_out) *num_blocks_out = (int)it->second.blocks.size();
  return PKV_OK;
}

int pkv_bm_block_tables(pkv_block_manager* m, const int64_t* seq_ids, int num_seqs,
                        int max_blocks_per_seq, int32_t* tables_out, int32_t* lens_out) {
  if (!m || num_seqs < 0 || max_blocks_per_seq <= 0 || (num_seqs > 0 && (!seq_ids || !tables_out)))
    return PKV_ERR_ARG;
  std::lock_guard<std::mutex> lock(m->mu);
  for (int i = 0; i < num_seqs; ++i) {
    auto it = m->seqs.find(seq_ids[i]);
    if (it == m->seqs.end()) return PKV_ERR_ARG;
    if ((int)it->second.blocks.size() > max_blocks_per_seq) return PKV_ERR_SHAPE;
  }
  for (int i = 0; i < num_seqs; ++i) {
    const auto& s = m->seqs.find(seq_ids[i])->second;
    int32_t* row = tables_out + (size_t)i * max_blocks_per_seq;
    for (int j = 0; j < max_blocks_per_seq; ++j)
      row[j] = j < (int)s.blocks.size() ? s.blocks[j] : -1;
    if (lens_out) lens_out[i] = (int32_t)s.len;
  }
  return PKV_OK;
}

// Moves sequence seq_id from `from` to `to`: its blocks are released in `from`
// and fresh blocks are taken in `to`; pairs_out[2*i], pairs_out[2*i+1] =
// (block in from, block in to) for every block, in table order.
static int move_sequence(pkv_block_manager* from, pkv_block_manager* to, int64_t seq_id,
                         int32_t* pairs_out, int capacity, int* num_pairs) {
  if (!from || !to || from == to || !num_pairs || from->block_size != to->block_size)
    return PKV_ERR_ARG;
  std::scoped_lock lock(from->mu, to->mu);
  auto it = from->seqs.find(seq_id);
  if (it == from->seqs.end() || to->seqs.count(seq_id)) return PKV_ERR_ARG;
  const auto& src = it->second;
  const int n = (int)src.blocks.size();
  if (n > capacity || (n > 0 && !pairs_out)) return PKV_ERR_ARG;
  if ((int)to->free_list.size() < n) return PKV_ERR_NO_BLOCKS;
  pkv_block_manager::Seq dst;
  dst.len = src.len;
  for (int i = 0; i < n; ++i) {
    const int32_t b = to->take();
    dst.blocks.push_back(b);
    pairs_out[2 * i] = src.blocks[i];
    pairs_out[2 * i + 1] = b;
  }
  for (int32_t b : src.blocks) from->drop(b);
  from->seqs.erase(it);
  to->seqs.emplace(seq_id, std::move(dst));
  *num_pairs = n;
  return PKV_OK;
}

int pkv_bm_swap_out(pkv_block_manager* device, pkv_block_manager* host, int64_t seq_id,
                    int32_t* pairs_out, int capacity, int* num_pairs) {
  return move_sequence(device, host, seq_id, pairs_out, capacity, num_pairs);
}

int pkv_bm_swap_in(pkv_block_manager* host, pkv_block_manager* device, int64_t seq_id,
                   int32_t* pairs_out, int capacity, int* num_pairs) {
  return move_sequence(host, device, seq_id, pairs_out, capacity, num_pairs);
}

}  // extern "C"
