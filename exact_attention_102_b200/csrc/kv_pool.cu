// kv_pool.cu — block pool of a paged KV cache (host) and the copy-on-write
// block copy (device).
//
// "FlashAttention系列优化" (johneyzheng.top), section PagedAttention: a
// sequence's KV cache is cut into fixed-size blocks, a block table maps its
// logical blocks to physical ones, physical blocks are allocated on demand as
// tokens arrive, and sequences of parallel sampling share physical blocks;
// sharing is kept safe by a reference count per block and copy-on-write.
//
// Policy (the pages give none; the plainest one, fixed here and in the test
// model): the free block handed out is the lowest-numbered one; an append to a
// sequence whose last block is partially filled and shared first copies that
// block to a new one (the pair is returned for the device copy), then takes new
// blocks in order; every operation is all-or-nothing.
#include <new>
#include <set>
#include <vector>

#include "fa.h"
#include "prim.cuh"

struct fa_kv_pool {
  int num_blocks, block_size, max_seqs, max_blocks;
  std::vector<int> ref;                     // references per physical block
  std::set<int> free_blocks;                // reference count 0, lowest first
  std::vector<int> len;                     // tokens per sequence, -1 when unused
  std::vector<std::vector<int>> table;      // physical block per logical block

  int take() {
    const int b = *free_blocks.begin();
    free_blocks.erase(free_blocks.begin());
    ref[b] = 1;
    return b;
  }
  void drop(int b) {
    if (--ref[b] == 0) free_blocks.insert(b);
  }
  bool live(int s) const { return s >= 0 && s < max_seqs && len[s] >= 0; }
};

namespace fa {
namespace {

// Copy block src[i] to dst[i] of both caches; one CTA row per pair, 16-byte
// vectors. Out-of-range indices are recorded and skipped.
__global__ void __launch_bounds__(256) kv_copy_kernel(uint4* k, uint4* v, int num_blocks,
                                                      const int* src, const int* dst, int n,
                                                      long long vec_per_block, uint32_t* err) {
  const int i = blockIdx.y;
  if (i >= n) return;
  const int s = src[i], d = dst[i];
  if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicCAS(err, 0u, kErrBadIndex + 3);
    return;
  }
  for (long long j = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
       j < vec_per_block; j += static_cast<long long>(gridDim.x) * blockDim.x) {
    k[d * vec_per_block + j] = k[s * vec_per_block + j];
    v[d * vec_per_block + j] = v[s * vec_per_block + j];
  }
}

}  // namespace

uint32_t* error_word_for_kv();   // api.cu

}  // namespace fa

extern "C" {

fa_status fa_kv_pool_create(int num_blocks, int block_size, int max_seqs, int max_blocks_per_seq,
                            fa_kv_pool** out) {
  if (out == nullptr || num_blocks < 1 || block_size < 1 || max_seqs < 1 ||
      max_blocks_per_seq < 1)
    return FA_ERR_INVALID_ARG;
  fa_kv_pool* p = new (std::nothrow) fa_kv_pool;
  if (p == nullptr) return FA_ERR_WORKSPACE;
  p->num_blocks = num_blocks;
  p->block_size = block_size;
  p->max_seqs = max_seqs;
  p->max_blocks = max_blocks_per_seq;
  p->ref.assign(num_blocks, 0);
  for (int b = 0; b < num_blocks; ++b) p->free_blocks.insert(p->free_blocks.end(), b);
  p->len.assign(max_seqs, -1);
  p->table.assign(max_seqs, {});
  *out = p;
  return FA_OK;
}

void fa_kv_pool_destroy(fa_kv_pool* pool) { delete pool; }

fa_status fa_kv_seq_add(fa_kv_pool* p, int seq) {
  if (p == nullptr || seq < 0 || seq >= p->max_seqs || p->len[seq] >= 0) return FA_ERR_INVALID_ARG;
  p->len[seq] = 0;
  p->table[seq].clear();
  return FA_OK;
}

fa_status fa_kv_seq_fork(fa_kv_pool* p, int parent, int child) {
  if (p == nullptr || !p->live(parent) || child < 0 || child >= p->max_seqs || p->len[child] >= 0)
    return FA_ERR_INVALID_ARG;
  for (int b : p->table[parent]) ++p->ref[b];
  p->table[child] = p->table[parent];
  p->len[child] = p->len[parent];
  return FA_OK;
}

fa_status fa_kv_seq_free(fa_kv_pool* p, int seq) {
  if (p == nullptr || !p->live(seq)) return FA_ERR_INVALID_ARG;
  for (int b : p->table[seq]) p->drop(b);
  p->table[seq].clear();
  p->len[seq] = -1;
  return FA_OK;
}

fa_status fa_kv_seq_append(fa_kv_pool* p, int seq, int n_tokens, int* copy_src, int* copy_dst,
                           int* n_copies) {
  if (p == nullptr || !p->live(seq) || n_tokens < 0 || copy_src == nullptr ||
      copy_dst == nullptr || n_copies == nullptr)
    return FA_ERR_INVALID_ARG;
  *n_copies = 0;
  std::vector<int>& blocks = p->table[seq];
  const long long len = p->len[seq];
  const long long new_len = len + n_tokens;
  const long long need = (new_len + p->block_size - 1) / p->block_size;
  if (new_len > 0x7fffffffll || need > p->max_blocks) return FA_ERR_INVALID_ARG;
  const bool cow = n_tokens > 0 && len % p->block_size != 0 && p->ref[blocks.back()] > 1;
  const long long take = need - static_cast<long long>(blocks.size()) + (cow ? 1 : 0);
  if (take > static_cast<long long>(p->free_blocks.size())) return FA_ERR_WORKSPACE;
  if (cow) {
    const int old = blocks.back();
    const int fresh = p->take();
    p->drop(old);
    blocks.back() = fresh;
    copy_src[0] = old;
    copy_dst[0] = fresh;
    *n_copies = 1;
  }
  while (static_cast<long long>(blocks.size()) < need) blocks.push_back(p->take());
  p->len[seq] = static_cast<int>(new_len);
  return FA_OK;
}

int fa_kv_num_free(const fa_kv_pool* p) {
  return p == nullptr ? -1 : static_cast<int>(p->free_blocks.size());
}

int fa_kv_refcount(const fa_kv_pool* p, int block) {
  return (p == nullptr || block < 0 || block >= p->num_blocks) ? -1 : p->ref[block];
}

int fa_kv_seq_len(const fa_kv_pool* p, int seq) {
  return (p == nullptr || seq < 0 || seq >= p->max_seqs) ? -1 : p->len[seq];
}

fa_status fa_kv_block_table(const fa_kv_pool* p, const int* seqs, int n, int* table,
                            int max_blocks_per_seq, int* lens) {
  if (p == nullptr || seqs == nullptr || table == nullptr || lens == nullptr || n < 0 ||
      max_blocks_per_seq < 1)
    return FA_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (!p->live(seqs[i]) ||
        static_cast<int>(p->table[seqs[i]].size()) > max_blocks_per_seq)
      return FA_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    const std::vector<int>& t = p->table[seqs[i]];
    int* row = table + static_cast<long long>(i) * max_blocks_per_seq;
    for (int j = 0; j < max_blocks_per_seq; ++j) row[j] = j < static_cast<int>(t.size()) ? t[j] : 0;
    lens[i] = p->len[seqs[i]];
  }
  return FA_OK;
}

fa_status fa_kv_copy_blocks(void* k_cache, void* v_cache, int num_blocks, const int* src,
                            const int* dst, int n, long long block_bytes, void* stream) {
  if (k_cache == nullptr || v_cache == nullptr || src == nullptr || dst == nullptr || n < 0 ||
      num_blocks < 1 || block_bytes < 16 || block_bytes % 16 != 0 ||
      (reinterpret_cast<uintptr_t>(k_cache) & 15u) || (reinterpret_cast<uintptr_t>(v_cache) & 15u))
    return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (n > 65535) return FA_ERR_UNSUPPORTED;
  uint32_t* err = fa::error_word_for_kv();
  if (err == nullptr) return FA_ERR_LAUNCH;
  const long long vec = block_bytes / 16;
  const long long want = (vec + 255) / 256;
  const dim3 grid(static_cast<unsigned>(want < 64 ? want : 64), static_cast<unsigned>(n));
  fa::kv_copy_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), num_blocks, src, dst, n, vec,
      err);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

}  // extern "C"
