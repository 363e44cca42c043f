// Host block allocator of the paged KV cache.
//
// "From FP8 KV cache to INT4 weight-only" (Core concepts 2, PagedAttention):
// the KV cache is a pool of fixed-size blocks, and each request holds only the
// blocks it needs, so requests of any length share one pool without
// fragmentation or over-allocation. "KV Cache compression" (6.2): with 8-bit
// K/V the same bytes hold twice the tokens per block.
//
// The pool hands out block ids only. Its byte counts follow the closed form of
// "KV Cache compression" section 1 (2 x layers x kv_heads x head_dim x tokens x
// bytes) for num_blocks x block_size tokens, with the per-token BF16 scales
// counted separately.

#include <algorithm>
#include <new>
#include <vector>

#include "kvq_internal.h"

struct kvq_pool {
  kvq_dims dims;
  kvq_fmt fmt;
  int32_t n_layers;
  std::vector<int32_t> free_ids;   // stack; back() is handed out next
  std::vector<uint8_t> in_use;     // per block
};

namespace kvq {

int check_dims(const kvq_dims* d) {
  if (!d) return KVQ_ERR_ARG;
  if (d->num_blocks <= 0 || d->n_kv_heads <= 0 || d->n_q_heads <= 0 ||
      d->max_blocks_per_seq <= 0 || d->head_dim <= 0 || d->block_size <= 0)
    return KVQ_ERR_ARG;
  if (d->n_q_heads % d->n_kv_heads != 0) return KVQ_ERR_ARG;
  const int g = d->n_q_heads / d->n_kv_heads;
  if (d->block_size != kBlockSize) return KVQ_ERR_UNSUPPORTED;
  if (d->head_dim != 64 && d->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
  if (g != 1 && g != 2 && g != 4 && g != 8) return KVQ_ERR_UNSUPPORTED;
  return KVQ_OK;
}

}  // namespace kvq

extern "C" {

int kvq_cache_bytes(const kvq_dims* dims, kvq_fmt fmt, size_t* cache_bytes, size_t* meta_bytes) {
  if (!(kvq::fmt_valid(fmt) || kvq::fmt_kivi(fmt)) || !cache_bytes || !meta_bytes) return KVQ_ERR_ARG;
  const int rc = kvq::check_dims(dims);
  if (rc != KVQ_OK) return rc;
  const size_t rows = size_t(dims->num_blocks) * dims->n_kv_heads * dims->block_size;
  if (kvq::fmt_kivi(fmt)) {
    // b-bit codes; 16 BF16 (s, z) pairs per (block, KV head): a token's for V,
    // D/8 channels' of the block's group for K (the same array size)
    *cache_bytes = rows * dims->head_dim * kvq::kivi_bits(fmt) / 8;
    *meta_bytes = rows * 2 * 2;
    return KVQ_OK;
  }
  *cache_bytes = rows * dims->head_dim * kvq::elem_bytes(fmt);
  if (fmt == KVQ_INT8_CHANNEL)
    *meta_bytes = size_t(dims->n_kv_heads) * dims->head_dim * 2;
  else if (fmt == KVQ_INT8_TENSOR)
    *meta_bytes = 16;                 // one BF16 value, padded to the 16-byte alignment
  else
    *meta_bytes = rows * kvq::meta_values(fmt) * 2;
  return KVQ_OK;
}

int kvq_pool_create(const kvq_dims* dims, kvq_fmt fmt, int32_t n_layers, kvq_pool** out) {
  if (!out || !(kvq::fmt_valid(fmt) || kvq::fmt_kivi(fmt)) || n_layers <= 0) return KVQ_ERR_ARG;
  const int rc = kvq::check_dims(dims);
  if (rc != KVQ_OK) return rc;
  kvq_pool* p = new (std::nothrow) kvq_pool;
  if (!p) return KVQ_ERR_ARG;
  p->dims = *dims;
  p->fmt = fmt;
  p->n_layers = n_layers;
  p->free_ids.resize(dims->num_blocks);
  for (int32_t i = 0; i < dims->num_blocks; ++i) p->free_ids[i] = dims->num_blocks - 1 - i;
  p->in_use.assign(dims->num_blocks, 0);
  *out = p;
  return KVQ_OK;
}

void kvq_pool_destroy(kvq_pool* pool) { delete pool; }

int kvq_pool_bytes(const kvq_pool* pool, size_t* element_bytes, size_t* meta_bytes) {
  if (!pool || !element_bytes || !meta_bytes) return KVQ_ERR_ARG;
  size_t cache = 0, meta = 0;
  const int rc = kvq_cache_bytes(&pool->dims, pool->fmt, &cache, &meta);
  if (rc != KVQ_OK) return rc;
  // K and V, every layer
  *element_bytes = 2 * size_t(pool->n_layers) * cache;
  *meta_bytes = 2 * size_t(pool->n_layers) * meta;
  return KVQ_OK;
}

int kvq_pool_num_free(const kvq_pool* pool, int32_t* n_free) {
  if (!pool || !n_free) return KVQ_ERR_ARG;
  *n_free = int32_t(pool->free_ids.size());
  return KVQ_OK;
}

int kvq_pool_alloc(kvq_pool* pool, int32_t n, int32_t* block_ids) {
  if (!pool || n < 0 || (n > 0 && !block_ids)) return KVQ_ERR_ARG;
  if (size_t(n) > pool->free_ids.size()) return KVQ_ERR_POOL_EXHAUSTED;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t id = pool->free_ids.back();
    pool->free_ids.pop_back();
    pool->in_use[id] = 1;
    block_ids[i] = id;
  }
  return KVQ_OK;
}

int kvq_pool_free(kvq_pool* pool, int32_t n, const int32_t* block_ids) {
  if (!pool || n < 0 || (n > 0 && !block_ids)) return KVQ_ERR_ARG;
  // validate everything before changing anything
  std::vector<int32_t> ids(block_ids, block_ids + n);
  std::sort(ids.begin(), ids.end());
  for (int32_t i = 0; i < n; ++i) {
    if (ids[i] < 0 || ids[i] >= pool->dims.num_blocks) return KVQ_ERR_ARG;
    if (i > 0 && ids[i] == ids[i - 1]) return KVQ_ERR_ARG;
    if (!pool->in_use[ids[i]]) return KVQ_ERR_ARG;
  }
  for (int32_t i = 0; i < n; ++i) {
    pool->in_use[block_ids[i]] = 0;
    pool->free_ids.push_back(block_ids[i]);
  }
  return KVQ_OK;
}

int kvq_pool_extend_seq(kvq_pool* pool, int32_t* row, int32_t cur_len, int32_t n_new,
                        int64_t* slots) {
  if (!pool || !row || cur_len < 0 || n_new < 0 || (n_new > 0 && !slots)) return KVQ_ERR_ARG;
  const int32_t bs = pool->dims.block_size;
  const int64_t new_len = int64_t(cur_len) + n_new;
  const int64_t have = (int64_t(cur_len) + bs - 1) / bs;
  const int64_t need = (new_len + bs - 1) / bs;
  if (need > pool->dims.max_blocks_per_seq) return KVQ_ERR_ARG;
  for (int64_t i = 0; i < have; ++i)
    if (row[i] < 0 || row[i] >= pool->dims.num_blocks || !pool->in_use[row[i]]) return KVQ_ERR_ARG;
  const int32_t extra = int32_t(need - have);
  if (size_t(extra) > pool->free_ids.size()) return KVQ_ERR_POOL_EXHAUSTED;
  if (extra > 0) {
    const int rc = kvq_pool_alloc(pool, extra, row + have);
    if (rc != KVQ_OK) return rc;
  }
  for (int32_t i = 0; i < n_new; ++i) {
    const int64_t p = int64_t(cur_len) + i;
    slots[i] = int64_t(row[p / bs]) * bs + p % bs;
  }
  return KVQ_OK;
}

}  // extern "C"
