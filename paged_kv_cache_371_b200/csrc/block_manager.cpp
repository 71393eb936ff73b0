// Host-side KV block manager: fixed-capacity physical block pool with
// reference counts, a LIFO free list, block-level copy-on-write and prefix
// sharing.
//
// Follows "LLM 推理优化：KV Cache、PagedAttention 与量化" §2.3:
//   (1) blocks are taken on demand when a token is written, returned to the
//       pool when a sequence ends and reused first; a full pool is the
//       preemption trigger (reported here as KV_ERR_OOM);
//   (2) a fork copies only the block table; the first write into a shared
//       block copies that block and repoints the writer's table;
//   (3) sharing a prefix means pointing several tables at the same blocks
//       (done with block_fork on the prefix's ids).
// Pool sizing follows the KV memory formula of "大模型推理加速：从 KV Cache 到
// 投机采样的工程实践" §"KV Cache的内存挑战".
#include <cstdint>
#include <cstring>
#include <new>
#include <string>
#include <unordered_map>
#include <vector>

#include "../../include/paged_kv.h"
#include "kv_pool_impl.h"
#include "kv_status.h"

namespace {

bool valid_config(const kv_pool_config* c)
{
    return c && c->num_blocks > 0 && (c->block_size == 8 || c->block_size == 16) &&
           c->num_kv_heads > 0 && c->head_dim > 0 && c->num_layers > 0 && c->dtype_bytes > 0;
}

int alloc_ids(kv_pool* p, int32_t n, int32_t* out)
{
    if (n < 0) return kv_fail(KV_ERR_INVALID, "block_alloc: negative count");
    if ((size_t)n > p->free_stack.size()) return kv_fail(KV_ERR_OOM, "block_alloc: pool exhausted");
    for (int32_t i = 0; i < n; ++i) {
        int32_t id = p->free_stack.back();
        p->free_stack.pop_back();
        p->refcount[id] = 1;
        out[i] = id;
    }
    return KV_OK;
}

}  // namespace

extern "C" {

int kv_version(void) { return 1; }

int kv_pool_bytes(const kv_pool_config* cfg, uint64_t* per_layer_bytes, uint64_t* total_bytes)
{
    if (!valid_config(cfg)) return kv_fail(KV_ERR_INVALID, "kv_pool_bytes: bad config");
    // 2 (K and V) x heads x head_dim x tokens x dtype, tokens = pool capacity.
    uint64_t per = 2ull * (uint64_t)cfg->num_kv_heads * (uint64_t)cfg->head_dim *
                   (uint64_t)cfg->num_blocks * (uint64_t)cfg->block_size *
                   (uint64_t)cfg->dtype_bytes;
    if (per_layer_bytes) *per_layer_bytes = per;
    if (total_bytes) *total_bytes = per * (uint64_t)cfg->num_layers;
    return KV_OK;
}

int kv_pool_create(const kv_pool_config* cfg, const int32_t* order, kv_pool** out)
{
    if (!out) return kv_fail(KV_ERR_INVALID, "kv_pool_create: null output");
    *out = nullptr;
    if (!valid_config(cfg)) return kv_fail(KV_ERR_INVALID, "kv_pool_create: bad config");
    const int32_t n = cfg->num_blocks;
    if (order) {
        std::vector<char> seen(n, 0);
        for (int32_t i = 0; i < n; ++i) {
            if (order[i] < 0 || order[i] >= n || seen[order[i]])
                return kv_fail(KV_ERR_INVALID, "kv_pool_create: order is not a permutation");
            seen[order[i]] = 1;
        }
    }
    kv_pool* p = new (std::nothrow) kv_pool;
    if (!p) return kv_fail(KV_ERR_OOM, "kv_pool_create: out of host memory");
    p->cfg = *cfg;
    p->refcount.assign(n, 0);
    p->free_stack.resize(n);
    // The first pop must return order[0] (or id 0): fill the stack reversed.
    for (int32_t i = 0; i < n; ++i) p->free_stack[n - 1 - i] = order ? order[i] : i;
    *out = p;
    return KV_OK;
}

int kv_pool_destroy(kv_pool* pool)
{
    delete pool;
    return KV_OK;
}

int kv_pool_num_free(const kv_pool* pool, int32_t* n_out)
{
    if (!pool || !n_out) return kv_fail(KV_ERR_INVALID, "kv_pool_num_free: null argument");
    *n_out = (int32_t)pool->free_stack.size();
    return KV_OK;
}

int block_alloc(kv_pool* pool, int32_t n, int32_t* ids_out)
{
    if (!pool || (n > 0 && !ids_out)) return kv_fail(KV_ERR_INVALID, "block_alloc: null argument");
    return alloc_ids(pool, n, ids_out);
}

int block_free(kv_pool* pool, const int32_t* ids, int32_t n)
{
    if (!pool || n < 0 || (n > 0 && !ids)) return kv_fail(KV_ERR_INVALID, "block_free: bad argument");
    std::unordered_map<int32_t, int32_t> need;
    for (int32_t i = 0; i < n; ++i) {
        if (ids[i] < 0 || ids[i] >= pool->cfg.num_blocks)
            return kv_fail(KV_ERR_INVALID, "block_free: id out of range");
        ++need[ids[i]];
    }
    for (const auto& kv : need)
        if (pool->refcount[kv.first] < kv.second)
            return kv_fail(KV_ERR_DOUBLE_FREE, "block_free: reference count would go below zero");
    for (int32_t i = 0; i < n; ++i) {
        if (--pool->refcount[ids[i]] == 0) pool->free_stack.push_back(ids[i]);
        kv_cache_recheck(pool, ids[i]);
    }
    return KV_OK;
}

int block_fork(kv_pool* pool, const int32_t* ids, int32_t n)
{
    if (!pool || n < 0 || (n > 0 && !ids)) return kv_fail(KV_ERR_INVALID, "block_fork: bad argument");
    for (int32_t i = 0; i < n; ++i)
        if (ids[i] < 0 || ids[i] >= pool->cfg.num_blocks || pool->refcount[ids[i]] == 0)
            return kv_fail(KV_ERR_INVALID, "block_fork: id is not a live block");
    for (int32_t i = 0; i < n; ++i) {
        ++pool->refcount[ids[i]];
        kv_cache_recheck(pool, ids[i]);
    }
    return KV_OK;
}

int block_refcount(const kv_pool* pool, int32_t id, int32_t* rc_out)
{
    if (!pool || !rc_out || id < 0 || id >= pool->cfg.num_blocks)
        return kv_fail(KV_ERR_INVALID, "block_refcount: bad argument");
    *rc_out = pool->refcount[id];
    return KV_OK;
}

int kv_seq_reserve_slot(kv_pool* pool, int32_t* table, int32_t table_capacity, int32_t* n_blocks,
                        int32_t ctx_len, int64_t* slot_out, int32_t* cow_src_out,
                        int32_t* cow_dst_out)
{
    if (!pool || !table || !n_blocks || !slot_out || !cow_src_out || !cow_dst_out || ctx_len < 0)
        return kv_fail(KV_ERR_INVALID, "kv_seq_reserve_slot: bad argument");
    const int32_t bs = pool->cfg.block_size;
    const int32_t nb = *n_blocks;
    if (nb != (ctx_len + bs - 1) / bs)
        return kv_fail(KV_ERR_INVALID, "kv_seq_reserve_slot: n_blocks does not match ctx_len");
    *cow_src_out = -1;
    *cow_dst_out = -1;
    const int32_t off = ctx_len % bs;
    if (off == 0) {
        if (nb >= table_capacity) return kv_fail(KV_ERR_INVALID, "kv_seq_reserve_slot: table full");
        int32_t id = -1;
        int rc = alloc_ids(pool, 1, &id);
        if (rc != KV_OK) return rc;
        table[nb] = id;
        *n_blocks = nb + 1;
        *slot_out = (int64_t)id * bs;
        return KV_OK;
    }
    const int32_t last = table[nb - 1];
    if (last < 0 || last >= pool->cfg.num_blocks || pool->refcount[last] == 0)
        return kv_fail(KV_ERR_INVALID, "kv_seq_reserve_slot: last block is not live");
    if (pool->refcount[last] > 1) {
        int32_t id = -1;
        int rc = alloc_ids(pool, 1, &id);
        if (rc != KV_OK) return rc;
        --pool->refcount[last];
        kv_cache_recheck(pool, last);
        table[nb - 1] = id;
        *cow_src_out = last;
        *cow_dst_out = id;
        *slot_out = (int64_t)id * bs + off;
        return KV_OK;
    }
    *slot_out = (int64_t)last * bs + off;
    return KV_OK;
}

int kv_batch_reserve_slots(kv_pool* pool, int32_t B, int32_t* tables, int32_t table_capacity,
                           int32_t* n_blocks, const int32_t* ctx_lens, int64_t* slots_out,
                           int32_t* cow_pairs_out, int32_t* n_cow_out, int32_t* n_done_out)
{
    if (!pool || B < 0 || !n_cow_out || !n_done_out ||
        (B > 0 && (!tables || !n_blocks || !ctx_lens || !slots_out || !cow_pairs_out)))
        return kv_fail(KV_ERR_INVALID, "kv_batch_reserve_slots: bad argument");
    *n_cow_out = 0;
    *n_done_out = 0;
    for (int32_t s = 0; s < B; ++s) {
        int32_t src, dst;
        int rc = kv_seq_reserve_slot(pool, tables + (size_t)s * table_capacity, table_capacity,
                                     n_blocks + s, ctx_lens[s], slots_out + s, &src, &dst);
        if (rc != KV_OK) return rc;
        if (src >= 0) {
            cow_pairs_out[2 * *n_cow_out] = src;
            cow_pairs_out[2 * *n_cow_out + 1] = dst;
            ++*n_cow_out;
        }
        *n_done_out = s + 1;
    }
    return KV_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Beam-search step ("LLM 推理优化：KV Cache、PagedAttention 与量化" §2.3 (2): a
// fork copies only the block table; blocks stay shared until a beam writes
// into one, then copy-on-write).  New beam i continues old beam parents[i];
// references are added for every new table before the old tables' are
// dropped (old beams released in order), so surviving blocks are never freed.
extern "C" int kv_beam_reorder(kv_pool* pool, const int32_t* tables, const int32_t* n_blocks,
                               int32_t n_beams, int32_t table_capacity, const int32_t* parents,
                               int32_t n_new, int32_t* new_tables, int32_t* new_n_blocks)
{
    if (!pool || n_beams < 0 || n_new < 0 || table_capacity < 1 ||
        (n_beams > 0 && (!tables || !n_blocks)) || (n_new > 0 && (!parents || !new_tables || !new_n_blocks)))
        return kv_fail(KV_ERR_INVALID, "kv_beam_reorder: bad argument");
    const size_t cap = static_cast<size_t>(table_capacity);
    if (n_new > 0 && n_beams > 0 && new_tables < tables + static_cast<size_t>(n_beams) * cap &&
        tables < new_tables + static_cast<size_t>(n_new) * cap)
        return kv_fail(KV_ERR_INVALID, "kv_beam_reorder: new_tables overlaps tables");
    for (int32_t i = 0; i < n_new; ++i)
        if (parents[i] < 0 || parents[i] >= n_beams)
            return kv_fail(KV_ERR_INVALID, "kv_beam_reorder: parent out of range");
    for (int32_t b = 0; b < n_beams; ++b) {
        if (n_blocks[b] < 0 || n_blocks[b] > table_capacity)
            return kv_fail(KV_ERR_INVALID, "kv_beam_reorder: bad block count");
        for (int32_t k = 0; k < n_blocks[b]; ++k) {
            const int32_t id = tables[b * cap + k];
            if (id < 0 || id >= pool->cfg.num_blocks || pool->refcount[id] == 0)
                return kv_fail(KV_ERR_INVALID, "kv_beam_reorder: table holds a block that is not live");
        }
    }
    for (int32_t i = 0; i < n_new; ++i) {
        const int32_t p = parents[i];
        const int32_t nb = n_blocks[p];
        for (int32_t k = 0; k < table_capacity; ++k) {
            const int32_t id = k < nb ? tables[p * cap + k] : -1;
            new_tables[i * cap + k] = id;
            if (id >= 0) {
                ++pool->refcount[id];
                kv_cache_recheck(pool, id);
            }
        }
        new_n_blocks[i] = nb;
    }
    for (int32_t b = 0; b < n_beams; ++b)
        for (int32_t k = 0; k < n_blocks[b]; ++k) {
            const int32_t id = tables[b * cap + k];
            if (--pool->refcount[id] == 0) pool->free_stack.push_back(id);
            kv_cache_recheck(pool, id);
        }
    return KV_OK;
}
