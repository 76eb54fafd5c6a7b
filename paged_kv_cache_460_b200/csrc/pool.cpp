// Host side of the paged KV pool: descriptor, free list, slot mapping, sizes.
//
// "为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427) s3.4: the KV cache is cut
// into fixed pages of 16 or 32 tokens; a request takes pages from the free list and
// returns them when it ends, so requests' pages interleave in one preallocated pool
// (s5.3: a preallocated pool instead of growing the cache by concatenation).
//
// No CUDA call is made in this file: the pool only describes caller-owned device
// memory, so everything here runs (and is tested) without a GPU.
#include <cstdint>
#include <vector>

#include "pagedkv.h"
#include "pkv_internal.h"

extern "C" const char* pkv_status_string(int status)
{
    switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_INVALID_ARG: return "invalid argument";
    case PKV_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case PKV_ERR_CUDA: return "CUDA error";
    case PKV_ERR_NO_SPACE: return "no space (free list or workspace too small)";
    default: return "unknown status";
    }
}

namespace {

int make_pool(int num_layers, int num_pages, int page_size, int kv_heads, int head_dim, int dtype, int storage,
              void* k_base, void* v_base, void* k_scales, void* v_scales, pkv_pool** out)
{
    if (!out) return PKV_ERR_INVALID_ARG;
    *out = nullptr;
    if (num_layers <= 0 || num_pages <= 0 || kv_heads <= 0 || !k_base || !v_base) return PKV_ERR_INVALID_ARG;
    if (storage == PKV_I8 && (!k_scales || !v_scales)) return PKV_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(k_base) | reinterpret_cast<uintptr_t>(v_base) |
         reinterpret_cast<uintptr_t>(k_scales) | reinterpret_cast<uintptr_t>(v_scales)) & 15u)
        return PKV_ERR_INVALID_ARG;
    if (page_size != 16 && page_size != 32) return PKV_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
    // the kernels index the 16-row blocks of a layer's (page, kv head) chunks with 32-bit ints
    if ((int64_t)num_pages * kv_heads * (page_size / 16) > INT32_MAX) return PKV_ERR_INVALID_ARG;
    pkv_pool* p = new (std::nothrow) pkv_pool;
    if (!p) return PKV_ERR_NO_SPACE;
    p->num_layers = num_layers;
    p->num_pages = num_pages;
    p->page_size = page_size;
    p->kv_heads = kv_heads;
    p->head_dim = head_dim;
    p->dtype = dtype;
    p->storage = storage;
    p->k_base = k_base;
    p->v_base = v_base;
    p->k_scale_base = k_scales;
    p->v_scale_base = v_scales;
    p->layer_elems = (int64_t)num_pages * kv_heads * page_size * head_dim;
    p->free_stack.resize((size_t)num_pages);
    for (int i = 0; i < num_pages; ++i) p->free_stack[(size_t)i] = num_pages - 1 - i;  // top = 0
    p->allocated.assign((size_t)num_pages, 0);
    *out = p;
    return PKV_OK;
}

}  // namespace

extern "C" int kv_pool_create(int num_layers, int num_pages, int page_size, int kv_heads,
                              int head_dim, int dtype, void* k_base, void* v_base, pkv_pool** out)
{
    return make_pool(num_layers, num_pages, page_size, kv_heads, head_dim, dtype, dtype, k_base, v_base, nullptr,
                     nullptr, out);
}

// int8 pages ([ENGINE] s3.4 compression): codes plus one fp32 scale per (token, head) row.
extern "C" int kv_pool_create_i8(int num_layers, int num_pages, int page_size, int kv_heads, int head_dim,
                                 int dtype, void* k_codes, void* v_codes, void* k_scales, void* v_scales,
                                 pkv_pool** out)
{
    return make_pool(num_layers, num_pages, page_size, kv_heads, head_dim, dtype, PKV_I8, k_codes, v_codes,
                     k_scales, v_scales, out);
}

extern "C" int kv_pool_storage(const pkv_pool* pool, int* storage_out)
{
    if (!pool || !storage_out) return PKV_ERR_INVALID_ARG;
    *storage_out = pool->storage;
    return PKV_OK;
}

extern "C" void kv_pool_destroy(pkv_pool* pool) { delete pool; }

extern "C" int kv_pool_alloc(pkv_pool* pool, int n, int32_t* page_ids_out)
{
    if (!pool || n < 0 || (n > 0 && !page_ids_out)) return PKV_ERR_INVALID_ARG;
    if ((size_t)n > pool->free_stack.size()) return PKV_ERR_NO_SPACE;
    for (int i = 0; i < n; ++i) {
        int32_t id = pool->free_stack.back();
        pool->free_stack.pop_back();
        pool->allocated[(size_t)id] = 1;
        page_ids_out[i] = id;
    }
    return PKV_OK;
}

extern "C" int kv_pool_free(pkv_pool* pool, int n, const int32_t* page_ids)
{
    if (!pool || n < 0 || (n > 0 && !page_ids)) return PKV_ERR_INVALID_ARG;
    // validate everything first so that a bad list changes nothing
    std::vector<uint8_t> seen;
    for (int i = 0; i < n; ++i) {
        int32_t id = page_ids[i];
        if (id < 0 || id >= pool->num_pages || !pool->allocated[(size_t)id]) return PKV_ERR_INVALID_ARG;
        if (seen.empty()) seen.assign((size_t)pool->num_pages, 0);
        if (seen[(size_t)id]) return PKV_ERR_INVALID_ARG;
        seen[(size_t)id] = 1;
    }
    for (int i = 0; i < n; ++i) {
        pool->allocated[(size_t)page_ids[i]] = 0;
        pool->free_stack.push_back(page_ids[i]);
    }
    return PKV_OK;
}

extern "C" int kv_pool_free_count(const pkv_pool* pool)
{
    return pool ? (int)pool->free_stack.size() : -1;
}

extern "C" int kv_pool_info(const pkv_pool* pool, int* num_layers, int* num_pages, int* page_size,
                            int* kv_heads, int* head_dim, int* dtype)
{
    if (!pool) return PKV_ERR_INVALID_ARG;
    if (num_layers) *num_layers = pool->num_layers;
    if (num_pages) *num_pages = pool->num_pages;
    if (page_size) *page_size = pool->page_size;
    if (kv_heads) *kv_heads = pool->kv_heads;
    if (head_dim) *head_dim = pool->head_dim;
    if (dtype) *dtype = pool->dtype;
    return PKV_OK;
}

extern "C" int64_t pkv_kv_cache_bytes(int num_layers, int kv_heads, int head_dim, int64_t tokens,
                                      int dtype)
{
    if (num_layers < 0 || kv_heads < 0 || head_dim < 0 || tokens < 0) return -1;
    if (dtype == PKV_I8) return (int64_t)num_layers * 2 * kv_heads * tokens * (head_dim + 4);
    if (dtype != PKV_F16 && dtype != PKV_BF16) return -1;
    const int64_t elt = 2;
    return (int64_t)num_layers * 2 * kv_heads * head_dim * tokens * elt;
}

extern "C" int pkv_slot_mapping(const int32_t* block_tables, int max_pages_per_seq,
                                const int32_t* positions, int n, int page_size, int64_t* slots_out)
{
    if (n < 0 || page_size <= 0 || max_pages_per_seq <= 0) return PKV_ERR_INVALID_ARG;
    if (n > 0 && (!block_tables || !positions || !slots_out)) return PKV_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        const int32_t pos = positions[i];
        if (pos < 0) {
            slots_out[i] = -1;
            continue;
        }
        const int lp = pos / page_size;
        if (lp >= max_pages_per_seq) return PKV_ERR_INVALID_ARG;
        const int32_t page = block_tables[(int64_t)i * max_pages_per_seq + lp];
        if (page < 0) return PKV_ERR_INVALID_ARG;
        slots_out[i] = (int64_t)page * page_size + pos % page_size;
    }
    return PKV_OK;
}
