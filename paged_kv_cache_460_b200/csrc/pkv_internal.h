// Internal definition of the pool descriptor shared by the host files of libpagedkv.
#ifndef PKV_INTERNAL_H_
#define PKV_INTERNAL_H_

#include <cstdint>
#include <new>
#include <vector>

constexpr int kStorageI8 = 2;   // PKV_I8

struct pkv_pool {
    // bytes of one layer's K (or V) pages
    int64_t layer_bytes() const { return layer_elems * (storage == kStorageI8 ? 1 : 2); }
    // fp32 scales of one layer's K (or V) pages (int8 pools)
    int64_t layer_rows() const { return layer_elems / head_dim; }

    int num_layers;
    int num_pages;
    int page_size;
    int kv_heads;
    int head_dim;
    int dtype;               // type of q, k, v and outputs (PKV_F16 / PKV_BF16)
    int storage;             // type of the pages: dtype, or PKV_I8
    void* k_base;            // device [layers][pages][kv_heads][page_size][head_dim]
    void* v_base;
    void* k_scale_base;      // int8 pools: device fp32 [layers][pages][kv_heads][page_size]
    void* v_scale_base;
    int64_t layer_elems;     // pages * kv_heads * page_size * head_dim
    std::vector<int32_t> free_stack;  // back() is handed out next
    std::vector<uint8_t> allocated;   // 1 while a page id is out of the free list
};

#endif  // PKV_INTERNAL_H_
