// Internal definition of the pool descriptor shared by the host files of libpagedkv.
#ifndef PKV_INTERNAL_H_
#define PKV_INTERNAL_H_

#include <cstdint>
#include <new>
#include <vector>

struct pkv_pool {
    int num_layers;
    int num_pages;
    int page_size;
    int kv_heads;
    int head_dim;
    int dtype;
    void* k_base;            // device [layers][pages][kv_heads][page_size][head_dim]
    void* v_base;
    int64_t layer_elems;     // pages * kv_heads * page_size * head_dim
    std::vector<int32_t> free_stack;  // back() is handed out next
    std::vector<uint8_t> allocated;   // 1 while a page id is out of the free list
};

#endif  // PKV_INTERNAL_H_
