// Chunked prefill attention: the parameters shared by the host launcher and the
// tensor-core kernel (prefill_attention_tc.cuh), and the tiled TMA load that stages K/V
// blocks from the pages.
//
// "为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427) s4.3: the forward of a chunk
// of seq_len new tokens at start_pos appends their k, v to the cache and applies the
// causal mask slice [start_pos : start_pos + seq_len, : start_pos + seq_len] -- query row i
// sees keys 0 .. start_pos + i.
#ifndef PKV_PREFILL_ATTENTION_CUH_
#define PKV_PREFILL_ATTENTION_CUH_

#include <cuda.h>
#include <type_traits>

#include "decode_attention_mma.cuh"

namespace pkv {

struct PrefillParams {
    // this layer's K and V pools [pages][kv_heads][P][D] as 4-D tensors (D, P, kv_heads,
    // pages; box 64 x P x 1 x 1, 128-byte swizzle): one copy lands one 64-column region of
    // one page in the canonical K-major layout
    CUtensorMap k_map;
    CUtensorMap v_map;
    const void* k;                 // this layer's K pool [pages][kv_heads][P][D]
    const void* v;
    const void* q;                 // [total_q][q_heads][D]
    void* out;                     // [total_q][q_heads][D]
    const int32_t* cu_q;           // [batch + 1]
    const int32_t* block_tables;   // [batch][max_pages]
    const int32_t* context_lens;   // [batch], the chunk included
    int batch;
    int max_pages;
    int q_heads;
    int kv_heads;
    int num_pages;
    float scale_log2;
};

// Tiled TMA load of box (x, y, z, w) of a 4-D tensor map into shared memory; completion is
// counted in bytes on `bar`.  x must be a multiple of 8 elements (16 bytes).
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int x, int y, int z, int w, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(
            smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_addr(bar))
        : "memory");
}

}  // namespace pkv

#endif  // PKV_PREFILL_ATTENTION_CUH_
