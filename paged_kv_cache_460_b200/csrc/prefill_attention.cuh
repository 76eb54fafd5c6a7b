// Chunked prefill attention: the parameters shared by the host launcher and the
// tensor-core kernel (prefill_attention_tc.cuh), and the zero-filling 16-byte copy used to
// stage K/V blocks from the pages.
//
// "为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427) s4.3: the forward of a chunk
// of seq_len new tokens at start_pos appends their k, v to the cache and applies the
// causal mask slice [start_pos : start_pos + seq_len, : start_pos + seq_len] -- query row i
// sees keys 0 .. start_pos + i.
#ifndef PKV_PREFILL_ATTENTION_CUH_
#define PKV_PREFILL_ATTENTION_CUH_

#include <type_traits>

#include "decode_attention_mma.cuh"

namespace pkv {

struct PrefillParams {
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

// 16-byte cp.async that writes zeros instead when `valid` is false (src-size 0: nothing is
// read from `src`, which must still be a mapped address).
__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src),
                 "r"(valid ? 16u : 0u)
                 : "memory");
}

}  // namespace pkv

#endif  // PKV_PREFILL_ATTENTION_CUH_
