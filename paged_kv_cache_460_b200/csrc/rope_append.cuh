// RoPE and KV-append kernels of the decode step.
//
// "为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427):
//   s4.2  RoPE writes the position into q and k with a rotation;
//   s4.3  apply_rotary_emb(q, k, start_pos), then the new k, v join the cache;
//   s5.3  the cache is a preallocated pool (no concatenation).
#ifndef PKV_ROPE_APPEND_CUH_
#define PKV_ROPE_APPEND_CUH_

#include "pkv_device.cuh"

namespace pkv {

// One CTA per token.  The head_dim/2 angles pos * theta^(-2i/d) and their cosines and
// sines are evaluated once per token in fp64 and shared through shared memory; every
// (head, pair) of q and k is then rotated in fp64 and rounded once to the storage type.
// Products and differences use explicit _rn intrinsics, so no fused multiply-add changes
// the rounding of the rotation.
template <typename T>
__global__ void __launch_bounds__(256) rope_kernel(T* __restrict__ q, T* __restrict__ k,
                                                   const int32_t* __restrict__ positions, int q_heads,
                                                   int kv_heads, int head_dim, double theta)
{
    __shared__ double cs[64][2];
    pdl_wait();
    pdl_launch_dependents();
    const int t = blockIdx.x;
    const int pos = positions[t];
    if (pos < 0) return;
    const int half = head_dim >> 1;
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
        const double freq = pow(theta, -2.0 * (double)i / (double)head_dim);
        double s, c;
        sincos((double)pos * freq, &s, &c);
        cs[i][0] = c;
        cs[i][1] = s;
    }
    __syncthreads();
    const int nq = q_heads * half;
    const int total = (q_heads + kv_heads) * half;
    for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
        T* x;
        int i;
        if (idx < nq) {
            const int h = idx / half;
            i = idx - h * half;
            x = q + ((size_t)t * q_heads + h) * head_dim + 2 * i;
        } else {
            const int rel = idx - nq;
            const int h = rel / half;
            i = rel - h * half;
            x = k + ((size_t)t * kv_heads + h) * head_dim + 2 * i;
        }
        const double x0 = Elt<T>::to_double(x[0]);
        const double x1 = Elt<T>::to_double(x[1]);
        const double c = cs[i][0], s = cs[i][1];
        const double y0 = __dsub_rn(__dmul_rn(x0, c), __dmul_rn(x1, s));
        const double y1 = __dadd_rn(__dmul_rn(x0, s), __dmul_rn(x1, c));
        x[0] = Elt<T>::from_double(y0);
        x[1] = Elt<T>::from_double(y1);
    }
}

// One CTA per token: copy the token's k and v rows (kv_heads x head_dim elements each,
// 16-byte vectors) into row slot % page_size of page slot / page_size.  A negative
// slot skips the token; a slot past the pool is skipped and flagged.
__global__ void __launch_bounds__(128) append_kernel(uint4* __restrict__ k_layer, uint4* __restrict__ v_layer,
                                                     const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                     const int64_t* __restrict__ slots, int kv_heads,
                                                     int head_dim, int page_size, int64_t num_slots)
{
    pdl_wait();
    pdl_launch_dependents();
    const int t = blockIdx.x;
    const int64_t s = slots[t];
    if (s < 0) return;
    if (s >= num_slots) {
        if (threadIdx.x == 0) atomicOr(&g_error_word, PKV_DEVERR_BAD_SLOT);
        return;
    }
    const int64_t page = s / page_size;
    const int row = (int)(s - page * page_size);
    const int vec_per_row = head_dim / 8;          // 8 two-byte elements per 16 bytes
    const int total = kv_heads * vec_per_row;
    for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
        const int h = idx / vec_per_row;
        const int c = idx - h * vec_per_row;
        const int64_t dst = ((page * kv_heads + h) * page_size + row) * vec_per_row + c;
        const int64_t src = ((int64_t)t * kv_heads + h) * vec_per_row + c;
        k_layer[dst] = k[src];
        v_layer[dst] = v[src];
    }
}

}  // namespace pkv

#endif  // PKV_ROPE_APPEND_CUH_
