// RoPE and KV append of the decode step's new token, one kernel for both.
//
// "为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427):
//   s4.2  RoPE writes the position into q and k with a rotation;
//   s4.3  apply_rotary_emb(q, k, start_pos), then the new k, v join the cache;
//   s5.3  the cache is a preallocated pool (no concatenation); fuse small kernels.
#ifndef PKV_ROPE_APPEND_CUH_
#define PKV_ROPE_APPEND_CUH_

#include "pkv_device.cuh"

namespace pkv {

constexpr int kRopeRotate = 1;   // turn q and k in place
constexpr int kRopeAppend = 2;   // write k and v into their pool slots
constexpr int kRopeQuantI8 = 4;  // ... as int8 codes plus a per-row fp32 scale
// Let the next kernel of the stream start before this one waits on its predecessor.  Only
// for launches that write no pool page: the decode kernels read cached pages before their
// own wait, so a launch that appends releases them only once its rows are written.
constexpr int kRopeEarlyRelease = 8;
// The decode step's form: token t is sequence t's newest token, at position
// context_lens[t] - 1, in the slot its page table gives that position.  Such a launch writes
// only pages that a decode kernel given the same lengths does not prefetch, so it may also
// release its dependent early.
constexpr int kRopeFromLens = 16;

struct RopeAppendParams {
    void* q;                 // [n][q_heads][d]   (rotated in place)
    void* k;                 // [n][kv_heads][d]  (rotated in place)
    const void* v;           // [n][kv_heads][d]
    const int32_t* positions;
    const int64_t* slots;
    const int32_t* context_lens;     // kRopeFromLens: [n] lengths (new token included)
    const int32_t* block_tables;     //   and page tables [n][max_pages]
    int max_pages;
    void* k_layer;           // this layer's K pool [pages][kv_heads][P][d]
    void* v_layer;
    float* ks_layer;         // int8 pools: this layer's row scales [pages][kv_heads][P]
    float* vs_layer;
    int q_heads;
    int kv_heads;
    int head_dim;
    int page_size;
    int64_t num_slots;
    double theta;
    int mode;
};

// Turn the four pairs of a 16-byte vector of T in place: pair k of the vector is pair
// i0 + k of the head, cs[2 i] = cos and cs[2 i + 1] = sin of its angle.  Each pair is turned
// in fp64 with explicit _rn products (no fused rounding) and rounded once to T.
template <typename T>
__device__ __forceinline__ void rope_rotate8(uint4& u, const double* cs, int i0)
{
    T* e = reinterpret_cast<T*>(&u);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const double x0 = Elt<T>::to_double(e[2 * k]);
        const double x1 = Elt<T>::to_double(e[2 * k + 1]);
        const double cn = cs[2 * (i0 + k)], sn = cs[2 * (i0 + k) + 1];
        e[2 * k] = Elt<T>::from_double(__dsub_rn(__dmul_rn(x0, cn), __dmul_rn(x1, sn)));
        e[2 * k + 1] = Elt<T>::from_double(__dadd_rn(__dmul_rn(x0, sn), __dmul_rn(x1, cn)));
    }
}

// Angles of the decode step's new tokens, shared by every layer of the step: for sequence b
// with L = context_lens[b] cached tokens (the new one included), position L - 1, and pair i,
// table[b][i] = (cos, sin)(pos * theta^(-2i/d)), evaluated in fp64 exactly as the RoPE
// kernel does.  Sequences with no token get zeros.  The kernel lets its successor start only
// after its rows are written and fenced: the fused layer reads the table before its own wait.
__global__ void __launch_bounds__(64) rope_table_kernel(const int32_t* __restrict__ context_lens, int head_dim,
                                                        double theta, double* __restrict__ table)
{
    pdl_wait();
    const int b = blockIdx.x, half = head_dim >> 1;
    const int pos = context_lens[b] - 1;
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
        double sn = 0.0, cn = 0.0;
        if (pos >= 0) {
            const double freq = pow(theta, -2.0 * (double)i / (double)head_dim);
            sincos((double)pos * freq, &sn, &cn);
        }
        table[((long long)b * half + i) * 2] = cn;
        table[((long long)b * half + i) * 2 + 1] = sn;
    }
    __threadfence();
    __syncthreads();
    pdl_launch_dependents();
}

// Grid: (token, part).  Each thread handles one 16-byte vector (8 elements, 4 pairs)
// of the token's q, k or v rows.  The head_dim/2 angles pos * theta^(-2i/d) and their
// cosines and sines are evaluated once per CTA in fp64 before griddepcontrol.wait, so
// this prologue overlaps the previous kernel on the stream; each pair is then turned in
// fp64 (explicit _rn products: no fused rounding) and rounded once to the storage type.
// A rotate-only launch lets the kernel after it start at once; a launch that appends lets
// it start only after every CTA has written its rows and fenced them at gpu scope, since
// the decode kernels prefetch cached pages (which an append of several tokens per
// sequence, or of any slots, may be writing) before their own wait.
// Appending copies the rotated k and the v vector bit for bit into row slot % P of page
// slot / P; a negative slot skips the token, a slot past the pool is skipped and flagged.
// On an int8 pool the head row is quantised instead ([ENGINE] s3.4 compression):
// amax = max |x| over the row's head_dim/8 threads (a shuffle reduction; a row's threads
// are consecutive lanes of one warp), codes round_half_even(x * (127 / amax)) clamped to
// +-127, scale amax / 127, every step a correctly rounded fp32 operation.
template <typename T>
__global__ void __launch_bounds__(256) rope_append_kernel(const RopeAppendParams p)
{
    __shared__ double cs[64][2];
    const int t = blockIdx.x;
    const int pos = (p.mode & kRopeFromLens) ? p.context_lens[t] - 1 : ((p.mode & kRopeRotate) ? p.positions[t] : -1);
    const int half = p.head_dim >> 1;
    if (pos >= 0) {
        for (int i = threadIdx.x; i < half; i += blockDim.x) {
            const double freq = pow(p.theta, -2.0 * (double)i / (double)p.head_dim);
            double sn, cn;
            sincos((double)pos * freq, &sn, &cn);
            cs[i][0] = cn;
            cs[i][1] = sn;
        }
    }
    __syncthreads();
    if (p.mode & kRopeEarlyRelease) pdl_launch_dependents();
    pdl_wait();
    int64_t slot = -1;
    if ((p.mode & kRopeAppend) && (p.mode & kRopeFromLens)) {
        if (pos >= 0) {            // the slot of position pos through the sequence's page table
            const int j = pos / p.page_size;
            const int page = j < p.max_pages ? p.block_tables[(int64_t)t * p.max_pages + j] : -1;
            if (page >= 0 && (int64_t)page * p.page_size < p.num_slots)
                slot = (int64_t)page * p.page_size + (pos - j * p.page_size);
            else if (blockIdx.y == 0 && threadIdx.x == 0)
                atomicOr(&g_error_word, PKV_DEVERR_BAD_PAGE);
        }
    } else if (p.mode & kRopeAppend) {
        slot = p.slots[t];
        if (slot >= p.num_slots) {
            if (blockIdx.y == 0 && threadIdx.x == 0) atomicOr(&g_error_word, PKV_DEVERR_BAD_SLOT);
            slot = -1;
        }
    }
    const int vph = p.head_dim / 8;                      // 16-byte vectors per head row
    const int nq = (p.mode & kRopeRotate) ? p.q_heads * vph : 0;
    const int nk = p.kv_heads * vph;
    const int total = nq + ((p.mode & kRopeAppend) ? 2 * nk : nk);
    const int64_t page = slot >= 0 ? slot / p.page_size : 0;
    const int row = slot >= 0 ? (int)(slot - page * p.page_size) : 0;
    for (int idx = blockIdx.y * blockDim.x + threadIdx.x; idx < total; idx += gridDim.y * blockDim.x) {
        uint4* src;
        int h, c;
        bool is_v = false;
        if (idx < nq) {
            h = idx / vph;
            c = idx - h * vph;
            src = reinterpret_cast<uint4*>(static_cast<T*>(p.q) + ((int64_t)t * p.q_heads + h) * p.head_dim) + c;
        } else if (idx < nq + nk) {
            h = (idx - nq) / vph;
            c = (idx - nq) - h * vph;
            src = reinterpret_cast<uint4*>(static_cast<T*>(p.k) + ((int64_t)t * p.kv_heads + h) * p.head_dim) + c;
        } else {
            h = (idx - nq - nk) / vph;
            c = (idx - nq - nk) - h * vph;
            src = const_cast<uint4*>(reinterpret_cast<const uint4*>(static_cast<const T*>(p.v) +
                                                                    ((int64_t)t * p.kv_heads + h) * p.head_dim)) + c;
            is_v = true;
        }
        uint4 u = *src;
        if (!is_v && pos >= 0) {
            rope_rotate8<T>(u, &cs[0][0], c * 4);
            *src = u;
        }
        if (slot >= 0 && idx >= nq) {      // uniform over the vph threads of a head row
            const int64_t row_id = (page * p.kv_heads + h) * p.page_size + row;
            if (p.mode & kRopeQuantI8) {
                float x[8];
                unpack8<T>(u, x);
                float amax = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[e]));
                const unsigned lane = threadIdx.x & 31u;
                const unsigned gmask = vph == 32 ? 0xffffffffu : ((1u << vph) - 1u) << (lane & ~(unsigned)(vph - 1));
                for (int m = vph >> 1; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, m));
                uint2 codes = make_uint2(0u, 0u);
                float sc = 0.f;
                if (amax > 0.f) {
                    const float inv = __fdiv_rn(127.f, amax);
                    uint32_t w[2] = {0u, 0u};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float r = fminf(fmaxf(rintf(__fmul_rn(x[e], inv)), -127.f), 127.f);
                        w[e >> 2] |= ((uint32_t)(int)r & 0xffu) << (8 * (e & 3));
                    }
                    codes = make_uint2(w[0], w[1]);
                    sc = __fdiv_rn(amax, 127.f);
                }
                *reinterpret_cast<uint2*>(static_cast<int8_t*>(is_v ? p.v_layer : p.k_layer) +
                                          row_id * p.head_dim + c * 8) = codes;
                if (c == 0) (is_v ? p.vs_layer : p.ks_layer)[row_id] = sc;
            } else {
                uint4* dst = static_cast<uint4*>(is_v ? p.v_layer : p.k_layer) + row_id * vph + c;
                *dst = u;
            }
        }
    }
    if (!(p.mode & kRopeEarlyRelease)) {
        __threadfence();            // this thread's pool and q/k writes, visible at gpu scope,
        __syncthreads();            // for every thread of the CTA, before the CTA releases
        pdl_launch_dependents();    // the next kernel
    }
}

}  // namespace pkv

#endif  // PKV_ROPE_APPEND_CUH_
