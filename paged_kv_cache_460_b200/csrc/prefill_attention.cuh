// Chunked prefill attention over the paged KV cache, on the tensor cores.
//
// "为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427) s4.3: the forward of a chunk
// of seq_len new tokens at start_pos appends their k, v to the cache and applies the
// causal mask slice [start_pos : start_pos + seq_len, : start_pos + seq_len] -- query row i
// sees keys 0 .. start_pos + i.  With a chunk of rows the contraction is dense (16 query
// rows per MMA), unlike the single-row decode step.
//
// Work: one CTA per (sequence, kv head, tile of 64 MMA rows), a row being one (query
// token, query head of the group) pair; warp w owns rows 16w .. 16w + 15.  The CTA streams
// the blocks of 64 keys that its last token can see through a two-stage shared-memory ring
// that all 128 threads fill with 16-byte cp.async copies (keys past the cache are
// zero-filled by the copy itself) and all four warps read, so a K/V block crosses the
// memory system once per 64 rows instead of once per 16.  Per block each warp computes
//   S[16 rows x 64 keys] = Q . K^T      (8 x D/16 mma.sync m16n8k16)
//   causal mask, fp32 online softmax per row (log2 domain)
//   O[16 x D] += P . V                 (4 x D/8 MMAs; P from the S accumulators in
//                                        registers, bf16 P as hi + lo)
// and finally writes O / l.  Rows past the chunk and keys past a row's position are
// masked; a warp whose rows all end before a block skips it (it still joins the barriers).
#ifndef PKV_PREFILL_ATTENTION_CUH_
#define PKV_PREFILL_ATTENTION_CUH_

#include <type_traits>

#include "decode_attention_mma.cuh"

namespace pkv {

constexpr int kPrefillWarps = 4;
constexpr int kPrefillThreads = kPrefillWarps * 32;
constexpr int kPrefillRows = kPrefillWarps * 16;   // MMA rows per CTA
constexpr int kPrefillKeys = 64;                    // keys per ring stage

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

template <int D>
struct PrefillShape {
    static constexpr int kBlock = kPrefillKeys * D * 2;      // bytes of 64 K (or V) rows
    static constexpr int kStage = 2 * kBlock;
    static constexpr int kRingBytes = 2 * kStage;
    static constexpr int kScanOffset = kRingBytes;            // item prefix [batch + 1]
    static int smem_bytes(int batch) { return kScanOffset + 4 * (batch + 1); }
};

// 16-byte cp.async that writes zeros instead when `valid` is false (src-size 0: nothing is
// read from `src`, which must still be a mapped address).
__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src),
                 "r"(valid ? 16u : 0u)
                 : "memory");
}

template <int D, int P, int G, typename T>
__global__ void __launch_bounds__(kPrefillThreads, 3) prefill_attention_kernel(const PrefillParams p)
{
    using S = PrefillShape<D>;
    constexpr int CPR = D / 8;             // 16-byte chunks per row
    constexpr int KS = D / 16;             // k-steps of Q.K^T
    constexpr int ND = D / 8;              // n-tiles of O
    constexpr int CT = kPrefillRows / G;   // query tokens per CTA tile
    constexpr int NKC = kPrefillKeys * CPR / kPrefillThreads;   // chunks per thread per block (K or V)
    static_assert(G >= 1 && G <= 16 && 16 % G == 0, "group size");
    extern __shared__ __align__(128) unsigned char smem[];
    int* items = reinterpret_cast<int*>(smem + S::kScanOffset);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Hkv = p.kv_heads;

    // prefix of work items over the sequences: Hkv * ceil(n_b * G / 64) per sequence
    if (tid == 0) {
        int run = 0;
        for (int b = 0; b < p.batch; ++b) {
            items[b] = run;
            const int n = p.cu_q[b + 1] - p.cu_q[b];
            run += n > 0 ? Hkv * ((n * G + kPrefillRows - 1) / kPrefillRows) : 0;
        }
        items[p.batch] = run;
    }
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();
    const int item = blockIdx.x;
    if (item >= items[p.batch]) return;
    int lo = 0, hi = p.batch - 1;         // sequence of the item: largest b with items[b] <= item
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (items[mid] <= item) lo = mid;
        else hi = mid - 1;
    }
    const int b = lo;
    const int q0 = p.cu_q[b], n_b = p.cu_q[b + 1] - q0;
    const int tiles = (n_b * G + kPrefillRows - 1) / kPrefillRows;
    const int g = (item - items[b]) / tiles, tile = (item - items[b]) % tiles;
    const int L = p.context_lens[b];
    const int start = L - n_b;
    const int cta_last = min(n_b - 1, tile * CT + CT - 1);
    const int n_blocks = (start + cta_last) / kPrefillKeys + 1;   // keys 0 .. position of the CTA's last token

    const int g4 = lane >> 2, t4 = lane & 3;
    // rows of this thread: r = 16 warp + g4 (+ 8) -> token tile * CT + r / G, head r % G
    int tok[2], pos[2];
    bool rvalid[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int r = 16 * warp + g4 + 8 * h;
        tok[h] = tile * CT + r / G;
        rvalid[h] = tok[h] < n_b;
        pos[h] = rvalid[h] ? start + tok[h] : -1;
    }
    const int warp_first = tile * CT + (16 * warp) / G;
    const int warp_maxpos = warp_first < n_b ? start + min(n_b - 1, tile * CT + (16 * warp + 15) / G) : -1;
    // Q as A fragments (rows x d)
    uint32_t qa[KS][4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int r = g4 + 8 * h;
        const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
            static_cast<const T*>(p.q) + ((long long)(q0 + (rvalid[h] ? tok[h] : 0)) * p.q_heads + g * G + r % G) * D);
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            qa[kk][h] = rvalid[h] ? qrow[(kk * 16 + 2 * t4) / 2] : 0u;
            qa[kk][2 + h] = rvalid[h] ? qrow[(kk * 16 + 8 + 2 * t4) / 2] : 0u;
        }
    }

    // ---- the CTA's two-stage ring of 64-key blocks (K then V, rows XOR-swizzled by chunk)
    const int32_t* table = p.block_tables + (long long)b * p.max_pages;
    auto issue = [&](int blk, int st) {
        unsigned char* kd = smem + st * S::kStage;
#pragma unroll
        for (int n = 0; n < NKC; ++n) {
            const int idx = n * kPrefillThreads + tid;
            const int t = idx / CPR, c = idx % CPR;
            const int key = blk * kPrefillKeys + t;
            bool valid = key < L;
            long long off = 0;
            if (valid) {
                const int pg = key / P;
                const int page = pg < p.max_pages ? table[pg] : -1;
                if ((unsigned)page < (unsigned)p.num_pages) {
                    off = (((long long)page * Hkv + g) * P + key % P) * D + c * 8;
                } else {
                    valid = false;
                    if (c == 0) atomicOr(&g_error_word, PKV_DEVERR_BAD_PAGE);   // never dereferenced
                }
            }
            const int dst = t * (2 * D) + ((c ^ (t & 7)) * 16);
            cp_async16_zfill(kd + dst, static_cast<const T*>(p.k) + off, valid);
            cp_async16_zfill(kd + S::kBlock + dst, static_cast<const T*>(p.v) + off, valid);
        }
    };
    issue(0, 0);
    cp_async_commit();
    if (n_blocks > 1) issue(1, 1);
    cp_async_commit();

    float oacc[ND][4], m_run[2], l_run[2];
#pragma unroll
    for (int n = 0; n < ND; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[n][e] = 0.f;
    m_run[0] = m_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.f;
    const int kb_row = (lane & 7) + 8 * (lane >> 4), kb_hi = (lane >> 3) & 1;      // K as B (keys x d)
    const int vb_row = (lane & 7) + 8 * ((lane >> 3) & 1), vb_hi = lane >> 4;      // V as B^T (keys x d)
    constexpr bool kSplitP = std::is_same<T, __nv_bfloat16>::value;

    for (int blk = 0; blk < n_blocks; ++blk) {
        cp_async_wait<1>();
        __syncthreads();                      // block blk visible to every warp
        const unsigned char* ks = smem + (blk & 1) * S::kStage;
        const unsigned char* vs = ks + S::kBlock;
        if (blk * kPrefillKeys <= warp_maxpos) {
            // ---- S = Q . K^T for the block's 64 keys (eight n-tiles of 8 keys)
            float sacc[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
                for (int kk = 0; kk < KS; ++kk) {
                    uint32_t kb[4];
                    const int ch = 2 * kk + kb_hi;
                    ldmatrix_x4(kb, ks + (16 * j + kb_row) * (2 * D) + ((ch ^ (kb_row & 7)) * 16));
                    MmaOps<T>::mma(sacc[2 * j], qa[kk], kb[0], kb[1]);
                    MmaOps<T>::mma(sacc[2 * j + 1], qa[kk], kb[2], kb[3]);
                }
            }
            // ---- causal mask and online softmax per row (rows g4: e = 0,1; g4 + 8: e = 2,3)
            float alpha[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float mx = -INFINITY;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const int key = blk * kPrefillKeys + nt * 8 + 2 * t4 + c;
                        float& sv = sacc[nt][2 * h + c];
                        sv = key <= pos[h] ? sv * p.scale_log2 : -INFINITY;
                        mx = fmaxf(mx, sv);
                    }
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float mn = fmaxf(m_run[h], mx);
                const bool none = mn == -INFINITY;       // row past the chunk: keep it empty
                alpha[h] = none ? 1.f : fast_exp2(m_run[h] - mn);
                m_run[h] = mn;
                float ls = 0.f;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        float& sv = sacc[nt][2 * h + c];
                        sv = none ? 0.f : fast_exp2(sv - mn);
                        ls += sv;
                    }
                l_run[h] = l_run[h] * alpha[h] + ls;
            }
#pragma unroll
            for (int n = 0; n < ND; ++n) {
                oacc[n][0] *= alpha[0];
                oacc[n][1] *= alpha[0];
                oacc[n][2] *= alpha[1];
                oacc[n][3] *= alpha[1];
            }
            // ---- O += P . V, 16 keys at a time (P as A fragments; bf16 P as hi + lo)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t pa[4], pl[4];
                pa[0] = MmaOps<T>::pack(sacc[2 * j][0], sacc[2 * j][1]);
                pa[1] = MmaOps<T>::pack(sacc[2 * j][2], sacc[2 * j][3]);
                pa[2] = MmaOps<T>::pack(sacc[2 * j + 1][0], sacc[2 * j + 1][1]);
                pa[3] = MmaOps<T>::pack(sacc[2 * j + 1][2], sacc[2 * j + 1][3]);
                if constexpr (kSplitP) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float* sv = &sacc[2 * j + (i >> 1)][2 * (i & 1)];
                        pl[i] = MmaOps<T>::pack(sv[0] - __uint_as_float(pa[i] << 16),
                                                sv[1] - __uint_as_float(pa[i] & 0xffff0000u));
                    }
                }
#pragma unroll
                for (int jt = 0; jt < ND / 2; ++jt) {
                    uint32_t vb[4];
                    const int ch = 2 * jt + vb_hi;
                    ldmatrix_x4_trans(vb, vs + (16 * j + vb_row) * (2 * D) + ((ch ^ (vb_row & 7)) * 16));
                    MmaOps<T>::mma(oacc[2 * jt], pa, vb[0], vb[1]);
                    MmaOps<T>::mma(oacc[2 * jt + 1], pa, vb[2], vb[3]);
                    if constexpr (kSplitP) {
                        MmaOps<T>::mma(oacc[2 * jt], pl, vb[0], vb[1]);
                        MmaOps<T>::mma(oacc[2 * jt + 1], pl, vb[2], vb[3]);
                    }
                }
            }
        }
        __syncthreads();                      // every warp is done with this stage
        if (blk + 2 < n_blocks) issue(blk + 2, blk & 1);
        cp_async_commit();
    }
    cp_async_wait<0>();
    // ---- out = O / l
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float lt = l_run[h];
        lt += __shfl_xor_sync(0xffffffffu, lt, 1);
        lt += __shfl_xor_sync(0xffffffffu, lt, 2);
        if (!rvalid[h]) continue;
        const float inv = 1.f / lt;
        const int r = g4 + 8 * h;
        T* orow = static_cast<T*>(p.out) + ((long long)(q0 + tok[h]) * p.q_heads + g * G + r % G) * D;
#pragma unroll
        for (int n = 0; n < ND; ++n) {
            T pair[2] = {Elt<T>::from_float(oacc[n][2 * h] * inv), Elt<T>::from_float(oacc[n][2 * h + 1] * inv)};
            *reinterpret_cast<uint32_t*>(orow + n * 8 + 2 * t4) = *reinterpret_cast<uint32_t*>(pair);
        }
    }
}

}  // namespace pkv

#endif  // PKV_PREFILL_ATTENTION_CUH_
