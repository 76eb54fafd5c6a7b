// Paged decode attention: a balanced streaming pass over all cached pages plus a
// log-sum-exp merge of the (sequence, kv head) pairs that a partition boundary cut.
//
// What is computed ("为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427) s4.3;
// "大模型推理全流程解析" (stapisi.com/news/4049481) s2.2.2): for the single new query of
// each sequence, softmax(scale * q . K^T) . V over its cached tokens, the K/V rows found
// through the page table (s3.4).  The causal mask keeps every cached token because the
// query is the last position.  The pages note that decode is bound by reading the KV
// cache ([FLOW] s2.2.2) and that fp16 q.k products can overflow (dpshk.com/news/4990443
// s3.2), so products are accumulated and the softmax is kept in fp32.
//
// Work layout (B200 design, not from the pages).  Flatten the batch's work into
// W = kv_heads * sum_b pages(b) "page-head" units in (sequence, kv head, page) order and
// cut it into num_splits equal contiguous ranges, one per CTA.  Every CTA therefore
// streams the same number of bytes whatever the length mix, and a (sequence, kv head)
// pair is cut at most at range boundaries.  Inside a CTA:
//   - a producer warp walks its range, reads the page table, and for each page issues
//     two 1-D bulk (TMA) copies -- the page's K and V chunks of page_size*head_dim
//     contiguous elements -- into a ring of shared-memory slots, plus the group's q
//     rows when a (sequence, kv head) segment begins;
//   - NW consumer warps all work on each page, warp w on its page_size/NW token rows:
//     q.k dot products with 16-byte shared loads and shuffle reductions, an online
//     softmax (running max m, running sum l, unnormalised output o), all in fp32 in
//     the log2 domain;
//   - at the end of a segment the warps' (m, l, o) are combined through shared memory;
//     a segment wholly inside the range is normalised and written as the output, a cut
//     one is written to one of the CTA's two partial slots (2c: the segment began before
//     the range, 2c+1: it continues after it) for the merge kernel.
#ifndef PKV_DECODE_ATTENTION_CUH_
#define PKV_DECODE_ATTENTION_CUH_

#include "pkv_device.cuh"

namespace pkv {

constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr int kRingBudgetBytes = 96 * 1024;
constexpr int kMetaHeaderBytes = 16;   // int64 chunk, int64 total units

struct DecodeParams {
    const void* k;              // this layer's K pool  [pages][kv_heads][P][D]
    const void* v;
    const void* q;              // [batch][q_heads][D]
    void* out;                  // [batch][q_heads][D]
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* part_o;              // [2 * num_splits][G][D]
    float* part_ml;             // [2 * num_splits][G][2]
    unsigned char* meta;        // chunk, W, prefix[batch + 1]
    int batch;
    int max_pages;
    int q_heads;
    int kv_heads;
    int num_pages;
    int num_splits;
    float scale_log2;           // scale * log2(e)
};

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

template <int D, int P, int G>
struct DecodeShape {
    static constexpr int kChunk = P * D * 2;                 // bytes of one (page, head)
    static constexpr int kQBytes = G * D * 2;
    static constexpr int kSlot = 2 * kChunk + kQBytes;
    static constexpr int kStagesRaw = kRingBudgetBytes / kSlot;
    static constexpr int kStages = kStagesRaw < 2 ? 2 : (kStagesRaw > 16 ? 16 : kStagesRaw);
    static constexpr int kRingBytes = kStages * kSlot;
    static constexpr int kBarOffset = kRingBytes;
    static constexpr int kFlagOffset = kBarOffset + 2 * kStages * 8;
    static constexpr int kCmbOffset = align_up(kFlagOffset + 16 + 8 * 4, 16);
    static constexpr int kCmbFloats = kConsumerWarps * G * (D + 2);
    static constexpr int kScanOffset = kCmbOffset + 2 * kCmbFloats * 4;
    // prefix[batch+1] and lens[batch] follow
    static int smem_bytes(int batch) { return kScanOffset + 4 * (2 * batch + 1); }
};

// Page prefix sums of the batch: prefix[b] = sum_{b' < b} ceil(len_b' / P); lens copied.
template <int P>
__device__ __forceinline__ void block_page_prefix(const int32_t* __restrict__ lens_g, int batch,
                                                  int* prefix, int* lens, int* warp_tot)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nt = blockDim.x;
    const int per = (batch + nt - 1) / nt;
    const int lo = min(batch, tid * per), hi = min(batch, lo + per);
    int sum = 0;
    for (int b = lo; b < hi; ++b) {
        const int L = max(lens_g[b], 0);
        lens[b] = L;
        sum += (L + P - 1) / P;
    }
    int x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    int run = x - sum;
    for (int w = 0; w < warp; ++w) run += warp_tot[w];
    for (int b = lo; b < hi; ++b) {
        run += (lens[b] + P - 1) / P;
        prefix[b + 1] = run;
    }
    if (tid == 0) prefix[0] = 0;
}

// Position `u` of the flattened (sequence, kv head, page) order -> (b, g, j).
__device__ __forceinline__ void locate_unit(long long u, const int* prefix, int batch, int kv_heads,
                                            int& b, int& g, int& j)
{
    int lo = 0, hi = batch - 1;           // largest b with kv_heads * prefix[b] <= u
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((long long)kv_heads * prefix[mid] <= u) lo = mid;
        else hi = mid - 1;
    }
    b = lo;
    const int np = prefix[b + 1] - prefix[b];
    const long long rem = u - (long long)kv_heads * prefix[b];
    g = (int)(rem / np);
    j = (int)(rem - (long long)g * np);
}

__device__ __forceinline__ void next_unit(int& b, int& g, int& j, int& np, const int* prefix, int kv_heads,
                                          int batch)
{
    if (++j < np) return;
    j = 0;
    if (++g < kv_heads) return;
    g = 0;
    do {
        ++b;
        np = b < batch ? prefix[b + 1] - prefix[b] : 1;
    } while (np == 0);
}

template <int D, int P, int G, typename T>
__global__ void __launch_bounds__(kDecodeThreads) decode_pass1_kernel(const DecodeParams p)
{
    using S = DecodeShape<D, P, G>;
    constexpr int NST = S::kStages;
    constexpr int NW = kConsumerWarps;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOffset);
    uint64_t* empty = full + NST;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kFlagOffset);
    int* issued = reinterpret_cast<int*>(smem + S::kFlagOffset + 4);
    volatile int* drain_abort = reinterpret_cast<volatile int*>(smem + S::kFlagOffset + 8);
    int* warp_tot = reinterpret_cast<int*>(smem + S::kFlagOffset + 16);
    float* cmb = reinterpret_cast<float*>(smem + S::kCmbOffset);
    int* prefix = reinterpret_cast<int*>(smem + S::kScanOffset);
    int* lens = prefix + p.batch + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NW);
        }
        *abort_flag = 0;
        *issued = 0;
        *drain_abort = 0;
        fence_barrier_init();
    }
    // The prologue reads only the caller's lengths; the pool and the workspace are
    // touched after pdl_wait, once the previous kernel on the stream has finished.
    block_page_prefix<P>(p.context_lens, p.batch, prefix, lens, warp_tot);
    __syncthreads();

    const int Hkv = p.kv_heads;
    const long long W = (long long)Hkv * prefix[p.batch];
    const long long chunk = W > 0 ? (W + p.num_splits - 1) / p.num_splits : 1;
    const long long r0 = (long long)blockIdx.x * chunk;
    const long long r1 = min(W, r0 + chunk);
    pdl_wait();
    pdl_launch_dependents();
    if (blockIdx.x == 0) {
        long long* hdr = reinterpret_cast<long long*>(p.meta);
        int* pre = reinterpret_cast<int*>(p.meta + kMetaHeaderBytes);
        if (tid == 0) {
            hdr[0] = chunk;
            hdr[1] = W;
        }
        for (int b = tid; b <= p.batch; b += blockDim.x) pre[b] = prefix[b];
    }
    if (r0 >= r1) return;

    if (warp == NW) {
        // ------------------------------------------------------------ producer
        const uint64_t policy = l2_policy_evict_first();
        int b, g, j;
        locate_unit(r0, prefix, p.batch, Hkv, b, g, j);
        int np = prefix[b + 1] - prefix[b];
        int win_b = -1, win_j0 = 0, bt = 0;
        int it = 0;
        for (long long u = r0; u < r1; ++u, ++it) {
            const int slot = it % NST;
            if (it >= NST && !mbar_wait_bounded(&empty[slot], ((it / NST) - 1) & 1, abort_flag)) break;
            if (b != win_b || j < win_j0 || j >= win_j0 + 32) {
                win_b = b;
                win_j0 = j & ~31;
                const int jj = win_j0 + lane;
                // a length beyond the table's width yields -1: flagged, never dereferenced
                bt = jj < np ? (jj < p.max_pages ? p.block_tables[(long long)b * p.max_pages + jj] : -1) : 0;
            }
            const int page = __shfl_sync(0xffffffffu, bt, j - win_j0);
            if (lane == 0) {
                unsigned char* s = smem + slot * S::kSlot;
                const bool ok = (unsigned)page < (unsigned)p.num_pages;
                const bool seg_start = (j == 0) || (it == 0);
                const uint32_t bytes = (ok ? 2u * S::kChunk : 0u) + (seg_start ? (uint32_t)S::kQBytes : 0u);
                if (!ok) atomicOr(&g_error_word, PKV_DEVERR_BAD_PAGE);
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(&full[slot], bytes);
                if (ok) {
                    const long long off = ((long long)page * Hkv + g) * (P * D);
                    bulk_load_evict_first(s, static_cast<const T*>(p.k) + off, S::kChunk, &full[slot], policy);
                    bulk_load_evict_first(s + S::kChunk, static_cast<const T*>(p.v) + off, S::kChunk, &full[slot],
                                          policy);
                }
                if (seg_start)
                    bulk_load(s + 2 * S::kChunk,
                              static_cast<const T*>(p.q) + ((long long)b * p.q_heads + (long long)g * G) * D,
                              S::kQBytes, &full[slot]);
            }
            __syncwarp();
            next_unit(b, g, j, np, prefix, Hkv, p.batch);
        }
        if (lane == 0) *issued = it;
    } else {
        // ------------------------------------------------------------ consumers
        constexpr int LPR = D / 8;            // lanes per K/V row (16 bytes each)
        constexpr int RPI = 32 / LPR;         // rows per warp-wide load
        constexpr int TPW = P / NW;           // token rows per warp per page
        constexpr int NIT = TPW / RPI;
        static_assert(TPW % RPI == 0, "page rows must split evenly over the warps");
        const int r = lane / LPR, c = lane % LPR;
        float qf[G][8], o[G][8], m[G], l[G];
        int b, g, j;
        locate_unit(r0, prefix, p.batch, Hkv, b, g, j);
        int np = prefix[b + 1] - prefix[b];
        int seg = 0;
        int it = 0;
        bool live = true;
        for (long long u = r0; u < r1; ++u, ++it) {
            const int slot = it % NST;
            if (live) live = mbar_wait_bounded(&full[slot], (it / NST) & 1, abort_flag);
            const unsigned char* s = smem + slot * S::kSlot;
            const bool seg_start = (j == 0) || (it == 0);
            if (seg_start) {
#pragma unroll
                for (int gi = 0; gi < G; ++gi) {
                    const uint4 qu = *reinterpret_cast<const uint4*>(s + 2 * S::kChunk + (gi * D + c * 8) * 2);
                    unpack8<T>(qu, qf[gi]);
                    m[gi] = -INFINITY;
                    l[gi] = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[gi][e] = 0.f;
                }
            }
            const int nvalid = min(P, lens[b] - j * P);
            float kf[NIT][8], vf[NIT][8];
#pragma unroll
            for (int n = 0; n < NIT; ++n) {
                const int tok = warp * TPW + n * RPI + r;
                const uint4 ku = *reinterpret_cast<const uint4*>(s + (tok * D + c * 8) * 2);
                const uint4 vu = *reinterpret_cast<const uint4*>(s + S::kChunk + (tok * D + c * 8) * 2);
                unpack8<T>(ku, kf[n]);
                unpack8<T>(vu, vf[n]);
                if (tok >= nvalid) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) vf[n][e] = 0.f;   // rows past the context may hold anything
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
#pragma unroll
            for (int gi = 0; gi < G; ++gi) {
                float sc[NIT];
                float pm = -INFINITY;
#pragma unroll
                for (int n = 0; n < NIT; ++n) {
                    float dot = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) dot = fmaf(qf[gi][e], kf[n][e], dot);
#pragma unroll
                    for (int mask = LPR / 2; mask > 0; mask >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, mask);
                    const int tok = warp * TPW + n * RPI + r;
                    sc[n] = tok < nvalid ? dot * p.scale_log2 : -INFINITY;
                    pm = fmaxf(pm, sc[n]);
                }
#pragma unroll
                for (int mask = LPR; mask < 32; mask <<= 1) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, mask));
                const float mn = fmaxf(m[gi], pm);
                if (mn == -INFINITY) continue;        // no valid token seen yet by this warp
                const float alpha = fast_exp2(m[gi] - mn);
                m[gi] = mn;
                float lsum = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) o[gi][e] *= alpha;
#pragma unroll
                for (int n = 0; n < NIT; ++n) {
                    const float pr = fast_exp2(sc[n] - mn);
                    lsum += pr;
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[gi][e] = fmaf(pr, vf[n][e], o[gi][e]);
                }
                l[gi] = l[gi] * alpha + lsum;
            }
            const bool seg_end = (j == np - 1) || (u == r1 - 1);
            if (seg_end) {
                float* buf = cmb + (seg & 1) * S::kCmbFloats;
#pragma unroll
                for (int gi = 0; gi < G; ++gi) {
                    float lt = l[gi];
#pragma unroll
                    for (int mask = LPR; mask < 32; mask <<= 1) lt += __shfl_xor_sync(0xffffffffu, lt, mask);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        float ot = o[gi][e];
#pragma unroll
                        for (int mask = LPR; mask < 32; mask <<= 1) ot += __shfl_xor_sync(0xffffffffu, ot, mask);
                        o[gi][e] = ot;
                    }
                    float* row = buf + (warp * G + gi) * (D + 2);
                    if (r == 0) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) row[c * 8 + e] = o[gi][e];
                        if (c == 0) {
                            row[D] = m[gi];
                            row[D + 1] = lt;
                        }
                    }
                }
                named_barrier(1, NW * 32);
                const long long seg0 = (long long)Hkv * prefix[b] + (long long)g * np;
                const bool complete = seg0 >= r0 && seg0 + np <= r1;
                const int pslot = seg0 < r0 ? 2 * blockIdx.x : 2 * blockIdx.x + 1;
                for (int idx = tid; idx < G * D; idx += NW * 32) {
                    const int gi = idx / D, dd = idx - gi * D;
                    float M = -INFINITY;
#pragma unroll
                    for (int w = 0; w < NW; ++w) M = fmaxf(M, buf[(w * G + gi) * (D + 2) + D]);
                    float num = 0.f, den = 0.f;
#pragma unroll
                    for (int w = 0; w < NW; ++w) {
                        const float* row = buf + (w * G + gi) * (D + 2);
                        const float wt = fast_exp2(row[D] - M);   // a warp with no tokens has m = -inf
                        num = fmaf(wt, row[dd], num);
                        den = fmaf(wt, row[D + 1], den);
                    }
                    if (complete) {
                        T* dst = static_cast<T*>(p.out) + ((long long)b * p.q_heads + (long long)g * G + gi) * D + dd;
                        *dst = Elt<T>::from_float(num / den);
                    } else {
                        p.part_o[((long long)pslot * G + gi) * D + dd] = num;
                        if (dd == 0) {
                            p.part_ml[((long long)pslot * G + gi) * 2 + 0] = M;
                            p.part_ml[((long long)pslot * G + gi) * 2 + 1] = den;
                        }
                    }
                }
                ++seg;
            }
            next_unit(b, g, j, np, prefix, Hkv, p.batch);
        }
    }
    __syncthreads();
    // Drain: a fill that no consumer waited for (only after a timeout) must land before
    // the CTA's shared memory is released.
    if (tid == 0) {
        const int n = *issued;
        for (int s = 0; s < NST && s < n; ++s) {
            const int last = (n - 1 - s) / NST;          // index of the last fill of slot s
            mbar_wait_bounded(&full[s], last & 1, drain_abort);
        }
    }
}

// One CTA per (sequence, kv head).  Sequences with no cached token get zeros; pairs
// finished inside one partition were written by pass 1; the others are merged from the
// partial slots of the partitions c0..c1 that cover them: M = max m_k,
// out = sum_k 2^(m_k - M) o_k / sum_k 2^(m_k - M) l_k.
template <int D, int G, typename T>
__global__ void __launch_bounds__(128) decode_merge_kernel(const DecodeParams p)
{
    pdl_wait();
    pdl_launch_dependents();
    const int Hkv = p.kv_heads;
    const int b = blockIdx.x / Hkv, g = blockIdx.x - b * Hkv;
    const long long chunk = reinterpret_cast<const long long*>(p.meta)[0];
    const int* pre = reinterpret_cast<const int*>(p.meta + kMetaHeaderBytes);
    const int np = pre[b + 1] - pre[b];
    T* out = static_cast<T*>(p.out) + ((long long)b * p.q_heads + (long long)g * G) * D;
    if (np == 0) {
        for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) out[idx] = Elt<T>::from_float(0.f);
        return;
    }
    const long long seg0 = (long long)Hkv * pre[b] + (long long)g * np;
    const int c0 = (int)(seg0 / chunk), c1 = (int)((seg0 + np - 1) / chunk);
    if (c0 == c1) return;
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int gi = idx / D, dd = idx - gi * D;
        float M = -INFINITY;
        for (int c = c0; c <= c1; ++c) {
            const int slot = c == c0 ? 2 * c0 + 1 : 2 * c;
            M = fmaxf(M, p.part_ml[((long long)slot * G + gi) * 2]);
        }
        float num = 0.f, den = 0.f;
        for (int c = c0; c <= c1; ++c) {
            const int slot = c == c0 ? 2 * c0 + 1 : 2 * c;
            const float wt = fast_exp2(p.part_ml[((long long)slot * G + gi) * 2] - M);
            num = fmaf(wt, p.part_o[((long long)slot * G + gi) * D + dd], num);
            den = fmaf(wt, p.part_ml[((long long)slot * G + gi) * 2 + 1], den);
        }
        out[idx] = Elt<T>::from_float(num / den);
    }
}

}  // namespace pkv

#endif  // PKV_DECODE_ATTENTION_CUH_
