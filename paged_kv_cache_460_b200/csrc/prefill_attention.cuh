// Chunked prefill attention over the paged KV cache, on the tensor cores.
//
// "为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427) s4.3: the forward of a chunk
// of seq_len new tokens at start_pos appends their k, v to the cache and applies the
// causal mask slice [start_pos : start_pos + seq_len, : start_pos + seq_len] -- query row i
// sees keys 0 .. start_pos + i.  With a chunk of rows the contraction is dense (16 query
// rows per MMA), unlike the single-row decode step.
//
// Work: one warp per (sequence, kv head, tile of 16 MMA rows), a row being one (query
// token, query head of the group) pair, so a tile holds 16 / G tokens x G heads.  The
// warp streams the key units (16 rows of K and V) that the tile's last token can see,
// 0 .. pos_max, through its own cp.async ring (chunks XOR-swizzled as in the decode
// tensor-core kernel), and per unit computes
//   S[16 rows x 16 keys] = Q . K^T      (2 x D/16 mma.sync m16n8k16)
//   causal mask, fp32 online softmax per row (log2 domain)
//   O[16 x D] += P . V                 (D/8 MMAs; P from the S accumulators in registers,
//                                        bf16 P as hi + lo)
// and finally writes O / l.  Rows past the chunk and keys past a row's position are
// masked; V rows past the cached length are zeroed before they meet a zero weight.
#ifndef PKV_PREFILL_ATTENTION_CUH_
#define PKV_PREFILL_ATTENTION_CUH_

#include <type_traits>

#include "decode_attention_mma.cuh"

namespace pkv {

constexpr int kPrefillWarps = 4;
constexpr int kPrefillThreads = kPrefillWarps * 32;
constexpr int kPrefillDepth = 2;

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
    static constexpr int kUnit = 16 * D * 2;                 // bytes of 16 K (or V) rows
    static constexpr int kSlot = 2 * kUnit;
    static constexpr int kRingBytes = kPrefillWarps * kPrefillDepth * kSlot;
    static constexpr int kScanOffset = kRingBytes;            // item prefix [batch + 1]
    static int smem_bytes(int batch) { return kScanOffset + 4 * (batch + 1); }
};

template <int D, int P, int G, typename T>
__global__ void __launch_bounds__(kPrefillThreads) prefill_attention_kernel(const PrefillParams p)
{
    using S = PrefillShape<D>;
    constexpr int DEPTH = kPrefillDepth;
    constexpr int CPR = D / 8;
    constexpr int U = P / 16;              // key units per page
    constexpr int KS = D / 16;             // k-steps of Q.K^T
    constexpr int ND = D / 8;              // n-tiles of O
    constexpr int TT = 16 / G;             // query tokens per tile
    static_assert(G >= 1 && G <= 16 && 16 % G == 0, "group size");
    extern __shared__ __align__(128) unsigned char smem[];
    int* items = reinterpret_cast<int*>(smem + S::kScanOffset);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Hkv = p.kv_heads;

    // prefix of work items over the sequences: Hkv * ceil(n_b * G / 16) per sequence
    for (int b = threadIdx.x; b <= p.batch; b += blockDim.x) items[b] = 0;
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int b = 0; b < p.batch; ++b) {
            items[b] = run;
            const int n = p.cu_q[b + 1] - p.cu_q[b];
            run += n > 0 ? Hkv * ((n * G + 15) / 16) : 0;
        }
        items[p.batch] = run;
    }
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();
    const int item = blockIdx.x * kPrefillWarps + warp;
    if (item >= items[p.batch]) return;
    int lo = 0, hi = p.batch - 1;         // sequence of the item: largest b with items[b] <= item
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (items[mid] <= item) lo = mid;
        else hi = mid - 1;
    }
    const int b = lo;
    const int q0 = p.cu_q[b], n_b = p.cu_q[b + 1] - q0;
    const int tiles = (n_b * G + 15) / 16;
    const int g = (item - items[b]) / tiles, tile = (item - items[b]) % tiles;
    const int L = p.context_lens[b];
    const int start = L - n_b;
    const int last_tok = min(n_b - 1, tile * TT + TT - 1);
    const int n_units = (start + last_tok) / 16 + 1;   // keys 0 .. position of the tile's last token

    const int g4 = lane >> 2, t4 = lane & 3;
    // rows of this thread: r = g4 and g4 + 8 -> token tile * TT + r / G, head r % G
    int tok[2], pos[2];
    bool rvalid[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int r = g4 + 8 * h;
        tok[h] = tile * TT + r / G;
        rvalid[h] = tok[h] < n_b;
        pos[h] = rvalid[h] ? start + tok[h] : -1;
    }
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

    // ---- per-warp ring of key units
    unsigned char* ring = smem + warp * DEPTH * S::kSlot;
    int win = 0, win0 = -1;
    auto issue = [&](int u) {
        if (win0 < 0 || u >= win0 + 32) {
            win0 = u;
            const int pg = (u + lane) / U;
            win = (u + lane < n_units && pg < p.max_pages) ? p.block_tables[(long long)b * p.max_pages + pg] : -1;
        }
        const int page = __shfl_sync(0xffffffffu, win, u - win0);
        unsigned char* slot = ring + (u % DEPTH) * S::kSlot;
        if ((unsigned)page < (unsigned)p.num_pages) {
            const long long off = (((long long)page * Hkv + g) * P + (u % U) * 16) * D;
            const unsigned char* ks = reinterpret_cast<const unsigned char*>(static_cast<const T*>(p.k) + off);
            const unsigned char* vs = reinterpret_cast<const unsigned char*>(static_cast<const T*>(p.v) + off);
#pragma unroll
            for (int n = 0; n < S::kUnit / 512; ++n) {
                const int gidx = n * 32 + lane;
                const int t = gidx / CPR, c = gidx % CPR;
                const int dst = t * (2 * D) + ((c ^ (t & 7)) * 16);
                cp_async16(slot + dst, ks + gidx * 16);
                cp_async16(slot + S::kUnit + dst, vs + gidx * 16);
            }
        } else if (lane == 0) {
            atomicOr(&g_error_word, PKV_DEVERR_BAD_PAGE);   // never dereferenced
        }
    };
#pragma unroll
    for (int u = 0; u < DEPTH; ++u) {
        if (u < n_units) issue(u);
        cp_async_commit();
    }

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

    for (int u = 0; u < n_units; ++u) {
        cp_async_wait<DEPTH - 1>();
        __syncwarp();
        unsigned char* s = ring + (u % DEPTH) * S::kSlot;
        const int kvalid = min(16, L - u * 16);
        if (kvalid < 16) {                    // rows past the cache: zero V (weights are 0 there)
            for (int x = lane; x < (16 - kvalid) * CPR; x += 32)
                reinterpret_cast<uint4*>(s + S::kUnit + kvalid * (2 * D))[x] = make_uint4(0, 0, 0, 0);
            __syncwarp();
        }
        // ---- S = Q . K^T for the unit's 16 keys (two n-tiles of 8 keys)
        float sacc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            uint32_t kb[4];
            const int ch = 2 * kk + kb_hi;
            ldmatrix_x4(kb, s + kb_row * (2 * D) + ((ch ^ (kb_row & 7)) * 16));
            MmaOps<T>::mma(sacc[0], qa[kk], kb[0], kb[1]);
            MmaOps<T>::mma(sacc[1], qa[kk], kb[2], kb[3]);
        }
        // ---- causal mask and online softmax per row (rows g4: e = 0,1; g4 + 8: e = 2,3)
        float alpha[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int key = u * 16 + nt * 8 + 2 * t4 + c;
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
            for (int nt = 0; nt < 2; ++nt)
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
        // ---- P as A fragments (rows x 16 keys); bf16 P as hi + lo
        uint32_t pa[4], pl[4];
        pa[0] = MmaOps<T>::pack(sacc[0][0], sacc[0][1]);
        pa[1] = MmaOps<T>::pack(sacc[0][2], sacc[0][3]);
        pa[2] = MmaOps<T>::pack(sacc[1][0], sacc[1][1]);
        pa[3] = MmaOps<T>::pack(sacc[1][2], sacc[1][3]);
        if constexpr (kSplitP) {
            const float* sv = &sacc[0][0];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                pl[i] = MmaOps<T>::pack(sv[2 * i] - __uint_as_float(pa[i] << 16),
                                        sv[2 * i + 1] - __uint_as_float(pa[i] & 0xffff0000u));
        }
        // ---- O += P . V (two n-tiles of 8 columns per ldmatrix)
#pragma unroll
        for (int jt = 0; jt < ND / 2; ++jt) {
            uint32_t vb[4];
            const int ch = 2 * jt + vb_hi;
            ldmatrix_x4_trans(vb, s + S::kUnit + vb_row * (2 * D) + ((ch ^ (vb_row & 7)) * 16));
            MmaOps<T>::mma(oacc[2 * jt], pa, vb[0], vb[1]);
            MmaOps<T>::mma(oacc[2 * jt + 1], pa, vb[2], vb[3]);
            if constexpr (kSplitP) {
                MmaOps<T>::mma(oacc[2 * jt], pl, vb[0], vb[1]);
                MmaOps<T>::mma(oacc[2 * jt + 1], pl, vb[2], vb[3]);
            }
        }
        __syncwarp();
        if (u + DEPTH < n_units) issue(u + DEPTH);
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
