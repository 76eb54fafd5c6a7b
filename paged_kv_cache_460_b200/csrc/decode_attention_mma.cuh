// Paged decode attention for grouped-query heads on the tensor cores.
//
// When G = q_heads / kv_heads query heads share one kv head ("为什么要自己动手写一个LLM
// 推理引擎" (wzjinhao.cn/news/61427) s4.3 n_kv_heads; dpshk.com/news/4990443 s5.1 GQA
// k_proj shape), every K and V row is used G times and the contraction becomes a small
// dense GEMM.  This kernel computes it with warp-level tensor-core MMAs (m16n8k16,
// bf16/fp16 inputs, fp32 accumulation); everything else -- the balanced partition of
// the batch's work, the per-warp cp.async rings, the prefetch before the PDL wait, the
// in-kernel merge -- is shared with the CUDA-core kernel in decode_attention.cuh.
//
// Work unit: 16 token rows of one (sequence, kv head) -- a 16-token page, or half of a
// 32-token page -- so 32-token pages keep the same shared-memory footprint per warp.
// Per unit a warp computes
//   S^T[16 tokens x 8 heads] = K[16 x D] . Q^T[D x 8]      (D/16 MMAs; heads >= G are zero)
//   online softmax per head (fp32, log2 domain)
//   O^T[D x 8] += V^T[D x 16] . P^T[16 x 8]               (D/16 MMAs)
// K and V land XOR-swizzled by 16-byte chunk (chunk c of row t at c ^ (t & 7)), so the
// ldmatrix reads of 8 rows at one column are conflict-free; P^T reaches the B-operand
// layout with movmatrix.trans.  P enters the second MMA in the input type -- fp16 as is,
// bf16 as a hi + lo pair -- and the softmax sums stay in fp32.
#ifndef PKV_DECODE_ATTENTION_MMA_CUH_
#define PKV_DECODE_ATTENTION_MMA_CUH_

#include <type_traits>

#include "decode_attention.cuh"

namespace pkv {

template <int D, int G>
struct MmaShape {
    static constexpr int kRows = 16;                          // token rows per unit
    static constexpr int kChunk = kRows * D * 2;              // bytes of one unit's K (or V)
    static constexpr int kQBytes = G * D * 2;
    static constexpr int kSlot = 2 * kChunk + kQBytes;
    static constexpr int kDepthRaw = kRingBudgetBytes / (kDecodeWarps * kSlot);
    static constexpr int kDepth = kDepthRaw < 2 ? 2 : (kDepthRaw > 8 ? 8 : kDepthRaw);
    static constexpr int kRingBytes = kDecodeWarps * kDepth * kSlot;
    static constexpr int kCmbOffset = kRingBytes;
    static constexpr int kCmbFloats = kDecodeWarps * G * (D + 2);
    static constexpr int kWarpTotOffset = kCmbOffset + 2 * kCmbFloats * 4;
    static constexpr int kScanOffset = kWarpTotOffset + 64;
    static int smem_bytes(int batch) { return kScanOffset + 4 * (2 * batch + 1); }
    static constexpr int kCtasPerSm = ctas_per_sm(kScanOffset + 4 * (2 * 64 + 1));
};

template <typename T> struct MmaOps;

template <> struct MmaOps<__nv_bfloat16> {
    static __device__ __forceinline__ void mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
    {
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                     "{%0,%1,%2,%3};"
                     : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                     : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    static __device__ __forceinline__ uint32_t pack(float lo, float hi)
    {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
};

template <> struct MmaOps<__half> {
    static __device__ __forceinline__ void mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
    {
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                     "{%0,%1,%2,%3};"
                     : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                     : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    static __device__ __forceinline__ uint32_t pack(float lo, float hi)
    {
        __half2 h = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
};

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* row_addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_addr(row_addr)));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void* row_addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_addr(row_addr)));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// Register cap from the CTAs per SM that shared memory admits (kCtasPerSm: two with two or four
// query heads per kv head at head_dim 128, one with eight).
template <int D, int P, int G, typename T>
__global__ void __launch_bounds__(kDecodeThreads, MmaShape<D, G>::kCtasPerSm) decode_pass1_mma_kernel(const DecodeParams p)
{
    using S = MmaShape<D, G>;
    constexpr int NW = kDecodeWarps;
    constexpr int DEPTH = S::kDepth;
    constexpr int CPR = D / 8;            // 16-byte chunks per row
    constexpr int U = P / 16;             // units per page
    constexpr int KS = D / 16;            // k-steps of q.k = m-tiles of p.V
    constexpr int QV = S::kQBytes / 16;
    static_assert(G >= 2 && G <= 8, "the MMA kernel serves 2 to 8 query heads per kv head");
    extern __shared__ __align__(128) unsigned char smem[];
    float* cmb = reinterpret_cast<float*>(smem + S::kCmbOffset);
    int* warp_tot = reinterpret_cast<int*>(smem + S::kWarpTotOffset);
    volatile int* last_flag = warp_tot + 8;
    int* prefix = reinterpret_cast<int*>(smem + S::kScanOffset);
    int* lens = prefix + p.batch + 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // Prologue before the PDL wait (as in decode_pass1_kernel): lengths, page table
    // window, and the first units' K/V except any unit holding a sequence's newest token.
    block_page_prefix<16>(p.context_lens, p.batch, prefix, lens, warp_tot);
    __syncthreads();
    const int Hkv = p.kv_heads;
    const long long W = (long long)Hkv * prefix[p.batch];
    const long long chunk = W > 0 ? (W + p.num_splits - 1) / p.num_splits : 1;
    const long long r0 = (long long)blockIdx.x * chunk;
    const long long r1 = min(W, r0 + chunk);
    const long long n_mine = r1 - r0 > warp ? (r1 - r0 - warp + NW - 1) / NW : 0;

    // lane l holds the index of the 16-row chunk (page, kv head, half of a 32-token page)
    // of this warp's unit win0 + l: (page * Hkv + head) * U + row block; -1 for a page
    // outside the table or the pool
    auto load_window = [&](long long win0) {
        const long long k = win0 + lane;
        int id = -1;
        if (k < n_mine) {
            int bb, gg, jj;
            locate_unit(r0 + warp + k * NW, prefix, p.batch, Hkv, bb, gg, jj);
            const int pg = jj / U;
            const int page = pg < p.max_pages ? p.block_tables[(long long)bb * p.max_pages + pg] : -1;
            if ((unsigned)page < (unsigned)p.num_pages) id = (page * Hkv + gg) * U + jj % U;
        }
        return id;
    };
    long long win0 = 0;
    int win = load_window(0);
    const int ring_off = warp * DEPTH * S::kSlot;

    int ib = 0, ig = 0, ij = 0, inp = 1, qb = -1, qg = -1;
    if (n_mine > 0) {
        locate_unit(r0 + warp, prefix, p.batch, Hkv, ib, ig, ij);
        inp = prefix[ib + 1] - prefix[ib];
    }
    auto issue_kv = [&](long long k) {
        if (k >= win0 + 32) {
            win0 = k;
            win = load_window(k);
        }
        const int ci = __shfl_sync(0xffffffffu, win, (int)(k - win0));
        unsigned char* slot = smem + ring_off + (int)(k % DEPTH) * S::kSlot;
        if (ci >= 0) {
            const long long off = (long long)ci * (16 * D);
            const unsigned char* ks = reinterpret_cast<const unsigned char*>(static_cast<const T*>(p.k) + off);
            const unsigned char* vs = reinterpret_cast<const unsigned char*>(static_cast<const T*>(p.v) + off);
#pragma unroll
            for (int n = 0; n < S::kChunk / 512; ++n) {
                const int gidx = n * 32 + lane;
                const int t = gidx / CPR, c = gidx % CPR;
                const int dst = t * (2 * D) + ((c ^ (t & 7)) * 16);
                cp_async16(slot + dst, ks + gidx * 16);
                cp_async16(slot + S::kChunk + dst, vs + gidx * 16);
            }
        } else if (lane == 0) {
            atomicOr(&g_error_word, PKV_DEVERR_BAD_PAGE);   // never dereferenced
        }
    };
    auto issue_q = [&](long long k, int bq, int gq) {
        unsigned char* slot = smem + ring_off + (int)(k % DEPTH) * S::kSlot;
        const unsigned char* qs = reinterpret_cast<const unsigned char*>(
            static_cast<const T*>(p.q) + ((long long)bq * p.q_heads + (long long)gq * G) * D);
        for (int n = lane; n < QV; n += 32) cp_async16(slot + 2 * S::kChunk + n * 16, qs + n * 16);
    };
    auto advance = [&]() {
        if (ij + NW < inp) {
            ij += NW;
        } else {
            for (int t = 0; t < NW; ++t) next_unit(ib, ig, ij, inp, prefix, Hkv, p.batch);
        }
    };
    auto issue = [&](long long k) {
        issue_kv(k);
        if (ib != qb || ig != qg) {
            qb = ib;
            qg = ig;
            issue_q(k, ib, ig);
        }
        advance();
    };
    if (n_mine > 0) prefetch_q_rows<D, G, T>(p, ib, ig, lane);     // this warp's first segment
    if (r0 < r1) prefetch_epilogue_lines<D, G>(p, r0, chunk, prefix, tid);
    int m_pre = 0, pre_qb[DEPTH], pre_qg[DEPTH];
    for (; m_pre < DEPTH && m_pre < n_mine; ++m_pre) {
        if (ij == inp - 1) break;
        issue_kv(m_pre);
        pre_qb[m_pre] = -1;
        if (ib != qb || ig != qg) {
            qb = ib;
            qg = ig;
            pre_qb[m_pre] = ib;
            pre_qg[m_pre] = ig;
        }
        advance();
        cp_async_commit();
    }

    pdl_wait();
    pdl_launch_dependents();
    for (int b = blockIdx.x; b < p.batch; b += gridDim.x) {
        if (prefix[b + 1] != prefix[b]) continue;
        T* row = static_cast<T*>(p.out) + (long long)b * p.q_heads * D;
        for (int idx = tid; idx < p.q_heads * D; idx += blockDim.x) row[idx] = Elt<T>::from_float(0.f);
    }
    if (r0 >= r1) return;

    unsigned char* ring = smem + ring_off;
    for (int k = 0; k < m_pre; ++k)
        if (pre_qb[k] >= 0) issue_q(k, pre_qb[k], pre_qg[k]);
    if (m_pre == DEPTH) cp_async_commit();
    for (int k = m_pre; k < DEPTH; ++k) {
        if (k < n_mine) issue(k);
        cp_async_commit();
    }
    cp_async_wait<0>();

    // ---- compute side (fragments of m16n8k16: g4 = lane / 4, t4 = lane % 4)
    const int g4 = lane >> 2, t4 = lane & 3;
    // ldmatrix row addresses: lane l supplies row (l & 7) + 8 * ((l >> 3) & 1) of matrix
    // l >> 3 for the K tile (A, non-transposed), row (l & 7) + 8 * (l >> 4) for V (A^T).
    const int k_row = (lane & 7) + 8 * ((lane >> 3) & 1), k_chunk_hi = lane >> 4;
    const int v_row = (lane & 7) + 8 * (lane >> 4), v_chunk_hi = (lane >> 3) & 1;
    uint32_t bq[KS][2];                       // Q^T fragments of the segment (heads >= G are 0)
    float oacc[KS][4], m_run[2], l_run[2];    // O^T[d][head], running max/sum of heads 2 t4 + j
#pragma unroll
    for (int mt = 0; mt < KS; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[mt][e] = 0.f;
    m_run[0] = m_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.f;
    long long kc = 0;
    int b, g, j;
    locate_unit(r0, prefix, p.batch, Hkv, b, g, j);
    int np = prefix[b + 1] - prefix[b];
    int seg = 0;
    for (long long u = r0; u < r1; ++seg) {
        const long long u_end = min(r1, u + (np - j));
        const long long first = u + ((warp - (int)((u - r0) % NW)) + NW) % NW;
        bool have_q = false;
        for (long long uu = first; uu < u_end; uu += NW) {
            cp_async_wait<DEPTH - 1>();
            __syncwarp();
            unsigned char* s = ring + (int)(kc % DEPTH) * S::kSlot;
            if (!have_q) {
                have_q = true;
                const unsigned char* qa = s + 2 * S::kChunk;
#pragma unroll
                for (int kk = 0; kk < KS; ++kk) {
                    bq[kk][0] = g4 < G ? *reinterpret_cast<const uint32_t*>(qa + (g4 * D + kk * 16 + 2 * t4) * 2) : 0u;
                    bq[kk][1] = g4 < G ? *reinterpret_cast<const uint32_t*>(qa + (g4 * D + kk * 16 + 8 + 2 * t4) * 2)
                                       : 0u;
                }
            }
            const int nvalid = min(16, lens[b] - (j + (int)(uu - u)) * 16);
            if (nvalid < 16) {
                // rows past the context may hold anything: zero them in V (their p is 0,
                // but 0 * NaN would poison the MMA)
                for (int x = lane; x < (16 - nvalid) * CPR; x += 32)
                    reinterpret_cast<uint4*>(s + S::kChunk + nvalid * (2 * D))[x] = make_uint4(0, 0, 0, 0);
                __syncwarp();
            }
            // ---- S^T = K . Q^T, the k-steps spread over kScoreChains independent accumulators
            //      so that consecutive MMAs do not wait on one another
            constexpr int SCH = KS < kScoreChains ? KS : kScoreChains;
            float sacc_c[SCH][4];
#pragma unroll
            for (int c = 0; c < SCH; ++c)
#pragma unroll
                for (int e = 0; e < 4; ++e) sacc_c[c][e] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                uint32_t a[4];
                const int ch = 2 * kk + k_chunk_hi;
                ldmatrix_x4(a, s + k_row * (2 * D) + ((ch ^ (k_row & 7)) * 16));
                MmaOps<T>::mma(sacc_c[kk % SCH], a, bq[kk][0], bq[kk][1]);
            }
            float sacc[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                sacc[e] = sacc_c[0][e];
#pragma unroll
                for (int c = 1; c < SCH; ++c) sacc[e] += sacc_c[c][e];
            }
            // ---- online softmax: sacc = (token g4, heads 2t4, 2t4+1), (token g4 + 8, same heads)
            float sc[4];
            sc[0] = g4 < nvalid ? sacc[0] * p.scale_log2 : -INFINITY;
            sc[1] = g4 < nvalid ? sacc[1] * p.scale_log2 : -INFINITY;
            sc[2] = g4 + 8 < nvalid ? sacc[2] * p.scale_log2 : -INFINITY;
            sc[3] = g4 + 8 < nvalid ? sacc[3] * p.scale_log2 : -INFINITY;
            float alpha[2], pr[4];
#pragma unroll
            for (int jh = 0; jh < 2; ++jh) {
                float pm = fmaxf(sc[jh], sc[jh + 2]);
#pragma unroll
                for (int m = 4; m < 32; m <<= 1) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, m));
                const float mn = fmaxf(m_run[jh], pm);         // finite: row 0 is always valid
                alpha[jh] = fast_exp2(m_run[jh] - mn);
                m_run[jh] = mn;
                pr[jh] = fast_exp2(sc[jh] - mn);
                pr[jh + 2] = fast_exp2(sc[jh + 2] - mn);
                l_run[jh] = l_run[jh] * alpha[jh] + pr[jh] + pr[jh + 2];
            }
            if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
                for (int mt = 0; mt < KS; ++mt) {
                    oacc[mt][0] *= alpha[0];
                    oacc[mt][1] *= alpha[1];
                    oacc[mt][2] *= alpha[0];
                    oacc[mt][3] *= alpha[1];
                }
            }
            // ---- P^T as the B operand: transpose the 8x8 blocks (tokens 0-7, 8-15).  With
            //      bf16 inputs P is carried as hi + lo bf16 parts (two MMAs on the same V
            //      fragments), keeping ~16 bits of P instead of bf16's 8.
            const uint32_t h01 = MmaOps<T>::pack(pr[0], pr[1]), h23 = MmaOps<T>::pack(pr[2], pr[3]);
            const uint32_t pb0 = movmatrix_trans(h01), pb1 = movmatrix_trans(h23);
            constexpr bool kSplitP = std::is_same<T, __nv_bfloat16>::value;
            uint32_t pl0 = 0, pl1 = 0;
            if constexpr (kSplitP) {
                pl0 = movmatrix_trans(MmaOps<T>::pack(pr[0] - __uint_as_float(h01 << 16),
                                                      pr[1] - __uint_as_float(h01 & 0xffff0000u)));
                pl1 = movmatrix_trans(MmaOps<T>::pack(pr[2] - __uint_as_float(h23 << 16),
                                                      pr[3] - __uint_as_float(h23 & 0xffff0000u)));
            }
            // ---- O^T += V^T . P^T
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                uint32_t a[4];
                const int ch = 2 * mt + v_chunk_hi;
                ldmatrix_x4_trans(a, s + S::kChunk + v_row * (2 * D) + ((ch ^ (v_row & 7)) * 16));
                MmaOps<T>::mma(oacc[mt], a, pb0, pb1);
                if constexpr (kSplitP) MmaOps<T>::mma(oacc[mt], a, pl0, pl1);
            }
            __syncwarp();
            if (kc + DEPTH < n_mine) issue(kc + DEPTH);
            cp_async_commit();
            ++kc;
        }
        // ---- publish this warp's state: o[head][d], m, l of the real heads
        float* buf = cmb + (seg & 1) * S::kCmbFloats;
#pragma unroll
        for (int jh = 0; jh < 2; ++jh) {
            float lt = l_run[jh];
#pragma unroll
            for (int m = 4; m < 32; m <<= 1) lt += __shfl_xor_sync(0xffffffffu, lt, m);
            const int head = 2 * t4 + jh;
            if (head < G) {
                float* row = buf + (warp * G + head) * (D + 2);
#pragma unroll
                for (int mt = 0; mt < KS; ++mt) {
                    row[mt * 16 + g4] = oacc[mt][jh];
                    row[mt * 16 + 8 + g4] = oacc[mt][2 + jh];
                }
                if (g4 == 0) {
                    row[D] = m_run[jh];
                    row[D + 1] = lt;
                }
            }
            m_run[jh] = -INFINITY;
            l_run[jh] = 0.f;
        }
#pragma unroll
        for (int mt = 0; mt < KS; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) oacc[mt][e] = 0.f;
        segment_epilogue<D, G, T>(p, buf, b, g, np, prefix, r0, r1, chunk, last_flag);
        u = u_end;
        j = 0;
        if (++g == Hkv) {
            g = 0;
            do {
                ++b;
                np = b < p.batch ? prefix[b + 1] - prefix[b] : 1;
            } while (np == 0);
        }
    }
    cp_async_wait<0>();
}

}  // namespace pkv

#endif  // PKV_DECODE_ATTENTION_MMA_CUH_
