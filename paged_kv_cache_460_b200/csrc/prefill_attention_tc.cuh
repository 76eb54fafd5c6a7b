// Chunked prefill attention over the paged KV cache on the fifth-generation tensor cores.
//
// "为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427) s4.3: the forward of a chunk
// of seq_len new tokens at start_pos appends their k, v to the cache and applies the
// causal mask slice [start_pos : start_pos + seq_len, : start_pos + seq_len] -- query row i
// sees keys 0 .. start_pos + i.  A chunk makes the contraction dense, so it runs on
// tcgen05: one elected lane issues the MMAs, operands come from shared memory, the
// accumulators live in tensor memory (TMEM).
//
// Work: one CTA (one per SM) per pair of 128-row tiles of one (sequence, kv head), a row
// being one (query token, query head of the group) pair, so each K/V block is staged once
// for 256 rows.  The warps specialise and meet only on mbarriers:
//   warps 0-3, 4-7  softmax of tile A, tile B: one thread per row (TMEM lane); per block of
//                   NK keys (64 for fp16; 32 for bf16, whose P takes two buffers) it reads
//                   its S row from TMEM, applies the causal mask, runs the fp32 online
//                   softmax (log2 domain) against a reference max that moves only when the
//                   row max passes it by more than 2^8 (so O is rarely rescaled), writes
//                   its P row to shared memory and signals P ready
//   warp 8          the MMAs, from one elected lane: S_X(b) = Q_X . K(b)^T (M 128, N NK,
//                   D/16 k-steps) into one of two S buffers per tile, and
//                   O_X += P_X(b) . V(b) (M 128, N D, NK/16 k-steps; bf16: P as hi + lo);
//                   S_X(b + 2) goes into the buffer block b emptied as soon as P_X(b) is
//                   ready, so the next scores are on hand when a softmax warp finishes
//   warp 9          tiled TMA copies of K and V blocks (a 64-column region of one page per
//                   copy) into three-stage rings, full and empty barriers per stage; the V
//                   rows past the cache in the last block are zeroed after they land
// TMEM (512 columns): O_A, O_B, then the two S buffers of each tile.  Shared memory holds
// the 128-byte-swizzle canonical layouts: Q, K and P K-major (rows of 128 bytes, 16-byte
// chunk c of row r at c ^ (r & 7), 8-row atoms 1024 bytes apart, a region per 64 columns),
// V MN-major -- the same bytes as K's layout read with the other major-ness.  Every wait is
// bounded and honours a CTA abort flag: on timeout the kernel sets PKV_DEVERR_TIMEOUT, the
// roles stop, wait (bounded) for their copies and MMAs in flight, skip the output and free
// the TMEM.
#ifndef PKV_PREFILL_ATTENTION_TC_CUH_
#define PKV_PREFILL_ATTENTION_TC_CUH_

#include <cuda/ptx>
#include <type_traits>

#include "prefill_attention.cuh"

namespace pkv {

constexpr int kTcRows = 128;          // query rows per tile (= TMEM lanes); two tiles per CTA
constexpr int kTcThreads = 320;       // 8 softmax warps, an MMA warp, a TMA warp
constexpr int kTcStages = 3;          // K and V ring stages
constexpr float kLazyLog2 = 8.f;      // the softmax reference max moves only by more than this (log2)

template <int D, bool kSplitP>
struct TcShape {
    static constexpr int kKeys = kSplitP ? 32 : 64;             // keys per block
    static constexpr int kQBytes = kTcRows * D * 2;             // one tile's Q
    static constexpr int kRegion = kKeys * 128;                 // one 64-column region of a K (or V) block
    static constexpr int kKvBytes = (D / 64) * kRegion;         // one K (or V) block
    static constexpr int kPBytes = kTcRows * 128;               // one P buffer
    static constexpr int kPParts = kSplitP ? 2 : 1;
    static constexpr int kQOff = 0;                             // Q_A, Q_B
    static constexpr int kKOff = kQOff + 2 * kQBytes;
    static constexpr int kVOff = kKOff + kTcStages * kKvBytes;
    static constexpr int kPOff = kVOff + kTcStages * kKvBytes;  // P_A (parts), P_B (parts)
    static constexpr int kBarOff = kPOff + 2 * kPParts * kPBytes;
    // k_full[3] k_empty[3] v_full[3] v_empty[3] v_tail s_full[4] p_ready[2] o_done[2] drain
    static constexpr int kNumBars = 4 * kTcStages + 1 + 4 + 2 + 2 + 1;
    static constexpr int kBytes = kBarOff + kNumBars * 8 + 16;  // + TMEM base, abort flag; then [batch + 1] ints
    static constexpr int kMinBytes = 120 * 1024;                // launched with at least this: one CTA per SM
};

// UMMA shared-memory descriptor, 128-byte swizzle (start, leading and stride byte offsets)
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// kind::f16 instruction descriptor: fp32 accumulator, A and B of the element type,
// A K-major, B K-major or MN-major, M x N
template <typename T>
__host__ __device__ constexpr uint32_t umma_idesc(int m, int n, bool b_mn_major)
{
    constexpr uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ bool mbar_wait_parity_bounded(uint64_t* bar, uint32_t parity)
{
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > kWaitLimitCycles) return false;
    }
}

// tcgen05.mma kind::f16 / tcgen05.commit issued by one elected lane of a converged warp; the
// whole warp computes the (warp-uniform) operands
__device__ __forceinline__ void umma_f16_elected(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 bool accumulate)
{
    asm volatile(
        "{\n\t.reg .pred e, p;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
        "}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit_elected(uint64_t* bar)
{
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t"
        "}" ::"r"(smem_addr(bar))
        : "memory");
}

template <int D, int P, int G, typename T>
__global__ void __launch_bounds__(kTcThreads, 1) prefill_tc_kernel(const __grid_constant__ PrefillParams p)
{
    namespace ptx = cuda::ptx;
    constexpr bool kSplitP = std::is_same<T, __nv_bfloat16>::value;
    using S = TcShape<D, kSplitP>;
    constexpr int CPR = D / 8;                 // 16-byte chunks per row
    constexpr int KS = D / 16;                 // k-steps of Q.K^T
    constexpr int CT = kTcRows / G;            // query tokens per tile
    constexpr int NK = S::kKeys;
    constexpr int NS = kTcStages;
    constexpr int NPB = NK / P;
    constexpr uint32_t kPageBytes = (D / 64) * P * 128;
    static_assert(G >= 1 && G <= 16 && 16 % G == 0, "group size");
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(NK % P == 0 && 2 * D + 4 * NK <= 512, "tiling");
    extern __shared__ __align__(1024) unsigned char tc_smem[];    // own name: other kernels align theirs to 128
    unsigned char* const smem = tc_smem;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
    uint64_t* k_full = bars;
    uint64_t* k_empty = bars + NS;
    uint64_t* v_full = bars + 2 * NS;
    uint64_t* v_empty = bars + 3 * NS;
    uint64_t* v_tail = bars + 4 * NS;
    uint64_t* s_full = bars + 4 * NS + 1;      // [tile * 2 + buffer]
    uint64_t* p_ready = bars + 4 * NS + 5;     // [tile]
    uint64_t* o_done = bars + 4 * NS + 7;      // [tile]
    uint64_t* drain = bars + 4 * NS + 9;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + S::kBarOff + S::kNumBars * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
    int* items = reinterpret_cast<int*>(smem + S::kBytes);
    const int Hkv = p.kv_heads;

    if (tid == 0) {
        int run = 0;
        for (int b = 0; b < p.batch; ++b) {
            items[b] = run;
            const int n = p.cu_q[b + 1] - p.cu_q[b];
            const int tiles = n > 0 ? (n * G + kTcRows - 1) / kTcRows : 0;
            run += Hkv * ((tiles + 1) / 2);
        }
        items[p.batch] = run;
        *abort_flag = (smem_addr(smem) & 1023u) != 0;
        for (int i = 0; i < 4 * NS; ++i) mbar_init(bars + i, 1);
        mbar_init(v_tail, 32);
        for (int i = 0; i < 4; ++i) mbar_init(s_full + i, 1);
        mbar_init(p_ready, kTcRows);
        mbar_init(p_ready + 1, kTcRows);
        mbar_init(o_done, 1);
        mbar_init(o_done + 1, 1);
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();
    const int item = blockIdx.x;
    if (item >= items[p.batch] || *abort_flag) {
        if (tid == 0 && *abort_flag) atomicOr(&g_error_word, PKV_DEVERR_TIMEOUT);
        return;
    }
    int lo = 0, hi = p.batch - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (items[mid] <= item) lo = mid;
        else hi = mid - 1;
    }
    const int b = lo;
    const int q0 = p.cu_q[b], n_b = p.cu_q[b + 1] - q0;
    const int tiles = (n_b * G + kTcRows - 1) / kTcRows;
    const int pairs = (tiles + 1) / 2;
    const int g = (item - items[b]) / pairs;
    const int pair = pairs - 1 - (item - items[b]) % pairs;     // later (longer) pairs first
    const int L = p.context_lens[b];
    const int start = L - n_b;
    // blocks each tile needs (0 for a tile past the chunk)
    auto tile_blocks = [&](int t) {
        if (t >= tiles) return 0;
        const int last = min(n_b - 1, t * CT + CT - 1);
        return (start + last) / NK + 1;
    };
    const int nbk[2] = {tile_blocks(2 * pair), tile_blocks(2 * pair + 1)};
    const int n_all = max(nbk[0], nbk[1]);

    unsigned char* kring = smem + S::kKOff;
    unsigned char* vring = smem + S::kVOff;
    const bool softmax = warp < 8;
    const int X = warp >> 2;                   // softmax: this warp's tile
    const int r = tid & (kTcRows - 1);         // softmax: this thread's row (TMEM lane)
    const int tile = 2 * pair + (softmax ? X : 0);
    const int tok = tile * CT + r / G;
    const bool rvalid = softmax && tile < tiles && tok < n_b;
    const int pos = rvalid ? start + tok : -1;
    const long long row_elt = ((long long)(q0 + (rvalid ? tok : 0)) * p.q_heads + g * G + r % G) * D;
    unsigned char* qs_x = smem + S::kQOff + (softmax ? X : 0) * S::kQBytes;
    unsigned char* ps_x = smem + S::kPOff + (softmax ? X : 0) * S::kPParts * S::kPBytes;

    // ---- Q rows -> shared memory (K-major, swizzled); rows past the chunk are zero
    if (softmax) {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(p.q) + row_elt);
#pragma unroll
        for (int c = 0; c < CPR; ++c) {
            const uint4 v = rvalid ? src[c] : make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(qs_x + (c / 8) * (kTcRows * 128) + r * 128 + (((c % 8) ^ (r & 7)) * 16)) = v;
        }
    }
    if (warp == 8) {
        ptx::tcgen05_alloc(ptx::cta_group_1, tslot, 512u);
        ptx::tcgen05_relinquish_alloc_permit(ptx::cta_group_1);
    }
    fence_proxy_async_smem();
    ptx::tcgen05_fence_before_thread_sync();
    __syncthreads();
    ptx::tcgen05_fence_after_thread_sync();
    const uint32_t tmem = *tslot;
    auto s_col = [&](int t, int blk) { return (uint32_t)(2 * D + (2 * t + (blk & 1)) * NK); };

    if (warp == 9) {
        // ===================== TMA loads =====================
        const int32_t* table = p.block_tables + (long long)b * p.max_pages;
        int issued_k = 0, issued_v = 0;
        for (int j = 0; j < n_all; ++j) {
            const int s = j % NS;
            bool ok = true;
            if (j >= NS) ok = mbar_wait_bounded(k_empty + s, ((j / NS) + 1) & 1, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            int ids[NPB];
#pragma unroll
            for (int jj = 0; jj < NPB; ++jj) {
                const int pg = j * NPB + jj;
                ids[jj] = pg * P < L ? (pg < p.max_pages ? table[pg] : -1) : -2;
            }
            uint32_t bytes = 0;
#pragma unroll
            for (int jj = 0; jj < NPB; ++jj) bytes += (unsigned)ids[jj] < (unsigned)p.num_pages ? kPageBytes : 0u;
            if (lane == 0) {
                mbar_arrive_expect_tx(k_full + s, bytes);
#pragma unroll
                for (int jj = 0; jj < NPB; ++jj) {
                    if ((unsigned)ids[jj] < (unsigned)p.num_pages) {
#pragma unroll
                        for (int rg = 0; rg < D / 64; ++rg)
                            tma_load_4d(kring + s * S::kKvBytes + rg * S::kRegion + jj * P * 128, &p.k_map, 64 * rg, 0, g,
                                        ids[jj], k_full + s);
                    } else if (ids[jj] != -2) {
                        atomicOr(&g_error_word, PKV_DEVERR_BAD_PAGE);
                    }
                }
            }
            ok = true;
            if (j >= NS) ok = mbar_wait_bounded(v_empty + s, ((j / NS) + 1) & 1, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            issued_k = j + 1;
            if (!ok) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(v_full + s, bytes);
#pragma unroll
                for (int jj = 0; jj < NPB; ++jj) {
                    if ((unsigned)ids[jj] < (unsigned)p.num_pages) {
#pragma unroll
                        for (int rg = 0; rg < D / 64; ++rg)
                            tma_load_4d(vring + s * S::kKvBytes + rg * S::kRegion + jj * P * 128, &p.v_map, 64 * rg, 0, g,
                                        ids[jj], v_full + s);
                    }
                }
            }
            issued_v = j + 1;
            // the block holding the end of the cache: its V rows past the cache become zeros
            const int past = L - j * NK;
            if (past < NK) {
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(v_full + s, (j / NS) & 1, abort_flag));
                if (!ok) break;
                unsigned char* vb = vring + s * S::kKvBytes;
                const int chunks = (NK - past) * 8 * (D / 64);
                for (int i = lane; i < chunks; i += 32) {
                    const int rg = i / ((NK - past) * 8), rest = i % ((NK - past) * 8);
                    *reinterpret_cast<uint4*>(vb + rg * S::kRegion + (past + rest / 8) * 128 + (rest % 8) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();
                mbar_arrive(v_tail);
            }
        }
        // copies in flight (only after an abort): wait, bounded, for the last ones into each stage
        for (int j = max(0, issued_k - NS); j < issued_k; ++j) mbar_wait_parity_bounded(k_full + j % NS, (j / NS) & 1);
        for (int j = max(0, issued_v - NS); j < issued_v; ++j) mbar_wait_parity_bounded(v_full + j % NS, (j / NS) & 1);
    } else if (warp == 8) {
        // ===================== MMAs (one elected lane) =====================
        const uint32_t idesc_s = umma_idesc<T>(kTcRows, NK, false);
        const uint32_t idesc_o = umma_idesc<T>(kTcRows, D, true);
        const uint64_t dk = umma_desc_sw128(smem_addr(kring), 16, 1024);
        const uint64_t dv = umma_desc_sw128(smem_addr(vring), S::kRegion, 1024);
        auto issue_s = [&](int t, int blk) {
            const uint64_t dq = umma_desc_sw128(smem_addr(smem + S::kQOff + t * S::kQBytes), 16, 1024);
            const uint32_t kst = (blk % NS) * S::kKvBytes;
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                const uint64_t ad = dq + (((kk / 4) * (kTcRows * 128) + (kk % 4) * 32) >> 4);
                const uint64_t bd = dk + ((kst + (kk / 4) * S::kRegion + (kk % 4) * 32) >> 4);
                umma_f16_elected(tmem + s_col(t, blk), ad, bd, idesc_s, kk > 0);
            }
            umma_commit_elected(s_full + 2 * t + (blk & 1));
        };
        auto issue_pv = [&](int t, int blk) {
            const uint64_t dp = umma_desc_sw128(smem_addr(smem + S::kPOff + t * S::kPParts * S::kPBytes), 16, 1024);
            const uint32_t vst = (blk % NS) * S::kKvBytes;
#pragma unroll
            for (int part = 0; part < S::kPParts; ++part) {
#pragma unroll
                for (int kk = 0; kk < NK / 16; ++kk) {
                    const uint64_t ad = dp + ((part * S::kPBytes + kk * 32) >> 4);
                    const uint64_t bd = dv + ((vst + kk * 2048) >> 4);
                    umma_f16_elected(tmem + t * D, ad, bd, idesc_o, blk > 0 || kk > 0 || part > 0);
                }
            }
            umma_commit_elected(o_done + t);
        };
        bool ok = true;
        // S of the first two blocks
        for (int j = 0; ok && j < min(n_all, 2); ++j) {
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(k_full + j % NS, (j / NS) & 1, abort_flag));
            if (!ok) break;
            ptx::tcgen05_fence_after_thread_sync();
            for (int t = 0; t < 2; ++t)
                if (j < nbk[t]) issue_s(t, j);
            umma_commit_elected(k_empty + j % NS);
        }
        for (int j = 0; ok && j < n_all; ++j) {
            bool v_ready = false;
            for (int t = 0; ok && t < 2; ++t) {
                if (j >= nbk[t]) continue;
                // P_X(j) written, S_X(j) read, O_X rescaled
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(p_ready + t, j & 1, abort_flag));
                if (!ok) break;
                if (!v_ready) {
                    ok = __all_sync(0xffffffffu, mbar_wait_bounded(v_full + j % NS, (j / NS) & 1, abort_flag));
                    if (ok && L - j * NK < NK)
                        ok = __all_sync(0xffffffffu, mbar_wait_bounded(v_tail, 0, abort_flag));
                    if (!ok) break;
                    v_ready = true;
                }
                ptx::tcgen05_fence_after_thread_sync();
                issue_pv(t, j);
            }
            if (!ok) break;
            umma_commit_elected(v_empty + j % NS);
            if (j + 2 < n_all) {
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(k_full + (j + 2) % NS, ((j + 2) / NS) & 1, abort_flag));
                if (!ok) break;
                for (int t = 0; t < 2; ++t)
                    if (j + 2 < nbk[t]) issue_s(t, j + 2);    // into the S buffer block j emptied
                umma_commit_elected(k_empty + (j + 2) % NS);
            }
        }
        // every MMA this warp issued has completed before TMEM is released
        umma_commit_elected(drain);
        mbar_wait_parity_bounded(drain, 0);
    } else {
        // ===================== softmax of tile X, one thread per row =====================
        const int nb = nbk[X];
        const uint32_t t_row = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        const float sc = p.scale_log2 != 0.f ? p.scale_log2 : 1e-30f;
        const float sgn_inf = sc >= 0.f ? -INFINITY : INFINITY;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = nb > 0;
        for (int j = 0; ok && j < nb; ++j) {
            ok = __all_sync(0xffffffffu, mbar_wait_bounded(s_full + 2 * X + (j & 1), (j >> 1) & 1, abort_flag));
            if (!ok) break;
            ptx::tcgen05_fence_after_thread_sync();
            float sv[NK];
            {
                uint32_t r0[32];
                ptx::tcgen05_ld_32x32b(r0, t_row + s_col(X, j));
                if constexpr (NK == 64) {
                    uint32_t r1[32];
                    ptx::tcgen05_ld_32x32b(r1, t_row + s_col(X, j) + 32);
                    ptx::tcgen05_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) sv[32 + i] = __uint_as_float(r1[i]);
                } else {
                    ptx::tcgen05_wait_ld();
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) sv[i] = __uint_as_float(r0[i]);
            }
            const int key0 = j * NK;
            if (__any_sync(0xffffffffu, key0 + NK - 1 > pos)) {
#pragma unroll
                for (int i = 0; i < NK; ++i) sv[i] = key0 + i <= pos ? sv[i] : sgn_inf;
            }
            float ext;
            {
                float e8[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) e8[k] = sv[k];
                if (sc >= 0.f) {
#pragma unroll
                    for (int i = 8; i < NK; i += 8)
#pragma unroll
                        for (int k = 0; k < 8; ++k) e8[k] = fmaxf(e8[k], sv[i + k]);
#pragma unroll
                    for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
                        for (int k = 0; k < w; ++k) e8[k] = fmaxf(e8[k], e8[k + w]);
                } else {
#pragma unroll
                    for (int i = 8; i < NK; i += 8)
#pragma unroll
                        for (int k = 0; k < 8; ++k) e8[k] = fminf(e8[k], sv[i + k]);
#pragma unroll
                    for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
                        for (int k = 0; k < w; ++k) e8[k] = fminf(e8[k], e8[k + w]);
                }
                ext = e8[0];
            }
            const float mt = fmaxf(m_run, ext * sc);
            float alpha = 1.f;
            if (mt > m_run + kLazyLog2) {
                alpha = fast_exp2(m_run - mt);
                m_run = mt;
            }
            const float mn = m_run;
            const bool none = mn == -INFINITY;
            float2 ls2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            if (none) {
#pragma unroll
                for (int i = 0; i < NK; ++i) sv[i] = 0.f;
            } else {
                const float2 c2 = make_float2(sc, sc), nm2 = make_float2(-mn, -mn);
#pragma unroll
                for (int i = 0; i < NK; i += 2) {
                    const float2 t = __ffma2_rn(make_float2(sv[i], sv[i + 1]), c2, nm2);
                    sv[i] = fast_exp2(t.x);
                    sv[i + 1] = fast_exp2(t.y);
                    ls2[(i >> 1) & 3] = __fadd2_rn(ls2[(i >> 1) & 3], make_float2(sv[i], sv[i + 1]));
                }
            }
            const float2 lsa = __fadd2_rn(__fadd2_rn(ls2[0], ls2[1]), __fadd2_rn(ls2[2], ls2[3]));
            l_run = l_run * alpha + (lsa.x + lsa.y);
            // P_X(j - 1) has been consumed and O_X is final for block j - 1
            if (j > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait_bounded(o_done + X, (j - 1) & 1, abort_flag));
                if (!ok) break;
                ptx::tcgen05_fence_after_thread_sync();
            }
#pragma unroll
            for (int c = 0; c < NK / 8; ++c) {
                uint32_t w[4], wl[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float a = sv[8 * c + 2 * e], bb = sv[8 * c + 2 * e + 1];
                    w[e] = MmaOps<T>::pack(a, bb);
                    if constexpr (kSplitP)
                        wl[e] = MmaOps<T>::pack(a - __uint_as_float(w[e] << 16), bb - __uint_as_float(w[e] & 0xffff0000u));
                }
                const int off = r * 128 + ((c ^ (r & 7)) * 16);
                *reinterpret_cast<uint4*>(ps_x + off) = make_uint4(w[0], w[1], w[2], w[3]);
                if constexpr (kSplitP)
                    *reinterpret_cast<uint4*>(ps_x + S::kPBytes + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
            }
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 64) {
                    uint32_t r0[32], r1[32];
                    ptx::tcgen05_ld_32x32b(r0, t_row + X * D + c0);
                    ptx::tcgen05_ld_32x32b(r1, t_row + X * D + c0 + 32);
                    ptx::tcgen05_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        r0[i] = __float_as_uint(__uint_as_float(r0[i]) * alpha);
                        r1[i] = __float_as_uint(__uint_as_float(r1[i]) * alpha);
                    }
                    ptx::tcgen05_st_32x32b(t_row + X * D + c0, r0);
                    ptx::tcgen05_st_32x32b(t_row + X * D + c0 + 32, r1);
                }
                ptx::tcgen05_wait_st();
            }
            fence_proxy_async_smem();
            ptx::tcgen05_fence_before_thread_sync();
            mbar_arrive(p_ready + X);
        }
        // ---- out = O / l
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(o_done + X, (nb - 1) & 1, abort_flag));
        if (ok) {
            ptx::tcgen05_fence_after_thread_sync();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            T* orow = static_cast<T*>(p.out) + row_elt;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t rr[32];
                ptx::tcgen05_ld_32x32b(rr, t_row + X * D + c0);
                ptx::tcgen05_wait_ld();
                if (rvalid) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 u;
                        uint32_t* uw = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
                        for (int h = 0; h < 4; ++h)
                            uw[h] = MmaOps<T>::pack(__uint_as_float(rr[e + 2 * h]) * inv,
                                                    __uint_as_float(rr[e + 2 * h + 1]) * inv);
                        *reinterpret_cast<uint4*>(orow + c0 + e) = u;
                    }
                }
            }
        }
    }
    ptx::tcgen05_fence_before_thread_sync();
    __syncthreads();
    if (warp == 8) {
        ptx::tcgen05_fence_after_thread_sync();
        ptx::tcgen05_dealloc(ptx::cta_group_1, tmem, 512u);
    }
}

}  // namespace pkv

#endif  // PKV_PREFILL_ATTENTION_TC_CUH_
