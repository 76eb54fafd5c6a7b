// Chunked prefill attention over the paged KV cache on the fifth-generation tensor cores.
//
// "为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427) s4.3: the forward of a chunk
// of seq_len new tokens at start_pos appends their k, v to the cache and applies the
// causal mask slice [start_pos : start_pos + seq_len, : start_pos + seq_len] -- query row i
// sees keys 0 .. start_pos + i.  A chunk makes the contraction dense, so it runs on
// tcgen05: one elected thread issues the MMAs, operands come from shared memory, the
// accumulators live in tensor memory (TMEM).
//
// Work: one CTA of 256 threads per (sequence, kv head, tile of 128 rows), a row being one
// (query token, query head of the group) pair.  Two threads share a row: thread t takes
// row t % 128 (TMEM lane t % 128, which warps w and w + 4 both reach) and half t / 128 of
// the row's key columns and of its O columns.  Per block of NK keys (64 for fp16; 32 for
// bf16, whose P takes two buffers):
//   S[128 x NK] = Q . K^T          tcgen05.mma kind::f16, M 128, N NK, D/16 k-steps -> TMEM
//   each thread: its half of the S row from TMEM, causal mask, its half's max, combined
//                with the partner's through a per-row shared-memory slot; fp32 online
//                softmax (log2 domain) against a reference max that moves only when the
//                row max passes it by more than 2^8, so O is rarely rescaled; its half of
//                P written to shared memory, its half of the O row rescaled in TMEM when
//                the reference moved
//   O[128 x D] += P . V            M 128, N D, NK/16 k-steps (bf16: P as hi + lo, twice)
// Shared memory uses the 128-byte-swizzle canonical layouts: Q, K and P K-major (rows of
// 128 bytes, 16-byte chunk c of row r at c ^ (r & 7), 8-row atoms 1024 bytes apart, a
// region per 64 columns), V MN-major -- which is the same bytes as K's layout read with
// the other major-ness, so K and V blocks are staged identically: one thread each issues
// tiled TMA copies (a 64-column region of one page per copy) into two-stage rings, counted
// in bytes on a barrier per stage.  K(b) is refilled as soon as S(b) is done, V(b) as soon
// as P.V(b) is; V rows past the cache are zeroed after their copy lands.  S has two TMEM
// buffers: at the end of block b warp 0 (one elected lane) issues P.V(b), then S(b + 2)
// into the buffer block b has emptied, so S of the next block is already on hand when its
// softmax starts.  Every wait on an MMA or a copy is bounded: on timeout the kernel sets
// PKV_DEVERR_TIMEOUT, skips its output, waits (bounded) for its copies in flight and still
// frees its TMEM.
#ifndef PKV_PREFILL_ATTENTION_TC_CUH_
#define PKV_PREFILL_ATTENTION_TC_CUH_

#include <cuda/ptx>
#include <type_traits>

#include "prefill_attention.cuh"

namespace pkv {

constexpr int kTcRows = 128;          // query rows per CTA (= TMEM lanes)
constexpr int kTcThreads = 256;       // two threads per row
constexpr float kLazyLog2 = 8.f;      // the softmax reference max moves only by more than this (log2)
template <int D, bool kSplitP>
struct TcShape {
    static constexpr int kKeys = kSplitP ? 32 : 64;             // keys per block
    static constexpr int kQBytes = kTcRows * D * 2;             // Q, D/64 regions of 128 rows x 128 B
    static constexpr int kRegion = kKeys * 128;                 // one 64-column region of a K (or V) block
    static constexpr int kKvBytes = (D / 64) * kRegion;         // one K (or V) block
    static constexpr int kPBytes = kTcRows * 128;               // one P buffer: 128 rows of 128 B
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQOff + kQBytes;               // K ring, 2 stages
    static constexpr int kVOff = kKOff + 2 * kKvBytes;          // V ring, 2 stages
    static constexpr int kPOff = kVOff + 2 * kKvBytes;
    static constexpr int kBarOff = kPOff + (kSplitP ? 2 : 1) * kPBytes;
    static constexpr int kBytes = kBarOff + 64;                 // 6 mbarriers, TMEM base, abort flag
    // after the fixed part: the work-item prefix [batch + 1] ints, reused once it has been
    // searched as the per-row max slots [kTcRows] (so at least kTcRows ints)
    static constexpr int kTailMin = kTcRows * 4;
    static constexpr uint32_t kTmemCols = D + 2 * kKeys <= 128 ? 128u : 256u;   // O at 0, S twice from D
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

// Order-preserving code of a float as an unsigned int (a > b as floats iff code(a) > code(b))
__device__ __forceinline__ uint32_t float_order_code(float f)
{
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float float_from_order_code(uint32_t c)
{
    return __uint_as_float((c & 0x80000000u) ? (c & 0x7fffffffu) : ~c);
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
__global__ void __launch_bounds__(kTcThreads, 2) prefill_tc_kernel(const __grid_constant__ PrefillParams p)
{
    namespace ptx = cuda::ptx;
    constexpr bool kSplitP = std::is_same<T, __nv_bfloat16>::value;
    using S = TcShape<D, kSplitP>;
    constexpr int CPR = D / 8;                 // 16-byte chunks per row
    constexpr int KS = D / 16;                 // k-steps of Q.K^T
    constexpr int CT = kTcRows / G;            // query tokens per CTA tile
    constexpr int NK = S::kKeys;               // keys per block
    constexpr int NKH = NK / 2;                // keys of a block per thread
    constexpr int DH = D / 2;                  // O columns per thread
    constexpr int NPB = NK / P;                // pages per block
    constexpr uint32_t kPageBytes = (D / 64) * P * 128;   // one page of one block (all its regions)
    static_assert(G >= 1 && G <= 16 && 16 % G == 0, "group size");
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(NK % P == 0 && NKH % 8 == 0 && DH % 32 == 0, "tiling");
    extern __shared__ __align__(1024) unsigned char tc_smem[];    // own name: other kernels align theirs to 128
    unsigned char* const smem = tc_smem;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int r = tid & (kTcRows - 1);         // this thread's row (TMEM lane)
    const int half = tid / kTcRows;            // which half of the key and O columns
    const int pair_bar = 1 + (warp & 3);       // named barrier of warps w and w + 4 (rows of one lane quarter)
    const bool k_loader = tid == 32, v_loader = tid == 64;
    uint64_t* bar_s = reinterpret_cast<uint64_t*>(smem + S::kBarOff);   // [2]: S buffer done
    uint64_t* bar_o = bar_s + 2;
    uint64_t* full_k = bar_s + 3;              // [2]: K stage landed
    uint64_t* full_v = bar_s + 5;              // [2]: V stage landed
    uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + S::kBarOff + 56);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kBarOff + 60);
    int* items = reinterpret_cast<int*>(smem + S::kBytes);   // [batch + 1] after the fixed part
    uint32_t* mslot = reinterpret_cast<uint32_t*>(smem + S::kBytes);   // the same bytes, later
    const int Hkv = p.kv_heads;

    if (tid == 0) {
        int run = 0;
        for (int b = 0; b < p.batch; ++b) {
            items[b] = run;
            const int n = p.cu_q[b + 1] - p.cu_q[b];
            run += n > 0 ? Hkv * ((n * G + kTcRows - 1) / kTcRows) : 0;
        }
        items[p.batch] = run;
        *abort_flag = (smem_addr(smem) & 1023u) != 0;     // the swizzle atoms need 1024-byte alignment
        for (int i = 0; i < 7; ++i) mbar_init(bar_s + i, 1);
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
    int lo = 0, hi = p.batch - 1;               // sequence of the item
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (items[mid] <= item) lo = mid;
        else hi = mid - 1;
    }
    const int b = lo;
    const int q0 = p.cu_q[b], n_b = p.cu_q[b + 1] - q0;
    const int tiles = (n_b * G + kTcRows - 1) / kTcRows;
    const int g = (item - items[b]) / tiles;
    const int tile = tiles - 1 - (item - items[b]) % tiles;     // later (longer) tiles first
    const int L = p.context_lens[b];
    const int start = L - n_b;
    const int cta_last = min(n_b - 1, tile * CT + CT - 1);
    const int n_blocks = (start + cta_last) / NK + 1;

    // this thread's row
    const int tok = tile * CT + r / G;
    const bool rvalid = tok < n_b;
    const int pos = rvalid ? start + tok : -1;
    const long long row_elt = ((long long)(q0 + (rvalid ? tok : 0)) * p.q_heads + g * G + r % G) * D;

    unsigned char* qs = smem + S::kQOff;
    unsigned char* kring = smem + S::kKOff;
    unsigned char* vring = smem + S::kVOff;
    unsigned char* ps = smem + S::kPOff;
    // ---- K and V blocks: one thread each issues the block's TMA copies, a 64-column region
    //      of a page at a time, into the stage's canonical swizzled layout, and counts the
    //      bytes on the stage's barrier.  Page ids are fetched a block ahead.  Pages past the
    //      cache are not read; a page id out of range is flagged and never read.
    const int32_t* table = p.block_tables + (long long)b * p.max_pages;
    auto fetch_ids = [&](int blk, int (&ids)[NPB]) {
#pragma unroll
        for (int j = 0; j < NPB; ++j) {
            const int pg = blk * NPB + j;
            ids[j] = pg * P < L ? (pg < p.max_pages ? table[pg] : -1) : -2;
        }
    };
    auto tma_block = [&](const CUtensorMap* map, unsigned char* dst_block, uint64_t* full, const int (&ids)[NPB]) {
        uint32_t bytes = 0;
#pragma unroll
        for (int j = 0; j < NPB; ++j) bytes += (unsigned)ids[j] < (unsigned)p.num_pages ? kPageBytes : 0u;
        mbar_arrive_expect_tx(full, bytes);
#pragma unroll
        for (int j = 0; j < NPB; ++j) {
            if ((unsigned)ids[j] < (unsigned)p.num_pages) {
#pragma unroll
                for (int rg = 0; rg < D / 64; ++rg)
                    tma_load_4d(dst_block + rg * S::kRegion + j * P * 128, map, 64 * rg, 0, g, ids[j], full);
            } else if (ids[j] != -2) {
                atomicOr(&g_error_word, PKV_DEVERR_BAD_PAGE);
            }
        }
    };
    int ids_a[NPB];                             // the next block the loader copies
    int issued = 0;                             // blocks this loader has copied: 0 .. issued - 1
    if (k_loader) {
        fetch_ids(0, ids_a);
        tma_block(&p.k_map, kring, full_k, ids_a);
        issued = 1;
        if (n_blocks > 1) {
            fetch_ids(1, ids_a);
            tma_block(&p.k_map, kring + S::kKvBytes, full_k + 1, ids_a);
            issued = 2;
        }
        fetch_ids(2, ids_a);
    }
    if (v_loader) {
        fetch_ids(0, ids_a);
        tma_block(&p.v_map, vring, full_v, ids_a);
        issued = 1;
        fetch_ids(1, ids_a);
    }
    // ---- this thread's half of its Q row -> shared memory (K-major, swizzled); rows past
    //      the chunk are zero
    {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(p.q) + row_elt);
#pragma unroll
        for (int cc = 0; cc < CPR / 2; ++cc) {
            const int c = half * (CPR / 2) + cc;
            const uint4 v = rvalid ? src[c] : make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(qs + (c / 8) * (kTcRows * 128) + r * 128 + (((c % 8) ^ (r & 7)) * 16)) = v;
        }
    }

    // ---- TMEM
    const uint32_t tmem_cols = S::kTmemCols;
    if (warp == 0) {
        ptx::tcgen05_alloc(ptx::cta_group_1, tslot, tmem_cols);
        ptx::tcgen05_relinquish_alloc_permit(ptx::cta_group_1);
    }
    const uint32_t idesc_s = umma_idesc<T>(kTcRows, NK, false);
    const uint32_t idesc_o = umma_idesc<T>(kTcRows, D, true);
    // Base descriptors; an operand's start moves by adding (bytes >> 4) to the low field
    // (every address stays below 256 KB, so the 14-bit field never carries).
    const uint64_t dq = umma_desc_sw128(smem_addr(qs), 16, 1024);
    const uint64_t dk = umma_desc_sw128(smem_addr(kring), 16, 1024);
    const uint64_t dv = umma_desc_sw128(smem_addr(vring), S::kRegion, 1024);
    const uint64_t dp = umma_desc_sw128(smem_addr(ps), 16, 1024);
    // S = Q . K^T of block blk into the S columns
    auto issue_s = [&](int blk, uint32_t tm) {
        const uint32_t kst = (blk & 1) * S::kKvBytes;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            const uint64_t ad = dq + (((kk / 4) * (kTcRows * 128) + (kk % 4) * 32) >> 4);
            const uint64_t bd = dk + ((kst + (kk / 4) * S::kRegion + (kk % 4) * 32) >> 4);
            umma_f16_elected(tm + D + (blk & 1) * NK, ad, bd, idesc_s, kk > 0);
        }
        umma_commit_elected(bar_s + (blk & 1));
    };
    int timed_out = 0;                           // this thread gave up on a wait; every exit is decided
                                                 // by a barrier over all threads, so it is uniform
    if (tid == 0 && (!mbar_wait_parity_bounded(full_k, 0) ||
                     (n_blocks > 1 && !mbar_wait_parity_bounded(full_k + 1, 0)))) {     // K0, K1 landed
        timed_out = 1;
        atomicOr(&g_error_word, PKV_DEVERR_TIMEOUT);
    }
    fence_proxy_async_smem();
    ptx::tcgen05_fence_before_thread_sync();
    bool ok = !__syncthreads_or(timed_out);      // Q, K0 and the TMEM base ready; items searched
    ptx::tcgen05_fence_after_thread_sync();
    const uint32_t tmem = *tslot;
    const uint32_t t_row = tmem + ((uint32_t)(32 * (warp & 3)) << 16);   // this warp's lane quarter
    if (warp == 0 && ok) {                       // the whole warp: one elected lane issues
        issue_s(0, tmem);
        if (n_blocks > 1) issue_s(1, tmem);
    }
    // The row's max slot holds the running max over both halves' blocks so far; it only
    // grows, so it needs no reset, and the CTA barrier that ends an iteration keeps either
    // half from raising it for the next block before its partner has read it.
    if (half == 0) mslot[r] = float_order_code(-INFINITY);
    named_barrier(pair_bar, 64);

    float m_run = -INFINITY, l_run = 0.f;        // l_run: this half's share of the row sum
    const float sc = p.scale_log2 != 0.f ? p.scale_log2 : 1e-30f;   // zero: uniform weights, no 0 * inf
    const float sgn_inf = sc >= 0.f ? -INFINITY : INFINITY;          // a masked score's raw value
    for (int blk = 0; ok && blk < n_blocks; ++blk) {
        // ---- this half of the S row of this block from TMEM
        if (!mbar_wait_parity_bounded(bar_s + (blk & 1), (blk >> 1) & 1)) {
            timed_out = 1;
            atomicOr(&g_error_word, PKV_DEVERR_TIMEOUT);
        }
        ptx::tcgen05_fence_after_thread_sync();
        float sv[NKH];
        {
            uint32_t r0[NKH];
            ptx::tcgen05_ld_32x32b(r0, t_row + D + (blk & 1) * NK + half * NKH);
            ptx::tcgen05_wait_ld();
#pragma unroll
            for (int i = 0; i < NKH; ++i) sv[i] = __uint_as_float(r0[i]);
        }
        // K stage blk & 1 is free again (S(blk) is done): fetch K(blk + 2) into it
        if (k_loader) {
            if (blk + 2 < n_blocks) {
                tma_block(&p.k_map, kring + (blk & 1) * S::kKvBytes, full_k + (blk & 1), ids_a);
                issued = blk + 3;
            }
            fetch_ids(blk + 3, ids_a);           // used an iteration from now
        }
        // ---- causal mask and this half's max.  The max is taken over the raw scores (max
        //      of s * c is max(s) * c for c > 0, min(s) * c otherwise).
        const int key0 = blk * NK + half * NKH;
        if (__any_sync(0xffffffffu, key0 + NKH - 1 > pos)) {    // some key of this half is past a row
#pragma unroll
            for (int i = 0; i < NKH; ++i) sv[i] = key0 + i <= pos ? sv[i] : sgn_inf;
        }
        float ext;
        {
            float e8[8];                         // eight independent chains, then a tree
#pragma unroll
            for (int k = 0; k < 8; ++k) e8[k] = sv[k];
            if (sc >= 0.f) {
#pragma unroll
                for (int i = 8; i < NKH; i += 8)
#pragma unroll
                    for (int k = 0; k < 8; ++k) e8[k] = fmaxf(e8[k], sv[i + k]);
#pragma unroll
                for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
                    for (int k = 0; k < w; ++k) e8[k] = fmaxf(e8[k], e8[k + w]);
            } else {
#pragma unroll
                for (int i = 8; i < NKH; i += 8)
#pragma unroll
                    for (int k = 0; k < 8; ++k) e8[k] = fminf(e8[k], sv[i + k]);
#pragma unroll
                for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
                    for (int k = 0; k < w; ++k) e8[k] = fminf(e8[k], e8[k + w]);
            }
            ext = e8[0];
        }
        // ---- the row's max: both halves raise the slot, then read it back.  The reference
        //      m_run the weights are taken against moves only when the max passes it by more
        //      than kLazyLog2 (the result does not depend on the reference; weights stay
        //      <= 2^kLazyLog2, well inside fp16), so O is rarely rescaled.
        atomicMax(&mslot[r], float_order_code(ext * sc));   // -inf when every key of the half is masked
        named_barrier(pair_bar, 64);
        const float mt = float_from_order_code(mslot[r]);
        float alpha = 1.f;
        if (mt > m_run + kLazyLog2) {            // never while mt is -inf
            alpha = fast_exp2(m_run - mt);       // 0 when m_run was -inf
            m_run = mt;
        }
        const float mn = m_run;
        const bool none = mn == -INFINITY;       // no visible key yet (or a row past the chunk)
        float2 ls2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        if (none) {
#pragma unroll
            for (int i = 0; i < NKH; ++i) sv[i] = 0.f;
        } else {
            const float2 c2 = make_float2(sc, sc), nm2 = make_float2(-mn, -mn);
#pragma unroll
            for (int i = 0; i < NKH; i += 2) {
                const float2 t = __ffma2_rn(make_float2(sv[i], sv[i + 1]), c2, nm2);
                sv[i] = fast_exp2(t.x);
                sv[i + 1] = fast_exp2(t.y);
                ls2[(i >> 1) & 3] = __fadd2_rn(ls2[(i >> 1) & 3], make_float2(sv[i], sv[i + 1]));
            }
        }
        const float2 lsa = __fadd2_rn(__fadd2_rn(ls2[0], ls2[1]), __fadd2_rn(ls2[2], ls2[3]));
        l_run = l_run * alpha + (lsa.x + lsa.y);
        // ---- the previous P.V must be done before P is rewritten, O rescaled and its V stage refilled
        if (blk > 0) {
            if (!mbar_wait_parity_bounded(bar_o, (blk - 1) & 1)) {
                timed_out = 1;
                atomicOr(&g_error_word, PKV_DEVERR_TIMEOUT);
            }
            ptx::tcgen05_fence_after_thread_sync();
        }
        // V stage (blk + 1) & 1 last held V(blk - 1), whose P.V is complete
        if (v_loader) {
            if (blk + 1 < n_blocks) {
                tma_block(&p.v_map, vring + ((blk + 1) & 1) * S::kKvBytes, full_v + ((blk + 1) & 1), ids_a);
                issued = blk + 2;
            }
            fetch_ids(blk + 2, ids_a);
        }
        // ---- this half of the row of P (and of its low part) -> shared memory, K-major swizzled
#pragma unroll
        for (int cc = 0; cc < NKH / 8; ++cc) {
            const int c = half * (NKH / 8) + cc;
            uint32_t w[4], wl[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a = sv[8 * cc + 2 * e], bb = sv[8 * cc + 2 * e + 1];
                w[e] = MmaOps<T>::pack(a, bb);
                if constexpr (kSplitP)
                    wl[e] = MmaOps<T>::pack(a - __uint_as_float(w[e] << 16), bb - __uint_as_float(w[e] & 0xffff0000u));
            }
            const int off = r * 128 + ((c ^ (r & 7)) * 16);
            *reinterpret_cast<uint4*>(ps + off) = make_uint4(w[0], w[1], w[2], w[3]);
            if constexpr (kSplitP)
                *reinterpret_cast<uint4*>(ps + S::kPBytes + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
        }
        // ---- rescale this half of the warp's O rows
        if (blk > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
            for (int c0 = half * DH; c0 < half * DH + DH; c0 += 64) {
                uint32_t r0[32], r1[32];
                ptx::tcgen05_ld_32x32b(r0, t_row + c0);
                if constexpr (DH >= 64) ptx::tcgen05_ld_32x32b(r1, t_row + c0 + 32);
                ptx::tcgen05_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) r0[i] = __float_as_uint(__uint_as_float(r0[i]) * alpha);
                ptx::tcgen05_st_32x32b(t_row + c0, r0);
                if constexpr (DH >= 64) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) r1[i] = __float_as_uint(__uint_as_float(r1[i]) * alpha);
                    ptx::tcgen05_st_32x32b(t_row + c0 + 32, r1);
                }
            }
            ptx::tcgen05_wait_st();
        }
        // ---- the block holding the end of the cache: its V rows past the cache (stale or
        //      never written) become zeros, so that their zero weights give exact zeros
        const int past = L - blk * NK;           // rows [past, NK) of this block lie past the cache
        if (past < NK) {
            if (!mbar_wait_parity_bounded(full_v + (blk & 1), (blk >> 1) & 1)) {
                timed_out = 1;
                atomicOr(&g_error_word, PKV_DEVERR_TIMEOUT);
            } else {
                unsigned char* vb = vring + (blk & 1) * S::kKvBytes;
                const int chunks = (NK - past) * 8 * (D / 64);
                for (int i = tid; i < chunks; i += kTcThreads) {
                    const int rg = i / ((NK - past) * 8), rest = i % ((NK - past) * 8);
                    *reinterpret_cast<uint4*>(vb + rg * S::kRegion + (past + rest / 8) * 128 + (rest % 8) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
            }
        }
        // ---- the MMA issuer: K(blk + 2) and V(blk) must have landed
        if (tid == 0) {
            if (blk + 2 < n_blocks && !mbar_wait_parity_bounded(full_k + (blk & 1), ((blk + 2) >> 1) & 1))
                timed_out = 1;
            if (!mbar_wait_parity_bounded(full_v + (blk & 1), (blk >> 1) & 1)) timed_out = 1;
            if (timed_out) atomicOr(&g_error_word, PKV_DEVERR_TIMEOUT);
        }
        fence_proxy_async_smem();
        ptx::tcgen05_fence_before_thread_sync();
        const int stop = __syncthreads_or(timed_out);   // P, rescaled O, S reads and block blk + 1 ready
        ptx::tcgen05_fence_after_thread_sync();
        if (stop) { ok = false; break; }
        if (warp == 0) {
            // O += P . V, then S two blocks ahead into the S buffer this block has emptied
            const uint32_t vst = (blk & 1) * S::kKvBytes;
#pragma unroll
            for (int part = 0; part < (kSplitP ? 2 : 1); ++part) {
#pragma unroll
                for (int kk = 0; kk < NK / 16; ++kk) {
                    const uint64_t ad = dp + ((part * S::kPBytes + kk * 32) >> 4);
                    const uint64_t bd = dv + ((vst + kk * 2048) >> 4);
                    umma_f16_elected(tmem, ad, bd, idesc_o, blk > 0 || kk > 0 || part > 0);
                }
            }
            umma_commit_elected(bar_o);
            if (blk + 2 < n_blocks) issue_s(blk + 2, tmem);
        }
    }
    // ---- out = O / l, l being the sum of the two halves' shares
    if (ok) {
        if (!mbar_wait_parity_bounded(bar_o, (n_blocks - 1) & 1)) timed_out = 1;
        ok = !__syncthreads_or(timed_out);
        if (!ok && tid == 0) atomicOr(&g_error_word, PKV_DEVERR_TIMEOUT);
        ptx::tcgen05_fence_after_thread_sync();
        float l_row = 0.f;
        if (ok) {                                // uniform; every MMA has completed, so P's bytes are free
            float* lx = reinterpret_cast<float*>(ps);
            lx[half * kTcRows + r] = l_run;
            named_barrier(pair_bar, 64);
            l_row = lx[r] + lx[kTcRows + r];
        }
        const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
        T* orow = static_cast<T*>(p.out) + row_elt;
#pragma unroll
        for (int c0 = half * DH; c0 < half * DH + DH; c0 += 32) {
            uint32_t rr[32];
            ptx::tcgen05_ld_32x32b(rr, t_row + c0);
            ptx::tcgen05_wait_ld();
            if (ok && rvalid) {
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    uint4 u;
                    uint32_t* uw = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
                    for (int h = 0; h < 4; ++h)
                        uw[h] = MmaOps<T>::pack(__uint_as_float(rr[e + 2 * h]) * inv, __uint_as_float(rr[e + 2 * h + 1]) * inv);
                    *reinterpret_cast<uint4*>(orow + c0 + e) = u;
                }
            }
        }
    }
    // ---- copies still in flight (only after a timeout): each loader waits, bounded, for the
    //      last copy it issued into each stage before the CTA's shared memory is released
    if (k_loader || v_loader) {
        uint64_t* full = k_loader ? full_k : full_v;
        for (int j = max(0, issued - 2); j < issued; ++j) mbar_wait_parity_bounded(full + (j & 1), (j >> 1) & 1);
    }
    ptx::tcgen05_fence_before_thread_sync();
    __syncthreads();
    if (warp == 0) ptx::tcgen05_dealloc(ptx::cta_group_1, tmem, tmem_cols);
}

}  // namespace pkv

#endif  // PKV_PREFILL_ATTENTION_TC_CUH_
