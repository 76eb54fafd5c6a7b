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
// pair is cut at most at range boundaries.  Inside a CTA, warp w takes units
// w, w + NW, w + 2 NW, ... of the range: a whole page-head per warp, so each per-page
// reduction covers P tokens.  Every warp streams its own pages through a private ring
// of DEPTH shared-memory slots with 16-byte cp.async copies (K chunk, V chunk and, when
// the warp enters a new (sequence, kv head), the group's q rows), DEPTH pages ahead of
// the one it computes; the page ids come from a 32-entry window of the page table that
// the lanes fetch together.  Many independent warp streams keep enough bytes in flight
// to saturate HBM; a single TMA-issuing thread per CTA could not (one bulk copy per
// thread-instruction issue slot capped it near 4 TB/s on this access pattern).
// Per page the warp computes q.k over its lanes' 16-byte column slices, reduces the
// partial dots with a transposed shuffle reduction (each lane ends with one row's
// score), updates an fp32 online softmax (running max m, sum l, unnormalised o) in
// the log2 domain, and accumulates p.V with packed fp32 FMAs.  At the end of a segment
// the warps' (m, l, o) are combined through shared memory: a segment wholly inside the
// range is normalised and written as the output; a cut one is written to one of the
// CTA's two partial slots (2c: it began before the range, 2c+1: it continues after it),
// and the CTA that delivers the last partial of a cut segment (counted with an atomic in
// the workspace, indexed by the segment's first CTA) merges them: M = max m_k,
// out = sum_k 2^(m_k - M) o_k / sum_k 2^(m_k - M) l_k, and resets the counter.
#ifndef PKV_DECODE_ATTENTION_CUH_
#define PKV_DECODE_ATTENTION_CUH_

#include "pkv_device.cuh"
#include "rope_append.cuh"

namespace pkv {

constexpr int kDecodeWarps = 4;
constexpr int kDecodeThreads = kDecodeWarps * 32;
// Two ring slots per warp at page 16 / head_dim 128, three CTAs per SM (the MHA kernel
// is held to 128 registers so that a RoPE/append CTA still fits beside them).  Deeper
// rings (3-5 slots) measured slower on the 10-request, 32-layer decode workload.
constexpr int kRingBudgetBytes = 68 * 1024;
// Partials loaded per merge round.  Eight per round measured slower on every workload: the
// merge is inlined in the segment loop and its registers cost the hot loop spills.
constexpr int kMaxMergeParts = 4;
// Independent accumulators over which the tensor-core kernels spread the k-steps of q.K^T
// (1, 2 and 4 measured within 1.5 % of one another; 2 was the best on the grouped-query and
// the fused int8 workloads).
constexpr int kScoreChains = 2;

struct DecodeParams {
    const void* k;              // this layer's K pool  [pages][kv_heads][P][D]
    const void* v;
    const void* q;              // [batch][q_heads][D]
    void* out;                  // [batch][q_heads][D]
    const int32_t* block_tables;
    const int32_t* context_lens;
    const float* k_scale;       // int8 pools: this layer's row scales [pages][kv_heads][P]
    const float* v_scale;
    const void* k_new;          // fused layer: the new token's k (not yet turned) and v,
    const void* v_new;          //   [batch][kv_heads][D]
    const double* rope;         // fused layer: (cos, sin) of the new token's angles, [batch][D/2][2]
    float* part_o;              // [2 * num_splits][G][D]
    float* part_ml;             // [2 * num_splits][G][2]
    int* counters;              // [num_splits]: partials delivered per cut segment (zero between calls)
    int batch;
    int max_pages;
    int q_heads;
    int kv_heads;
    int num_pages;
    int num_splits;
    int cluster;                // cluster variant: CTAs per (sequence, kv head) cluster
    float scale_log2;           // scale * log2(e)
};

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

// CTAs of `smem` dynamic shared-memory bytes that fit on one SM (228 KB, 1 KB reserved per
// CTA), between 1 and 3 (three is the most the decode kernels are tuned for).
__host__ __device__ constexpr int ctas_per_sm(int smem)
{
    return (228 * 1024) / (smem + 1024) >= 3 ? 3 : ((228 * 1024) / (smem + 1024) < 1 ? 1 : (228 * 1024) / (smem + 1024));
}

// kFused: the fused layer also keeps, per CTA, the angle-table rows of the first two
// sequences its range touches and the new k and v rows of the first two sequence ends in its
// range (kNewRows rows of D elements), so that turning q at a segment's start and the append
// at a sequence's end read shared memory instead of waiting on global loads; the ids of those
// rows follow (kFusedIds ints).
// kCluster: the cluster variant also keeps the CTA's combined state of its piece of the
// segment ([G][D + 2] floats: o, m, l), which the cluster's first CTA reads through
// distributed shared memory.
template <int D, int P, int G, bool kFused = false, bool kCluster = false>
struct DecodeShape {
    static constexpr int kChunk = P * D * 2;                 // bytes of one (page, head)
    static constexpr int kQBytes = G * D * 2;
    static constexpr int kSlot = 2 * kChunk + kQBytes;
    static constexpr int kDepthRaw = kRingBudgetBytes / (kDecodeWarps * kSlot);
    static constexpr int kDepth = kDepthRaw < 2 ? 2 : (kDepthRaw > 8 ? 8 : kDepthRaw);
    static constexpr int kRingBytes = kDecodeWarps * kDepth * kSlot;
    static constexpr int kCmbOffset = kRingBytes;
    static constexpr int kCmbFloats = kDecodeWarps * G * (D + 2);
    static constexpr int kPbufOffset = kCmbOffset + 2 * kCmbFloats * 4;     // [warps][G][P] floats
    static constexpr int kWarpTotOffset = kPbufOffset + kDecodeWarps * G * P * 4;
    static constexpr int kRopeRows = kFused ? 2 : 0;
    static constexpr int kRopeOffset = kWarpTotOffset + 64;                 // [kRopeRows][D/2][2] doubles
    static constexpr int kNewOffset = kRopeOffset + kRopeRows * D * 8;      // [2][k, v][D] of T
    static constexpr int kNewRows = kFused ? 4 : 0;
    static constexpr int kIdsOffset = kNewOffset + kNewRows * D * 2;        // rope b[2], append (b*Hkv+g)[2]
    static constexpr int kPartOffset = kIdsOffset + (kFused ? 16 : 0);     // [G][D + 2] floats (kCluster)
    static constexpr int kScanOffset = kPartOffset + (kCluster ? G * (D + 2) * 4 : 0);
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

// A release/acquire fence at gpu scope: with the CTA barrier before it, the partials that
// the CTA's threads wrote are visible to whichever CTA reads the delivery counter after it.
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Before the PDL wait, pull into L2 the q rows of (b, g)'s query heads (G x D elements of T,
// one 128-byte line per lane), which the kernel reads right after the wait, so that read
// finds them in L2 instead of DRAM.  If the kernel ahead is still writing q, the prefetched
// lines are only an older copy in L2, which its writes update (L2 is the coherence point);
// nothing is read into registers or shared memory before the wait.
template <int D, int G, typename T>
__device__ __forceinline__ void prefetch_q_rows(const DecodeParams& p, int b, int g, int lane)
{
    constexpr int kLines = (G * D * (int)sizeof(T) + 127) / 128;
    const unsigned char* q = reinterpret_cast<const unsigned char*>(static_cast<const T*>(p.q) +
                                                                    ((long long)b * p.q_heads + (long long)g * G) * D);
    if (lane < kLines) prefetch_l2(q + lane * 128);
}

// Before the PDL wait, pull into L2 with the evict-last priority the workspace lines this
// CTA writes at its segment ends -- its two partial slots, and the delivery counters of the
// segments its range cuts (its own index and its first segment's first CTA).  The workspace
// is touched once per call, so the KV stream of a call would otherwise push those lines out
// and the partial stores and counter atomics at the CTA's end, on the kernel's critical path,
// would go to DRAM.  Only L2 lines move; nothing is read or written before the wait.
template <int D, int G>
__device__ __forceinline__ void prefetch_epilogue_lines(const DecodeParams& p, long long r0, long long chunk,
                                                        const int* prefix, int tid)
{
    constexpr int kSlotBytes = 2 * G * D * 4;                       // both partial slots of this CTA
    if (tid < kSlotBytes / 128) {
        prefetch_l2_evict_last(reinterpret_cast<const unsigned char*>(p.part_o + (long long)blockIdx.x * 2 * G * D) +
                               tid * 128);
    } else if (tid == kSlotBytes / 128) {
        prefetch_l2_evict_last(p.part_ml + (long long)blockIdx.x * 2 * G * 2);
    } else if (tid == kSlotBytes / 128 + 1) {
        prefetch_l2_evict_last(p.counters + blockIdx.x);
    } else if (tid == kSlotBytes / 128 + 2) {
        int b, g, j;                                                // the first segment's first CTA
        locate_unit(r0, prefix, p.batch, p.kv_heads, b, g, j);
        const long long seg0 = (long long)p.kv_heads * prefix[b] + (long long)g * (prefix[b + 1] - prefix[b]);
        prefetch_l2_evict_last(p.counters + seg0 / chunk);
    }
}

// End of a segment, after every warp has published its (m, l, o) of it in `buf`
// ([warps][G][D + 2]: o, then m and l): combine the warps; a segment wholly inside the
// CTA's range [r0, r1) is normalised and written as the output, a cut one leaves a
// partial in one of the CTA's two slots (2c: it began before the range, 2c+1: it goes on
// after it), and the CTA that delivers the last partial of a segment merges them:
// M = max m_k, out = sum_k 2^(m_k - M) o_k / sum_k 2^(m_k - M) l_k.  The delivery is
// counted with an atomic in the workspace (indexed by the segment's first CTA); one
// thread publishes the CTA's writes with a gpu-scope release fence (cumulative over the
// barrier) and the merging CTA, after an acquire fence, reads the other partials through
// L2, then resets the counter.
// kCluster: a cut segment's combined state goes to `cpart` ([G][D + 2] in this CTA's shared
// memory) for the cluster's merge (cluster_merge) instead of the workspace.
template <int D, int G, typename T, bool kCluster = false>
__device__ __forceinline__ void segment_epilogue(const DecodeParams& p, const float* buf, int b, int g, int np,
                                                 const int* prefix, long long r0, long long r1, long long chunk,
                                                 volatile int* last_flag, float* cpart = nullptr)
{
    constexpr int NW = kDecodeWarps;
    const int tid = threadIdx.x;
    named_barrier(1, kDecodeThreads);
    const long long seg0 = (long long)p.kv_heads * prefix[b] + (long long)g * np;
    const bool complete = seg0 >= r0 && seg0 + np <= r1;
    const int pslot = seg0 < r0 ? 2 * blockIdx.x : 2 * blockIdx.x + 1;
    for (int idx = tid; idx < G * D; idx += kDecodeThreads) {
        const int gi = idx / D, dd = idx - gi * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, buf[(w * G + gi) * (D + 2) + D]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float* row = buf + (w * G + gi) * (D + 2);
            const float wt = fast_exp2(row[D] - M);   // a warp with no page here has m = -inf
            num = fmaf(wt, row[dd], num);
            den = fmaf(wt, row[D + 1], den);
        }
        if (complete) {
            T* dst = static_cast<T*>(p.out) + ((long long)b * p.q_heads + (long long)g * G + gi) * D + dd;
            *dst = Elt<T>::from_float(num / den);
        } else if constexpr (kCluster) {
            cpart[gi * (D + 2) + dd] = num;
            if (dd == 0) {
                cpart[gi * (D + 2) + D] = M;
                cpart[gi * (D + 2) + D + 1] = den;
            }
        } else {
            p.part_o[((long long)pslot * G + gi) * D + dd] = num;
            if (dd == 0) {
                p.part_ml[((long long)pslot * G + gi) * 2 + 0] = M;
                p.part_ml[((long long)pslot * G + gi) * 2 + 1] = den;
            }
        }
    }
    if (!kCluster && !complete) {
        // Deliver this partial; the CTA that delivers the last one merges the segment.
        // One thread publishes the CTA's writes (a gpu-scope release fence is cumulative
        // over the barrier) and counts them in; the merging CTA reads the other partials
        // through L2.
        const int c0 = (int)(seg0 / chunk), c1 = (int)((seg0 + np - 1) / chunk);
        named_barrier(1, kDecodeThreads);
        if (tid == 0) {
            fence_acq_rel_gpu();          // release: the CTA's partial (ordered by the barrier)
            const bool last = atomicAdd(&p.counters[c0], 1) == c1 - c0;
            if (last) fence_acq_rel_gpu();   // acquire: the other CTAs' partials
            *last_flag = last;
        }
        named_barrier(1, kDecodeThreads);
        if (*last_flag) {
            for (int idx = tid; idx < G * D; idx += kDecodeThreads) {
                const int gi = idx / D, dd = idx - gi * D;
                float mk[kMaxMergeParts], lk[kMaxMergeParts], ok[kMaxMergeParts];
                float M = -INFINITY, num = 0.f, den = 0.f;
                for (int c = c0; c <= c1; c += kMaxMergeParts) {
                    const int n = min(kMaxMergeParts, c1 + 1 - c);
#pragma unroll
                    for (int q = 0; q < kMaxMergeParts; ++q) {      // independent loads
                        if (q < n) {
                            const int sl = c + q == c0 ? 2 * c0 + 1 : 2 * (c + q);
                            mk[q] = __ldcg(&p.part_ml[((long long)sl * G + gi) * 2]);
                            lk[q] = __ldcg(&p.part_ml[((long long)sl * G + gi) * 2 + 1]);
                            ok[q] = __ldcg(&p.part_o[((long long)sl * G + gi) * D + dd]);
                        }
                    }
#pragma unroll
                    for (int q = 0; q < kMaxMergeParts; ++q) {      // running log-sum-exp
                        if (q < n) {
                            const float Mn = fmaxf(M, mk[q]);
                            const float a = fast_exp2(M - Mn), w = fast_exp2(mk[q] - Mn);
                            num = num * a + w * ok[q];
                            den = den * a + w * lk[q];
                            M = Mn;
                        }
                    }
                }
                T* dst = static_cast<T*>(p.out) + ((long long)b * p.q_heads + (long long)g * G + gi) * D + dd;
                *dst = Elt<T>::from_float(num / den);
            }
            if (tid == 0) p.counters[c0] = 0;   // ready for the next call
        }
    }
}

// Thread-block cluster helpers (sm_90+): a barrier over all threads of the cluster with
// release/acquire semantics, and loads from another CTA's shared memory.
__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float ld_dsmem_f32(const float* local, uint32_t rank)
{
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// The cluster variant's merge, after every CTA of the cluster has stored its piece's state in
// `cpart` (empty pieces: m = -inf, l = 0): the cluster's first CTA combines the C states,
// M = max m_k, out = sum_k 2^(m_k - M) o_k / sum_k 2^(m_k - M) l_k, and writes the output;
// every CTA then waits for it, so that no CTA leaves while its state is still being read.
template <int D, int G, typename T>
__device__ __forceinline__ void cluster_merge(const DecodeParams& p, const float* cpart, int b, int g, bool cut,
                                              int rank, int C)
{
    cluster_sync_all();
    if (rank == 0 && cut) {
        for (int idx = threadIdx.x; idx < G * D; idx += kDecodeThreads) {
            const int gi = idx / D, dd = idx - gi * D;
            float M = -INFINITY;
            for (int r = 0; r < C; ++r) M = fmaxf(M, ld_dsmem_f32(cpart + gi * (D + 2) + D, r));
            float num = 0.f, den = 0.f;
            for (int r = 0; r < C; ++r) {
                const float m = ld_dsmem_f32(cpart + gi * (D + 2) + D, r);
                if (m == -INFINITY) continue;                     // an empty piece
                const float w = fast_exp2(m - M);
                num = fmaf(w, ld_dsmem_f32(cpart + gi * (D + 2) + dd, r), num);
                den = fmaf(w, ld_dsmem_f32(cpart + gi * (D + 2) + D + 1, r), den);
            }
            T* dst = static_cast<T*>(p.out) + ((long long)b * p.q_heads + (long long)g * G + gi) * D + dd;
            *dst = Elt<T>::from_float(num / den);
        }
    }
    cluster_sync_all();
}

// kFused: the whole decode layer in one kernel ("为什么要自己动手写一个LLM推理引擎"
// (wzjinhao.cn/news/61427) s4.3 rotate q and k, append k and v, attend; s5.3 fuse small
// kernels).  q arrives unturned and each warp turns its segment's q rows in shared memory
// from the step's angle table; the warp that owns a sequence's last page (which holds the
// new token at position L - 1) turns the new k, writes k and v into the pool (the append)
// and into its staged copy of the page.  No other kernel writes the pool meanwhile, so every
// page may be prefetched before the PDL wait.
// Register cap: 128 for the attention kernel alone (three of its CTAs and a RoPE/append CTA fit
// on one SM); the fused layer has no such neighbour and takes the cap of three CTAs per SM.
//
// kCluster: one cluster of p.cluster CTAs per (sequence, kv head) -- for batches whose
// (sequence, kv head) pairs are too few to fill the GPU -- each CTA taking an equal share
// of its pages; the pieces are merged through distributed shared memory (cluster_merge)
// instead of the workspace, so no CTA waits on global fences, atomics or loads at its end.
template <int D, int P, int G, typename T, bool kFused = false, bool kCluster = false>
__global__ void __launch_bounds__(kDecodeThreads, G == 1 ? (kFused ? 3 : 4) : 1) decode_pass1_kernel(const DecodeParams p)
{
    using S = DecodeShape<D, P, G, kFused, kCluster>;
    constexpr int NW = kDecodeWarps;
    constexpr int DEPTH = S::kDepth;
    constexpr int CPR = D / 8;            // 16-byte chunks per K/V row
    constexpr int LPRK = 2;               // lanes sharing one K row in q.k
    constexpr int RPL = P / 16;           // K rows per lane per page (rows t and t + 16)
    constexpr int CPL = CPR / LPRK;       // K chunks per lane per row
    constexpr int EPL = D / 32;           // output columns owned by each lane in p.V
    constexpr int QV = S::kQBytes / 16;   // 16-byte pieces of the group's q rows
    static_assert(P == 16 || P == 32, "page size");
    static_assert(EPL == 2 || EPL == 4, "head_dim");
    extern __shared__ __align__(128) unsigned char smem[];
    float* cmb = reinterpret_cast<float*>(smem + S::kCmbOffset);
    float* pbuf_all = reinterpret_cast<float*>(smem + S::kPbufOffset);
    int* warp_tot = reinterpret_cast<int*>(smem + S::kWarpTotOffset);
    volatile int* last_flag = warp_tot + 8;
    int* prefix = reinterpret_cast<int*>(smem + S::kScanOffset);
    int* lens = prefix + p.batch + 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // Prologue, before waiting on the previous kernel of the stream: the caller's lengths
    // and page table, and the first cached pages (see below).  A library kernel that
    // appends rows lets its successor start only once they are written and fenced, and
    // every other library kernel only after its own predecessor has finished; the one
    // exception, the fused layer, writes nothing but each sequence's newest token, whose
    // page is not prefetched here.  So none of these is still being written; q, the
    // newest tokens, the outputs and the workspace are touched only after pdl_wait.
    block_page_prefix<P>(p.context_lens, p.batch, prefix, lens, warp_tot);
    __syncthreads();
    const int Hkv = p.kv_heads;
    const long long W = (long long)Hkv * prefix[p.batch];
    const long long chunk = W > 0 ? (W + p.num_splits - 1) / p.num_splits : 1;
    long long r0 = (long long)blockIdx.x * chunk;
    long long r1 = min(W, r0 + chunk);
    // cluster variant: this CTA's share of its cluster's (sequence, kv head)
    const int c_rank = kCluster ? (int)(blockIdx.x % p.cluster) : 0;
    const int c_b = kCluster ? (int)(blockIdx.x / p.cluster) / Hkv : 0;
    const int c_g = kCluster ? (int)(blockIdx.x / p.cluster) % Hkv : 0;
    const int c_np = kCluster ? prefix[c_b + 1] - prefix[c_b] : 0;
    float* cpart = reinterpret_cast<float*>(smem + S::kPartOffset);
    if constexpr (kCluster) {
        const long long seg0 = (long long)Hkv * prefix[c_b] + (long long)c_g * c_np;
        r0 = seg0 + (long long)c_rank * c_np / p.cluster;
        r1 = seg0 + (long long)(c_rank + 1) * c_np / p.cluster;
        for (int i = tid; i < G; i += kDecodeThreads) {      // an empty piece's state
            cpart[i * (D + 2) + D] = -INFINITY;
            cpart[i * (D + 2) + D + 1] = 0.f;
        }
    }
    const long long n_mine = r1 - r0 > warp ? (r1 - r0 - warp + NW - 1) / NW : 0;   // this warp's pages

    // lane l holds the (page, kv head) chunk index page * Hkv + head of this warp's page
    // win0 + l; -1 for a page outside the table or the pool
    auto load_window = [&](long long win0) {
        const long long k = win0 + lane;
        int id = -1;
        if (k < n_mine) {
            int bb, gg, jj;
            locate_unit(r0 + warp + k * NW, prefix, p.batch, Hkv, bb, gg, jj);
            const int page = jj < p.max_pages ? p.block_tables[(long long)bb * p.max_pages + jj] : -1;
            if ((unsigned)page < (unsigned)p.num_pages) id = page * Hkv + gg;
        }
        return id;
    };
    long long win0 = 0;
    int win = load_window(0);
    const int ring_off = warp * DEPTH * S::kSlot;

    // ---- issue side: this warp's page k (iterator at unit r0 + warp + k NW).
    // K rows land XOR-swizzled by 16-byte chunk -- chunk c of row t at position
    // c ^ ((2 t + c / CPL) & 7) -- so that the lanes reading different rows at the same
    // column hit different banks; V rows land as they are.
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
        const int ph = __shfl_sync(0xffffffffu, win, (int)(k - win0));
        unsigned char* slot = smem + ring_off + (int)(k % DEPTH) * S::kSlot;
        if (ph >= 0) {
            const long long off = (long long)ph * (P * D);
            const unsigned char* ks = reinterpret_cast<const unsigned char*>(static_cast<const T*>(p.k) + off);
            const unsigned char* vs = reinterpret_cast<const unsigned char*>(static_cast<const T*>(p.v) + off);
#pragma unroll
            for (int n = 0; n < S::kChunk / 512; ++n) {
                const int gidx = n * 32 + lane;               // 16-byte chunk of the page
                const int t = gidx / CPR, c = gidx % CPR;
                const int pos = c ^ ((t * LPRK + c / CPL) & 7);
                cp_async16(slot + t * (2 * D) + pos * 16, ks + gidx * 16);
                cp_async16(slot + S::kChunk + gidx * 16, vs + gidx * 16);
            }
        } else if (lane == 0) {
            atomicOr(&g_error_word, PKV_DEVERR_BAD_PAGE);   // never dereferenced
        }
    };
    auto issue_q = [&](long long k, int bq, int gq) {    // the group's q rows into page k's slot
        unsigned char* slot = smem + ring_off + (int)(k % DEPTH) * S::kSlot;
        const unsigned char* qs = reinterpret_cast<const unsigned char*>(
            static_cast<const T*>(p.q) + ((long long)bq * p.q_heads + (long long)gq * G) * D);
        for (int n = lane; n < QV; n += 32) cp_async16(slot + 2 * S::kChunk + n * 16, qs + n * 16);
    };
    auto advance = [&]() {
        if (ij + NW < inp) {
            ij += NW;                          // common case: same (sequence, kv head)
        } else {
            for (int t = 0; t < NW; ++t) next_unit(ib, ig, ij, inp, prefix, Hkv, p.batch);
        }
    };
    auto issue = [&](long long k) {
        issue_kv(k);
        if (ib != qb || ig != qg) {           // first page of a (sequence, kv head) for this warp
            qb = ib;
            qg = ig;
            issue_q(k, ib, ig);
        }
        advance();
    };
    // Fused layer: which angle-table rows and new k, v rows this CTA keeps (see DecodeShape),
    // and the angle rows themselves, fetched before the PDL wait -- the table is written once
    // per step by rope_table, which releases its successor only after writing it.
    int* fids = reinterpret_cast<int*>(smem + S::kIdsOffset);
    double* rope_c = reinterpret_cast<double*>(smem + S::kRopeOffset);
    T* new_c = reinterpret_cast<T*>(smem + S::kNewOffset);
    if constexpr (kFused) {
        if (tid == 0) {
            int nr = 0, na = 0;
            fids[0] = fids[1] = fids[2] = fids[3] = -1;
            if (r0 < r1) {
                int sb, sg, sj;
                locate_unit(r0, prefix, p.batch, Hkv, sb, sg, sj);
                int snp = prefix[sb + 1] - prefix[sb];
                for (long long su = r0; su < r1 && (nr < 2 || na < 2);) {
                    const long long s_end = (long long)Hkv * prefix[sb] + (long long)(sg + 1) * snp;
                    if (nr < 2 && (nr == 0 || fids[nr - 1] != sb)) fids[nr++] = sb;
                    if (na < 2 && s_end <= r1) fids[2 + na++] = sb * Hkv + sg;
                    su = s_end;
                    if (++sg == Hkv) {
                        sg = 0;
                        do {
                            ++sb;
                            snp = sb < p.batch ? prefix[sb + 1] - prefix[sb] : 1;
                        } while (snp == 0);
                    }
                }
            }
        }
        __syncthreads();
        constexpr int RV = D * 8 / 16;                       // 16-byte pieces of one angle row
        for (int i = tid; i < 2 * RV; i += kDecodeThreads)
            if (fids[i / RV] >= 0)
                cp_async16(reinterpret_cast<unsigned char*>(rope_c) + i * 16,
                           reinterpret_cast<const unsigned char*>(p.rope + (long long)fids[i / RV] * D) + (i % RV) * 16);
        cp_async_commit();                   // the oldest group: waited for before the PDL wait
    }
    auto rope_row = [&](int bb) -> const double* {
        if constexpr (kFused) {
            if (fids[0] == bb) return rope_c;
            if (fids[1] == bb) return rope_c + D;
        }
        return p.rope + (long long)bb * D;
    };
    // Before waiting on the previous kernel: prefetch this warp's first pages, except a
    // page holding a sequence's newest token (a fused layer before this kernel may still
    // be writing it) and the q rows (the kernel before may still be producing them).
    if (n_mine > 0) prefetch_q_rows<D, G, T>(p, ib, ig, lane);     // this warp's first segment
    if (!kCluster && r0 < r1) prefetch_epilogue_lines<D, G>(p, r0, chunk, prefix, tid);
    if constexpr (kFused) {                   // the new k, v rows of the kept sequence ends
        constexpr int kRowLines = (D * (int)sizeof(T) + 127) / 128;
        if (warp == 0 && lane < 4 * kRowLines && fids[2 + lane / (2 * kRowLines)] >= 0) {
            const int a = lane / (2 * kRowLines), kv = (lane / kRowLines) & 1;
            prefetch_l2(reinterpret_cast<const unsigned char*>(static_cast<const T*>(kv ? p.v_new : p.k_new) +
                                                               (long long)fids[2 + a] * D) + (lane % kRowLines) * 128);
        }
    }
    int m_pre = 0, pre_qb[DEPTH], pre_qg[DEPTH];
    for (; m_pre < DEPTH && m_pre < n_mine; ++m_pre) {
        if (!kFused && ij == inp - 1) break;
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
    if constexpr (kFused) {
        // every warp reads both angle rows: let them land (the m_pre page groups may stay in
        // flight) and make them visible to the CTA before the wait, so that no CTA barrier
        // sits between the wait and the first page
        cp_async_wait_upto(m_pre);
        __syncthreads();
    }

    pdl_wait();
    pdl_launch_dependents();
    // rows with no cached token get zeros (spread over the CTAs)
    for (int b = blockIdx.x; b < p.batch; b += gridDim.x) {
        if (prefix[b + 1] != prefix[b]) continue;
        T* row = static_cast<T*>(p.out) + (long long)b * p.q_heads * D;
        for (int idx = tid; idx < p.q_heads * D; idx += blockDim.x) row[idx] = Elt<T>::from_float(0.f);
    }
    if (!kCluster && r0 >= r1) return;       // (a cluster's CTAs all reach its merge)

    unsigned char* ring = smem + ring_off;
    float* pbuf = pbuf_all + warp * G * P;
    for (int k = 0; k < m_pre; ++k)
        if (pre_qb[k] >= 0) issue_q(k, pre_qb[k], pre_qg[k]);
    if constexpr (kFused) {
        // the new k, v rows of the kept sequence ends, each copied by the warp that owns the
        // sequence's last page (the one that appends it), so only that warp waits for them
        constexpr int NV = D * 2 / 16;        // 16-byte pieces of one row
#pragma unroll
        for (int a = 0; a < 2; ++a) {
            const int bg = fids[2 + a];
            if (bg < 0) continue;
            const int bb = bg / Hkv, gg = bg - bb * Hkv, nb = prefix[bb + 1] - prefix[bb];
            const long long u_last = (long long)Hkv * prefix[bb] + (long long)gg * nb + nb - 1;
            if ((int)((u_last - r0) % NW) != warp) continue;
            for (int i = lane; i < 2 * NV; i += 32) {
                const int kv = i / NV;
                cp_async16(reinterpret_cast<unsigned char*>(new_c) + (a * 2 * NV + i) * 16,
                           reinterpret_cast<const unsigned char*>(static_cast<const T*>(kv ? p.v_new : p.k_new) +
                                                                  (long long)bg * D) + (i % NV) * 16);
            }
        }
    }
    if (m_pre == DEPTH) cp_async_commit();
    for (int k = m_pre; k < DEPTH; ++k) {
        if (k < n_mine) issue(k);
        cp_async_commit();
    }
    cp_async_wait<0>();

    // ---- compute side.  q.k: lane (t, h) = (lane / 2, lane % 2) dots rows t (and t + 16
    // at P = 32) over chunks h*CPL .. h*CPL+CPL-1; p.V: lane owns output columns
    // lane*EPL .. lane*EPL+EPL-1.
    const int t_own = lane / LPRK, h_own = lane % LPRK;
    const int sw_own = (t_own * LPRK + h_own) & 7;
    uint4 qraw[G][CPL];
    float o[G][EPL], m_run[G], l_run[G];
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
        m_run[gi] = -INFINITY;
        l_run[gi] = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) o[gi][e] = 0.f;
    }
    long long kc = 0;                         // this warp's pages consumed
    int b = 0, g = 0, j = 0, np = 1;
    if (r0 < r1) {
        locate_unit(r0, prefix, p.batch, Hkv, b, g, j);
        np = prefix[b + 1] - prefix[b];
    }
    int seg = 0;
    // One pass per segment (the range's part of one (sequence, kv head)): this warp's
    // pages of it, then the combine of all warps.
    for (long long u = r0; u < r1; ++seg) {
        const long long u_end = min(r1, u + (np - j));
        const long long first = u + ((warp - (int)((u - r0) % NW)) + NW) % NW;
        bool have_q = false;
        for (long long uu = first; uu < u_end; uu += NW) {
            cp_async_wait<DEPTH - 1>();         // page kc has landed (this lane's copies)
            __syncwarp();                       // ... and every lane's
            unsigned char* s = ring + (int)(kc % DEPTH) * S::kSlot;
            if constexpr (kFused) {
                if (j + (int)(uu - u) == np - 1) {
                    // the new token: row L - 1 of the sequence, in this (its last) page
                    const int tn = lens[b] - 1 - (np - 1) * P;
                    const int page = p.block_tables[(long long)b * p.max_pages + np - 1];
                    if (lane < 2 * CPR) {
                        const bool is_v = lane >= CPR;
                        const int c = is_v ? lane - CPR : lane;
                        const int bg = b * Hkv + g;
                        const T* src = fids[2] == bg ? new_c : fids[3] == bg ? new_c + 2 * D
                                                                              : static_cast<const T*>(p.k_new) + (long long)bg * D;
                        if (is_v)
                            src = fids[2] == bg ? new_c + D : fids[3] == bg ? new_c + 3 * D
                                                                             : static_cast<const T*>(p.v_new) + (long long)bg * D;
                        uint4 w = reinterpret_cast<const uint4*>(src)[c];
                        if (!is_v) rope_rotate8<T>(w, rope_row(b), 4 * c);
                        if (is_v)
                            *reinterpret_cast<uint4*>(s + S::kChunk + tn * (2 * D) + c * 16) = w;
                        else
                            *reinterpret_cast<uint4*>(s + tn * (2 * D) + ((c ^ ((tn * LPRK + c / CPL) & 7)) * 16)) = w;
                        if ((unsigned)page < (unsigned)p.num_pages)      // the append
                            reinterpret_cast<uint4*>(const_cast<T*>(static_cast<const T*>(is_v ? p.v : p.k)) +
                                                     (((long long)page * Hkv + g) * P + tn) * D)[c] = w;
                    }
                    __syncwarp();
                }
            }
            if (!have_q) {                      // first page of this segment for this warp
                have_q = true;
                if constexpr (kFused) {         // turn the group's q rows in place
                    for (int n = lane; n < G * CPR; n += 32) {
                        uint4* qv = reinterpret_cast<uint4*>(s + 2 * S::kChunk) + n;
                        uint4 w = *qv;
                        rope_rotate8<T>(w, rope_row(b), 4 * (n % CPR));
                        *qv = w;
                    }
                    __syncwarp();
                }
#pragma unroll
                for (int gi = 0; gi < G; ++gi)
#pragma unroll
                    for (int i = 0; i < CPL; ++i)
                        qraw[gi][i] = *reinterpret_cast<const uint4*>(s + 2 * S::kChunk + gi * (2 * D) +
                                                                      (h_own * CPL + i) * 16);
            }
            const int nvalid = min(P, lens[b] - (j + (int)(uu - u)) * P);
            // ---- scores: lane's partial dots over its chunks of rows t_own (+ 16)
            float sc[G][RPL];
#pragma unroll
            for (int rr = 0; rr < RPL; ++rr) {
                float acc[G];
#pragma unroll
                for (int gi = 0; gi < G; ++gi) acc[gi] = 0.f;
                const int t = t_own + 16 * rr;
#pragma unroll
                for (int i = 0; i < CPL; ++i) {
                    const int pos = (h_own * CPL + i) ^ sw_own;
                    const uint4 ku = *reinterpret_cast<const uint4*>(s + t * (2 * D) + pos * 16);
#pragma unroll
                    for (int gi = 0; gi < G; ++gi) acc[gi] += dot8<T>(qraw[gi][i], ku);
                }
#pragma unroll
                for (int gi = 0; gi < G; ++gi) {
                    acc[gi] += __shfl_xor_sync(0xffffffffu, acc[gi], 1);
                    sc[gi][rr] = t < nvalid ? acc[gi] * p.scale_log2 : -INFINITY;
                }
            }
            // ---- online softmax update; p of every row published to the warp's buffer
            float alpha[G];
            bool rescale = false;
#pragma unroll
            for (int gi = 0; gi < G; ++gi) {
                float pm = sc[gi][0];
#pragma unroll
                for (int rr = 1; rr < RPL; ++rr) pm = fmaxf(pm, sc[gi][rr]);
#pragma unroll
                for (int m = 16; m >= 2; m >>= 1) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, m));
                const float mn = fmaxf(m_run[gi], pm);   // finite: row 0 of a page is always valid
                alpha[gi] = fast_exp2(m_run[gi] - mn);
                rescale |= m_run[gi] != mn;
                m_run[gi] = mn;
                float ls = 0.f;
#pragma unroll
                for (int rr = 0; rr < RPL; ++rr) {
                    const float pr = fast_exp2(sc[gi][rr] - mn);   // 0 for rows past the context
                    ls += pr;
                    if (h_own == 0) pbuf[gi * P + t_own + 16 * rr] = pr;
                }
                l_run[gi] = l_run[gi] * alpha[gi] + (h_own == 0 ? ls : 0.f);
            }
            if (rescale) {
#pragma unroll
                for (int gi = 0; gi < G; ++gi)
#pragma unroll
                    for (int e = 0; e < EPL; e += 2) {
                        const float2 t2 = __fmul2_rn(make_float2(o[gi][e], o[gi][e + 1]), make_float2(alpha[gi], alpha[gi]));
                        o[gi][e] = t2.x;
                        o[gi][e + 1] = t2.y;
                    }
            }
            __syncwarp();                         // p of all rows visible to the warp
            // ---- o += p V: row t's EPL columns of this lane (rows past the context skipped)
            const unsigned char* vbase = s + S::kChunk + lane * (EPL * 2);
            auto pv_row = [&](int t) {
                float vf[EPL];
                if constexpr (EPL == 4) {
                    const uint2 w = *reinterpret_cast<const uint2*>(vbase + t * (2 * D));
                    const float2 a = Elt<T>::to_float2(w.x), c2 = Elt<T>::to_float2(w.y);
                    vf[0] = a.x; vf[1] = a.y; vf[2] = c2.x; vf[3] = c2.y;
                } else {
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(vbase + t * (2 * D));
                    const float2 a = Elt<T>::to_float2(w);
                    vf[0] = a.x; vf[1] = a.y;
                }
#pragma unroll
                for (int gi = 0; gi < G; ++gi) {
                    const float pt = pbuf[gi * P + t];
#pragma unroll
                    for (int e = 0; e < EPL; e += 2) {
                        const float2 r2 = __ffma2_rn(make_float2(pt, pt), make_float2(vf[e], vf[e + 1]),
                                                     make_float2(o[gi][e], o[gi][e + 1]));
                        o[gi][e] = r2.x;
                        o[gi][e + 1] = r2.y;
                    }
                }
            };
            if (nvalid == P) {
#pragma unroll
                for (int t = 0; t < P; ++t) pv_row(t);
            } else {
                for (int t = 0; t < nvalid; ++t) pv_row(t);   // last page of a sequence
            }
            __syncwarp();                         // every lane is done with the slot and p
            if (kc + DEPTH < n_mine) issue(kc + DEPTH);
            cp_async_commit();
            ++kc;
        }
        // ---- every warp publishes its (possibly empty) state of this segment
        float* buf = cmb + (seg & 1) * S::kCmbFloats;
#pragma unroll
        for (int gi = 0; gi < G; ++gi) {
            float lt = l_run[gi];
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) lt += __shfl_xor_sync(0xffffffffu, lt, m);
            float* row = buf + (warp * G + gi) * (D + 2);
#pragma unroll
            for (int e = 0; e < EPL; ++e) row[lane * EPL + e] = o[gi][e];
            if (lane == 0) {
                row[D] = m_run[gi];
                row[D + 1] = lt;
            }
            m_run[gi] = -INFINITY;
            l_run[gi] = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) o[gi][e] = 0.f;
        }
        segment_epilogue<D, G, T, kCluster>(p, buf, b, g, np, prefix, r0, r1, chunk, last_flag, cpart);
        // next segment: the next kv head of this sequence, or the next non-empty sequence
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
    if constexpr (kCluster) cluster_merge<D, G, T>(p, cpart, c_b, c_g, c_np >= 2, c_rank, p.cluster);
}

}  // namespace pkv

#endif  // PKV_DECODE_ATTENTION_CUH_
