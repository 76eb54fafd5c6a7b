// Paged decode attention over int8 KV pages on the tensor cores.
//
// The pages' KV strategy pairs paging with compression of the cached values ("为什么要
// 自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427) s3.4).  Here every cached (token, kv
// head) row of K and V is head_dim int8 codes c with one fp32 scale s, the value being
// c * s.  The kernel computes the same softmax(scale q.K^T) V as the 16-bit kernels, with
// the balanced partition, per-warp cp.async rings, PDL prologue and in-kernel merge of
// decode_attention.cuh, over 32-token units (a 32-token page or two 16-token pages),
// each two 16-token tiles:
//   S^T[32 tokens x 8 heads] = C_K[32 x D] . Q^T[D x 8]          (fp16 MMAs, fp32 sums)
//   scores = S^T * s_K(token) * scale                             (heads >= G are zero)
//   O^T[D x 8] += C_V^T[D x 32] . (p * s_V * 2^E)^T[32 x 8]       (fp16 MMAs)
// A 32-token unit halves, per token, the fixed cost of a unit (softmax reductions, ring
// and page-table bookkeeping) next to the 16-token tiles of the 16-bit MMA kernel.
// Decoding: the codes are read with ldmatrix as 16-bit pairs (non-transposed for K,
// transposed for V) and each byte becomes an exact fp16 value: the byte offset by 128 is
// placed under the exponent of 1024 with one byte permute (1152 + code); for V one packed
// fp16 subtraction of 1152 leaves the code, for K the constant stays in the MMA operand and
// 1152 * sum_d q_d is subtracted from each score (q is fixed for the whole segment, and the
// offset sum spans only head_dim terms, unlike the output sums over the whole context).  Which bytes of a fragment register feed which
// MMA operand slot fixes a permutation of the contraction index (head_dim for K, the
// output column order for V); q's fragments are loaded in the same permuted order and
// the output columns are written back in place, so no data is moved to undo it.
// fp16 for both data types: codes are exact in fp16; bf16 q is scaled by a power of two
// per head row (none unless max |q| >= 2^15) so that it converts exactly; P times the V
// scale is scaled by 2^E per unit (E from the unit's largest V scale), which keeps it in
// fp16's normal range, and the accumulated output is rescaled when E changes.  A row whose
// V scale lies more than 2^14 below the unit's largest one gets a subnormal fp16 weight:
// its absolute error stays under 2^-25 of the unit's largest possible weight.
#ifndef PKV_DECODE_ATTENTION_I8_CUH_
#define PKV_DECODE_ATTENTION_I8_CUH_

#include "decode_attention_mma.cuh"

namespace pkv {

template <int D, int G>
struct I8Shape {
    static constexpr int kRows = 32;                          // token rows per unit
    static constexpr int kChunk = kRows * D;                  // code bytes of one unit's K (or V)
    static constexpr int kScaleBytes = kRows * 4;             // its fp32 row scales
    static constexpr int kQOffset = 2 * kChunk + 2 * kScaleBytes;
    static constexpr int kQBytes = G * D * 2;
    static constexpr int kSlot = kQOffset + kQBytes;
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

// Position of 16-byte chunk c of token row t in shared memory: c ^ swizzle(t), so that the
// eight rows of one ldmatrix (consecutive tokens, same chunk) fall in distinct banks
// (rows of 128 bytes: eight chunks; rows of 64 bytes: two rows per 128-byte line).
template <int D>
__device__ __forceinline__ int i8_swizzle(int t)
{
    return D == 128 ? (t & 7) : ((t >> 1) & 3);
}

// Two exact fp16 codes from the bytes of x picked by `sel` (a byte-permute selector whose
// odd nibbles pick 0x64): ((0x64 << 8) | (byte ^ 0x80)) is 1024 + code + 128.
__device__ __forceinline__ uint32_t i8_pair_to_f16x2(uint32_t x_biased, uint32_t sel)
{
    const uint32_t h = __byte_perm(x_biased, 0x64646464u, sel);
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h), "r"(0x64806480u));   // 1152 = 0x6480
    return r;
}

// Bytes 0,1 / 2,3 (K fragments: consecutive head_dim columns of one token) as fp16
// 1152 + code: the constant is removed after the MMA (1152 * sum(q) per head).
__device__ __forceinline__ void i8_lo_hi_biased(uint32_t w, uint32_t& lo, uint32_t& hi)
{
    const uint32_t x = w ^ 0x80808080u;
    lo = __byte_perm(x, 0x64646464u, 0x5140u);
    hi = __byte_perm(x, 0x64646464u, 0x5342u);
}

// Bytes 0,2 / 1,3 (transposed V fragments: tokens 2i, 2i+1 of an even / odd column)
__device__ __forceinline__ void i8_even_odd(uint32_t w, uint32_t& ev, uint32_t& od)
{
    const uint32_t x = w ^ 0x80808080u;
    ev = i8_pair_to_f16x2(x, 0x5240u);
    od = i8_pair_to_f16x2(x, 0x5341u);
}

// Quantise one head row held as 16-byte vectors of T by `vpr` consecutive lanes (vector c of
// the row in lane c of the group): the row's amax by a shuffle reduction within the group,
// codes round_half_even(x * (127 / amax)) clamped to +-127, scale amax / 127 -- every step the
// correctly rounded fp32 operation of the append kernel, so the results are identical.
// Lanes outside any group take part in the shuffles with amax 0.
template <typename T>
__device__ __forceinline__ uint2 i8_quantise_vec(const uint4& u, int vpr, bool active, float& scale)
{
    float x[8];
    unpack8<T>(u, x);
    float amax = 0.f;
    if (active) {
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[e]));
    }
    for (int m = vpr >> 1; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    uint32_t w[2] = {0u, 0u};
    scale = 0.f;
    if (amax > 0.f) {
        const float inv = __fdiv_rn(127.f, amax);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float r = fminf(fmaxf(rintf(__fmul_rn(x[e], inv)), -127.f), 127.f);
            w[e >> 2] |= ((uint32_t)(int)r & 0xffu) << (8 * (e & 3));
        }
        scale = __fdiv_rn(amax, 127.f);
    }
    return make_uint2(w[0], w[1]);
}

// kFused: the whole decode layer in one kernel, as for the 16-bit CUDA-core kernel: q turned
// in shared memory from the step's angle table at each segment's first unit; the warp that
// owns a sequence's last unit turns the new k, quantises k and v, appends codes and scales to
// the pool and patches its staged copy; every unit may be prefetched before the PDL wait.
// Register cap from the CTAs per SM that shared memory admits (kCtasPerSm: three with one query
// head per kv head at head_dim 128, two with two or four, one with eight): a tighter cap would
// only cost registers, not add residency.
template <int D, int P, int G, typename T, bool kFused = false>
__global__ void __launch_bounds__(kDecodeThreads, I8Shape<D, G>::kCtasPerSm) decode_i8_kernel(const DecodeParams p)
{
    using S = I8Shape<D, G>;
    using Mma = MmaOps<__half>;
    constexpr int NW = kDecodeWarps;
    constexpr int DEPTH = S::kDepth;
    constexpr int CPR = D / 16;           // 16-byte chunks per token row
    constexpr int PPU = 32 / P;           // pages per 32-token unit
    constexpr int WIN = 32 / PPU;         // units whose page ids one window holds
    constexpr int KS = D / 16;            // k-steps of q.k = m-tiles of p.V
    constexpr int QV = S::kQBytes / 16;
    static_assert(P == 16 || P == 32, "page size");
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(G >= 1 && G <= 8, "1 to 8 query heads per kv head");
    extern __shared__ __align__(128) unsigned char smem[];
    float* cmb = reinterpret_cast<float*>(smem + S::kCmbOffset);
    int* warp_tot = reinterpret_cast<int*>(smem + S::kWarpTotOffset);
    volatile int* last_flag = warp_tot + 8;
    int* prefix = reinterpret_cast<int*>(smem + S::kScanOffset);
    int* lens = prefix + p.batch + 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // Prologue before the PDL wait, as in the 16-bit kernels; units are 32 tokens.
    block_page_prefix<32>(p.context_lens, p.batch, prefix, lens, warp_tot);
    __syncthreads();
    const int Hkv = p.kv_heads;
    const long long W = (long long)Hkv * prefix[p.batch];
    const long long chunk = W > 0 ? (W + p.num_splits - 1) / p.num_splits : 1;
    const long long r0 = (long long)blockIdx.x * chunk;
    const long long r1 = min(W, r0 + chunk);
    const int n_mine = r1 - r0 > warp ? (int)((r1 - r0 - warp + NW - 1) / NW) : 0;

    // lane l holds, for page l % PPU of this warp's unit win0 + l / PPU, its (page, kv head)
    // index page * Hkv + head: -1 when the page table has no such entry or it is outside
    // the pool, -2 when the unit's tokens end before that page
    auto load_window = [&](int win0) {
        const int k = win0 + lane / PPU;
        int id = -2;
        if (k < n_mine) {
            int bb, gg, jj;
            locate_unit(r0 + warp + (long long)k * NW, prefix, p.batch, Hkv, bb, gg, jj);
            const int pg = jj * PPU + lane % PPU;
            if (pg * P < lens[bb]) {
                const int page = pg < p.max_pages ? p.block_tables[(long long)bb * p.max_pages + pg] : -1;
                id = (unsigned)page < (unsigned)p.num_pages ? page * Hkv + gg : -1;
            }
        }
        return id;
    };
    int win0 = 0;
    int win = load_window(0);
    unsigned char* ring = smem + warp * DEPTH * S::kSlot;

    int ib = 0, ig = 0, ij = 0, inp = 1, qb = -1, qg = -1;
    if (n_mine > 0) {
        locate_unit(r0 + warp, prefix, p.batch, Hkv, ib, ig, ij);
        inp = prefix[ib + 1] - prefix[ib];
    }
    // unit k of this warp into ring slot `sl` (= k mod DEPTH): its P-token pages land at
    // unit rows pp * P ..
    auto issue_kv = [&](int k, int sl) {
        if (k >= win0 + WIN) {
            win0 = k;
            win = load_window(k);
        }
        unsigned char* slot = ring + sl * S::kSlot;
#pragma unroll
        for (int pp = 0; pp < PPU; ++pp) {
            const int ph = __shfl_sync(0xffffffffu, win, (k - win0) * PPU + pp);
            if (ph == -2) continue;                          // past the sequence's last token
            if (ph >= 0) {
                const long long row0 = (long long)ph * P;   // first token row
                const unsigned char* ks = static_cast<const unsigned char*>(p.k) + row0 * D;
                const unsigned char* vs = static_cast<const unsigned char*>(p.v) + row0 * D;
#pragma unroll
                for (int n = 0; n < P * D / 512; ++n) {
                    const int gidx = n * 32 + lane;
                    const int t = pp * P + gidx / CPR, c = gidx % CPR;
                    const int dst = t * D + ((c ^ i8_swizzle<D>(t)) * 16);
                    cp_async16(slot + dst, ks + gidx * 16);
                    cp_async16(slot + S::kChunk + dst, vs + gidx * 16);
                }
                constexpr int SC = P / 4;                    // 16-byte pieces of P scales
                if (lane < SC)
                    cp_async16(slot + 2 * S::kChunk + pp * P * 4 + lane * 16,
                               reinterpret_cast<const unsigned char*>(p.k_scale + row0) + lane * 16);
                else if (lane >= 16 && lane < 16 + SC)
                    cp_async16(slot + 2 * S::kChunk + S::kScaleBytes + pp * P * 4 + (lane - 16) * 16,
                               reinterpret_cast<const unsigned char*>(p.v_scale + row0) + (lane - 16) * 16);
            } else if (lane == 0) {
                atomicOr(&g_error_word, PKV_DEVERR_BAD_PAGE);   // never dereferenced
            }
        }
    };
    auto issue_q = [&](int sl, int bq, int gq) {
        unsigned char* slot = ring + sl * S::kSlot;
        const unsigned char* qs = reinterpret_cast<const unsigned char*>(
            static_cast<const T*>(p.q) + ((long long)bq * p.q_heads + (long long)gq * G) * D);
        for (int n = lane; n < QV; n += 32) cp_async16(slot + S::kQOffset + n * 16, qs + n * 16);
    };
    auto advance = [&]() {
        if (ij + NW < inp) {
            ij += NW;
        } else {
            for (int t = 0; t < NW; ++t) next_unit(ib, ig, ij, inp, prefix, Hkv, p.batch);
        }
    };
    auto issue = [&](int k, int sl) {
        issue_kv(k, sl);
        if (ib != qb || ig != qg) {
            qb = ib;
            qg = ig;
            issue_q(sl, ib, ig);
        }
        advance();
    };
    if (n_mine > 0) prefetch_q_rows<D, G, T>(p, ib, ig, lane);     // this warp's first segment
    if (r0 < r1) prefetch_epilogue_lines<D, G>(p, r0, chunk, prefix, tid);
    int m_pre = 0, pre_qb[DEPTH], pre_qg[DEPTH];
    for (; m_pre < DEPTH && m_pre < n_mine; ++m_pre) {
        if (!kFused && ij == inp - 1) break;
        issue_kv(m_pre, m_pre);
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

    for (int k = 0; k < m_pre; ++k)
        if (pre_qb[k] >= 0) issue_q(k, pre_qb[k], pre_qg[k]);
    if (m_pre == DEPTH) cp_async_commit();
    for (int k = m_pre; k < DEPTH; ++k) {
        if (k < n_mine) issue(k, k);
        cp_async_commit();
    }
    cp_async_wait<0>();

    // ---- compute side (fragments of m16n8k16: g4 = lane / 4, t4 = lane % 4).  A unit is
    // two 16-token tiles; ldmatrix x4 rows: lane l supplies token ((l >> 3) & 1) * 8 + (l & 7)
    // of the tile, chunk 2x + (l >> 4).
    const int g4 = lane >> 2, t4 = lane & 3;
    const int lm_tok = ((lane >> 3) & 1) * 8 + (lane & 7);
    const int lm_off = lm_tok * D;
    const int lm_chunk = lane >> 4, lm_swz = i8_swizzle<D>(lm_tok);   // same for tile 1 (rows + 16)
    uint32_t bq[KS][2];                       // Q^T fragments: head g4, columns 16kk + 4t4 + {0,1 | 2,3}
    float qscale[2];                          // 2^s(head) * scale * log2(e) for heads 2 t4 + j
    float qbias[2];                           // 1152 * sum_d q_d (fp16 operand) of heads 2 t4 + j
    float oacc[KS][4], m_run[2], l_run[2];    // O^T * 2^E: rows 16 mt + 2 g4 (+1), heads 2 t4 + j
#pragma unroll
    for (int mt = 0; mt < KS; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[mt][e] = 0.f;
    m_run[0] = m_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.f;
    int e_cur = 127;                          // biased exponent of 2^-E (the unit scale in use)
    int kc = 0;
    int cs = 0;                               // ring slot of unit kc
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
            unsigned char* s = ring + cs * S::kSlot;
            if constexpr (kFused) {
                if (j + (int)(uu - u) == np - 1) {
                    // the new token: position L - 1 of the sequence, row tn of this (its last) unit
                    const int last = lens[b] - 1;
                    const int tn = last - (np - 1) * 32;
                    const int page = p.block_tables[(long long)b * p.max_pages + last / P];
                    constexpr int VPR = D / 8;                  // 16-byte vectors of T per row
                    const bool active = lane < 2 * VPR;
                    const bool is_v = lane >= VPR;
                    const int c = lane % VPR;
                    uint4 w = make_uint4(0u, 0u, 0u, 0u);
                    if (active) {
                        w = reinterpret_cast<const uint4*>(static_cast<const T*>(is_v ? p.v_new : p.k_new) +
                                                           ((long long)b * Hkv + g) * D)[c];
                        if (!is_v) rope_rotate8<T>(w, p.rope + (long long)b * D, 4 * c);
                    }
                    float sc;
                    const uint2 codes = i8_quantise_vec<T>(w, VPR, active, sc);
                    if (active) {
                        unsigned char* row = s + (is_v ? S::kChunk : 0) + tn * D;
                        *reinterpret_cast<uint2*>(row + (((c >> 1) ^ i8_swizzle<D>(tn)) * 16) + 8 * (c & 1)) = codes;
                        if (c == 0)
                            reinterpret_cast<float*>(s + 2 * S::kChunk + (is_v ? S::kScaleBytes : 0))[tn] = sc;
                        if ((unsigned)page < (unsigned)p.num_pages) {           // the append
                            const long long rid = ((long long)page * Hkv + g) * P + last % P;
                            *reinterpret_cast<uint2*>(const_cast<unsigned char*>(
                                static_cast<const unsigned char*>(is_v ? p.v : p.k)) + rid * D + 8 * c) = codes;
                            if (c == 0) const_cast<float*>(is_v ? p.v_scale : p.k_scale)[rid] = sc;
                        }
                    }
                    __syncwarp();
                }
            }
            if (!have_q) {
                have_q = true;
                if constexpr (kFused) {         // turn the group's q rows in place
                    for (int n = lane; n < G * (D / 8); n += 32) {
                        uint4* qv = reinterpret_cast<uint4*>(s + S::kQOffset) + n;
                        uint4 w = *qv;
                        rope_rotate8<T>(w, p.rope + (long long)b * D, 4 * (n % (D / 8)));
                        *qv = w;
                    }
                    __syncwarp();
                }
                const T* qa = reinterpret_cast<const T*>(s + S::kQOffset);
                int shift = 0;                // power of two that brings the head row's max under 2^15
                float qs = 0.f;               // this lane's part of sum_d q_d (of the fp16 operand)
                if constexpr (std::is_same<T, __half>::value) {
#pragma unroll
                    for (int kk = 0; kk < KS; ++kk) {
                        const uint2 w = g4 < G ? *reinterpret_cast<const uint2*>(qa + g4 * D + kk * 16 + 4 * t4)
                                               : make_uint2(0u, 0u);
                        bq[kk][0] = w.x;
                        bq[kk][1] = w.y;
                        const float2 a = Elt<__half>::to_float2(w.x), c2 = Elt<__half>::to_float2(w.y);
                        qs += (a.x + a.y) + (c2.x + c2.y);
                    }
                } else {
                    float qf[KS][4];
                    float mx = 0.f;
#pragma unroll
                    for (int kk = 0; kk < KS; ++kk) {
                        const uint2 w = g4 < G ? *reinterpret_cast<const uint2*>(qa + g4 * D + kk * 16 + 4 * t4)
                                               : make_uint2(0u, 0u);
                        const float2 a = Elt<T>::to_float2(w.x), c2 = Elt<T>::to_float2(w.y);
                        qf[kk][0] = a.x; qf[kk][1] = a.y; qf[kk][2] = c2.x; qf[kk][3] = c2.y;
#pragma unroll
                        for (int e = 0; e < 4; ++e) mx = fmaxf(mx, fabsf(qf[kk][e]));
                    }
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                    shift = max(0, (int)((__float_as_uint(mx) >> 23) & 0xff) - 141);   // 141 = 127 + 14
                    const float down = __uint_as_float((uint32_t)(127 - shift) << 23);   // 2^-shift
#pragma unroll
                    for (int kk = 0; kk < KS; ++kk) {
                        bq[kk][0] = Mma::pack(qf[kk][0] * down, qf[kk][1] * down);
                        bq[kk][1] = Mma::pack(qf[kk][2] * down, qf[kk][3] * down);
                        const float2 a = Elt<__half>::to_float2(bq[kk][0]), c2 = Elt<__half>::to_float2(bq[kk][1]);
                        qs += (a.x + a.y) + (c2.x + c2.y);
                    }
                }
                qs += __shfl_xor_sync(0xffffffffu, qs, 1);
                qs += __shfl_xor_sync(0xffffffffu, qs, 2);
#pragma unroll
                for (int jh = 0; jh < 2; ++jh) {
                    const int src = (2 * t4 + jh) * 4;
                    const int sh = __shfl_sync(0xffffffffu, shift, src);
                    qscale[jh] = __uint_as_float((uint32_t)(127 + sh) << 23) * p.scale_log2;
                    qbias[jh] = 1152.f * __shfl_sync(0xffffffffu, qs, src);
                }
            }
            const int nvalid = (int)min(32LL, (long long)lens[b] - (j + (uu - u)) * 32);
            const unsigned char* kb = s;
            const unsigned char* vb = s + S::kChunk;
            const float* ksc = reinterpret_cast<const float*>(s + 2 * S::kChunk);
            const float* vsc = reinterpret_cast<const float*>(s + 2 * S::kChunk + S::kScaleBytes);
            // ---- S^T = C_K . Q^T for the two 16-token tiles
            // (each tile's k-steps spread over kScoreChains independent accumulators)
            constexpr int SCH = KS < kScoreChains ? KS : kScoreChains;
            float sacc_c[2][SCH][4];
#pragma unroll
            for (int tau = 0; tau < 2; ++tau)
#pragma unroll
                for (int c = 0; c < SCH; ++c)
#pragma unroll
                    for (int e = 0; e < 4; ++e) sacc_c[tau][c][e] = 0.f;
#pragma unroll
            for (int tau = 0; tau < 2; ++tau) {
#pragma unroll
                for (int x = 0; x < KS / 2; ++x) {
                    uint32_t r[4];
                    ldmatrix_x4(r, kb + tau * 16 * D + lm_off + (((2 * x + lm_chunk) ^ lm_swz) * 16));
#pragma unroll
                    for (int h = 0; h < 2; ++h) {         // k-step 2x + h: r[2h] tokens 0-7, r[2h+1] 8-15
                        uint32_t a[4];
                        i8_lo_hi_biased(r[2 * h], a[0], a[2]);
                        i8_lo_hi_biased(r[2 * h + 1], a[1], a[3]);
                        Mma::mma(sacc_c[tau][(2 * x + h) % SCH], a, bq[2 * x + h][0], bq[2 * x + h][1]);
                    }
                }
            }
            float sacc[2][4];
#pragma unroll
            for (int tau = 0; tau < 2; ++tau)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    sacc[tau][e] = sacc_c[tau][0][e];
#pragma unroll
                    for (int c = 1; c < SCH; ++c) sacc[tau][e] += sacc_c[tau][c][e];
                }
            // ---- scores of tokens 16 tau + g4 (+8), heads 2t4, 2t4+1; the unit's 2^E
            float sc[2][4], w[2][2];
            float smax = 0.f;
#pragma unroll
            for (int tau = 0; tau < 2; ++tau)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int tok = 16 * tau + 8 * hh + g4;
                    const bool ok = tok < nvalid;
                    const float kscale = ksc[tok];
                    sc[tau][2 * hh] = ok ? (sacc[tau][2 * hh] - qbias[0]) * kscale * qscale[0] : -INFINITY;
                    sc[tau][2 * hh + 1] = ok ? (sacc[tau][2 * hh + 1] - qbias[1]) * kscale * qscale[1] : -INFINITY;
                    w[tau][hh] = ok ? vsc[tok] : 0.f;
                    smax = fmaxf(smax, w[tau][hh]);
                }
#pragma unroll
            for (int m = 4; m < 32; m <<= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, m));
            const int e_unit = (int)(__float_as_uint(smax) >> 23);        // 0 for an all-zero unit
            const int e_new = e_unit > 0 ? e_unit : e_cur;
            const float up = __uint_as_float((uint32_t)(254 - e_new) << 23);            // 2^E
            // O' = O * 2^E: rescale by 2^(E_new - E_old) = 2^(e_cur - e_new) (clamped to
            // fp32's normal range)
            const float ratio = __uint_as_float((uint32_t)min(254, max(1, 127 + e_cur - e_new)) << 23);
            float alpha[2], pr[2][4];
#pragma unroll
            for (int jh = 0; jh < 2; ++jh) {
                float pm = fmaxf(fmaxf(sc[0][jh], sc[0][jh + 2]), fmaxf(sc[1][jh], sc[1][jh + 2]));
#pragma unroll
                for (int m = 4; m < 32; m <<= 1) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, m));
                const float mn = fmaxf(m_run[jh], pm);         // finite: row 0 is always valid
                alpha[jh] = fast_exp2(m_run[jh] - mn);
                m_run[jh] = mn;
                float ls = 0.f;
#pragma unroll
                for (int tau = 0; tau < 2; ++tau) {
                    pr[tau][jh] = fast_exp2(sc[tau][jh] - mn);
                    pr[tau][jh + 2] = fast_exp2(sc[tau][jh + 2] - mn);
                    ls += pr[tau][jh] + pr[tau][jh + 2];
                }
                l_run[jh] = l_run[jh] * alpha[jh] + ls;
            }
            if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f || e_new != e_cur)) {
                const float f0 = alpha[0] * ratio, f1 = alpha[1] * ratio;
#pragma unroll
                for (int mt = 0; mt < KS; ++mt) {
                    oacc[mt][0] *= f0;
                    oacc[mt][1] *= f1;
                    oacc[mt][2] *= f0;
                    oacc[mt][3] *= f1;
                }
            }
            e_cur = e_new;
            // ---- (p * s_V * 2^E)^T as B operands (fp16): movmatrix.trans of the 8x8 blocks
            //      of tokens 16 tau + 0-7 and 16 tau + 8-15
            uint32_t pb[2][2];
#pragma unroll
            for (int tau = 0; tau < 2; ++tau) {
                const float w0 = w[tau][0] * up, w1 = w[tau][1] * up;
                pb[tau][0] = movmatrix_trans(Mma::pack(pr[tau][0] * w0, pr[tau][1] * w0));
                pb[tau][1] = movmatrix_trans(Mma::pack(pr[tau][2] * w1, pr[tau][3] * w1));
            }
            // ---- O^T += C_V^T . P'^T over both tiles; m-tile mt holds columns 16 mt + 2 g4
            //      (row g4) and 16 mt + 2 g4 + 1 (row g4 + 8)
#pragma unroll
            for (int x = 0; x < KS / 2; ++x) {
#pragma unroll
                for (int tau = 0; tau < 2; ++tau) {
                    uint32_t r[4];
                    ldmatrix_x4_trans(r, vb + tau * 16 * D + lm_off + (((2 * x + lm_chunk) ^ lm_swz) * 16));
#pragma unroll
                    for (int h = 0; h < 2; ++h) {         // m-tile 2x + h: r[2h] tokens 0-7, r[2h+1] 8-15
                        uint32_t a[4];
                        i8_even_odd(r[2 * h], a[0], a[1]);
                        i8_even_odd(r[2 * h + 1], a[2], a[3]);
                        Mma::mma(oacc[2 * x + h], a, pb[tau][0], pb[tau][1]);
                    }
                }
            }
            __syncwarp();
            if (kc + DEPTH < n_mine) issue(kc + DEPTH, cs);
            cp_async_commit();
            ++kc;
            cs = cs + 1 == DEPTH ? 0 : cs + 1;
        }
        // ---- publish this warp's state: o[head][d] (2^-E applied), m, l of the real heads
        float* buf = cmb + (seg & 1) * S::kCmbFloats;
        const float down = __uint_as_float((uint32_t)e_cur << 23);                 // 2^-E
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
                    row[mt * 16 + 2 * g4] = oacc[mt][jh] * down;
                    row[mt * 16 + 2 * g4 + 1] = oacc[mt][2 + jh] * down;
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
        e_cur = 127;
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

#endif  // PKV_DECODE_ATTENTION_I8_CUH_
