/*
 * pagedkv.h -- C ABI of libpagedkv.so: one autoregressive decode step of
 * LLaMA-style attention against a paged KV cache, on NVIDIA B200 (sm_100a).
 *
 * Sources, cited by page title and section:
 *   [ENGINE] "为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427), chapter 1
 *            s3.4  KV-cache management: size formula; the cache cut into fixed pages of
 *                  16 or 32 tokens, allocated from a free list and given back when a
 *                  request ends; attention locates a token's block through a page index.
 *            s4.2  RoPE: position enters q and k through a rotation; RMSNorm with eps
 *                  added to the mean square before the root.
 *            s4.3  forward with a cache: n_heads / n_kv_heads views,
 *                  apply_rotary_emb(q, k, start_pos), cache update, q k^T / sqrt(head_dim)
 *                  plus causal mask, softmax, times v.
 *            s5.3  replace concatenation with a preallocated cache pool; fused attention.
 *   [FLOW]   "大模型推理全流程解析" (stapisi.com/news/4049481) s2.2.2: decode attention of
 *            the new token against every cached K/V; KV read bandwidth is the bottleneck.
 *
 * Conventions for every entry point
 *   - Return value: PKV_OK (0) or one of the PKV_ERR_* codes below;
 *     pkv_status_string() names it.  Arguments are validated on the host before any
 *     launch; a call that returns an error has launched nothing.
 *   - Memory: every device pointer is owned by the caller (allocated by any CUDA
 *     allocator, e.g. PyTorch).  The library allocates no device memory on any path;
 *     scratch comes from a caller-provided workspace (paged_decode_attention_noalloc
 *     instead uses a fixed array compiled into the library).
 *   - Streams: device work is enqueued asynchronously on the caller's stream (a
 *     cudaStream_t; NULL = legacy default stream); no entry point synchronises the
 *     host except kv_get_device_error().  Consecutive kernels of the library use
 *     programmatic dependent launch, so a kernel's prologue may overlap the tail of the
 *     library kernel before it on the same stream.  The decode calls read cached pages
 *     in that prologue, all but the page of each sequence's newest token; so the calls
 *     that write pages (paged_kv_append, rope_append) let the next kernel start only once
 *     their rows are written, whatever tokens and slots they are given, while
 *     rope_append_step and paged_decode_layer, which let it start earlier, write only the
 *     newest token of each sequence (position context_lens[b] - 1).  A decode call that
 *     directly follows one of these two on the same layer must be given the same
 *     context_lens and block tables.
 *   - Layouts are row-major, innermost index last.  Element type: PKV_F16 (IEEE
 *     binary16) or PKV_BF16 (bfloat16), the same for q, k, v, the pool and the output.
 *   - Device-side index checks: an out-of-range page id or slot is never dereferenced;
 *     the access is skipped and a bit is set in a device error word that
 *     kv_get_device_error() returns.  Bounded waits inside the kernels set a bit there
 *     too instead of spinning forever.
 */
#ifndef PAGEDKV_H_
#define PAGEDKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define PKV_OK 0
#define PKV_ERR_INVALID_ARG 1   /* null pointer, negative or inconsistent size */
#define PKV_ERR_UNSUPPORTED 2   /* a shape/dtype combination with no compiled kernel */
#define PKV_ERR_CUDA 3          /* a CUDA runtime call or launch failed */
#define PKV_ERR_NO_SPACE 4      /* free list too short, or workspace too small */

/* element types */
#define PKV_F16 0
#define PKV_BF16 1
#define PKV_I8 2     /* KV storage only: int8 codes with one fp32 scale per (token, head) row */

/* Largest num_splits that paged_decode_attention and paged_decode_layer accept.  A decode
 * workspace starts with a counter region of this many int32 slots whatever num_splits is. */
#define PKV_MAX_DECODE_SPLITS 4096

/* device error word bits (kv_get_device_error) */
#define PKV_DEVERR_BAD_PAGE 0x1u     /* block-table entry outside [0, num_pages) */
#define PKV_DEVERR_BAD_SLOT 0x2u     /* slot_mapping entry >= num_pages * page_size */
#define PKV_DEVERR_TIMEOUT 0x4u      /* a bounded wait on a shared-memory barrier gave up */

typedef struct CUstream_st* pkv_stream_t; /* identical to cudaStream_t */
typedef struct pkv_pool pkv_pool;         /* opaque host-side pool descriptor */

/* Human-readable name of a status code (static string, never NULL). */
const char* pkv_status_string(int status);

/* ------------------------------------------------------------------------
 * KV pool  ([ENGINE] s3.4, s5.3)
 * ---------------------------------------------------------------------- */

/*
 * Describe a preallocated paged KV pool and create its host free list.
 *   k_base, v_base: device arrays of [num_layers][num_pages][kv_heads][page_size][head_dim]
 *                   elements of `dtype`; one (page, head) is page_size*head_dim contiguous
 *                   elements.  Both must be 16-byte aligned.  The caller keeps ownership and
 *                   must keep them alive while the pool is used; nothing is read or written
 *                   here.
 *   page_size: 16 or 32 tokens; head_dim: 64 or 128; dtype: PKV_F16 or PKV_BF16.
 * The free list starts with every page id 0..num_pages-1, handed out in increasing order.
 * Errors: INVALID_ARG for null/non-positive/misaligned arguments, and for a pool with
 * num_pages * kv_heads * page_size / 16 above 2^31 - 1 (the kernels index 16-token blocks
 * of a layer with 32-bit integers; such a layer would hold terabytes), UNSUPPORTED for
 * other page sizes, head dims or dtypes.
 */
int kv_pool_create(int num_layers, int num_pages, int page_size, int kv_heads, int head_dim,
                   int dtype, void* k_base, void* v_base, pkv_pool** out);

/*
 * Describe a preallocated int8 paged KV pool ([ENGINE] s3.4: the KV strategy pairs paging
 * with compression of the cached values).  Each cached (token, kv head) row x of head_dim
 * values is held as int8 codes c and one fp32 scale s with x ~ c * s:
 *   s = amax / 127 and c_i = round_half_even(x_i * (127 / amax)) clamped to [-127, 127],
 *   amax = max_i |x_i|, every step one correctly rounded fp32 operation (amax = 0 gives
 *   s = 0 and c = 0).  The scale is per row, not per page, because the cache grows one
 *   token at a time and a page's later tokens may exceed the range of its earlier ones.
 *   k_codes, v_codes: device int8 [num_layers][num_pages][kv_heads][page_size][head_dim];
 *   k_scales, v_scales: device fp32 [num_layers][num_pages][kv_heads][page_size];
 *   all four 16-byte aligned and caller-owned, as for kv_pool_create.
 *   dtype: PKV_F16 or PKV_BF16, the type of q, k, v and the output of the calls on this pool.
 * paged_kv_append and rope_append quantise the new rows as they write them;
 * paged_decode_attention reads k = c * s, v = c * s (every q_heads / kv_heads in {1, 2, 4, 8},
 * on the tensor cores); paged_prefill_attention returns UNSUPPORTED on such a pool.
 * Errors as for kv_pool_create.
 */
int kv_pool_create_i8(int num_layers, int num_pages, int page_size, int kv_heads, int head_dim,
                      int dtype, void* k_codes, void* v_codes, void* k_scales, void* v_scales,
                      pkv_pool** out);

/* Storage type of the pool's pages: PKV_I8 for kv_pool_create_i8 pools, else the element
 * type.  INVALID_ARG for a NULL pool or output. */
int kv_pool_storage(const pkv_pool* pool, int* storage_out);

/* Free the host descriptor (not the caller's device arrays).  NULL is ignored. */
void kv_pool_destroy(pkv_pool* pool);

/*
 * Take n page ids from the free list into page_ids_out[0..n) (host array).  All or
 * nothing: NO_SPACE, with nothing taken, when fewer than n pages are free.
 */
int kv_pool_alloc(pkv_pool* pool, int n, int32_t* page_ids_out);

/*
 * Give n page ids back (host array).  INVALID_ARG, with nothing returned, if any id is out of
 * range, not currently allocated, or repeated in the list.  Freed pages are handed out again
 * before never-used ones, most recently freed first.
 */
int kv_pool_free(pkv_pool* pool, int n, const int32_t* page_ids);

/* Number of free pages, or -1 for a NULL pool. */
int kv_pool_free_count(const pkv_pool* pool);

/* Shape of the pool: writes any of the non-NULL outputs; INVALID_ARG for a NULL pool. */
int kv_pool_info(const pkv_pool* pool, int* num_layers, int* num_pages, int* page_size,
                 int* kv_heads, int* head_dim, int* dtype);

/*
 * KV-cache bytes for `tokens` tokens ([ENGINE] s3.4):
 * layers x 2 (K and V) x kv_heads x head_dim x tokens x element bytes; for PKV_I8,
 * layers x 2 x kv_heads x tokens x (head_dim + 4) (codes and the row's fp32 scale).
 * -1 on bad input.
 */
int64_t pkv_kv_cache_bytes(int num_layers, int kv_heads, int head_dim, int64_t tokens, int dtype);

/*
 * Slot of each new token (host arrays; [ENGINE] s3.4 page index):
 *   slots_out[i] = block_tables[i][positions[i] / page_size] * page_size + positions[i] % page_size
 * block_tables: [n][max_pages_per_seq] int32; positions[i] < 0 marks a padded row and
 * gives slot -1.  INVALID_ARG if a position's page lies beyond max_pages_per_seq or its
 * table entry is negative.
 */
int pkv_slot_mapping(const int32_t* block_tables, int max_pages_per_seq, const int32_t* positions,
                     int n, int page_size, int64_t* slots_out);

/* ------------------------------------------------------------------------
 * Decode step kernels
 * ---------------------------------------------------------------------- */

/*
 * RoPE on the new token's q and k, in place ([ENGINE] s4.2, s4.3 apply_rotary_emb(q, k,
 * start_pos)).
 *   q: device [n_tokens][q_heads][head_dim]; k: device [n_tokens][kv_heads][head_dim];
 *   positions: device [n_tokens] int32, the position of each token; rows with a negative
 *   position are left untouched.
 * Pair i = (x[2i], x[2i+1]) of every head turns by pos * theta^(-2i/head_dim).  The angle,
 * its cosine and sine and the rotation are evaluated in fp64 and rounded once to the
 * element type.  head_dim: 64 or 128.  Either q or k may be NULL (with its head count 0);
 * q and k 16-byte aligned.
 */
int rope_apply(void* q, void* k, const int32_t* positions, int n_tokens, int q_heads,
               int kv_heads, int head_dim, double theta, int dtype, pkv_stream_t stream);

/*
 * Cache update of one layer ([ENGINE] s4.3 append to the cache, s5.3 preallocated pool):
 * for each token i with slot s = slot_mapping[i] >= 0, copies k[i][h][:] and v[i][h][:]
 * bit for bit into page s / page_size, row s % page_size of kv head h of `layer`.
 *   k, v: device [n_tokens][kv_heads][head_dim] (pool's dtype), 16-byte aligned;
 *   slot_mapping: device [n_tokens] int64 (negative = skip the row).
 * A slot >= num_pages * page_size is skipped and sets PKV_DEVERR_BAD_SLOT.
 * On an int8 pool (kv_pool_create_i8) each written row is quantised instead of copied.
 */
int paged_kv_append(const pkv_pool* pool, int layer, const void* k, const void* v,
                    const int64_t* slot_mapping, int n_tokens, pkv_stream_t stream);

/*
 * rope_apply followed by paged_kv_append in one launch ([ENGINE] s4.3 rotate then append;
 * s5.3 fuse small kernels and cut launch overhead): q [n_tokens][q_heads][head_dim] and
 * k [n_tokens][kv_heads][head_dim] are rotated in place at positions[i] (fp64, one rounding),
 * and the rotated k and v [n_tokens][kv_heads][head_dim] are copied bit for bit into the
 * pool slots slot_mapping[i] of `layer` (negative = skip; past the pool = skip and set
 * PKV_DEVERR_BAD_SLOT).  kv_heads, head_dim and the element type are the pool's.  Results
 * are identical to the two separate calls (on an int8 pool the rows are quantised as in
 * paged_kv_append).  q, k, v 16-byte aligned.
 */
int rope_append(const pkv_pool* pool, int layer, void* q, void* k, const void* v,
                const int32_t* positions, const int64_t* slot_mapping, int n_tokens, int q_heads,
                double theta, pkv_stream_t stream);

/*
 * rope_append in the decode step's form ([ENGINE] s4.3 rotate the new token, append it):
 * one new token per sequence, sequence b's at position L - 1 with L = context_lens[b] (the
 * new token counted); q[b] [q_heads][head_dim] and k[b] [kv_heads][head_dim] are turned in
 * place at that position (fp64, one rounding) and the turned k[b] and v[b] are copied bit
 * for bit (int8 pool: quantised) into row (L - 1) % page_size of page
 * block_tables[b][(L - 1) / page_size] of `layer`.  Results are identical to rope_append
 * given positions L - 1 and the slots pkv_slot_mapping gives them; sequences with L <= 0 are
 * left untouched.  A table entry outside [0, num_pages), or a position past
 * max_pages_per_seq pages, is skipped and sets PKV_DEVERR_BAD_PAGE.
 *   q, k, v: device, 16-byte aligned; block_tables [batch][max_pages_per_seq] and
 *   context_lens [batch]: device int32, as for paged_decode_attention.
 * Since it writes nothing but each sequence's newest token, it lets the next kernel on the
 * stream start at once: a paged_decode_attention given the same context_lens and
 * block_tables prefetches every other page while this call runs.
 */
int rope_append_step(const pkv_pool* pool, int layer, void* q, void* k, const void* v,
                     const int32_t* block_tables, int max_pages_per_seq, const int32_t* context_lens,
                     int batch, int q_heads, double theta, pkv_stream_t stream);

/*
 * RMSNorm of each row of the decode hidden state ([ENGINE] s4.2: root mean square only,
 * eps added to the mean square before the root):
 *   out[r][i] = h[r][i] * rsqrt(mean_i(h[r][i]^2) + eps) * weight[i]
 * with h = x, or, when `residual` is not NULL, h = x + residual rounded once to the element
 * type and written back to `residual` (the fused residual add of a decoder block).
 *   out, x, residual: device [rows][hidden]; weight: device [hidden]; all 16-byte aligned;
 *   out may be x.  hidden a multiple of 8, at most 16384; sum of squares and scaling in fp32,
 *   one rounding of the result.
 */
int rms_norm(void* out, const void* x, void* residual, const void* weight, int rows, int hidden,
             float eps, int dtype, pkv_stream_t stream);

/*
 * Number of work partitions paged_decode_attention uses when called with num_splits = 0 on
 * the current device (SM count x resident CTAs per SM for this shape, at most
 * PKV_MAX_DECODE_SPLITS).  Needs a CUDA device; PKV_ERR_CUDA without one.
 */
int pkv_decode_default_splits(int q_heads, int kv_heads, int head_dim, int page_size, int dtype,
                              int* num_splits_out);

/*
 * The split count paged_decode_attention and paged_decode_layer use for num_splits = 0 on
 * this pool and shape: pkv_decode_default_splits (a full wave of CTAs), or fewer when
 * kv_heads x batch x the work units of max_pages_per_seq pages (a unit is a page for one
 * query head per kv head, 16 tokens for grouped heads, 32 tokens on int8 pages) would leave
 * a CTA fewer than 16 units: ceil(units / 16), at least 1.  Never above
 * pkv_decode_default_splits, so a workspace sized for that serves every automatic call.
 * Needs a CUDA device (PKV_ERR_CUDA without one); INVALID_ARG / UNSUPPORTED as for
 * paged_decode_attention.
 */
int pkv_decode_auto_splits(const pkv_pool* pool, int batch, int max_pages_per_seq, int q_heads, int kv_heads,
                           int* num_splits_out);

/*
 * Whether num_splits = 0 runs the cluster variant on this pool and shape, and its cluster
 * size: *cluster_out = C >= 2, or 0 for the partitioned kernel.  The cluster variant serves
 * 16-bit pools with one query head per kv head when batch x kv_heads is at most half of
 * pkv_decode_default_splits: one thread-block cluster of C = min(8, default_splits /
 * (batch x kv_heads), max_pages_per_seq) CTAs per (sequence, kv head), each CTA taking an
 * equal share of that pair's pages, the shares merged through distributed shared memory
 * (no workspace is touched).  Needs a CUDA device (PKV_ERR_CUDA without one); INVALID_ARG /
 * UNSUPPORTED as for paged_decode_attention.
 */
int pkv_decode_cluster_size(const pkv_pool* pool, int batch, int max_pages_per_seq, int q_heads, int kv_heads,
                            int* cluster_out);

/*
 * Workspace bytes paged_decode_attention needs for `num_splits` (1 .. PKV_MAX_DECODE_SPLITS)
 * partitions: a fixed region of PKV_MAX_DECODE_SPLITS int32 counters (16 KiB), then per
 * partition two fp32 partial results (running max, sum and the unnormalised output of every
 * query head of a kv-head group).  The counters do not move with num_splits, so one
 * workspace serves calls with any split count up to the one it was sized for.  `batch` is
 * accepted for compatibility and does not change the size.  0 on bad input.
 */
size_t pkv_decode_workspace_size(int batch, int q_heads, int kv_heads, int head_dim,
                                 int num_splits);

/*
 * Decode attention of one new query token per sequence over its paged cache
 * ([ENGINE] s4.3, [FLOW] s2.2.2):
 *   out[b][h][:] = sum_t softmax_t(scale * <q[b][h], K_b[t][g]>) * V_b[t][g],
 *   g = h / (q_heads / kv_heads), t over the context_lens[b] cached tokens, token t of
 *   sequence b read from page block_tables[b][t / page_size], row t % page_size.
 * The query sits at the last position, so the causal mask keeps every cached token.
 *   out, q: device [batch][q_heads][head_dim] (pool's dtype), 16-byte aligned; out is
 *           written once, rounded to nearest-even from fp32; rows with context_lens[b] <= 0
 *           get zeros.
 *   block_tables: device [batch][max_pages_per_seq] int32; entries past a row's
 *           ceil(context_lens[b] / page_size) pages are not read.
 *   context_lens: device [batch] int32, the new token included.
 *   kv_heads must equal the pool's; q_heads a multiple of it with q_heads / kv_heads in
 *   {1, 2, 4, 8}.
 *   num_splits: number of work partitions, at most PKV_MAX_DECODE_SPLITS
 *           (0 = pkv_decode_auto_splits for this shape, or the cluster variant where
 *           pkv_decode_cluster_size gives one).  The batch's
 *           pages x kv heads are laid end to end and cut into num_splits equal ranges, one
 *           per CTA; a (sequence, kv head) cut by a range boundary is finished by the CTA
 *           that delivers its last partial, which rescales the partial softmax sums
 *           (log-sum-exp).  One kernel launch per call.
 *   workspace: device scratch of >= pkv_decode_workspace_size(batch, q_heads, kv_heads,
 *           head_dim, num_splits) bytes, 256-byte aligned, zero-filled before its first use
 *           (pkv_decode_workspace_clear or any memset); every call leaves its counter region
 *           at zero, so the next call may use any split count the workspace is large enough
 *           for.  Calls that share a workspace must be ordered on one stream.
 * Errors: INVALID_ARG (bad pointer/shape/layer, num_splits above PKV_MAX_DECODE_SPLITS),
 * UNSUPPORTED (group/head_dim/page/dtype
 * combination), NO_SPACE (workspace too small), CUDA (launch failure).
 */
int paged_decode_attention(const pkv_pool* pool, int layer, void* out, const void* q,
                           const int32_t* block_tables, int max_pages_per_seq,
                           const int32_t* context_lens, int batch, int q_heads, int kv_heads,
                           float scale, int num_splits, void* workspace, size_t workspace_bytes,
                           pkv_stream_t stream);

/*
 * paged_decode_attention for callers that cannot allocate device memory.  The pages have
 * no counterpart: this is a library convenience, not part of the method.
 * Who needs it: a plugin whose host application owns all device memory and gives the
 * plugin no allocator, a runtime whose caching allocator has already reserved the whole
 * GPU, or a serving loop that may not call cudaMalloc (it synchronises the device).
 * Arguments, results and errors are those of paged_decode_attention, without the
 * workspace: the scratch is a fixed 4 MiB array inside the library, in device memory
 * that every GPU which loads the library holds until the process exits.
 *   - A call whose scratch would exceed 4 MiB (the 16 KiB counter region plus
 *     2 x num_splits x (q_heads / kv_heads) x (head_dim + 2) fp32 values, each part rounded
 *     up to 256 bytes) is rejected with PKV_ERR_NO_SPACE and launches nothing; the pool,
 *     layer and shape are checked first, as in paged_decode_attention.  On B200 the
 *     automatic split count (num_splits = 0) fits for every shape the kernels accept.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call before any
 *     stream capture begins.
 *   - All calls on a device share the one array, which keeps the previous call's
 *     contents; nothing in it needs clearing (its counter region is zero when the library
 *     is loaded, every call leaves it at zero, and no call's partial results overlap it,
 *     whatever the split counts of consecutive calls).  Calls that overlap on the GPU
 *     (different streams, or several host threads) race on it: order them on one stream.
 *   - No cudaMalloc, cudaFree or allocating library routine is called.
 */
int paged_decode_attention_noalloc(const pkv_pool* pool, int layer, void* out, const void* q,
                                   const int32_t* block_tables, int max_pages_per_seq,
                                   const int32_t* context_lens, int batch, int q_heads, int kv_heads,
                                   float scale, int num_splits, pkv_stream_t stream);

/*
 * Chunked prefill attention over the paged cache ([ENGINE] s4.3: a chunk of seq_len tokens
 * at start_pos with the causal mask slice [start_pos : start_pos + seq_len]).  The chunk's
 * k and v must already be in the pool (rope_apply / paged_kv_append take any number of
 * tokens with their positions and slots).
 *   q, out: device [total_q][q_heads][head_dim] (pool's dtype), 16-byte aligned; the rows of
 *           sequence b are cu_q[b] .. cu_q[b+1] - 1 (cu_q: device [batch + 1] int32, cu_q[0] = 0,
 *           cu_q[batch] = total_q, non-decreasing).
 *   context_lens: device [batch] int32, the cached tokens of each sequence with the chunk
 *           included (L_b >= n_b); row i of sequence b sits at position L_b - n_b + i and
 *           attends to tokens 0 .. L_b - n_b + i.
 *   block_tables, max_pages_per_seq, kv_heads, scale: as for paged_decode_attention;
 *   q_heads / kv_heads in {1, 2, 4, 8}.
 * One CTA per (sequence, kv head, two tiles of 128 query rows) on the fifth-generation
 * tensor cores (tcgen05.mma, S and O accumulated in tensor memory; fp32 online softmax;
 * softmax, MMA and copy warps meet on mbarriers); K and V pages
 * are staged by tiled TMA through tensor maps of this layer's pools, encoded on the host
 * for each call; no workspace.
 * Errors as for paged_decode_attention; PKV_ERR_CUDA also when the driver's tensor-map
 * encoder cannot be found or rejects the pool; on an int8 pool, UNSUPPORTED.  A CTA keeps
 * one int per sequence (batch + 1) in shared memory beside its tiles, so batch is bounded
 * (about 8900 sequences at head_dim 128 fp16, 13000 bf16, 27000-29000 at head_dim 64):
 * UNSUPPORTED above.
 */
int paged_prefill_attention(const pkv_pool* pool, int layer, void* out, const void* q, const int32_t* cu_q,
                            int total_q, const int32_t* block_tables, int max_pages_per_seq,
                            const int32_t* context_lens, int batch, int q_heads, int kv_heads, float scale,
                            pkv_stream_t stream);

/*
 * Angles of a decode step's new tokens, shared by all layers of the step ([ENGINE] s4.2):
 * table[b][i] = (cos, sin)(pos_b * theta^(-2i/head_dim)) in fp64 for pos_b = context_lens[b] - 1
 * (the new token's position; zeros when context_lens[b] <= 0), evaluated exactly as
 * rope_apply does.
 *   context_lens: device [batch] int32; table: device [batch][head_dim / 2][2] double,
 *   16-byte aligned, written by the call.  head_dim 64 or 128.
 */
int rope_table(const int32_t* context_lens, int batch, int head_dim, double theta, double* table,
               pkv_stream_t stream);

/*
 * One whole decode layer in one launch ([ENGINE] s4.3 rotate, append, attend; s5.3 fuse small
 * kernels): for each sequence b with L = context_lens[b] > 0 the new token sits at position
 * L - 1 of its page table; its k is turned by RoPE and written with v into that slot of
 * `layer` (the append, bit for bit as rope_append would), q is turned likewise, and `out`
 * receives the same attention as paged_decode_attention over the L tokens.
 *   q: device [batch][q_heads][head_dim] and k, v: device [batch][kv_heads][head_dim], not yet
 *      turned and left unchanged; rope: the step's rope_table; every other argument as for
 *      paged_decode_attention (workspace sized by pkv_decode_workspace_size).
 * Supported: 16-bit pools with q_heads == kv_heads, and int8 pools (kv_pool_create_i8) with
 * q_heads / kv_heads in {1, 2, 4, 8}, whose new rows are quantised as paged_kv_append does
 * (UNSUPPORTED otherwise).  A page id out of range is skipped and flagged as in
 * paged_decode_attention.
 */
int paged_decode_layer(const pkv_pool* pool, int layer, void* out, const void* q, const void* k,
                       const void* v, const double* rope, const int32_t* block_tables, int max_pages_per_seq,
                       const int32_t* context_lens, int batch, int q_heads, int kv_heads, float scale,
                       int num_splits, void* workspace, size_t workspace_bytes, pkv_stream_t stream);

/*
 * Zero-fill a decode workspace (cudaMemsetAsync on `stream`) before its first use with
 * paged_decode_attention.  INVALID_ARG for a NULL workspace with a non-zero size.
 */
int pkv_decode_workspace_clear(void* workspace, size_t workspace_bytes, pkv_stream_t stream);

/*
 * Read and clear the device error word (PKV_DEVERR_* bits) of the current device.
 * Synchronises the device.  PKV_ERR_CUDA if the read fails.
 */
int kv_get_device_error(uint32_t* err_out);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H_ */
