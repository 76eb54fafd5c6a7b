// libpagedkv: C-ABI entry points that launch the decode-step kernels on sm_100a.
//
// Every entry point validates its arguments on the host, launches asynchronously on
// the caller's stream and returns a PKV_* status.  Kernels are launched with
// programmatic stream serialization (programmatic dependent launch), so the next
// library kernel on the stream can start its prologue while the previous one drains;
// each kernel waits (griddepcontrol.wait) before touching data the previous kernel
// may write.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "decode_attention.cuh"
#include "decode_attention_i8.cuh"
#include "decode_attention_mma.cuh"
#include "prefill_attention_tc.cuh"
#include "pagedkv.h"
#include "pkv_internal.h"
#include "rms_norm.cuh"
#include "rope_append.cuh"

namespace pkv {
namespace {

template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args)
{
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

int status_of(cudaError_t e) { return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA; }

// As launch_pdl, in thread-block clusters of `cluster` CTAs along x.
template <typename Kernel, typename... Args>
cudaError_t launch_pdl_cluster(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, int cluster,
                               Args... args)
{
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

constexpr int kMaxDevices = 64;

// Raise a kernel's dynamic shared-memory limit once per device (and size).
template <typename Kernel>
cudaError_t ensure_smem(Kernel kernel, int bytes, int* configured)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (configured[dev] >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) configured[dev] = bytes;
    return e;
}

constexpr int kMaxSmemPerCta = 227 * 1024;

struct DecodeOps {
    int (*launch)(const DecodeParams&, cudaStream_t);
    int (*splits)(int*);
    int group;
    int unit_tokens;    // tokens of one work unit: a page (CUDA cores), 16 (MMA), 32 (int8)
};

// The automatic split count: the device's full wave (SMs x resident CTAs), unless the
// batch's work is too small to give every CTA at least kMinUnitsPerCta units; then fewer,
// fuller CTAs -- each CTA pays a fixed cost (lengths scan, first page-table window, ring
// fill, merge of its cut segments) that a few units do not amortise.  The host knows only
// an upper bound of the work: kv_heads x batch x the units of max_pages_per_seq pages.
constexpr long long kMinUnitsPerCta = 16;

int auto_splits(int full_wave, long long max_units)
{
    const long long n = (max_units + kMinUnitsPerCta - 1) / kMinUnitsPerCta;
    return n < 1 ? 1 : (n < full_wave ? (int)n : full_wave);
}

long long max_decode_units(int kv_heads, int batch, int max_pages, int page_size, int unit_tokens)
{
    const long long per_seq = ((long long)max_pages * page_size + unit_tokens - 1) / unit_tokens;
    return (long long)kv_heads * batch * per_seq;
}

// One query head per kv head: the CUDA-core kernel; 2 to 8 heads sharing a kv head: the
// tensor-core kernel.  Int8 pages (I8): the int8 tensor-core kernel for every group size.
template <int D, int P, int G, typename T, bool I8, bool kMma = (G > 1)>
struct DecodeKernel {
    static constexpr auto fn = decode_pass1_kernel<D, P, G, T>;
    static int smem(int batch) { return DecodeShape<D, P, G>::smem_bytes(batch); }
};
template <int D, int P, int G, typename T, bool kMma>
struct DecodeKernel<D, P, G, T, true, kMma> {
    static constexpr auto fn = decode_i8_kernel<D, P, G, T>;
    static int smem(int batch) { return I8Shape<D, G>::smem_bytes(batch); }
};
template <int D, int P, int G, typename T>
struct DecodeKernel<D, P, G, T, false, true> {
    static constexpr auto fn = decode_pass1_mma_kernel<D, P, G, T>;
    static int smem(int batch) { return MmaShape<D, G>::smem_bytes(batch); }
};

template <int D, int P, int G, typename T, bool I8>
struct DecodeImpl {
    using K = DecodeKernel<D, P, G, T, I8>;
    static int configured[kMaxDevices];

    static int launch(const DecodeParams& prm, cudaStream_t st)
    {
        const int smem = K::smem(prm.batch);
        if (smem > kMaxSmemPerCta) return PKV_ERR_UNSUPPORTED;
        cudaError_t e = ensure_smem(K::fn, smem, configured);
        if (e != cudaSuccess) return PKV_ERR_CUDA;
        e = launch_pdl(K::fn, dim3(prm.num_splits), dim3(kDecodeThreads), smem, st, prm);
        return status_of(e);
    }

    // SMs x resident CTAs per SM (at the shared-memory size of a 64-row batch), at most
    // three per SM: a fourth did not fit beside the RoPE/append kernel and ran slower.
    static int splits(int* out)
    {
        int dev = 0, sms = 0, per_sm = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return PKV_ERR_CUDA;
        const int smem = K::smem(64);
        if (ensure_smem(K::fn, smem, configured) != cudaSuccess) return PKV_ERR_CUDA;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, K::fn, kDecodeThreads, smem) != cudaSuccess)
            return PKV_ERR_CUDA;
        const int n = sms * (per_sm > 3 ? 3 : (per_sm > 0 ? per_sm : 1));
        *out = n < PKV_MAX_DECODE_SPLITS ? n : PKV_MAX_DECODE_SPLITS;
        return PKV_OK;
    }
};

template <int D, int P, int G, typename T, bool I8>
int DecodeImpl<D, P, G, T, I8>::configured[kMaxDevices] = {0};

// Tokens of one work unit of the decode kernel for this page size, group and storage.
constexpr int unit_tokens(int P, int group, bool i8) { return i8 ? 32 : (group == 1 ? P : 16); }

template <int D, int P, typename T, bool I8>
bool pick_group(int group, DecodeOps& ops)
{
    const int ut = unit_tokens(P, group, I8);
    switch (group) {
    case 1: ops = {DecodeImpl<D, P, 1, T, I8>::launch, DecodeImpl<D, P, 1, T, I8>::splits, 1, ut}; return true;
    case 2: ops = {DecodeImpl<D, P, 2, T, I8>::launch, DecodeImpl<D, P, 2, T, I8>::splits, 2, ut}; return true;
    case 4: ops = {DecodeImpl<D, P, 4, T, I8>::launch, DecodeImpl<D, P, 4, T, I8>::splits, 4, ut}; return true;
    case 8: ops = {DecodeImpl<D, P, 8, T, I8>::launch, DecodeImpl<D, P, 8, T, I8>::splits, 8, ut}; return true;
    default: return false;
    }
}

template <typename T, bool I8>
bool pick_shape(int head_dim, int page_size, int group, DecodeOps& ops)
{
    if (head_dim == 128 && page_size == 16) return pick_group<128, 16, T, I8>(group, ops);
    if (head_dim == 128 && page_size == 32) return pick_group<128, 32, T, I8>(group, ops);
    if (head_dim == 64 && page_size == 16) return pick_group<64, 16, T, I8>(group, ops);
    if (head_dim == 64 && page_size == 32) return pick_group<64, 32, T, I8>(group, ops);
    return false;
}

// dtype: the type of q and the output; storage: the pages' type (dtype or PKV_I8)
bool pick_decode(int head_dim, int page_size, int group, int dtype, int storage, DecodeOps& ops)
{
    const bool i8 = storage == PKV_I8;
    if (!i8 && storage != dtype) return false;
    if (dtype == PKV_F16)
        return i8 ? pick_shape<__half, true>(head_dim, page_size, group, ops)
                  : pick_shape<__half, false>(head_dim, page_size, group, ops);
    if (dtype == PKV_BF16)
        return i8 ? pick_shape<__nv_bfloat16, true>(head_dim, page_size, group, ops)
                  : pick_shape<__nv_bfloat16, false>(head_dim, page_size, group, ops);
    return false;
}

// The cluster variant of the CUDA-core kernel (16-bit pages, one query head per kv head):
// one cluster of C CTAs per (sequence, kv head), used for num_splits = 0 when the batch's
// (sequence, kv head) pairs number at most half the full wave; C = min(8, wave / pairs,
// max_pages_per_seq), at least 2.  0 when the variant does not apply.
int cluster_size(int full_wave, int batch, int kv_heads, int max_pages)
{
    const long long pairs = (long long)batch * kv_heads;
    if (pairs <= 0 || 2 * pairs > full_wave) return 0;
    int c = (int)(full_wave / pairs);
    c = c < 8 ? c : 8;
    c = c < max_pages ? c : max_pages;
    return c >= 2 ? c : 0;
}

template <int D, int P, typename T, bool kFused>
int launch_cluster(const DecodeParams& prm, cudaStream_t st)
{
    static int configured[kMaxDevices] = {0};
    constexpr auto fn = decode_pass1_kernel<D, P, 1, T, kFused, true>;
    const int smem = DecodeShape<D, P, 1, kFused, true>::smem_bytes(prm.batch);
    if (smem > kMaxSmemPerCta) return PKV_ERR_UNSUPPORTED;
    if (ensure_smem(fn, smem, configured) != cudaSuccess) return PKV_ERR_CUDA;
    const int grid = prm.batch * prm.kv_heads * prm.cluster;
    return status_of(launch_pdl_cluster(fn, dim3(grid), dim3(kDecodeThreads), smem, st, prm.cluster, prm));
}

template <typename T, bool kFused>
int cluster_shape(int head_dim, int page_size, const DecodeParams& prm, cudaStream_t st)
{
    if (head_dim == 128 && page_size == 16) return launch_cluster<128, 16, T, kFused>(prm, st);
    if (head_dim == 128 && page_size == 32) return launch_cluster<128, 32, T, kFused>(prm, st);
    if (head_dim == 64 && page_size == 16) return launch_cluster<64, 16, T, kFused>(prm, st);
    if (head_dim == 64 && page_size == 32) return launch_cluster<64, 32, T, kFused>(prm, st);
    return PKV_ERR_UNSUPPORTED;
}

template <bool kFused>
int launch_cluster_variant(const pkv_pool* pool, const DecodeParams& prm, cudaStream_t st)
{
    if (pool->dtype == PKV_F16) return cluster_shape<__half, kFused>(pool->head_dim, pool->page_size, prm, st);
    return cluster_shape<__nv_bfloat16, kFused>(pool->head_dim, pool->page_size, prm, st);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WorkspaceLayout {
    size_t counters, part_o, part_ml, total;
};

// The per-partition counters sit in a region of fixed size at the start of the
// workspace, whatever num_splits is: a call with more partitions than the previous call
// on the same scratch must find zeros there, never the previous call's partial results.
WorkspaceLayout workspace_layout(int batch, int group, int head_dim, int num_splits)
{
    (void)batch;
    WorkspaceLayout w;
    w.counters = 0;
    w.part_o = align256(sizeof(int) * (size_t)PKV_MAX_DECODE_SPLITS);
    w.part_ml = w.part_o + align256(sizeof(float) * 2 * (size_t)num_splits * group * head_dim);
    w.total = w.part_ml + align256(sizeof(float) * 2 * (size_t)num_splits * group * 2);
    return w;
}

}  // namespace
}  // namespace pkv

using namespace pkv;

namespace pkv {
namespace {

int launch_rope_append(const RopeAppendParams& prm, int n_tokens, int dtype, cudaStream_t st)
{
    const int vph = prm.head_dim / 8;
    const int nq = (prm.mode & kRopeRotate) ? prm.q_heads * vph : 0;
    const int total = nq + ((prm.mode & kRopeAppend) ? 2 : 1) * prm.kv_heads * vph;
    const int parts = (total + 255) / 256;
    const dim3 grid(n_tokens, parts > 0 ? parts : 1);
    cudaError_t e;
    if (dtype == PKV_F16)
        e = launch_pdl(rope_append_kernel<__half>, grid, dim3(256), 0, st, prm);
    else
        e = launch_pdl(rope_append_kernel<__nv_bfloat16>, grid, dim3(256), 0, st, prm);
    return status_of(e);
}

RopeAppendParams pool_params(const pkv_pool* pool, int layer)
{
    RopeAppendParams prm;
    std::memset(&prm, 0, sizeof(prm));
    const size_t off = (size_t)layer * pool->layer_bytes();
    prm.k_layer = static_cast<char*>(pool->k_base) + off;
    prm.v_layer = static_cast<char*>(pool->v_base) + off;
    if (pool->storage == kStorageI8) {
        prm.ks_layer = static_cast<float*>(pool->k_scale_base) + (size_t)layer * pool->layer_rows();
        prm.vs_layer = static_cast<float*>(pool->v_scale_base) + (size_t)layer * pool->layer_rows();
        prm.mode = kRopeQuantI8;
    }
    prm.kv_heads = pool->kv_heads;
    prm.head_dim = pool->head_dim;
    prm.page_size = pool->page_size;
    prm.num_slots = (int64_t)pool->num_pages * pool->page_size;
    return prm;
}

bool misaligned16(const void* a, const void* b = nullptr, const void* c = nullptr)
{
    return ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b) | reinterpret_cast<uintptr_t>(c)) & 15u) != 0;
}

}  // namespace
}  // namespace pkv

extern "C" int rope_apply(void* q, void* k, const int32_t* positions, int n_tokens, int q_heads, int kv_heads,
                          int head_dim, double theta, int dtype, pkv_stream_t stream)
{
    if (n_tokens < 0 || q_heads < 0 || kv_heads < 0 || !(theta > 0.0)) return PKV_ERR_INVALID_ARG;
    if ((q_heads > 0 && !q) || (kv_heads > 0 && !k)) return PKV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
    if (n_tokens == 0 || q_heads + kv_heads == 0) return PKV_OK;
    if (!positions || misaligned16(q, k)) return PKV_ERR_INVALID_ARG;
    RopeAppendParams prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.q = q;
    prm.k = k;
    prm.positions = positions;
    prm.q_heads = q_heads;
    prm.kv_heads = kv_heads;
    prm.head_dim = head_dim;
    prm.theta = theta;
    prm.mode = kRopeRotate | kRopeEarlyRelease;     // writes no pool page
    return launch_rope_append(prm, n_tokens, dtype, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int paged_kv_append(const pkv_pool* pool, int layer, const void* k, const void* v,
                               const int64_t* slot_mapping, int n_tokens, pkv_stream_t stream)
{
    if (!pool || layer < 0 || layer >= pool->num_layers || n_tokens < 0) return PKV_ERR_INVALID_ARG;
    if (n_tokens == 0) return PKV_OK;
    if (!k || !v || !slot_mapping) return PKV_ERR_INVALID_ARG;
    if (misaligned16(k, v)) return PKV_ERR_INVALID_ARG;
    RopeAppendParams prm = pool_params(pool, layer);
    prm.k = const_cast<void*>(k);    // read only: no rotation in this mode
    prm.v = v;
    prm.slots = slot_mapping;
    prm.mode |= kRopeAppend;
    return launch_rope_append(prm, n_tokens, pool->dtype, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int rope_append(const pkv_pool* pool, int layer, void* q, void* k, const void* v,
                           const int32_t* positions, const int64_t* slot_mapping, int n_tokens, int q_heads,
                           double theta, pkv_stream_t stream)
{
    if (!pool || layer < 0 || layer >= pool->num_layers || n_tokens < 0 || q_heads < 0 || !(theta > 0.0))
        return PKV_ERR_INVALID_ARG;
    if (n_tokens == 0) return PKV_OK;
    if (!k || !v || !positions || !slot_mapping || (q_heads > 0 && !q)) return PKV_ERR_INVALID_ARG;
    if (misaligned16(q, k, v)) return PKV_ERR_INVALID_ARG;
    RopeAppendParams prm = pool_params(pool, layer);
    prm.q = q;
    prm.k = k;
    prm.v = v;
    prm.positions = positions;
    prm.slots = slot_mapping;
    prm.q_heads = q_heads;
    prm.theta = theta;
    prm.mode |= kRopeRotate | kRopeAppend;
    return launch_rope_append(prm, n_tokens, pool->dtype, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int rope_append_step(const pkv_pool* pool, int layer, void* q, void* k, const void* v,
                                const int32_t* block_tables, int max_pages_per_seq, const int32_t* context_lens,
                                int batch, int q_heads, double theta, pkv_stream_t stream)
{
    if (!pool || layer < 0 || layer >= pool->num_layers || batch < 0 || q_heads < 0 || !(theta > 0.0))
        return PKV_ERR_INVALID_ARG;
    if (max_pages_per_seq <= 0) return PKV_ERR_INVALID_ARG;
    if (batch == 0) return PKV_OK;
    if (!k || !v || !block_tables || !context_lens || (q_heads > 0 && !q)) return PKV_ERR_INVALID_ARG;
    if (misaligned16(q, k, v)) return PKV_ERR_INVALID_ARG;
    RopeAppendParams prm = pool_params(pool, layer);
    prm.q = q;
    prm.k = k;
    prm.v = v;
    prm.context_lens = context_lens;
    prm.block_tables = block_tables;
    prm.max_pages = max_pages_per_seq;
    prm.q_heads = q_heads;
    prm.theta = theta;
    // writes only each sequence's newest token: the next kernel may start at once
    prm.mode |= kRopeRotate | kRopeAppend | kRopeFromLens | kRopeEarlyRelease;
    return launch_rope_append(prm, batch, pool->dtype, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int rms_norm(void* out, const void* x, void* residual, const void* weight, int rows, int hidden,
                        float eps, int dtype, pkv_stream_t stream)
{
    if (rows < 0 || hidden <= 0 || hidden % 8 || !(eps >= 0.f)) return PKV_ERR_INVALID_ARG;
    if (hidden > kNormThreads * kNormMaxVecPerThread * 8) return PKV_ERR_UNSUPPORTED;
    if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
    if (rows == 0) return PKV_OK;
    if (!out || !x || !weight) return PKV_ERR_INVALID_ARG;
    if (misaligned16(out, x, weight) || misaligned16(residual)) return PKV_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (dtype == PKV_F16)
        e = launch_pdl(rms_norm_kernel<__half>, dim3(rows), dim3(kNormThreads), 0, st, static_cast<__half*>(out),
                       static_cast<const __half*>(x), static_cast<__half*>(residual),
                       static_cast<const __half*>(weight), hidden, eps);
    else
        e = launch_pdl(rms_norm_kernel<__nv_bfloat16>, dim3(rows), dim3(kNormThreads), 0, st,
                       static_cast<__nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(x),
                       static_cast<__nv_bfloat16*>(residual), static_cast<const __nv_bfloat16*>(weight), hidden, eps);
    return status_of(e);
}

extern "C" int pkv_decode_default_splits(int q_heads, int kv_heads, int head_dim, int page_size, int dtype,
                                         int* num_splits_out)
{
    if (!num_splits_out || q_heads <= 0 || kv_heads <= 0 || q_heads % kv_heads) return PKV_ERR_INVALID_ARG;
    DecodeOps ops;
    const int act = dtype == PKV_I8 ? PKV_F16 : dtype;     // int8 pages: split count of the f16 kernel
    if (!pick_decode(head_dim, page_size, q_heads / kv_heads, act, dtype, ops)) return PKV_ERR_UNSUPPORTED;
    return ops.splits(num_splits_out);
}

extern "C" int pkv_decode_auto_splits(const pkv_pool* pool, int batch, int max_pages_per_seq, int q_heads,
                                      int kv_heads, int* num_splits_out)
{
    if (!pool || !num_splits_out || batch < 0 || max_pages_per_seq <= 0 || q_heads <= 0 || kv_heads != pool->kv_heads ||
        q_heads % kv_heads)
        return PKV_ERR_INVALID_ARG;
    DecodeOps ops;
    if (!pick_decode(pool->head_dim, pool->page_size, q_heads / kv_heads, pool->dtype, pool->storage, ops))
        return PKV_ERR_UNSUPPORTED;
    int full = 0;
    const int st = ops.splits(&full);
    if (st != PKV_OK) return st;
    *num_splits_out = auto_splits(full, max_decode_units(kv_heads, batch, max_pages_per_seq, pool->page_size,
                                                         ops.unit_tokens));
    return PKV_OK;
}

extern "C" int pkv_decode_cluster_size(const pkv_pool* pool, int batch, int max_pages_per_seq, int q_heads,
                                       int kv_heads, int* cluster_out)
{
    if (!pool || !cluster_out || batch < 0 || max_pages_per_seq <= 0 || q_heads <= 0 || kv_heads != pool->kv_heads ||
        q_heads % kv_heads)
        return PKV_ERR_INVALID_ARG;
    DecodeOps ops;
    if (!pick_decode(pool->head_dim, pool->page_size, q_heads / kv_heads, pool->dtype, pool->storage, ops))
        return PKV_ERR_UNSUPPORTED;
    int full = 0;
    const int st = ops.splits(&full);
    if (st != PKV_OK) return st;
    *cluster_out = (pool->storage != kStorageI8 && ops.group == 1)
                       ? cluster_size(full, batch, kv_heads, max_pages_per_seq) : 0;
    return PKV_OK;
}

extern "C" size_t pkv_decode_workspace_size(int batch, int q_heads, int kv_heads, int head_dim, int num_splits)
{
    if (batch < 0 || q_heads <= 0 || kv_heads <= 0 || q_heads % kv_heads || head_dim <= 0 || num_splits <= 0 ||
        num_splits > PKV_MAX_DECODE_SPLITS)
        return 0;
    return workspace_layout(batch, q_heads / kv_heads, head_dim, num_splits).total;
}

extern "C" int paged_decode_attention(const pkv_pool* pool, int layer, void* out, const void* q,
                                      const int32_t* block_tables, int max_pages_per_seq,
                                      const int32_t* context_lens, int batch, int q_heads, int kv_heads, float scale,
                                      int num_splits, void* workspace, size_t workspace_bytes, pkv_stream_t stream)
{
    if (!pool || layer < 0 || layer >= pool->num_layers) return PKV_ERR_INVALID_ARG;
    if (batch < 0 || q_heads <= 0 || kv_heads != pool->kv_heads || q_heads % kv_heads) return PKV_ERR_INVALID_ARG;
    if (num_splits < 0 || num_splits > PKV_MAX_DECODE_SPLITS || max_pages_per_seq <= 0 || !(scale == scale))
        return PKV_ERR_INVALID_ARG;
    if (batch == 0) return PKV_OK;
    if (!out || !q || !block_tables || !context_lens || !workspace) return PKV_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(q)) & 15u) return PKV_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return PKV_ERR_INVALID_ARG;
    DecodeOps ops;
    if (!pick_decode(pool->head_dim, pool->page_size, q_heads / kv_heads, pool->dtype, pool->storage, ops))
        return PKV_ERR_UNSUPPORTED;
    int cluster = 0;
    if (num_splits == 0) {
        const int st = ops.splits(&num_splits);
        if (st != PKV_OK) return st;
        if (pool->storage != kStorageI8 && ops.group == 1)
            cluster = cluster_size(num_splits, batch, kv_heads, max_pages_per_seq);
        num_splits = auto_splits(num_splits, max_decode_units(kv_heads, batch, max_pages_per_seq, pool->page_size,
                                                              ops.unit_tokens));
    }
    const WorkspaceLayout wl = workspace_layout(batch, ops.group, pool->head_dim, num_splits);
    if (workspace_bytes < wl.total) return PKV_ERR_NO_SPACE;
    DecodeParams prm;
    prm.cluster = cluster;
    prm.k = static_cast<const char*>(pool->k_base) + (size_t)layer * pool->layer_bytes();
    prm.v = static_cast<const char*>(pool->v_base) + (size_t)layer * pool->layer_bytes();
    prm.k_scale = nullptr;
    prm.v_scale = nullptr;
    if (pool->storage == kStorageI8) {
        prm.k_scale = static_cast<const float*>(pool->k_scale_base) + (size_t)layer * pool->layer_rows();
        prm.v_scale = static_cast<const float*>(pool->v_scale_base) + (size_t)layer * pool->layer_rows();
    }
    prm.q = q;
    prm.out = out;
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    prm.counters = reinterpret_cast<int*>(ws + wl.counters);
    prm.part_o = reinterpret_cast<float*>(ws + wl.part_o);
    prm.part_ml = reinterpret_cast<float*>(ws + wl.part_ml);
    prm.batch = batch;
    prm.max_pages = max_pages_per_seq;
    prm.q_heads = q_heads;
    prm.kv_heads = kv_heads;
    prm.num_pages = pool->num_pages;
    prm.num_splits = num_splits;
    prm.scale_log2 = scale * 1.4426950408889634f;
    if (cluster) return launch_cluster_variant<false>(pool, prm, reinterpret_cast<cudaStream_t>(stream));
    return ops.launch(prm, reinterpret_cast<cudaStream_t>(stream));
}

namespace pkv {
namespace {

// The fused decode layer: the attention kernels with RoPE and the append folded in --
// the CUDA-core kernel for 16-bit pages with one query head per kv head, the int8 kernel
// for int8 pages with any group size.
template <int D, int P, int G, typename T, bool I8>
struct FusedKernel {      // 16-bit pages: the CUDA-core kernel (one query head per kv head)
    static constexpr auto fn = decode_pass1_kernel<D, P, G, T, true>;
    static int smem(int batch) { return DecodeShape<D, P, G, true>::smem_bytes(batch); }
};
template <int D, int P, int G, typename T>
struct FusedKernel<D, P, G, T, true> {
    static constexpr auto fn = decode_i8_kernel<D, P, G, T, true>;
    static int smem(int batch) { return I8Shape<D, G>::smem_bytes(batch); }
};

template <int D, int P, int G, typename T, bool I8>
int launch_fused(const DecodeParams& prm, cudaStream_t st)
{
    static int configured[kMaxDevices] = {0};
    constexpr auto fn = FusedKernel<D, P, G, T, I8>::fn;
    const int smem = FusedKernel<D, P, G, T, I8>::smem(prm.batch);
    if (smem > kMaxSmemPerCta) return PKV_ERR_UNSUPPORTED;
    if (ensure_smem(fn, smem, configured) != cudaSuccess) return PKV_ERR_CUDA;
    return status_of(launch_pdl(fn, dim3(prm.num_splits), dim3(kDecodeThreads), smem, st, prm));
}

template <int D, int P, typename T>
int fused_group(int group, bool i8, const DecodeParams& prm, cudaStream_t st)
{
    if (!i8) return group == 1 ? launch_fused<D, P, 1, T, false>(prm, st) : PKV_ERR_UNSUPPORTED;
    switch (group) {
    case 1: return launch_fused<D, P, 1, T, true>(prm, st);
    case 2: return launch_fused<D, P, 2, T, true>(prm, st);
    case 4: return launch_fused<D, P, 4, T, true>(prm, st);
    case 8: return launch_fused<D, P, 8, T, true>(prm, st);
    default: return PKV_ERR_UNSUPPORTED;
    }
}

template <typename T>
int fused_shape(int head_dim, int page_size, int group, bool i8, const DecodeParams& prm, cudaStream_t st)
{
    if (head_dim == 128 && page_size == 16) return fused_group<128, 16, T>(group, i8, prm, st);
    if (head_dim == 128 && page_size == 32) return fused_group<128, 32, T>(group, i8, prm, st);
    if (head_dim == 64 && page_size == 16) return fused_group<64, 16, T>(group, i8, prm, st);
    if (head_dim == 64 && page_size == 32) return fused_group<64, 32, T>(group, i8, prm, st);
    return PKV_ERR_UNSUPPORTED;
}

}  // namespace
}  // namespace pkv

extern "C" int rope_table(const int32_t* context_lens, int batch, int head_dim, double theta, double* table,
                          pkv_stream_t stream)
{
    if (batch < 0 || !(theta > 0.0)) return PKV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (batch == 0) return PKV_OK;
    if (!context_lens || !table || (reinterpret_cast<uintptr_t>(table) & 15u)) return PKV_ERR_INVALID_ARG;
    return status_of(launch_pdl(rope_table_kernel, dim3(batch), dim3(64), 0, reinterpret_cast<cudaStream_t>(stream),
                                context_lens, head_dim, theta, table));
}

extern "C" int paged_decode_layer(const pkv_pool* pool, int layer, void* out, const void* q, const void* k,
                                  const void* v, const double* rope, const int32_t* block_tables, int max_pages_per_seq,
                                  const int32_t* context_lens, int batch, int q_heads, int kv_heads, float scale,
                                  int num_splits, void* workspace, size_t workspace_bytes, pkv_stream_t stream)
{
    if (!pool || layer < 0 || layer >= pool->num_layers) return PKV_ERR_INVALID_ARG;
    if (batch < 0 || q_heads <= 0 || kv_heads != pool->kv_heads || q_heads % kv_heads) return PKV_ERR_INVALID_ARG;
    if (num_splits < 0 || num_splits > PKV_MAX_DECODE_SPLITS || max_pages_per_seq <= 0 || !(scale == scale))
        return PKV_ERR_INVALID_ARG;
    const bool i8 = pool->storage == kStorageI8;
    const int group = q_heads / kv_heads;
    if (!i8 && group != 1) return PKV_ERR_UNSUPPORTED;
    if (batch == 0) return PKV_OK;
    if (!out || !q || !k || !v || !rope || !block_tables || !context_lens || !workspace) return PKV_ERR_INVALID_ARG;
    if (misaligned16(out, q, k) || misaligned16(v, rope)) return PKV_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return PKV_ERR_INVALID_ARG;
    DecodeOps ops;
    if (!pick_decode(pool->head_dim, pool->page_size, group, pool->dtype, pool->storage, ops))
        return PKV_ERR_UNSUPPORTED;
    int cluster = 0;
    if (num_splits == 0) {
        const int st = ops.splits(&num_splits);
        if (st != PKV_OK) return st;
        if (!i8) cluster = cluster_size(num_splits, batch, kv_heads, max_pages_per_seq);
        num_splits = auto_splits(num_splits, max_decode_units(kv_heads, batch, max_pages_per_seq, pool->page_size,
                                                              ops.unit_tokens));
    }
    const WorkspaceLayout wl = workspace_layout(batch, group, pool->head_dim, num_splits);
    if (workspace_bytes < wl.total) return PKV_ERR_NO_SPACE;
    DecodeParams prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.k = static_cast<const char*>(pool->k_base) + (size_t)layer * pool->layer_bytes();
    prm.v = static_cast<const char*>(pool->v_base) + (size_t)layer * pool->layer_bytes();
    prm.q = q;
    prm.out = out;
    prm.k_new = k;
    prm.v_new = v;
    prm.rope = rope;
    if (i8) {
        prm.k_scale = static_cast<const float*>(pool->k_scale_base) + (size_t)layer * pool->layer_rows();
        prm.v_scale = static_cast<const float*>(pool->v_scale_base) + (size_t)layer * pool->layer_rows();
    }
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    prm.counters = reinterpret_cast<int*>(ws + wl.counters);
    prm.part_o = reinterpret_cast<float*>(ws + wl.part_o);
    prm.part_ml = reinterpret_cast<float*>(ws + wl.part_ml);
    prm.batch = batch;
    prm.max_pages = max_pages_per_seq;
    prm.q_heads = q_heads;
    prm.kv_heads = kv_heads;
    prm.num_pages = pool->num_pages;
    prm.num_splits = num_splits;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.cluster = cluster;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cluster) return launch_cluster_variant<true>(pool, prm, st);
    if (pool->dtype == PKV_F16) return fused_shape<__half>(pool->head_dim, pool->page_size, group, i8, prm, st);
    return fused_shape<__nv_bfloat16>(pool->head_dim, pool->page_size, group, i8, prm, st);
}

namespace pkv {
namespace {

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    return fn;
}

// One layer's K or V pool [pages][kv_heads][P][D] as a 4-D tensor (D, P, kv_heads, pages),
// box 64 x P x 1 x 1 with the 128-byte swizzle: one copy is one 64-column region of a page.
template <int D, int P, typename T>
bool encode_page_map(CUtensorMap* map, const void* base, int kv_heads, int num_pages)
{
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)P, (cuuint64_t)kv_heads, (cuuint64_t)num_pages};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)P * D * 2, (cuuint64_t)kv_heads * P * D * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)P, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapDataType dt =
        std::is_same<T, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    return enc(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int P, int G, typename T>
int launch_prefill(const PrefillParams& prm_in, int grid, cudaStream_t st)
{
    static int configured[kMaxDevices] = {0};
    using S = TcShape<D, std::is_same<T, __nv_bfloat16>::value>;
    const int smem = std::max(S::kBytes + 4 * (prm_in.batch + 1), S::kMinBytes);
    if (smem > kMaxSmemPerCta) return PKV_ERR_UNSUPPORTED;
    PrefillParams prm = prm_in;
    if (!encode_page_map<D, P, T>(&prm.k_map, prm.k, prm.kv_heads, prm.num_pages) ||
        !encode_page_map<D, P, T>(&prm.v_map, prm.v, prm.kv_heads, prm.num_pages))
        return PKV_ERR_CUDA;
    if (ensure_smem(prefill_tc_kernel<D, P, G, T>, smem, configured) != cudaSuccess) return PKV_ERR_CUDA;
    return status_of(launch_pdl(prefill_tc_kernel<D, P, G, T>, dim3(grid), dim3(kTcThreads), smem, st, prm));
}

template <int D, int P, typename T>
int prefill_group(int group, const PrefillParams& prm, int grid, cudaStream_t st)
{
    switch (group) {
    case 1: return launch_prefill<D, P, 1, T>(prm, grid, st);
    case 2: return launch_prefill<D, P, 2, T>(prm, grid, st);
    case 4: return launch_prefill<D, P, 4, T>(prm, grid, st);
    case 8: return launch_prefill<D, P, 8, T>(prm, grid, st);
    default: return PKV_ERR_UNSUPPORTED;
    }
}

template <typename T>
int prefill_shape(int head_dim, int page_size, int group, const PrefillParams& prm, int grid, cudaStream_t st)
{
    if (head_dim == 128 && page_size == 16) return prefill_group<128, 16, T>(group, prm, grid, st);
    if (head_dim == 128 && page_size == 32) return prefill_group<128, 32, T>(group, prm, grid, st);
    if (head_dim == 64 && page_size == 16) return prefill_group<64, 16, T>(group, prm, grid, st);
    if (head_dim == 64 && page_size == 32) return prefill_group<64, 32, T>(group, prm, grid, st);
    return PKV_ERR_UNSUPPORTED;
}

}  // namespace
}  // namespace pkv

extern "C" int paged_prefill_attention(const pkv_pool* pool, int layer, void* out, const void* q, const int32_t* cu_q,
                                       int total_q, const int32_t* block_tables, int max_pages_per_seq,
                                       const int32_t* context_lens, int batch, int q_heads, int kv_heads, float scale,
                                       pkv_stream_t stream)
{
    if (!pool || layer < 0 || layer >= pool->num_layers) return PKV_ERR_INVALID_ARG;
    if (batch < 0 || total_q < 0 || q_heads <= 0 || kv_heads != pool->kv_heads || q_heads % kv_heads)
        return PKV_ERR_INVALID_ARG;
    if (max_pages_per_seq <= 0 || !(scale == scale)) return PKV_ERR_INVALID_ARG;
    if (pool->storage != pool->dtype) return PKV_ERR_UNSUPPORTED;    // int8 pages: decode only
    if (batch == 0 || total_q == 0) return PKV_OK;
    if (!out || !q || !cu_q || !block_tables || !context_lens) return PKV_ERR_INVALID_ARG;
    if (misaligned16(out, q)) return PKV_ERR_INVALID_ARG;
    const int group = q_heads / kv_heads;
    PrefillParams prm;
    const size_t elt = 2;
    prm.k = static_cast<const char*>(pool->k_base) + (size_t)layer * pool->layer_elems * elt;
    prm.v = static_cast<const char*>(pool->v_base) + (size_t)layer * pool->layer_elems * elt;
    prm.q = q;
    prm.out = out;
    prm.cu_q = cu_q;
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    prm.batch = batch;
    prm.max_pages = max_pages_per_seq;
    prm.q_heads = q_heads;
    prm.kv_heads = kv_heads;
    prm.num_pages = pool->num_pages;
    prm.scale_log2 = scale * 1.4426950408889634f;
    // work items (one CTA each): kv_heads * sum_b ceil(ceil(n_b * group / R) / 2), R = kTcRows
    // (a CTA takes two row tiles), at most kv_heads * ((total_q * group + (2R - 1) * batch) / 2R + 1)
    const long long grid = (long long)kv_heads * (((long long)total_q * group + (long long)(2 * kTcRows - 1) * batch) /
                                                      (2 * kTcRows) + 1);
    if (grid > 0x7fffffffLL) return PKV_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (pool->dtype == PKV_F16)
        return prefill_shape<__half>(pool->head_dim, pool->page_size, group, prm, (int)grid, st);
    return prefill_shape<__nv_bfloat16>(pool->head_dim, pool->page_size, group, prm, (int)grid, st);
}

extern "C" int pkv_decode_workspace_clear(void* workspace, size_t workspace_bytes, pkv_stream_t stream)
{
    if (!workspace && workspace_bytes) return PKV_ERR_INVALID_ARG;
    if (!workspace_bytes) return PKV_OK;
    return status_of(cudaMemsetAsync(workspace, 0, workspace_bytes, reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" int kv_get_device_error(uint32_t* err_out)
{
    if (!err_out) return PKV_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return PKV_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof(v)) != cudaSuccess) return PKV_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return PKV_ERR_CUDA;
    *err_out = v;
    return PKV_OK;
}

// ---------------------------------------------------------------------------
// Decode attention with library-owned scratch, for callers that cannot allocate.
//
// Some callers have no way to obtain device memory of their own: a plugin whose host
// application owns every device allocation and hands the plugin none, a runtime whose
// caching allocator has already reserved the whole device, or a latency-critical
// serving loop that forbids cudaMalloc because it synchronises the device.  This entry
// point serves them: its scratch is one fixed array in the library's device memory.
namespace pkv {
namespace {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;   // 4 MiB per device

// Held by every GPU that loads the library, until the process exits.  In host code
// this name is only a stand-in for the symbol; its device address comes from
// cudaGetSymbolAddress below.
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_static_scratch_mutex;
void* g_static_scratch_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device, looked up once per device.
int static_scratch_address(void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
    if (!g_static_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return PKV_ERR_CUDA;
        g_static_scratch_addr[dev] = p;
    }
    *out = g_static_scratch_addr[dev];
    return PKV_OK;
}

}  // namespace
}  // namespace pkv

extern "C" int paged_decode_attention_noalloc(const pkv_pool* pool, int layer, void* out, const void* q,
                                              const int32_t* block_tables, int max_pages_per_seq,
                                              const int32_t* context_lens, int batch, int q_heads, int kv_heads,
                                              float scale, int num_splits, pkv_stream_t stream)
{
    // the same argument checks as paged_decode_attention, before the size check
    if (!pool || layer < 0 || layer >= pool->num_layers) return PKV_ERR_INVALID_ARG;
    if (batch < 0 || q_heads <= 0 || kv_heads != pool->kv_heads || q_heads % kv_heads) return PKV_ERR_INVALID_ARG;
    if (num_splits < 0 || num_splits > PKV_MAX_DECODE_SPLITS) return PKV_ERR_INVALID_ARG;
    if (num_splits > 0 && workspace_layout(batch, q_heads / kv_heads, pool->head_dim, num_splits).total >
                              kStaticScratchBytes)
        return PKV_ERR_NO_SPACE;
    void* scratch = nullptr;
    const int st = static_scratch_address(&scratch);
    if (st != PKV_OK) return st;
    // The scratch's only state that outlives a call is its counter region, which is zero
    // when the library is loaded, which every call leaves at zero, and which no call's
    // partial results overlap, whatever its split count.
    return paged_decode_attention(pool, layer, out, q, block_tables, max_pages_per_seq, context_lens, batch,
                                  q_heads, kv_heads, scale, num_splits, scratch, kStaticScratchBytes, stream);
}
