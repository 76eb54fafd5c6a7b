// RMSNorm of the decode hidden state, optionally fused with the residual add.
//
// "为什么要自己动手写一个LLM推理引擎" (wzjinhao.cn/news/61427) s4.2: RMSNorm scales by the
// root mean square only (no mean subtraction), and eps is added to the mean square
// before the root is taken: y = x * rsqrt(mean(x^2) + eps) * w.
#ifndef PKV_RMS_NORM_CUH_
#define PKV_RMS_NORM_CUH_

#include "pkv_device.cuh"

namespace pkv {

constexpr int kNormThreads = 256;
constexpr int kNormMaxVecPerThread = 8;              // hidden <= 256 * 8 * 8 = 16384

// One CTA per row; each thread keeps its 16-byte vectors of the row in registers.  With a
// residual, h = x + residual is rounded once to the storage type, written back to the
// residual and normalised; the sum of squares and the scaling are fp32.
template <typename T>
__global__ void __launch_bounds__(kNormThreads) rms_norm_kernel(T* __restrict__ out, const T* __restrict__ x,
                                                                T* __restrict__ residual, const T* __restrict__ w,
                                                                int hidden, float eps)
{
    __shared__ float red[kNormThreads / 32];
    pdl_wait();
    pdl_launch_dependents();
    const int row = blockIdx.x;
    const int nvec = hidden / 8;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (long long)row * hidden);
    uint4* rr = residual ? reinterpret_cast<uint4*>(residual + (long long)row * hidden) : nullptr;
    float v[kNormMaxVecPerThread][8];
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < kNormMaxVecPerThread; ++k) {
        const int idx = threadIdx.x + k * kNormThreads;
        if (idx < nvec) {
            unpack8<T>(xr[idx], v[k]);
            if (rr) {
                float r[8];
                unpack8<T>(rr[idx], r);
                uint4 packed;
                T* pe = reinterpret_cast<T*>(&packed);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    pe[e] = Elt<T>::from_float(v[k][e] + r[e]);      // one rounding of the sum
                    v[k][e] = static_cast<float>(pe[e]);
                }
                rr[idx] = packed;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(v[k][e], v[k][e], ss);
        }
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < kNormThreads / 32; ++i) tot += red[i];
    const float inv = rsqrtf(tot / (float)hidden + eps);
    const uint4* wr = reinterpret_cast<const uint4*>(w);
    uint4* orow = reinterpret_cast<uint4*>(out + (long long)row * hidden);
#pragma unroll
    for (int k = 0; k < kNormMaxVecPerThread; ++k) {
        const int idx = threadIdx.x + k * kNormThreads;
        if (idx < nvec) {
            float wf[8];
            unpack8<T>(wr[idx], wf);
            uint4 packed;
            T* pe = reinterpret_cast<T*>(&packed);
#pragma unroll
            for (int e = 0; e < 8; ++e) pe[e] = Elt<T>::from_float(v[k][e] * inv * wf[e]);
            orow[idx] = packed;
        }
    }
}

}  // namespace pkv

#endif  // PKV_RMS_NORM_CUH_
