// norm.cu -- pre-norm of the MoE block input (RMSNorm).
//
// Source of the operation: "Xiaohongshu dots3 note Open Source Deep Dive",
// §3.3 layer diagram ("Residual + RMSNorm" ahead of the MoE FFN); "Transformers
// 中的 dots.llm1（Dots1）模型" (blog.gitcode.com), config table (rms_norm_eps =
// 1e-6) and source notes (variance in fp32, reciprocal-square-root scaling,
// then the weight).
//
//   u[t, :] = bf16( gamma * (h[t, :] * r_t) ),  r_t = 1 / sqrt(sum(h[t, :]^2) / H + eps)
//
// One 128-thread block per row: a strided pass of 16-byte loads accumulates
// the sum of squares (fp32, fixed tree order), a second pass (the row is
// then in L1/L2) scales and writes 16-byte stores.  Divide and square root
// are the correctly rounded ones.  HBM traffic: the row read once, u written once.
#include "kernels.cuh"

#include <cuda_bf16.h>

namespace moe {

namespace {

constexpr int kNormThreads = 128;

__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(p[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

}  // namespace

__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(const NormArgs a) {
    __shared__ float part[kNormThreads / 32];
    __shared__ float r_sh;
    const int t = blockIdx.x;
    const int nch = a.H / 8;
    const uint4* row = reinterpret_cast<const uint4*>(a.h + (size_t)t * a.H);
    float ss = 0.0f;
    for (int c = threadIdx.x; c < nch; c += kNormThreads) {
        float f[8];
        unpack8(__ldg(row + c), f);
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
        float tot = 0.0f;
#pragma unroll
        for (int w = 0; w < kNormThreads / 32; ++w) tot += part[w];
        const float ms = __fdiv_rn(tot, (float)a.H);
        r_sh = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, a.eps)));
    }
    __syncthreads();
    const float r = r_sh;
    const uint4* g = reinterpret_cast<const uint4*>(a.gamma);
    uint4* out = reinterpret_cast<uint4*>(a.u + (size_t)t * a.H);
    for (int c = threadIdx.x; c < nch; c += kNormThreads) {
        float f[8], w[8];
        unpack8(__ldg(row + c), f);
        unpack8(__ldg(g + c), w);
        uint4 o;
        __nv_bfloat162* q = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            q[i] = __floats2bfloat162_rn(__fmul_rn(w[2 * i], __fmul_rn(f[2 * i], r)),
                                         __fmul_rn(w[2 * i + 1], __fmul_rn(f[2 * i + 1], r)));
        out[c] = o;
    }
}

cudaError_t launch_rmsnorm(const NormArgs& a, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    rmsnorm_kernel<<<a.T, kNormThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
