// quant.cu -- step a0 of the FP8 layer (per-token, per-128-column e4m3
// quantisation of the activations) and the row gather of e4m3 codes.
//
// FP8 deployment of the dots3-note weights: "dots3-note 架构深度解析" (mlqm.cn),
// 部署实战 (dots3-note-prev-fp8, single 8-card node) and the architecture table
// (BF16, FP8); "Xiaohongshu dots3 note Open Source Deep Dive" §3.2 (FP8 fits one
// 8xH100 node).  The pages name FP8 only; the recipe implemented here is
// weights in e4m3 with one fp32 scale per 128x128 block, activations in e4m3
// with one fp32 scale per token and 128 columns:
//   scale = amax / 448  (448: largest finite e4m3), or 1 for an all-zero block
//   code  = e4m3(x / scale), round to nearest even, saturating to +-448.
// The scale and every code are decided with correctly rounded binary32
// operations (__fdiv_rn and the RN-satfinite conversion), so they are fixed
// by the arithmetic and match any other IEEE implementation of the recipe.
#include "kernels.cuh"

#include <cuda_bf16.h>
#include <cuda_fp8.h>

namespace moe {

// One warp per (row, 128-column block): lane l owns columns 4l .. 4l+3.
__global__ void __launch_bounds__(256) quant_act_kernel(const QuantArgs a) {
    const int lane = threadIdx.x & 31;
    const int nb = a.cols / 128;
    const long long task = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (task >= (long long)a.rows * nb) return;
    const int r = (int)(task / nb), b = (int)(task % nb);
    const uint16_t* src = a.x + (size_t)r * a.cols + b * 128 + 4 * lane;
    const uint2 raw = *reinterpret_cast<const uint2*>(src);
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
    const float2 v01 = __bfloat1622float2(p[0]), v23 = __bfloat1622float2(p[1]);
    float v[4] = {v01.x, v01.y, v23.x, v23.y};
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_fp8_storage_t q = __nv_cvt_float_to_fp8(__fdiv_rn(v[i], s), __NV_SATFINITE, __NV_E4M3);
        packed |= (uint32_t)q << (8 * i);
    }
    *reinterpret_cast<uint32_t*>(a.q + (size_t)r * a.cols + b * 128 + 4 * lane) = packed;
    if (lane == 0) a.scale[(size_t)r * nb + b] = s;
}

cudaError_t launch_quant_act(const QuantArgs& a, cudaStream_t s) {
    const long long tasks = (long long)a.rows * (a.cols / 128);
    if (tasks == 0) return cudaSuccess;
    quant_act_kernel<<<(unsigned)((tasks + 7) / 8), 256, 0, s>>>(a);
    return cudaGetLastError();
}

// Exclusive scan of v[0..n) in shared memory (n <= 4 * blockDim.x).
__device__ static int scan_excl(int* v, int n, int* tmp) {
    const int tid = threadIdx.x, nt = blockDim.x;
    const int per = (n + nt - 1) / nt, b = tid * per;
    int local = 0;
    for (int i = 0; i < per; ++i)
        if (b + i < n) local += v[b + i];
    tmp[tid] = local;
    __syncthreads();
    for (int off = 1; off < nt; off <<= 1) {
        const int add = tid >= off ? tmp[tid - off] : 0;
        __syncthreads();
        tmp[tid] += add;
        __syncthreads();
    }
    const int total = tmp[nt - 1];
    int run = tmp[tid] - local;
    for (int i = 0; i < per; ++i)
        if (b + i < n) {
            const int x = v[b + i];
            v[b + i] = run;
            run += x;
        }
    __syncthreads();
    return total;
}

// One warp per slot: codes (16-byte chunks) and scales of row s / k to the
// sorted row pos[s].  The extra last block builds the token-tile prefix.
__global__ void __launch_bounds__(256) gather_q_kernel(const GatherQArgs a, int gather_blocks) {
    if (blockIdx.x == gather_blocks) {
        extern __shared__ int sm[];
        int* v = sm;
        int* tmp = sm + a.E;
        for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
            const int ne = a.offsets[e + 1] - a.offsets[e];
            v[e] = (ne + a.bn - 1) / a.bn;
        }
        __syncthreads();
        const int total = scan_excl(v, a.E, tmp);
        for (int e = threadIdx.x; e < a.E; e += blockDim.x) a.tok_start[e] = v[e];
        if (threadIdx.x == 0) a.tok_start[a.E] = total;
        return;
    }
    const int n = a.T * a.k, lane = threadIdx.x & 31;
    const int chunks = a.H / 16, nb = a.H / 128;
    for (int s = blockIdx.x * 8 + (threadIdx.x >> 5); s < n; s += gather_blocks * 8) {
        const int row = a.pos[s];
        if (row < 0) continue;
        const int t = s / a.k;
        const uint4* src = reinterpret_cast<const uint4*>(a.xq + (size_t)t * a.H);
        uint4* dst = reinterpret_cast<uint4*>(a.xq_perm + (size_t)row * a.H);
        for (int c = lane; c < chunks; c += 32) dst[c] = __ldg(src + c);
        for (int c = lane; c < nb; c += 32) a.sx_perm[(size_t)row * nb + c] = __ldg(a.sx + (size_t)t * nb + c);
        if (lane == 0) a.w_perm[row] = a.topk_w[s];
    }
}

cudaError_t launch_gather_q(const GatherQArgs& a, cudaStream_t s) {
    const int n = a.T * a.k;
    int blocks = (n + 7) / 8;
    if (blocks > 4096) blocks = 4096;
    gather_q_kernel<<<blocks + 1, 256, (a.E + 256) * sizeof(int), s>>>(a, blocks);
    return cudaGetLastError();
}

}  // namespace moe
