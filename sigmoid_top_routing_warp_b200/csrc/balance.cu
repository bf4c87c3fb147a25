// balance.cu -- the expert-bias update of noaux_tc routing (moe_bias_update).
//
// Source: "dots3-note 架构深度解析" (mlqm.cn), 稀疏激活: noaux_tc routing, a
// per-expert bias that steers the top-k choice and is kept out of the
// routing weights, with no auxiliary balancing loss.  The pages give no rule
// for updating the bias; the one built here is the plainest reading: after a
// routed batch every expert above the mean load loses gamma, every expert
// below gains gamma, an expert exactly at the mean keeps its bias.
//
// One block: an integer histogram of the batch's T*k choices in shared
// memory (atomic increments, whose final counts do not depend on their
// order), then one thread per expert compares load_e * E with T * k exactly
// and applies one correctly rounded fp32 addition.
#include "moe.h"
#include "kernels.cuh"

#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>

namespace moe {
moe_status_t api_check_config(const moe_config_t* c);
moe_status_t api_fail(moe_status_t st, const char* msg);
void api_clear_error();
}  // namespace moe

namespace {

constexpr int kBalMaxE = 1024;  // the configuration's bound on E
constexpr int kBalThreads = 1024;

__global__ void __launch_bounds__(kBalThreads) bias_update_kernel(const int32_t* __restrict__ idx,
                                                                   long long n, int E,
                                                                   float* __restrict__ bias,
                                                                   float gamma) {
    __shared__ int load[kBalMaxE];
    for (int e = threadIdx.x; e < E; e += blockDim.x) load[e] = 0;
    __syncthreads();
    for (long long i = threadIdx.x; i < n; i += blockDim.x) {
        const int e = __ldg(idx + i);
        if ((unsigned)e < (unsigned)E) atomicAdd(&load[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const long long d = n - (long long)load[e] * E;  // sign(mean - load) * E
        if (d > 0)
            bias[e] = __fadd_rn(bias[e], gamma);
        else if (d < 0)
            bias[e] = __fsub_rn(bias[e], gamma);
    }
}

}  // namespace

extern "C" moe_status_t moe_bias_update(const moe_config_t* cfg, const int32_t* topk_idx,
                                        float* bias, float gamma, moe_stream_t stream) {
    moe::api_clear_error();
    moe_status_t st = moe::api_check_config(cfg);
    if (st != MOE_OK) return st;
    if (!(gamma >= 0.0f) || std::isinf(gamma))
        return moe::api_fail(MOE_ERR_INVALID_ARG, "gamma must be finite and >= 0");
    if (!topk_idx) return moe::api_fail(MOE_ERR_INVALID_ARG, "topk_idx is NULL");
    if (!bias) return moe::api_fail(MOE_ERR_INVALID_ARG, "bias is NULL");
    if (cfg->E > kBalMaxE) return moe::api_fail(MOE_ERR_UNSUPPORTED, "E above 1024");
    if (cfg->T == 0) return MOE_OK;
    bias_update_kernel<<<1, kBalThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        topk_idx, (long long)cfg->T * cfg->k, cfg->E, bias, gamma);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        char msg[160];
        snprintf(msg, sizeof(msg), "bias update launch: %s", cudaGetErrorString(e));
        return moe::api_fail(MOE_ERR_CUDA, msg);
    }
    return MOE_OK;
}
