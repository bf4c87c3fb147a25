// ep.cu -- the sending side of the expert-parallel form of the layer
// (moe_ep_pack): the routed rows of a rank's tokens, in expert order, packed
// into one send buffer whose chunks go to the ranks that own the experts.
//
// The production deployment the pages describe splits the experts over
// accelerators and moves tokens to them and back ("Xiaohongshu dots3 note Open
// Source Deep Dive", §8.2: FUSED_MC2 "dispatch -> gmm1 -> swiglu -> gmm2 ->
// combine"; §10.2: expert parallelism with an all-to-all backend).  With the
// experts of rank d the contiguous range [d E_loc, (d+1) E_loc), the stable
// expert order of moe_permute is also destination order: row r of the send
// buffer is sorted row r of the permutation, and the chunk for rank d is
// rows [offsets[d E_loc], offsets[(d+1) E_loc]).  Each row carries its token's
// activation, its routing weight and its expert's index on the destination.
#include "moe.h"
#include "kernels.cuh"

#include <cuda_runtime.h>

#include <cstdio>

namespace moe {
moe_status_t api_check_config(const moe_config_t* c);
moe_status_t api_fail(moe_status_t st, const char* msg);
void api_clear_error();
}  // namespace moe

namespace {

struct PackArgs {
    const uint16_t* x;        // [T, H]
    const int32_t* idx;       // [T * k]
    const float* topk_w;      // [T * k]
    const int32_t* offsets;   // [E + 1]
    const int32_t* pos;       // [T * k]
    uint16_t* x_send;         // [T * k, H]
    float* w_send;            // [T * k]
    int32_t* e_send;          // [T * k]
    int32_t* send_counts;     // [ep_size]
    int T, k, H, E, ep_size;
};

// Warps 0 .. T*k-1: one slot each; the warp after them writes the counts.
__global__ void __launch_bounds__(256) ep_pack_kernel(const PackArgs a) {
    const int warp = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    const int n = a.T * a.k;
    const int el = a.E / a.ep_size;
    if (warp < n) {
        const int e = a.idx[warp];
        if (e < 0 || e >= a.E) return;  // not a valid choice: its row is left as is
        const int r = a.pos[warp];
        if (lane == 0) {
            a.w_send[r] = a.topk_w[warp];
            a.e_send[r] = e - (e / el) * el;
        }
        const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)(warp / a.k) * a.H);
        uint4* dst = reinterpret_cast<uint4*>(a.x_send + (size_t)r * a.H);
        for (int v = lane; v < a.H / 8; v += 32) dst[v] = __ldg(src + v);
    } else if (warp == n) {
        for (int d = lane; d < a.ep_size; d += 32)
            a.send_counts[d] = a.offsets[(d + 1) * el] - a.offsets[d * el];
    }
}

moe_status_t pfail(moe_status_t st, const char* fmt, long long a = 0, long long b = 0) {
    char msg[256];
    snprintf(msg, sizeof(msg), fmt, a, b);
    return moe::api_fail(st, msg);
}

}  // namespace

extern "C" moe_status_t moe_ep_pack(const moe_config_t* cfg, int32_t ep_size, const void* x,
                                    const int32_t* topk_idx, const float* topk_w,
                                    const int32_t* offsets, const int32_t* pos, void* x_send,
                                    float* w_send, int32_t* e_send, int32_t* send_counts,
                                    moe_stream_t stream) {
    moe::api_clear_error();
    moe_status_t st = moe::api_check_config(cfg);
    if (st != MOE_OK) return st;
    if (ep_size < 1 || ep_size > 1024 || cfg->E % ep_size)
        return pfail(MOE_ERR_INVALID_ARG, "ep_size=%lld must divide E=%lld", ep_size, cfg->E);
    if (!x || !topk_idx || !topk_w || !offsets || !pos || !x_send || !w_send || !e_send ||
        !send_counts)
        return moe::api_fail(MOE_ERR_INVALID_ARG, "moe_ep_pack: a buffer is NULL");
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(x_send)) & 15u)
        return moe::api_fail(MOE_ERR_INVALID_ARG, "x and x_send must be 16-byte aligned");
    PackArgs a{static_cast<const uint16_t*>(x), topk_idx, topk_w, offsets, pos,
               static_cast<uint16_t*>(x_send), w_send, e_send, send_counts,
               cfg->T, cfg->k, cfg->H, cfg->E, ep_size};
    const long long warps = (long long)cfg->T * cfg->k + 1;
    ep_pack_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return moe::api_fail(MOE_ERR_CUDA, cudaGetErrorString(e));
    return MOE_OK;
}
