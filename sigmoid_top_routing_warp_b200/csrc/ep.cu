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

#include <cuda_bf16.h>
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

// ---------------------------------------------------------------------------
// The same exchange over peer memory: the sender stores each routed row
// straight into its owner's receive buffer, already in the owner's expert
// order, and after the owners' expert GEMMs the sender's combine loads its
// rows' outputs from the owners' buffers.  No all-to-all of rows remains;
// the caller exchanges only the per-expert counts and orders the steps
// across ranks (a barrier after the dispatch and after the expert GEMMs).
//
// Receive layout on rank d: for each of its experts e (in order), the rows
// of every source rank (in rank order), each source's rows in its own
// sorted order.  With cnt[src][e] the rows source src sends to expert e:
//   exp_base[e] = sum over the owner's experts e' < e of sum_src cnt[src][e']
//   src_base[e] = sum over src < rank of cnt[src][e]
// and the row of slot s (expert e, position q in the sender's segment of e)
// lands at row exp_base[e] + src_base[e] + q of the owner's buffer.
namespace {

struct CountArgs {
    const int32_t* offsets;
    int32_t* counts;
    int E;
};

__global__ void ep_counts_kernel(const CountArgs a) {
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) a.counts[e] = a.offsets[e + 1] - a.offsets[e];
}

struct PlanArgs {
    const int32_t* cnt;       // [ep_size][E]
    int32_t* exp_base;        // [E]
    int32_t* src_base;        // [E]
    int32_t* recv_offsets;    // [E / ep_size + 1]: this rank's experts' segments
    int32_t* recv_ident;      // [recv_cap]: 0, 1, 2, ... (rows of the k = 1 layer)
    int recv_cap;
    int* status;              // status word: DEV_STATUS_CAPACITY if the rows exceed recv_cap
    int E, ep_size, rank;
};

// One block of 1024 threads (E <= 1024).
__global__ void __launch_bounds__(1024) ep_plan_kernel(const PlanArgs a) {
    __shared__ int tot[1024];
    const int e = threadIdx.x;
    const int el = a.E / a.ep_size;
    int t = 0, sb = 0;
    if (e < a.E) {
        for (int src = 0; src < a.ep_size; ++src) {
            const int c = a.cnt[(size_t)src * a.E + e];
            t += c;
            if (src < a.rank) sb += c;
        }
        a.src_base[e] = sb;
    }
    tot[e] = t;
    __syncthreads();
    // exclusive scan of the totals inside each owner's block of el experts
    if (e < a.E) {
        const int first = (e / el) * el;
        int base = 0;
        for (int i = first; i < e; ++i) base += tot[i];
        a.exp_base[e] = base;
        if (e / el == a.rank) {
            a.recv_offsets[e - first] = base;
            if (e == first + el - 1) a.recv_offsets[el] = base + tot[e];
        }
    }
    __syncthreads();
    int rows = 0;
    for (int i = a.rank * el; i < (a.rank + 1) * el; ++i) rows += tot[i];
    if (rows > a.recv_cap) {
        if (threadIdx.x == 0 && a.status) atomicOr(a.status, moe::DEV_STATUS_CAPACITY);
        rows = a.recv_cap;
    }
    for (int r = threadIdx.x; r < rows; r += blockDim.x) a.recv_ident[r] = r;
}

struct PutArgs {
    const uint16_t* x;               // [T, H]
    const int32_t* idx;              // [T * k]
    const float* topk_w;             // [T * k]
    const int32_t* offsets;          // [E + 1]
    const int32_t* pos;              // [T * k]
    const int32_t* exp_base;         // [E]
    const int32_t* src_base;         // [E]
    uint16_t* const* x_recv;         // [ep_size] owners' row buffers [recv_cap, H]
    float* const* w_recv;            // [ep_size] owners' weight buffers [recv_cap]
    int T, k, H, E, ep_size, recv_cap;
};

// One warp per slot: 16-byte stores of the token's row into the owner's buffer.
__global__ void __launch_bounds__(256) ep_put_kernel(const PutArgs a) {
    const int warp = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (warp >= a.T * a.k) return;
    const int e = a.idx[warp];
    if (e < 0 || e >= a.E) return;
    const int el = a.E / a.ep_size;
    const int d = e / el;
    const int row = a.exp_base[e] + a.src_base[e] + (a.pos[warp] - a.offsets[e]);
    if (row >= a.recv_cap) return;  // the plan flagged the overflow
    if (lane == 0) a.w_recv[d][row] = a.topk_w[warp];
    const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)(warp / a.k) * a.H);
    uint4* dst = reinterpret_cast<uint4*>(a.x_recv[d] + (size_t)row * a.H);
    for (int v = lane; v < a.H / 8; v += 32) dst[v] = __ldg(src + v);
}

struct PullArgs {
    const int32_t* idx;              // [T * k]
    const int32_t* offsets;          // [E + 1]
    const int32_t* pos;              // [T * k]
    const int32_t* exp_base;         // [E]
    const int32_t* src_base;         // [E]
    const float* const* y_recv;      // [ep_size] owners' fp32 output rows [recv_cap, H]
    const float* y_shared;           // [T, H] fp32 or null
    uint16_t* out;                   // [T, H]
    int T, k, H, E, ep_size, recv_cap;
};

// out_t = sum over slots j (in order) of the row's output, rounded to bf16
// first when k > 1 (as the single-device layer stores routed rows), plus the
// shared expert's fp32 row; one bf16 rounding.  One thread per 8 columns.
__global__ void __launch_bounds__(64) ep_pull_kernel(const PullArgs a) {
    const int t = blockIdx.x;
    const int c = blockIdx.y * blockDim.x + threadIdx.x;  // 8-column chunk
    if (c >= a.H / 8) return;
    const int el = a.E / a.ep_size;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int j = 0; j < a.k; ++j) {
        const int s = t * a.k + j;
        const int e = a.idx[s];
        if (e < 0 || e >= a.E) continue;
        const int row = a.exp_base[e] + a.src_base[e] + (a.pos[s] - a.offsets[e]);
        if (row >= a.recv_cap) continue;
        const float4* yr = reinterpret_cast<const float4*>(a.y_recv[e / el] + (size_t)row * a.H) + 2 * c;
        const float4 v0 = yr[0], v1 = yr[1];
        float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
            acc[i] += a.k > 1 ? __bfloat162float(__float2bfloat16_rn(v[i])) : v[i];
    }
    if (a.y_shared) {
        const float4* ys = reinterpret_cast<const float4*>(a.y_shared + (size_t)t * a.H) + 2 * c;
        const float4 v0 = ys[0], v1 = ys[1];
        acc[0] += v0.x; acc[1] += v0.y; acc[2] += v0.z; acc[3] += v0.w;
        acc[4] += v1.x; acc[5] += v1.y; acc[6] += v1.z; acc[7] += v1.w;
    }
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        o[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i])) |
               ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i + 1])) << 16);
    *reinterpret_cast<uint4*>(a.out + (size_t)t * a.H + 8 * c) = make_uint4(o[0], o[1], o[2], o[3]);
}

moe_status_t ep_check(const moe_config_t* cfg, int32_t ep_size, int32_t ep_rank) {
    moe_status_t st = moe::api_check_config(cfg);
    if (st != MOE_OK) return st;
    if (ep_size < 1 || ep_size > 1024 || cfg->E % ep_size)
        return pfail(MOE_ERR_INVALID_ARG, "ep_size=%lld must divide E=%lld", ep_size, cfg->E);
    if (ep_rank < 0 || ep_rank >= ep_size)
        return pfail(MOE_ERR_INVALID_ARG, "ep_rank=%lld outside [0, ep_size=%lld)", ep_rank, ep_size);
    return MOE_OK;
}

moe_status_t launched(const char* what) {
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) return MOE_OK;
    char msg[256];
    snprintf(msg, sizeof(msg), "%s: %s", what, cudaGetErrorString(e));
    return moe::api_fail(MOE_ERR_CUDA, msg);
}

}  // namespace

extern "C" moe_status_t moe_ep_expert_counts(const moe_config_t* cfg, const int32_t* offsets,
                                             int32_t* counts, moe_stream_t stream) {
    moe::api_clear_error();
    moe_status_t st = moe::api_check_config(cfg);
    if (st != MOE_OK) return st;
    if (!offsets || !counts) return moe::api_fail(MOE_ERR_INVALID_ARG, "offsets and counts must be non-NULL");
    ep_counts_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(CountArgs{offsets, counts, cfg->E});
    return launched("expert counts launch");
}

extern "C" moe_status_t moe_ep_plan(const moe_config_t* cfg, int32_t ep_size, int32_t ep_rank,
                                    const int32_t* counts_all, int32_t* exp_base,
                                    int32_t* src_base, int32_t* recv_offsets, int32_t* recv_ident,
                                    int32_t recv_cap, void* ws, moe_stream_t stream) {
    moe::api_clear_error();
    moe_status_t st = ep_check(cfg, ep_size, ep_rank);
    if (st != MOE_OK) return st;
    if (!counts_all || !exp_base || !src_base || !recv_offsets || !recv_ident || recv_cap < 0)
        return moe::api_fail(MOE_ERR_INVALID_ARG, "moe_ep_plan: a buffer is NULL or recv_cap < 0");
    PlanArgs a{counts_all, exp_base, src_base, recv_offsets, recv_ident, recv_cap,
               static_cast<int*>(ws), cfg->E, ep_size, ep_rank};
    ep_plan_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(a);
    return launched("exchange plan launch");
}

extern "C" moe_status_t moe_ep_dispatch_peer(const moe_config_t* cfg, int32_t ep_size,
                                             int32_t ep_rank, const void* x,
                                             const int32_t* topk_idx, const float* topk_w,
                                             const int32_t* offsets, const int32_t* pos,
                                             const int32_t* exp_base, const int32_t* src_base,
                                             void* const* x_recv, float* const* w_recv,
                                             int32_t recv_cap, moe_stream_t stream) {
    moe::api_clear_error();
    moe_status_t st = ep_check(cfg, ep_size, ep_rank);
    if (st != MOE_OK) return st;
    if (!x || !topk_idx || !topk_w || !offsets || !pos || !exp_base || !src_base || !x_recv ||
        !w_recv)
        return moe::api_fail(MOE_ERR_INVALID_ARG, "moe_ep_dispatch_peer: a buffer is NULL");
    if (reinterpret_cast<uintptr_t>(x) & 15u)
        return moe::api_fail(MOE_ERR_INVALID_ARG, "x must be 16-byte aligned");
    if (cfg->T == 0) return MOE_OK;
    PutArgs a{static_cast<const uint16_t*>(x), topk_idx, topk_w, offsets, pos, exp_base, src_base,
              reinterpret_cast<uint16_t* const*>(x_recv), w_recv, cfg->T, cfg->k, cfg->H, cfg->E,
              ep_size, recv_cap};
    const long long warps = (long long)cfg->T * cfg->k;
    ep_put_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
    return launched("peer dispatch launch");
}

extern "C" moe_status_t moe_ep_combine_peer(const moe_config_t* cfg, int32_t ep_size,
                                            int32_t ep_rank, const int32_t* topk_idx,
                                            const int32_t* offsets, const int32_t* pos,
                                            const int32_t* exp_base, const int32_t* src_base,
                                            const float* const* y_recv, const float* y_shared,
                                            void* out, int32_t recv_cap, moe_stream_t stream) {
    moe::api_clear_error();
    moe_status_t st = ep_check(cfg, ep_size, ep_rank);
    if (st != MOE_OK) return st;
    if (!topk_idx || !offsets || !pos || !exp_base || !src_base || !y_recv || !out)
        return moe::api_fail(MOE_ERR_INVALID_ARG, "moe_ep_combine_peer: a buffer is NULL");
    if ((reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(y_shared)) & 15u)
        return moe::api_fail(MOE_ERR_INVALID_ARG, "out and y_shared must be 16-byte aligned");
    if (cfg->T == 0) return MOE_OK;
    PullArgs a{topk_idx, offsets, pos, exp_base, src_base, y_recv, y_shared,
               static_cast<uint16_t*>(out), cfg->T, cfg->k, cfg->H, cfg->E, ep_size, recv_cap};
    const dim3 grid(cfg->T, (cfg->H / 8 + 63) / 64);
    ep_pull_kernel<<<grid, 64, 0, static_cast<cudaStream_t>(stream)>>>(a);
    return launched("peer combine launch");
}
