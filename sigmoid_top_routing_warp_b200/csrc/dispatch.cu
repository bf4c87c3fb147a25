// dispatch.cu -- step a5 (dispatch order), the row gather that feeds the
// grouped GEMM, and step a9 (combine).
//
// Dispatch ("Xiaohongshu dots3 note Open Source Deep Dive", §8.2, FUSED_MC2
// "dispatch -> gmm1 -> swiglu -> gmm2 -> combine"; §3.1 notes the production
// path uses grouped GEMM): a counting sort of the T*k (token, slot) pairs by
// expert.  It is stable in the flattened slot s = t*k + j, so the rows of one
// expert are in token order and the result does not depend on thread timing.
// Integer atomics only count; every position comes from prefix sums and
// warp-level ranks (__match_any_sync), so the output is deterministic.
//
// Combine (§3.3 layer diagram, "Weighted sum" then shared "add"): per token,
// a fixed-order fp32 sum of its k routed rows and the shared-expert row, with
// no float atomics.
#include "kernels.cuh"

#include <cuda_bf16.h>

namespace moe {

constexpr int kSmallMax = 4096;   // slots handled by the single-block path
constexpr int kChunk = 2048;      // slots per block in the multi-block path
constexpr int kChunkWarps = 8;

int permute_chunks(int n_slots) {
    return n_slots <= kSmallMax ? 0 : (n_slots + kChunk - 1) / kChunk;
}

// Exclusive prefix sum of v[0..n) in place (n <= 4 * blockDim.x); returns
// the total to every thread.  Uses `tmp` (blockDim.x ints of shared memory).
__device__ int block_exclusive_scan(int* v, int n, int* tmp) {
    const int tid = threadIdx.x, nt = blockDim.x;
    const int per = (n + nt - 1) / nt;
    const int b = tid * per;
    int local = 0;
    for (int i = 0; i < per; ++i)
        if (b + i < n) local += v[b + i];
    tmp[tid] = local;
    __syncthreads();
    // Hillis-Steele inclusive scan over the per-thread sums
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

// Ranks a batch of 32 slots (one per lane) among equal experts and places
// them: row = fill[e] + (number of lower lanes with the same expert).
__device__ __forceinline__ void place_batch(const PermuteArgs& a, int s, int n, int* fill) {
    const int lane = threadIdx.x & 31;
    int e = -1;
    if (s < n) {
        e = a.idx[s];
        if (e < 0 || e >= a.E) {
            a.pos[s] = -1;  // out-of-range expert: slot dropped
            e = -1;
        }
    }
    const int key = e >= 0 ? e : -1 - lane;  // invalid lanes never match
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    int row = 0;
    if (e >= 0) {
        row = fill[e] + __popc(peers & ((1u << lane) - 1u));
        a.rows[row] = s / a.k;
        a.pos[s] = row;
    }
    __syncwarp();
    if (e >= 0 && lane == 31 - __clz(peers)) fill[e] += __popc(peers);
    __syncwarp();
}

// Single block: histogram, scan and scatter for small T*k.
__global__ void __launch_bounds__(1024) permute_small_kernel(const PermuteArgs a) {
    extern __shared__ int sm[];
    int* cnt = sm;              // [E + 1]
    int* tmp = sm + a.E + 1;    // [blockDim.x]
    const int n = a.T * a.k;
    for (int e = threadIdx.x; e <= a.E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    for (int s = threadIdx.x; s < n; s += blockDim.x) {
        const int e = a.idx[s];
        if (e >= 0 && e < a.E) atomicAdd(&cnt[e], 1);
    }
    __syncthreads();
    const int total = block_exclusive_scan(cnt, a.E, tmp);
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) a.offsets[e] = cnt[e];
    if (threadIdx.x == 0) a.offsets[a.E] = total;
    __syncthreads();
    if (threadIdx.x < 32)
        for (int b = 0; b < n; b += 32) place_batch(a, b + threadIdx.x, n, cnt);
}

// Multi-block pass 1: per-chunk expert counts into chunk_base[chunk][e].
__global__ void __launch_bounds__(256) permute_count_kernel(const PermuteArgs a) {
    extern __shared__ int cnt[];
    const int n = a.T * a.k;
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    const int s0 = blockIdx.x * kChunk;
    for (int s = s0 + threadIdx.x; s < min(n, s0 + kChunk); s += blockDim.x) {
        const int e = a.idx[s];
        if (e >= 0 && e < a.E) atomicAdd(&cnt[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += blockDim.x)
        a.chunk_base[(size_t)blockIdx.x * a.E + e] = cnt[e];
}

// Multi-block pass 2 (one block): chunk_base[c][e] <- first row of chunk c's
// rows of expert e; offsets.
__global__ void __launch_bounds__(1024) permute_scan_kernel(const PermuteArgs a, int n_chunks) {
    extern __shared__ int sm[];
    int* tot = sm;            // [E]
    int* tmp = sm + a.E;      // [blockDim.x]
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int run = 0;
        for (int c = 0; c < n_chunks; ++c) {
            const int v = a.chunk_base[(size_t)c * a.E + e];
            a.chunk_base[(size_t)c * a.E + e] = run;
            run += v;
        }
        tot[e] = run;
    }
    __syncthreads();
    const int total = block_exclusive_scan(tot, a.E, tmp);
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        a.offsets[e] = tot[e];
        for (int c = 0; c < n_chunks; ++c) a.chunk_base[(size_t)c * a.E + e] += tot[e];
    }
    if (threadIdx.x == 0) a.offsets[a.E] = total;
}

// Multi-block pass 3: stable placement inside each chunk.  Warp w of a chunk
// owns slots [s0 + w*256, s0 + (w+1)*256): count per warp, prefix over warps,
// then rank within 32-slot batches.
__global__ void __launch_bounds__(kChunkWarps * 32) permute_scatter_kernel(const PermuteArgs a) {
    extern __shared__ int wcnt[];  // [kChunkWarps][E]
    const int n = a.T * a.k;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < kChunkWarps * a.E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    constexpr int per_warp = kChunk / kChunkWarps;
    const int s0 = blockIdx.x * kChunk + w * per_warp;
    int* my = wcnt + w * a.E;
    for (int b = 0; b < per_warp; b += 32) {
        const int s = s0 + b + lane;
        int e = -1;
        if (s < n) {
            e = a.idx[s];
            if (e < 0 || e >= a.E) e = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e >= 0 ? e : -1 - lane);
        if (e >= 0 && lane == 31 - __clz(peers)) my[e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int run = a.chunk_base[(size_t)blockIdx.x * a.E + e];
        for (int v = 0; v < kChunkWarps; ++v) {
            const int c = wcnt[v * a.E + e];
            wcnt[v * a.E + e] = run;
            run += c;
        }
    }
    __syncthreads();
    for (int b = 0; b < per_warp; b += 32) place_batch(a, s0 + b + lane, n, my);
}

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s) {
    const int n = a.T * a.k;
    const int chunks = permute_chunks(n);
    if (chunks == 0) {
        const int threads = 1024;
        permute_small_kernel<<<1, threads, (a.E + 1 + threads) * sizeof(int), s>>>(a);
        return cudaGetLastError();
    }
    permute_count_kernel<<<chunks, 256, a.E * sizeof(int), s>>>(a);
    permute_scan_kernel<<<1, 1024, (a.E + 1024) * sizeof(int), s>>>(a, chunks);
    permute_scatter_kernel<<<chunks, kChunkWarps * 32, kChunkWarps * a.E * sizeof(int), s>>>(a);
    return cudaGetLastError();
}

// Row gather: x_perm[pos[s]] = x[s / k] and w_perm[pos[s]] = topk_w[s], one
// warp per slot with 16-byte accesses.  The extra last block builds the
// token-tile prefix of the grouped GEMM: tok_start[e] = sum over e' < e of
// ceil(n_e' / bn).
__global__ void __launch_bounds__(256) gather_kernel(const GatherArgs a, int gather_blocks) {
    if (blockIdx.x == gather_blocks) {
        extern __shared__ int sm[];
        int* v = sm;              // [E]
        int* tmp = sm + a.E;      // [blockDim.x]
        for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
            const int ne = a.offsets[e + 1] - a.offsets[e];
            v[e] = (ne + a.bn - 1) / a.bn;
        }
        __syncthreads();
        const int total = block_exclusive_scan(v, a.E, tmp);
        for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
            a.tok_start[e] = v[e];
            // token-tile table: one entry per bn-row tile of expert e
            const int r0 = a.offsets[e], ne = a.offsets[e + 1] - r0;
            for (int tt = 0; tt * a.bn < ne; ++tt)
                a.tok_tiles[v[e] + tt] = make_int4(e, r0 + tt * a.bn, min(a.bn, ne - tt * a.bn), 0);
        }
        if (threadIdx.x == 0) a.tok_start[a.E] = total;
        return;
    }
    const int n = a.T * a.k;
    const int lane = threadIdx.x & 31;
    const int chunks = a.H / 8;  // 16-byte chunks per row
    for (int s = blockIdx.x * 8 + (threadIdx.x >> 5); s < n; s += gather_blocks * 8) {
        const int row = a.pos[s];
        if (row < 0) continue;
        const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)(s / a.k) * a.H);
        uint4* dst = reinterpret_cast<uint4*>(a.x_perm + (size_t)row * a.H);
        // four chunks per lane in flight before their stores
        int c = lane;
        for (; c + 96 < chunks; c += 128) {
            const uint4 v0 = __ldg(src + c), v1 = __ldg(src + c + 32), v2 = __ldg(src + c + 64),
                        v3 = __ldg(src + c + 96);
            dst[c] = v0;
            dst[c + 32] = v1;
            dst[c + 64] = v2;
            dst[c + 96] = v3;
        }
        for (; c < chunks; c += 32) dst[c] = __ldg(src + c);
        if (lane == 0) a.w_perm[row] = a.topk_w[s];
    }
}

cudaError_t launch_gather(const GatherArgs& a, cudaStream_t s) {
    const int n = a.T * a.k;
    int blocks = (n + 7) / 8;
    if (blocks > 4096) blocks = 4096;
    gather_kernel<<<blocks + 1, 256, (a.E + 256) * sizeof(int), s>>>(a, blocks);
    return cudaGetLastError();
}

// out[t] = bf16( sum_j y[pos[t*k + j]] + y_shared[t] (+ residual[t]) ), 8 columns per
// thread, one fp32 sum in that order and one rounding.  y is bf16, or fp32
// when k = 1 (a single routed row per token: its rounding to bf16 would not be
// averaged with other experts' and would be the largest error of the sum).
__global__ void __launch_bounds__(64) combine_kernel(const CombineArgs a) {
    const int t = blockIdx.x;
    const int c = blockIdx.y * blockDim.x + threadIdx.x;  // 16-byte chunk
    if (c >= a.H / 8) return;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    if (a.y_f32) {
        for (int j = 0; j < a.k; ++j) {
            const int r = a.pos[(size_t)t * a.k + j];
            if (r < 0) continue;
            const float4* yr = reinterpret_cast<const float4*>(
                                   static_cast<const float*>(a.y) + (size_t)r * a.H) + 2 * c;
            const float4 v0 = __ldg(yr), v1 = __ldg(yr + 1);
            acc[0] += v0.x; acc[1] += v0.y; acc[2] += v0.z; acc[3] += v0.w;
            acc[4] += v1.x; acc[5] += v1.y; acc[6] += v1.z; acc[7] += v1.w;
        }
    } else {
        // eight slots at a time: their rows' loads are all issued before the
        // sums, which still run in slot order
        for (int j0 = 0; j0 < a.k; j0 += 8) {
            int r[8];
            uint4 v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) r[i] = j0 + i < a.k ? __ldg(a.pos + (size_t)t * a.k + j0 + i) : -1;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (r[i] >= 0)
                    v[i] = __ldg(reinterpret_cast<const uint4*>(
                                     static_cast<const uint16_t*>(a.y) + (size_t)r[i] * a.H) + c);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (r[i] < 0) continue;
                const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v[i]);
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float2 f = __bfloat1622float2(p[h]);
                    acc[2 * h] += f.x;
                    acc[2 * h + 1] += f.y;
                }
            }
        }
    }
    if (a.y_shared) {
        const float4* ys = reinterpret_cast<const float4*>(a.y_shared + (size_t)t * a.H) + 2 * c;
        const float4 v0 = __ldg(ys), v1 = __ldg(ys + 1);
        acc[0] += v0.x; acc[1] += v0.y; acc[2] += v0.z; acc[3] += v0.w;
        acc[4] += v1.x; acc[5] += v1.y; acc[6] += v1.z; acc[7] += v1.w;
    }
    if (a.residual) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.residual + (size_t)t * a.H) + c);
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(p[i]);
            acc[2 * i] += f.x;
            acc[2 * i + 1] += f.y;
        }
    }
    uint4 o;
    __nv_bfloat162* q = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    reinterpret_cast<uint4*>(a.out + (size_t)t * a.H)[c] = o;
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    dim3 grid(a.T, (a.H / 8 + 63) / 64);
    combine_kernel<<<grid, 64, 0, s>>>(a);
    return cudaGetLastError();
}

// Zero the tile-claim words of a workspace status block, in stream order
// before a claiming launch (a memset node when captured in a graph).
cudaError_t reset_claim_counters(int* status, cudaStream_t s) {
    return cudaMemsetAsync(status + kSchedFirstWord, 0,
                           (kStatusWords - kSchedFirstWord) * sizeof(int), s);
}

}  // namespace moe
