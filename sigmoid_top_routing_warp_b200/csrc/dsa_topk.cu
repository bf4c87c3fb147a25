// dsa_topk.cu -- top-k keys per query row of DSA indexer scores.
//
// Source of the operation: "Xiaohongshu dots3 note Open Source Deep Dive",
// §4.2 "How DSA Works" (the indexer keeps the top-k keys of each query);
// "dots3-note 架构深度解析" (mlqm.cn), 混合注意力 paragraph (index_topk = 2048).
//
// One CTA per row.  Scores become order-preserving 32-bit keys (a larger
// float gives a larger key; -inf and NaN give 0, which is never selected).
// Four 8-bit radix passes (most significant first, shared-memory histograms)
// find the key T of the k-th largest score.  Every key above T is taken,
// and of the keys equal to T those with the lowest indices (contiguous
// per-thread index chunks and block-wide prefix sums keep index order).  The
// chosen (key, index) pairs are sorted by key descending, index ascending
// (one bitonic sort in shared memory) and written as indices; rows with
// fewer valid keys than k are padded with -1.  All decisions are integer
// comparisons, so equal scores give equal results on any device.
//
// Rows of up to kTKCacheKeys scores are staged once in shared memory; longer
// rows are re-read from global memory on every pass (L2-resident per row).
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kTKThreads = 512;
constexpr int kTKCacheKeys = 32768;    // 128 KB of keys staged in shared memory

__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    if (!(f > -INFINITY)) return 0u;               // -inf and NaN: never selected
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive block-wide sum of one int per thread (kTKThreads threads);
// `tmp` holds kTKThreads / 32 ints.  Returns the exclusive prefix and
// writes the total to *total.
__device__ __forceinline__ int block_scan(int v, int* tmp, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kTKThreads / 32 ? tmp[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
        }
        if (lane < kTKThreads / 32) tmp[lane] = w;
    }
    __syncthreads();
    const int before = (warp > 0 ? tmp[warp - 1] : 0) + x - v;
    *total = tmp[kTKThreads / 32 - 1];
    __syncthreads();
    return before;
}

}  // namespace

__global__ void __launch_bounds__(kTKThreads) dsa_topk_kernel(const DsaTopkArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    unsigned long long* sortbuf = reinterpret_cast<unsigned long long*>(smem_raw);  // [kDsaMaxTopk]
    int* hist = reinterpret_cast<int*>(sortbuf + kDsaMaxTopk);                       // [256]
    int* tmp = hist + 256;                                                           // [32]
    int* sh = tmp + 32;                                                              // [4]
    uint32_t* cache = reinterpret_cast<uint32_t*>(sh + 4);                           // [Sk] or none
    const int t = blockIdx.x;
    const int Sk = a.Sk;
    const float* row = a.scores + (size_t)t * a.ld;
    const bool cached = Sk <= kTKCacheKeys;
    auto key_at = [&](int s) -> uint32_t { return cached ? cache[s] : order_key(__ldg(row + s)); };

    // stage keys, count valid ones
    int nv = 0;
    for (int s = threadIdx.x; s < Sk; s += kTKThreads) {
        const uint32_t k = order_key(__ldg(row + s));
        if (cached) cache[s] = k;
        nv += k != 0u;
    }
    int n_valid = 0;
    block_scan(nv, tmp, &n_valid);   // also a barrier for the cache
    const int want = min(a.topk, n_valid);

    // threshold key T and how many keys equal to T to take
    uint32_t T = 1u;
    int take_eq = 0;
    if (n_valid > a.topk) {
        uint32_t prefix = 0u, mask = 0u;
        int remaining = a.topk;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int b = threadIdx.x; b < 256; b += kTKThreads) hist[b] = 0;
            __syncthreads();
            for (int s = threadIdx.x; s < Sk; s += kTKThreads) {
                const uint32_t k = key_at(s);
                if (k != 0u && (k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1);
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                int cum = 0, digit = 0;
                for (int b = 255; b >= 0; --b) {
                    if (cum + hist[b] >= remaining) { digit = b; break; }
                    cum += hist[b];
                }
                sh[0] = digit;
                sh[1] = remaining - cum;
            }
            __syncthreads();
            prefix |= (uint32_t)sh[0] << shift;
            mask |= 255u << shift;
            remaining = sh[1];
            __syncthreads();
        }
        T = prefix;
        take_eq = remaining;
    }

    // collect: keys > T anywhere, keys == T by index order up to take_eq
    const int chunk = (Sk + kTKThreads - 1) / kTKThreads;
    const int c0 = min(Sk, threadIdx.x * chunk), c1 = min(Sk, c0 + chunk);
    int gt = 0, eq = 0;
    for (int s = c0; s < c1; ++s) {
        const uint32_t k = key_at(s);
        gt += k > T;
        eq += k == T;
    }
    int n_gt = 0, n_eq = 0;
    const int gt_off = block_scan(gt, tmp, &n_gt);
    const int eq_off = block_scan(eq, tmp, &n_eq);
    (void)n_eq;
    int pg = gt_off, pe = eq_off;
    for (int s = c0; s < c1; ++s) {
        const uint32_t k = key_at(s);
        const unsigned long long packed =
            ((unsigned long long)k << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)s);
        if (k > T) {
            sortbuf[pg++] = packed;
        } else if (k == T && k != 0u) {
            if (pe < take_eq) sortbuf[n_gt + pe] = packed;
            ++pe;
        }
    }
    // pad to a power of two with zeros (they sort last) and sort descending
    int P = 32;
    while (P < want) P <<= 1;
    for (int i = want + threadIdx.x; i < P; i += kTKThreads) sortbuf[i] = 0ull;
    __syncthreads();
    for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < P / 2; i += kTKThreads) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const unsigned long long x = sortbuf[lo], y = sortbuf[hi];
                if ((x < y) == desc) {
                    sortbuf[lo] = y;
                    sortbuf[hi] = x;
                }
            }
            __syncthreads();
        }
    }
    int32_t* out = a.idx + (size_t)t * a.topk;
    for (int j = threadIdx.x; j < a.topk; j += kTKThreads)
        out[j] = j < want ? (int32_t)(0xFFFFFFFFu - (uint32_t)(sortbuf[j] & 0xFFFFFFFFull)) : -1;
}

size_t dsa_topk_smem(int Sk) {
    return (size_t)kDsaMaxTopk * 8 + (256 + 32 + 4) * 4 + (Sk <= kTKCacheKeys ? (size_t)Sk * 4 : 0);
}

cudaError_t launch_dsa_topk(const DsaTopkArgs& a, cudaStream_t s) {
    if (a.Sq == 0) return cudaSuccess;
    const size_t smem = dsa_topk_smem(a.Sk);
    cudaError_t e = cudaFuncSetAttribute(dsa_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dsa_topk_kernel<<<a.Sq, kTKThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
