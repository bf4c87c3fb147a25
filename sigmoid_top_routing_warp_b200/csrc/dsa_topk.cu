// dsa_topk.cu -- top-k keys per query row of DSA indexer scores.
//
// Source of the operation: "Xiaohongshu dots3 note Open Source Deep Dive",
// §4.2 "How DSA Works" (the indexer keeps the top-k keys of each query);
// "dots3-note 架构深度解析" (mlqm.cn), 混合注意力 paragraph (index_topk = 2048).
//
// One CTA per row.  Scores become order-preserving 32-bit keys (a larger
// float gives a larger key; -inf and NaN give 0, which is never selected).
// Four 8-bit radix digits, most significant first, find the key T of the
// k-th largest score: shared-memory histograms with warp-aggregated counts.
// The first pass stages the row and counts the top digit; the second keeps
// the keys of the chosen top digit as candidates (compacted into the sort
// buffer) and counts their next digit; the last two digits count only the
// candidates.  Every key above T is taken, and of the keys equal to T those
// with the lowest indices (per-warp index segments and block-wide prefix
// sums keep index order).  For sorted output the chosen (key, index) pairs
// are sorted by key descending, index ascending (one bitonic network: steps
// inside 128-element chunks in registers, the rest in shared memory); when
// every key equal to T is taken they are gathered unordered first, since the
// sort fixes the order.  Rows with fewer valid keys than k are padded with
// -1.  All decisions are integer comparisons, so equal scores give equal
// results on any device.  Under a causal mask a row reads only the keys the
// mask leaves (the others are -inf by construction).
//
// Rows of up to kTKCacheKeys scores are staged once in shared memory; longer
// rows are re-read from global memory (L2-resident per row).
#include "dsa_kernels.cuh"

namespace moe {

namespace {

constexpr int kTKThreads = 512;
constexpr int kTKCacheKeys = 32768;    // 128 KB of keys staged in shared memory
constexpr int kTKCandCap = kDsaMaxTopk * 2;  // candidate keys (uint32) in the sort buffer
constexpr int kTKBatch = 6;                  // keys loaded per thread before they are used

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

__device__ __forceinline__ unsigned long long shfl_xor64(unsigned long long v, int m) {
    const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
    return ((unsigned long long)hi << 32) | lo;
}

__device__ __forceinline__ void reg_cmpswap(unsigned long long& x, unsigned long long& y, bool desc) {
    const unsigned long long hi = x > y ? x : y, lo = x > y ? y : x;
    x = desc ? hi : lo;
    y = desc ? lo : hi;
}

// The descending bitonic network on the 128 elements a warp holds (element
// base + 4 * lane + r is v[r]).  A pair (lo, lo + stride) of the step for
// block size `size` is ordered descending when (lo & size) == 0, ascending
// otherwise: the network of a plain shared-memory bitonic sort, with every
// step whose partner lies inside the 128-element chunk done in registers.
// For size >= 8 the bit `size` of an index does not depend on r, so the
// direction is one flag per lane; strides >= 4 exchange with lane ^ stride/4,
// strides 2 and 1 stay inside the thread.
template <int LSTRIDE>
__device__ __forceinline__ void warp_bitonic_step(unsigned long long (&v)[4], int lane, bool desc) {
    constexpr int stride = 1 << LSTRIDE;
    if constexpr (stride >= 4) {
        const bool keep_max = ((lane & (stride >> 2)) == 0) == desc;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const unsigned long long o = shfl_xor64(v[r], stride >> 2);
            v[r] = ((v[r] > o) == keep_max) ? v[r] : o;
        }
    } else if constexpr (stride == 2) {
        reg_cmpswap(v[0], v[2], desc);
        reg_cmpswap(v[1], v[3], desc);
    } else {
        reg_cmpswap(v[0], v[1], desc);
        reg_cmpswap(v[2], v[3], desc);
    }
}

// Merge steps of block size 2^LSIZE with strides 2^(LTOP) .. 1, in registers.
template <int LTOP>
__device__ __forceinline__ void warp_bitonic_merge(unsigned long long (&v)[4], int lane, bool desc) {
    warp_bitonic_step<LTOP>(v, lane, desc);
    if constexpr (LTOP > 0) warp_bitonic_merge<LTOP - 1>(v, lane, desc);
}

// Sizes 2 .. 128: the chunk ends descending for even base / 128 and
// ascending for odd (what the first cross-chunk merge needs).
__device__ __forceinline__ void warp_bitonic_chunk(unsigned long long (&v)[4], int base, int lane) {
    reg_cmpswap(v[0], v[1], true);   // size 2: pair (4l, 4l+1) descending,
    reg_cmpswap(v[2], v[3], false);  //         pair (4l+2, 4l+3) ascending
    const int i0 = base + 4 * lane;
    warp_bitonic_merge<1>(v, lane, ((i0 >> 2) & 1) == 0);
    warp_bitonic_merge<2>(v, lane, ((i0 >> 3) & 1) == 0);
    warp_bitonic_merge<3>(v, lane, ((i0 >> 4) & 1) == 0);
    warp_bitonic_merge<4>(v, lane, ((i0 >> 5) & 1) == 0);
    warp_bitonic_merge<5>(v, lane, ((i0 >> 6) & 1) == 0);
    warp_bitonic_merge<6>(v, lane, ((i0 >> 7) & 1) == 0);
}

// Adds one to hist[bin] for every lane with `act`: one shared-memory atomic
// per distinct bin of the warp (scores cluster in few top digits).
__device__ __forceinline__ void hist_add(bool act, uint32_t bin, int* hist) {
    const uint32_t am = __ballot_sync(0xffffffffu, act);
    if (act) {
        const uint32_t peers = __match_any_sync(am, bin);
        if ((int)(__ffs(peers) - 1) == (int)(threadIdx.x & 31)) atomicAdd(&hist[bin], __popc(peers));
    }
}

// The digit of the `remaining`-th largest key: the highest bin whose suffix
// count reaches it (thread i reads bin 255 - i; an inclusive scan gives
// suffix counts).  Sets sh[0] = the digit, sh[1] = the rank still wanted
// inside that bin, sh[2] = the bin's count; returns the sum of all bins.
// Ends with a barrier, after which sh is valid.
__device__ __forceinline__ int digit_search(const int* hist, int remaining, int* tmp, int* sh) {
    const int hb = threadIdx.x < 256 ? hist[255 - threadIdx.x] : 0;
    int tot = 0;
    const int above = block_scan(hb, tmp, &tot);
    if (threadIdx.x < 256 && above < remaining && above + hb >= remaining) {
        sh[0] = 255 - threadIdx.x;
        sh[1] = remaining - above;
        sh[2] = hb;
    }
    __syncthreads();
    return tot;
}

// Appends the keys of the lanes with `act` at buf[*count ...]: one atomic per
// warp, order across warps unspecified.  Positions at or past `cap` are not
// written (the count still grows, so the caller sees the overflow).
__device__ __forceinline__ void append_key(bool act, uint32_t k, uint32_t* buf, int* count, int cap) {
    const uint32_t am = __ballot_sync(0xffffffffu, act);
    if (am == 0u) return;
    const int lane = threadIdx.x & 31;
    const int leader = __ffs(am) - 1;
    int base = 0;
    if (lane == leader) base = atomicAdd(count, __popc(am));
    base = __shfl_sync(0xffffffffu, base, leader);
    const int pos = base + __popc(am & ((1u << lane) - 1u));
    if (act && pos < cap) buf[pos] = k;
}

}  // namespace

__global__ void __launch_bounds__(kTKThreads, 4) dsa_topk_kernel(const DsaTopkArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // sortbuf holds the candidate keys of the radix passes first, then the
    // chosen (key, index) pairs
    unsigned long long* sortbuf = reinterpret_cast<unsigned long long*>(smem_raw);  // [kDsaMaxTopk]
    uint32_t* cand = reinterpret_cast<uint32_t*>(sortbuf);                          // [kTKCandCap]
    int* hist = reinterpret_cast<int*>(sortbuf + kDsaMaxTopk);                       // [256]
    int* tmp = hist + 256;                                                           // [32]
    int* sh = tmp + 32;                                                              // [8]
    uint32_t* cache = reinterpret_cast<uint32_t*>(sh + 8);                           // [Sk] or none
    const int t = blockIdx.x;
    const int Sk = a.Sk;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lt = (1u << lane) - 1u;
    // keys past the causal limit are the score kernel's -inf: not read
    const int L = a.causal ? max(0, min(Sk, a.q_offset + t + 1)) : Sk;
    const float* row = a.scores + (size_t)t * a.ld;
    const bool cached = Sk <= kTKCacheKeys;
    auto key_at = [&](int s) -> uint32_t { return cached ? cache[s] : order_key(__ldg(row + s)); };
    // keys s_first + j * step (j < kTKBatch), 0 at or past `lim`; the loads
    // are issued before any is used
    auto load_keys = [&](uint32_t(&kb)[kTKBatch], int s_first, int step, int lim) {
        if (cached) {
#pragma unroll
            for (int j = 0; j < kTKBatch; ++j) {
                const int s = s_first + j * step;
                kb[j] = s < lim ? cache[s] : 0u;
            }
        } else {
            float f[kTKBatch];
#pragma unroll
            for (int j = 0; j < kTKBatch; ++j) {
                const int s = s_first + j * step;
                f[j] = s < lim ? __ldg(row + s) : -INFINITY;
            }
#pragma unroll
            for (int j = 0; j < kTKBatch; ++j) kb[j] = order_key(f[j]);
        }
    };

    for (int b = threadIdx.x; b < 256; b += kTKThreads) hist[b] = 0;
    if (threadIdx.x == 0) sh[3] = sh[4] = 0;
    __syncthreads();
    // pass 1: stage the keys, histogram of the top digit (its total counts
    // the valid keys)
    // (kTKBatch independent loads in flight per thread before any ballot)
    for (int s0 = 0; s0 < L; s0 += kTKThreads * kTKBatch) {
        float f[kTKBatch];
#pragma unroll
        for (int j = 0; j < kTKBatch; ++j) {
            const int s = s0 + j * kTKThreads + threadIdx.x;
            f[j] = s < L ? __ldg(row + s) : -INFINITY;
        }
#pragma unroll
        for (int j = 0; j < kTKBatch; ++j) {
            const int s = s0 + j * kTKThreads + threadIdx.x;
            const uint32_t k = order_key(f[j]);
            if (cached && s < L) cache[s] = k;
            hist_add(k != 0u, k >> 24, hist);
        }
    }
    __syncthreads();
    const int n_valid = digit_search(hist, a.topk, tmp, sh);
    const int want = min(a.topk, n_valid);

    // threshold key T, how many keys equal T (n_eq) and how many of them to
    // take (take_eq, lowest indices first)
    uint32_t T = 1u;
    int take_eq = 0, n_eq = 0;
    if (n_valid > a.topk) {
        uint32_t prefix = (uint32_t)sh[0] << 24, mask = 0xFF000000u;
        int remaining = sh[1];
        for (int b = threadIdx.x; b < 256; b += kTKThreads) hist[b] = 0;
        __syncthreads();
        // pass 2: the keys of the chosen top digit become candidates;
        // histogram of their second digit
        for (int s0 = 0; s0 < L; s0 += kTKThreads * kTKBatch) {
            uint32_t kb[kTKBatch];
            load_keys(kb, s0 + threadIdx.x, kTKThreads, L);
#pragma unroll
            for (int j = 0; j < kTKBatch; ++j) {
                const uint32_t k = kb[j];
                const bool act = k != 0u && (k & mask) == prefix;
                append_key(act, k, cand, &sh[3], kTKCandCap);
                hist_add(act, (k >> 16) & 255u, hist);
            }
        }
        __syncthreads();
        const int n_cand = sh[3];
        digit_search(hist, remaining, tmp, sh);
        prefix |= (uint32_t)sh[0] << 16;
        mask |= 0x00FF0000u;
        remaining = sh[1];
        // passes 3 and 4 over the candidates (over the row if they overflowed)
        const bool from_cand = n_cand <= kTKCandCap;
        const int n = from_cand ? n_cand : L;
        for (int shift = 8; shift >= 0; shift -= 8) {
            for (int b = threadIdx.x; b < 256; b += kTKThreads) hist[b] = 0;
            __syncthreads();
            for (int i0 = 0; i0 < n; i0 += kTKThreads) {
                const int i = i0 + threadIdx.x;
                uint32_t k = 0u;
                if (i < n) k = from_cand ? cand[i] : key_at(i);
                const bool act = k != 0u && (k & mask) == prefix;
                hist_add(act, (k >> shift) & 255u, hist);
            }
            __syncthreads();
            digit_search(hist, remaining, tmp, sh);
            prefix |= (uint32_t)sh[0] << shift;
            mask |= 255u << shift;
            remaining = sh[1];
            n_eq = sh[2];
        }
        T = prefix;
        take_eq = remaining;
    }

    int32_t* out = a.idx + (size_t)t * a.topk;
    int n_sel = want;
    if (a.sorted && n_eq == take_eq) {
        // every key >= T is chosen: place the pairs in any order, the sort
        // below orders them
        for (int s0 = 0; s0 < L; s0 += kTKThreads * kTKBatch) {
            uint32_t kb[kTKBatch];
            load_keys(kb, s0 + threadIdx.x, kTKThreads, L);
#pragma unroll
            for (int j = 0; j < kTKBatch; ++j) {
                const int s = s0 + j * kTKThreads + threadIdx.x;
                const uint32_t k = kb[j];
                const bool act = k != 0u && k >= T;
                const uint32_t am = __ballot_sync(0xffffffffu, act);
                if (am == 0u) continue;
                const int leader = __ffs(am) - 1;
                int base = 0;
                if (lane == leader) base = atomicAdd(&sh[4], __popc(am));
                base = __shfl_sync(0xffffffffu, base, leader);
                if (act)
                    sortbuf[base + __popc(am & lt)] =
                        ((unsigned long long)k << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)s);
            }
        }
    } else {
        // in index order: each warp walks its own contiguous segment of keys
        // with the lanes side by side (coalesced); ballots place each chosen
        // key.  Keys > T are all taken, keys == T while their rank < take_eq.
        const int seg = ((L + kTKThreads / 32 - 1) / (kTKThreads / 32) + 31) & ~31;
        const int s_beg = min(L, warp * seg), s_end = min(L, s_beg + seg);
        int gt = 0, eq = 0;
        for (int s0 = s_beg; s0 < s_end; s0 += 32 * kTKBatch) {
            uint32_t kb[kTKBatch];
            load_keys(kb, s0 + lane, 32, s_end);
#pragma unroll
            for (int j = 0; j < kTKBatch; ++j) {
                gt += __popc(__ballot_sync(0xffffffffu, kb[j] > T));
                eq += __popc(__ballot_sync(0xffffffffu, kb[j] == T && kb[j] != 0u));
            }
        }
        int n_gt = 0, n_eq_all = 0;
        const int gt_off = __shfl_sync(0xffffffffu, block_scan(lane == 0 ? gt : 0, tmp, &n_gt), 0);
        const int eq_off = __shfl_sync(0xffffffffu, block_scan(lane == 0 ? eq : 0, tmp, &n_eq_all), 0);
        (void)n_eq_all;
        const int eq_take = max(0, min(eq, take_eq - eq_off));
        const int sel_off = __shfl_sync(0xffffffffu, block_scan(lane == 0 ? gt + eq_take : 0, tmp, &n_sel), 0);
        int pg = gt_off, pe = eq_off, ps = sel_off;
        for (int s0 = s_beg; s0 < s_end; s0 += 32 * kTKBatch) {
          uint32_t kb[kTKBatch];
          load_keys(kb, s0 + lane, 32, s_end);
#pragma unroll
          for (int j = 0; j < kTKBatch; ++j) {
            const int s = s0 + 32 * j + lane;
            const uint32_t k = kb[j];
            const uint32_t bg = __ballot_sync(0xffffffffu, k > T);
            const uint32_t be = __ballot_sync(0xffffffffu, k == T && k != 0u);
            const int erank = pe + __popc(be & lt);
            const bool take_e = ((be >> lane) & 1u) && erank < take_eq;
            const uint32_t bt = __ballot_sync(0xffffffffu, take_e);
            if (a.sorted) {
                const unsigned long long packed =
                    ((unsigned long long)k << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)s);
                if ((bg >> lane) & 1u) sortbuf[pg + __popc(bg & lt)] = packed;
                if (take_e) sortbuf[n_gt + erank] = packed;
            } else {
                const uint32_t bsel = bg | bt;
                if ((bsel >> lane) & 1u) out[ps + __popc(bsel & lt)] = s;
                ps += __popc(bsel);
            }
            pg += __popc(bg);
            pe += __popc(be);
          }
        }
    }
    if (!a.sorted) {
        for (int j = n_sel + threadIdx.x; j < a.topk; j += kTKThreads) out[j] = -1;
        return;
    }
    // pad to a power of two (>= 128) with zeros (they sort last) and sort
    // descending: bitonic network, in-chunk steps in registers, the rest in
    // shared memory
    int P = 128;
    while (P < want) P <<= 1;
    for (int i = want + threadIdx.x; i < P; i += kTKThreads) sortbuf[i] = 0ull;
    __syncthreads();
    const int base = warp * 128;
    const bool wact = base < P;
    unsigned long long v[4];
    if (wact) {
#pragma unroll
        for (int r = 0; r < 4; ++r) v[r] = sortbuf[base + 4 * lane + r];
        warp_bitonic_chunk(v, base, lane);
#pragma unroll
        for (int r = 0; r < 4; ++r) sortbuf[base + 4 * lane + r] = v[r];
    }
    __syncthreads();
    for (int size = 256; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride >= 128; stride >>= 1) {
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
        if (wact) {
#pragma unroll
            for (int r = 0; r < 4; ++r) v[r] = sortbuf[base + 4 * lane + r];
            warp_bitonic_merge<6>(v, lane, (base & size) == 0);
#pragma unroll
            for (int r = 0; r < 4; ++r) sortbuf[base + 4 * lane + r] = v[r];
        }
        __syncthreads();
    }
    for (int j = threadIdx.x; j < a.topk; j += kTKThreads)
        out[j] = j < want ? (int32_t)(0xFFFFFFFFu - (uint32_t)(sortbuf[j] & 0xFFFFFFFFull)) : -1;
}

size_t dsa_topk_smem(int Sk) {
    return (size_t)kDsaMaxTopk * 8 + (256 + 32 + 8) * 4 + (Sk <= kTKCacheKeys ? (size_t)Sk * 4 : 0);
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
