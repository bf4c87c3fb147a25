// tiles.cuh -- the static tile walk and bounded waits shared by the
// single-CTA grouped GEMM kernels (bf16 and fp8).
#pragma once
#include "kernels.cuh"
#include "ptx.cuh"

namespace moe {

constexpr long long kWaitLimit = 1ll << 31;    // cycles (about one second)

struct Tile {
    int prob, exp, row0, nvalid, f0, kslice;
};

// fsz: output features per tile (128, or 256 for the token-major fp8 kernel).
__device__ __forceinline__ int problem_tiles(const GemmProblem& p, int bn, int fsz = 128) {
    const int nf = (p.n_feat + fsz - 1) / fsz;
    if (p.seg == nullptr) return nf * ((p.n_rows + bn - 1) / bn) * max(p.k_split, 1);
    return nf * __ldg(p.tok_start + p.n_exp);
}

// Tile t of the launch -> (problem, expert, token rows, feature tile).
// Order inside a problem: expert, then feature tile, then token tile, so that
// CTAs working at the same time share weight tiles through L2.
__device__ __forceinline__ bool tile_at(const GemmParams& P, int bn, int t, Tile& o,
                                        int fsz = 128) {
    for (int pi = 0; pi < P.n_problems; ++pi) {
        const GemmProblem& p = P.p[pi];
        const int n = problem_tiles(p, bn, fsz);
        if (t >= n) {
            t -= n;
            continue;
        }
        const int nf = (p.n_feat + fsz - 1) / fsz;
        int e = 0, first = 0, ntok, seg0, seg1;
        o.kslice = 0;
        if (p.seg == nullptr && p.k_split > 1) {
            o.kslice = t % p.k_split;
            t /= p.k_split;
        }
        if (p.seg == nullptr) {
            ntok = (p.n_rows + bn - 1) / bn;
            seg0 = 0;
            seg1 = p.n_rows;
        } else {
            // largest e with nf * tok_start[e] <= t
            int lo = 0, hi = p.n_exp - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (nf * __ldg(p.tok_start + mid) <= t) lo = mid; else hi = mid - 1;
            }
            e = lo;
            first = nf * __ldg(p.tok_start + e);
            ntok = __ldg(p.tok_start + e + 1) - __ldg(p.tok_start + e);
            seg0 = __ldg(p.seg + e);
            seg1 = __ldg(p.seg + e + 1);
        }
        const int local = t - first;
        const int ft = local / ntok, tt = local - ft * ntok;
        o.prob = pi;
        o.exp = e;
        o.f0 = ft * fsz;
        o.row0 = seg0 + tt * bn;
        o.nvalid = min(bn, seg1 - o.row0);
        return true;
    }
    return false;
}

__device__ __forceinline__ int total_tiles(const GemmParams& P, int bn, int fsz = 128) {
    int n = 0;
    for (int pi = 0; pi < P.n_problems; ++pi) n += problem_tiles(P.p[pi], bn, fsz);
    return n;
}

// Bounded mbarrier wait.  Returns false when this CTA is aborting (unless
// `drain`, used for the final waits on work already in flight, which only
// stop at the time limit).
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         int* status, bool drain = false) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (!drain && *abort_flag) return false;
        if (clock64() - t0 > kWaitLimit) {
            *abort_flag = 1;
            if (status) atomicOr(status, DEV_STATUS_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + __expf(-g)); }

}  // namespace moe
