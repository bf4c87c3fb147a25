// route.cu -- router selection: sigmoid scores, noaux_tc biased choice with
// optional group limit, top-k and renormalised weights (steps a2-a4), one
// warp per token, everything in registers and warp shuffles.
//
// Method: "dots3-note 架构深度解析" (mlqm.cn), section 稀疏激活：Top-8 路由 --
// sigmoid scoring function, noaux_tc routing, top-8 of 256, norm_topk_prob;
// "Transformers 中的 dots.llm1（Dots1）模型" (blog.gitcode.com), table
// MoE 路由与专家相关字段 -- n_group / topk_group (choose groups by group score,
// then the top-k inside them), routed_scaling_factor;
// "Xiaohongshu dots3 note Open Source Deep Dive", §3.1 -- weights are the
// chosen scores divided by their sum.
//
// Every floating-point step that decides a choice is an explicitly rounded
// binary32 operation (__fadd_rn, __fmul_rn, __fmaf_rn, __fdiv_rn, rintf), so
// the result is fixed by IEEE-754 and does not depend on compiler
// contraction.  The exponential is Cody & Waite reduction plus a degree-7
// Taylor polynomial (see dev_exp).
#include "kernels.cuh"


namespace moe {

// e^x: x = n ln2 + r, ln2 split into a 16-bit head (n * head exact for
// |n| < 256) and a binary32 tail; e^r by its Taylor series to r^7/7! in
// Horner form; times 2^n built from the exponent bits.  x is clamped to
// [-86, 86] so that every value stays a normal binary32 number.
__device__ __forceinline__ float dev_exp(float x) {
    x = fminf(fmaxf(x, -86.0f), 86.0f);
    const float nf = rintf(__fmul_rn(x, 0x1.715476p+0f));   // x / ln2
    float r = __fmaf_rn(-nf, 0x1.62e4p-1f, x);               // - n * ln2 head
    r = __fmaf_rn(-nf, 0x1.7f7d1cp-20f, r);                  // - n * ln2 tail
    float p = 0x1.a01a02p-13f;                               // 1/7!
    p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);                    // 1/6!
    p = __fmaf_rn(p, r, 0x1.111112p-7f);                     // 1/5!
    p = __fmaf_rn(p, r, 0x1.555556p-5f);                     // 1/4!
    p = __fmaf_rn(p, r, 0x1.555556p-3f);                     // 1/3!
    p = __fmaf_rn(p, r, 0x1.0p-1f);                          // 1/2!
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    const int n = static_cast<int>(nf);
    return __fmul_rn(p, __int_as_float((n + 127) << 23));
}

// Router score s = 1 / (1 + e^{-l}).
__device__ __forceinline__ float dev_sigmoid(float l) {
    return __fdiv_rn(1.0f, __fadd_rn(1.0f, dev_exp(-l)));
}

// (key, index) order of every top-k here: larger key first, then lower index.
__device__ __forceinline__ bool better(float a, int ia, float b, int ib) {
    return a > b || (a == b && ia < ib);
}

// Warp-wide arg-best; every lane ends with the winner.
__device__ __forceinline__ void warp_best(float& v, int& i) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, off);
        const int oi = __shfl_xor_sync(0xffffffffu, i, off);
        if (better(ov, oi, v, i)) {
            v = ov;
            i = oi;
        }
    }
}

// One warp per token; lane l owns experts l*VPL .. l*VPL + VPL - 1.
template <int VPL>
__global__ void __launch_bounds__(256) route_select_kernel(const RouteArgs a) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= a.T) return;
    const int E = a.E, k = a.k;
    const int e0 = lane * VPL;
    const float* row = a.logits + (size_t)t * E + e0;
    const size_t slice = (size_t)a.T * E;

    float lg[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) lg[i] = __ldg(row + i);
    if (a.n_split > 1) {
        // K-slice partials of the router GEMM, summed in slice order
        for (int sp = 1; sp < a.n_split; ++sp) {
            float part[VPL];
#pragma unroll
            for (int i = 0; i < VPL; ++i) part[i] = __ldg(row + sp * slice + i);
#pragma unroll
            for (int i = 0; i < VPL; ++i) lg[i] = __fadd_rn(lg[i], part[i]);
        }
#pragma unroll
        for (int i = 0; i < VPL; ++i) a.logits_out[(size_t)t * E + e0 + i] = lg[i];
    }

    float s[VPL], c[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const float l = lg[i];
        s[i] = dev_sigmoid(l);
        c[i] = __fadd_rn(s[i], __ldg(a.bias + e0 + i));  // bias steers the choice only
        if (isnan(c[i])) c[i] = -INFINITY;                // NaN ranks below numbers
    }

    uint32_t eligible = (VPL == 32) ? 0xffffffffu : ((1u << VPL) - 1u);
    if (a.n_group > 1) {
        // Group score: sum of the group_topn largest keys, largest first.
        const int gsz = E / a.n_group;
        float my_gs = -INFINITY;
        for (int g = 0; g < a.n_group; ++g) {
            uint32_t used = 0;
            float acc = 0.0f;
            for (int j = 0; j < a.group_topn; ++j) {
                float bv = -INFINITY;
                int bi = 0x7fffffff;
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    const int e = e0 + i;
                    if (e / gsz == g && !(used >> i & 1u) && better(c[i], e, bv, bi)) {
                        bv = c[i];
                        bi = e;
                    }
                }
                warp_best(bv, bi);
                if (bi >= e0 && bi < e0 + VPL) used |= 1u << (bi - e0);
                acc = (j == 0) ? bv : __fadd_rn(acc, bv);
            }
            if (lane == g) my_gs = isnan(acc) ? -INFINITY : acc;
        }
        // Keep the topk_group best groups (lower group index on ties).
        uint32_t keep = 0;
        bool chosen = lane >= a.n_group;
        for (int j = 0; j < a.topk_group; ++j) {
            float bv = chosen ? -INFINITY : my_gs;
            int bi = chosen ? 0x7fffffff : lane;
            warp_best(bv, bi);
            keep |= 1u << bi;
            if (lane == bi) chosen = true;
        }
        eligible = 0;
#pragma unroll
        for (int i = 0; i < VPL; ++i)
            if (keep >> ((e0 + i) / gsz) & 1u) eligible |= 1u << i;
    }

    // Top-k: k rounds of a warp arg-best over the remaining eligible keys.
    int my_idx = 0;
    float my_s = 0.0f;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < VPL; ++i)
            if ((eligible >> i & 1u) && better(c[i], e0 + i, bv, bi)) {
                bv = c[i];
                bi = e0 + i;
            }
        warp_best(bv, bi);
        const int owner = bi / VPL;
        float sv = 0.0f;
#pragma unroll
        for (int i = 0; i < VPL; ++i)
            if (e0 + i == bi) {
                sv = s[i];
                eligible &= ~(1u << i);
            }
        sv = __shfl_sync(0xffffffffu, sv, owner & 31);
        if (lane == j) {
            my_idx = bi;
            my_s = sv;
        }
    }
    // Renormalise: sum of the chosen scores in slot order.
    float sum = 0.0f;
    for (int j = 0; j < k; ++j) sum = __fadd_rn(sum, __shfl_sync(0xffffffffu, my_s, j));
    if (lane < k) {
        float w = a.norm ? __fdiv_rn(my_s, sum) : my_s;
        w = __fmul_rn(w, a.rsf);
        a.idx[(size_t)t * k + lane] = my_idx;
        a.w[(size_t)t * k + lane] = w;
    }
}

template <int VPL>
static cudaError_t launch_vpl(const RouteArgs& a, cudaStream_t s) {
    const int warps = 8;
    const int grid = (a.T + warps - 1) / warps;
    route_select_kernel<VPL><<<grid, warps * 32, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_route_select(const RouteArgs& a, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    switch (a.E / 32) {
        case 1: return launch_vpl<1>(a, s);
        case 2: return launch_vpl<2>(a, s);
        case 3: return launch_vpl<3>(a, s);
        case 4: return launch_vpl<4>(a, s);
        case 5: return launch_vpl<5>(a, s);
        case 6: return launch_vpl<6>(a, s);
        case 8: return launch_vpl<8>(a, s);
        case 10: return launch_vpl<10>(a, s);
        case 12: return launch_vpl<12>(a, s);
        case 16: return launch_vpl<16>(a, s);
        case 24: return launch_vpl<24>(a, s);
        case 32: return launch_vpl<32>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
