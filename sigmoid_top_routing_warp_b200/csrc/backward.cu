// backward.cu -- the layer's backward pass with the expert choice held fixed
// (moe_backward): gradients of a loss through the routed SwiGLU experts, the
// shared expert, the renormalised routing weights and the sigmoid router.
//
// The pages give the forward pass only ("Xiaohongshu dots3 note Open Source
// Deep Dive", §3.1 Expert Routing Mechanism and §8.2 gmm1 -> swiglu -> gmm2;
// "dots3-note 架构深度解析" (mlqm.cn), 稀疏激活: sigmoid scores, noaux_tc,
// norm_topk_prob); the backward pass is the chain rule through it:
//   y_r = SiLU(g_r) u_r W2_e^T,  out_t = sum_j w_tj y_tj + shared(x_t)
//   dw_tj = <dout_t, y_tj> = sum_i a_tj[i] (dout_t W2_e)[i]
//   with w_j = rsf s_j / S (S = sum of the chosen scores s = sigmoid(L)):
//     ds_j = rsf (dw_j / S - sum_i dw_i s_i / S^2),  dL = ds s (1 - s)
//   dx = sum_j dX_j + dx_shared + dL W_g,  dW_g = dL^T x
// The choice (top-k of s + bias) is piecewise constant: no gradient flows
// through it, and the expert bias gets none.
//
// Sequence on one stream:
//   1. permute (as the forward) -> expert segments
//   2. plan: segments padded to 16 rows (pstart) and their 256-row tile
//      prefix (tstart); a weight-gradient GEMM contracts over a padded
//      segment, and 16 rows is one MMA's K
//   3. gather: X and dout rows into the padded order, routing weight per
//      padded row, zero pad rows
//   4. GEMM  G|U = X W13^T (gate/up recomputed in fp32; shared expert beside it)
//   5. GEMM  dA' = dY W2_e, epilogue: SwiGLU backward -> dG|dU, w SiLU(g) u,
//      and partial sums of dw
//   6. router: dw -> ds -> dL (one warp per token)
//   7. GEMM  dX = dG|dU W13_e (routed, shared) and dL W_g
//   8. GEMM  dW2_e, dW13_e (K = the expert's padded rows), dW2s, dW13s, dW_g
//   9. combine: dx_t = sum_j dX[row(t, j)] + dx_shared + dx_router, fp32 sum
//      in slot order, one bf16 rounding
#include "moe.h"
#include "kernels.cuh"

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>

namespace moe {
moe_status_t api_check_config(const moe_config_t* c);
moe_status_t api_fail(moe_status_t st, const char* msg);
void api_clear_error();
moe_status_t api_sm_count(int* n);
moe_status_t api_make_map_2d_bf16(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols,
                                  uint32_t box_cols, uint32_t box_rows, const char* what);
moe_status_t api_make_map_3d_bf16(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1,
                                  uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t b0,
                                  uint32_t b1, uint32_t b2, const char* what);
moe_status_t api_make_map_store_3d(CUtensorMap* m, const void* ptr, int f32, uint64_t d0,
                                   uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2,
                                   uint32_t b0, uint32_t b1, const char* what);
}  // namespace moe

namespace {

constexpr int kPadRows = 16;   // segment padding: one MMA's K
constexpr int kRowTile = 256;  // token rows per tile of the rows-as-N GEMMs

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Workspace of moe_backward (256-byte aligned regions).
struct BLayout {
    size_t status, offsets, rows, pos, chunk, pstart, tstart, ttab, prow, wpad, xpad, dypad, gu, dgu, aw,
        dwpart, dxpad, gus, dgus, as, dxsh, dxr, dl, total;
    size_t rmax;  // rows of the padded buffers
};

BLayout blayout(const moe_config_t* c) {
    BLayout L{};
    const size_t T = c->T, E = c->E, k = c->k, H = c->H, I = c->I, Is = (size_t)c->n_shared * c->I;
    const size_t n = T * k;
    // padded rows: every segment rounded up to 16, plus one row tile of slack
    // that rows-as-N tiles may read past the last segment (never stored)
    L.rmax = n + (kPadRows - 1) * E + kRowTile;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + bytes, 256);
        return at;
    };
    L.status = take(256);
    L.offsets = take((E + 1) * 4);
    L.rows = take(n * 4);
    L.pos = take(n * 4);
    L.chunk = take((size_t)moe::permute_chunks((int)n) * E * 4);
    L.pstart = take((E + 1) * 4);
    L.tstart = take((E + 1) * 4);
    L.ttab = take((L.rmax / kRowTile + E) * 4);
    L.prow = take(n * 4);
    L.wpad = take(L.rmax * 4);
    L.xpad = take(L.rmax * H * 2);
    L.dypad = take(L.rmax * H * 2);
    L.gu = take(L.rmax * 2 * I * 4);  // fp32 pre-activations
    L.dgu = take(L.rmax * 2 * I * 2);
    L.aw = take(L.rmax * I * 2);
    L.dwpart = take(L.rmax * (I / 32) * 4);
    L.dxpad = take(L.rmax * H * 2);
    L.gus = take(T * 2 * Is * 4);
    L.dgus = take(T * 2 * Is * 2);
    L.as = take(T * Is * 2);
    L.dxsh = take(T * H * 4);
    L.dxr = take(T * H * 4);
    L.dl = take(T * align_up(E, 64) * 2);  // rows padded to 64 columns (zeros)
    L.total = off;
    return L;
}

template <typename Tp>
Tp* at(void* ws, size_t off) {
    return reinterpret_cast<Tp*>(static_cast<char*>(ws) + off);
}

moe_status_t bfail(moe_status_t st, const char* fmt, long long a = 0, long long b = 0) {
    char msg[256];
    snprintf(msg, sizeof(msg), fmt, a, b);
    return moe::api_fail(st, msg);
}

moe_status_t bcuda(cudaError_t e, const char* what) {
    char msg[256];
    snprintf(msg, sizeof(msg), "%s: %s", what, cudaGetErrorString(e));
    return moe::api_fail(MOE_ERR_CUDA, msg);
}

#define BW_TRY(x)                          \
    do {                                   \
        moe_status_t st_ = (x);            \
        if (st_ != MOE_OK) return st_;     \
    } while (0)
#define BW_CUDA(call, what)                             \
    do {                                                \
        cudaError_t e_ = (call);                        \
        if (e_ != cudaSuccess) return bcuda(e_, what);  \
    } while (0)

// ---------------------------------------------------------------- kernels

struct PlanArgs {
    const int32_t* offsets;
    int32_t* pstart;  // [E + 1] padded segment starts
    int32_t* tstart;  // [E + 1] prefix of 256-row tiles over the padded segments
    int32_t* ttab;    // [tstart[E]] the expert of each row tile
    int E;
};

// One block: two exclusive scans over the experts (E <= 1024).
__global__ void __launch_bounds__(1024) bwd_plan_kernel(const PlanArgs a) {
    __shared__ int sp[1024], st[1024];
    const int e = threadIdx.x;
    int np = 0, nt = 0;
    if (e < a.E) {
        const int ne = a.offsets[e + 1] - a.offsets[e];
        np = (ne + kPadRows - 1) / kPadRows * kPadRows;
        nt = (np + kRowTile - 1) / kRowTile;
    }
    sp[e] = np;
    st[e] = nt;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
        const int vp = e >= off ? sp[e - off] : 0;
        const int vt = e >= off ? st[e - off] : 0;
        __syncthreads();
        sp[e] += vp;
        st[e] += vt;
        __syncthreads();
    }
    if (e < a.E) {
        a.pstart[e] = sp[e] - np;
        a.tstart[e] = st[e] - nt;
    }
    if (e == a.E - 1) {
        a.pstart[a.E] = sp[e];
        a.tstart[a.E] = st[e];
    }
    // the expert of each row tile
    for (int r = 0; r < nt; ++r) a.ttab[st[e] - nt + r] = e;
}

struct BGatherArgs {
    const uint16_t* x;       // [T, H]
    const uint16_t* dout;    // [T, H]
    const int32_t* idx;      // [T * k]
    const float* topk_w;     // [T * k]
    const int32_t* pos;      // [T * k] sorted row of each slot
    const int32_t* offsets;  // [E + 1]
    const int32_t* pstart;   // [E + 1]
    int32_t* prow;           // [T * k] padded row of each slot
    float* wpad;             // [rows]
    uint16_t* xpad;          // [rows, H]
    uint16_t* dypad;         // [rows, H]
    int T, k, H, E;
};

// Warps 0 .. T*k-1: one slot each (copy x and dout rows into its padded row);
// warps T*k .. T*k+E-1: zero the pad rows of one expert.
__global__ void __launch_bounds__(256) bwd_gather_kernel(const BGatherArgs a) {
    const int warp = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    const int n = a.T * a.k;
    const int hv = a.H / 8;  // 16-byte vectors per row
    if (warp < n) {
        const int e = a.idx[warp];
        if (e < 0 || e >= a.E) {  // not a valid choice: the slot takes no part
            if (lane == 0) a.prow[warp] = -1;
            return;
        }
        const int r = a.pstart[e] + (a.pos[warp] - a.offsets[e]);
        const int t = warp / a.k;
        if (lane == 0) {
            a.prow[warp] = r;
            a.wpad[r] = a.topk_w[warp];
        }
        const uint4* xs = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.H);
        const uint4* ds = reinterpret_cast<const uint4*>(a.dout + (size_t)t * a.H);
        uint4* xd = reinterpret_cast<uint4*>(a.xpad + (size_t)r * a.H);
        uint4* dd = reinterpret_cast<uint4*>(a.dypad + (size_t)r * a.H);
        for (int v = lane; v < hv; v += 32) {
            xd[v] = __ldg(xs + v);
            dd[v] = __ldg(ds + v);
        }
    } else if (warp < n + a.E) {
        const int e = warp - n;
        const int r0 = a.pstart[e] + (a.offsets[e + 1] - a.offsets[e]);
        const int r1 = a.pstart[e + 1];
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int r = r0; r < r1; ++r) {
            if (lane == 0) a.wpad[r] = 0.0f;
            uint4* xd = reinterpret_cast<uint4*>(a.xpad + (size_t)r * a.H);
            uint4* dd = reinterpret_cast<uint4*>(a.dypad + (size_t)r * a.H);
            for (int v = lane; v < hv; v += 32) {
                xd[v] = z;
                dd[v] = z;
            }
        }
    }
}

struct BRouterArgs {
    const float* logits;   // [T, E]
    const int32_t* idx;    // [T, k]
    const int32_t* prow;   // [T * k]
    const float* dwpart;   // [rows, nparts]
    int nparts;
    uint16_t* dl;          // bf16 [T, ld_dl], zero in columns E .. ld_dl - 1
    int ld_dl;
    float* dlogits;        // fp32 [T, E] or null
    int T, E, k, norm;
    float rsf;
};

// One warp per token: the routing-weight gradient of each slot (its partial
// sums added in a fixed order), through the renormalisation and the sigmoid
// to the logits; zero off the chosen experts.
__global__ void __launch_bounds__(256) bwd_router_kernel(const BRouterArgs a) {
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= a.T) return;
    const int k = a.k;
    // lane j < k: slot j
    float s = 0.0f, dw = 0.0f;
    int e = -1;
    if (lane < k) {
        const int pr = a.prow[(size_t)t * k + lane];
        if (pr >= 0) {
            e = a.idx[(size_t)t * k + lane];
            s = 1.0f / (1.0f + expf(-a.logits[(size_t)t * a.E + e]));
            const float* p = a.dwpart + (size_t)pr * a.nparts;
            for (int c = 0; c < a.nparts; ++c) dw += p[c];
        }
    }
    // S = sum of the chosen scores, Q = sum dw_j s_j (fixed slot order)
    // (explicitly rounded operations: no contraction into fused multiply-adds)
    float S = 0.0f, Q = 0.0f;
    for (int j = 0; j < k; ++j) {
        const float sj = __shfl_sync(0xffffffffu, s, j);
        const float dj = __shfl_sync(0xffffffffu, dw, j);
        S = __fadd_rn(S, sj);
        Q = __fadd_rn(Q, __fmul_rn(dj, sj));
    }
    float ds = 0.0f;
    // (dw_j S - Q) / S^2: with k = 1 the numerator is exactly zero, as the
    // derivative of a weight fixed at rsf
    if (lane < k)
        ds = a.norm ? a.rsf * (__fsub_rn(__fmul_rn(dw, S), Q) / __fmul_rn(S, S)) : a.rsf * dw;
    const float dlv = ds * s * (1.0f - s);
    for (int c = lane; c < a.ld_dl; c += 32) {
        float v = 0.0f;
        for (int j = 0; j < k; ++j) {
            const int ej = __shfl_sync(0xffffffffu, e, j);
            const float vj = __shfl_sync(0xffffffffu, dlv, j);
            if (ej == c) v = vj;
        }
        a.dl[(size_t)t * a.ld_dl + c] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
        if (a.dlogits && c < a.E) a.dlogits[(size_t)t * a.E + c] = v;
    }
}

struct BCombineArgs {
    const uint16_t* dxpad;   // [rows, H]
    const int32_t* prow;     // [T * k]
    const float* dxsh;       // [T, H] or null
    const float* dxr;        // [T, H]
    uint16_t* dx;            // [T, H]
    int T, k, H;
};

// dx_t = sum_j dX[prow(t, j)] (slot order) + dx_shared_t + dx_router_t, fp32,
// one bf16 rounding; one thread per 8 columns.
__global__ void __launch_bounds__(256) bwd_combine_kernel(const BCombineArgs a) {
    const int hv = a.H / 8;
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)a.T * hv) return;
    const int t = (int)(i / hv), v = (int)(i % hv);
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
    for (int j = 0; j < a.k; ++j) {
        const int r = a.prow[(size_t)t * a.k + j];
        if (r < 0) continue;
        const uint4 q = *reinterpret_cast<const uint4*>(a.dxpad + (size_t)r * a.H + 8 * v);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            acc[2 * c] += __uint_as_float(w[c] << 16);
            acc[2 * c + 1] += __uint_as_float(w[c] & 0xffff0000u);
        }
    }
    const float* srcs[2] = {a.dxsh, a.dxr};
    for (int s = 0; s < 2; ++s) {
        if (!srcs[s]) continue;
        const float4* p = reinterpret_cast<const float4*>(srcs[s] + (size_t)t * a.H + 8 * v);
        const float4 f0 = p[0], f1 = p[1];
        acc[0] += f0.x; acc[1] += f0.y; acc[2] += f0.z; acc[3] += f0.w;
        acc[4] += f1.x; acc[5] += f1.y; acc[6] += f1.z; acc[7] += f1.w;
    }
    uint32_t o[4];
#pragma unroll
    for (int c = 0; c < 4; ++c)
        o[c] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * c])) |
               ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * c + 1])) << 16);
    *reinterpret_cast<uint4*>(a.dx + (size_t)t * a.H + 8 * v) = make_uint4(o[0], o[1], o[2], o[3]);
}

moe_status_t need(const void* p, const char* name) {
    if (p) return MOE_OK;
    char msg[128];
    snprintf(msg, sizeof(msg), "%s is NULL", name);
    return moe::api_fail(MOE_ERR_INVALID_ARG, msg);
}

moe_status_t need16(const void* p, const char* name) {
    BW_TRY(need(p, name));
    if (reinterpret_cast<uintptr_t>(p) & 15u) {
        char msg[128];
        snprintf(msg, sizeof(msg), "%s must be 16-byte aligned", name);
        return moe::api_fail(MOE_ERR_INVALID_ARG, msg);
    }
    return MOE_OK;
}

using moe::api_make_map_2d_bf16;

// K-major operand maps: [rows, cols] bf16, box {64, 128}.
moe_status_t kmap(CUtensorMap* m, const void* p, size_t rows, size_t cols, const char* what) {
    return api_make_map_2d_bf16(m, p, rows, cols, 64, 128, what);
}
// MN-major operand map of a row-major [K rows, MN cols] bf16 matrix: the 3-D
// view {64, rows, MN / 64} (strides: a row, 64 elements), box {64, 64, 2}:
// one copy brings 64 K rows of 128 consecutive MN elements as two 8 KB
// chunks.  MN is a multiple of 64 for every operand here.
moe_status_t mnmap(CUtensorMap* m, const void* p, size_t rows, size_t cols, const char* what) {
    return moe::api_make_map_3d_bf16(m, p, 64, rows, (cols + 63) / 64, cols * 2, 128, 64, 64, 2,
                                     what);
}

}  // namespace

extern "C" {

size_t moe_backward_workspace_size(const moe_config_t* cfg) {
    if (moe::api_check_config(cfg) != MOE_OK) return 0;
    return blayout(cfg).total;
}

moe_status_t moe_backward(const moe_config_t* cfg, const void* x, const void* w_router,
                          const float* logits, const int32_t* topk_idx, const float* topk_w,
                          const void* w13, const void* w2, const void* w13s, const void* w2s,
                          const void* dout, void* dx, float* dw_router, float* dw13, float* dw2,
                          float* dw13s, float* dw2s, float* dlogits, void* ws, size_t ws_bytes,
                          void* const* stage_events, moe_stream_t stream) {
    moe::api_clear_error();
    BW_TRY(moe::api_check_config(cfg));
    if (cfg->dtype != MOE_DTYPE_BF16)
        return moe::api_fail(MOE_ERR_UNSUPPORTED, "moe_backward: bf16 layers only");
    BW_TRY(need16(x, "x"));
    BW_TRY(need16(w_router, "w_router"));
    BW_TRY(need(logits, "logits"));
    BW_TRY(need(topk_idx, "topk_idx"));
    BW_TRY(need(topk_w, "topk_w"));
    BW_TRY(need16(w13, "w13"));
    BW_TRY(need16(w2, "w2"));
    BW_TRY(need16(dout, "dout"));
    BW_TRY(need16(dx, "dx"));
    BW_TRY(need16(dw_router, "dw_router"));
    BW_TRY(need16(dw13, "dw13"));
    BW_TRY(need16(dw2, "dw2"));
    if (cfg->n_shared > 0) {
        BW_TRY(need16(w13s, "w13s"));
        BW_TRY(need16(w2s, "w2s"));
        BW_TRY(need16(dw13s, "dw13s"));
        BW_TRY(need16(dw2s, "dw2s"));
    }
    if (!ws) return moe::api_fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
    if (reinterpret_cast<uintptr_t>(ws) & 255u)
        return moe::api_fail(MOE_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const BLayout L = blayout(cfg);
    if (ws_bytes < L.total)
        return bfail(MOE_ERR_WORKSPACE, "workspace has %lld bytes, needs %lld", (long long)ws_bytes,
                     (long long)L.total);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int T = cfg->T, E = cfg->E, k = cfg->k, H = cfg->H, I = cfg->I;
    const int Is = cfg->n_shared * cfg->I;
    const size_t n = (size_t)T * k;
    if (T == 0) {
        // no token: every weight gradient is zero
        BW_CUDA(cudaMemsetAsync(dw_router, 0, (size_t)E * H * 4, s), "memset");
        BW_CUDA(cudaMemsetAsync(dw13, 0, (size_t)E * 2 * I * H * 4, s), "memset");
        BW_CUDA(cudaMemsetAsync(dw2, 0, (size_t)E * H * I * 4, s), "memset");
        if (Is > 0) {
            BW_CUDA(cudaMemsetAsync(dw13s, 0, (size_t)2 * Is * H * 4, s), "memset");
            BW_CUDA(cudaMemsetAsync(dw2s, 0, (size_t)H * Is * 4, s), "memset");
        }
        return MOE_OK;
    }
    int* status = at<int>(ws, L.status);
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* pos = at<int32_t>(ws, L.pos);
    int32_t* pstart = at<int32_t>(ws, L.pstart);
    int32_t* tstart = at<int32_t>(ws, L.tstart);
    int32_t* ttab = at<int32_t>(ws, L.ttab);
    int32_t* prow = at<int32_t>(ws, L.prow);
    float* wpad = at<float>(ws, L.wpad);
    uint16_t* xpad = at<uint16_t>(ws, L.xpad);
    uint16_t* dypad = at<uint16_t>(ws, L.dypad);
    float* gu = at<float>(ws, L.gu);
    uint16_t* dgu = at<uint16_t>(ws, L.dgu);
    uint16_t* aw = at<uint16_t>(ws, L.aw);
    float* dwpart = at<float>(ws, L.dwpart);
    uint16_t* dxpad = at<uint16_t>(ws, L.dxpad);
    float* gus = at<float>(ws, L.gus);
    uint16_t* dgus = at<uint16_t>(ws, L.dgus);
    uint16_t* as = at<uint16_t>(ws, L.as);
    float* dxsh = at<float>(ws, L.dxsh);
    float* dxr = at<float>(ws, L.dxr);
    uint16_t* dl = at<uint16_t>(ws, L.dl);
    const size_t R = L.rmax;
    const int ld_dl = (int)align_up(E, 64);
    int sms = 0;
    BW_TRY(moe::api_sm_count(&sms));
    // K-major B maps: boxes of 128 rows and of 16, 32 and 64 rows for the
    // ragged row tiles
    auto kB = [&](moe::BwdProblem& q, const void* ptr, size_t r, size_t c, const char* w) {
        for (int i = 0; i < 3; ++i) BW_TRY(api_make_map_2d_bf16(&q.tbs[i], ptr, r, c, 64, 16u << i, w));
        return kmap(&q.tb, ptr, r, c, w);
    };
    // Launch one backward GEMM; a store epilogue first gets the store map of
    // each problem's output: 16-row boxes over padded segments (whose row
    // tiles end on a multiple of 16), 32-row boxes elsewhere.
    auto gemm = [&](int epi, moe::BwdParams& P, const char* what) -> moe_status_t {
        if (epi == moe::BEPI_STORE)
            for (int i = 0; i < P.n_problems; ++i) {
                moe::BwdProblem& p = P.p[i];
                const size_t rows = p.rows_as_k ? (size_t)p.N : p.seg ? R : (size_t)p.n_rows;
                const size_t groups = p.rows_as_k ? (size_t)p.n_grp : 1;
                const size_t es = p.out_f32 ? 4 : 2;
                const size_t gstride = groups > 1 ? (size_t)p.out_grp * es : rows * p.ld_out * es;
                BW_TRY(moe::api_make_map_store_3d(&p.to, p.out, p.out_f32, p.M, rows, groups,
                                                  (size_t)p.ld_out * es, gstride, 32,
                                                  (p.rows_as_k || !p.seg) ? 32 : 16,
                                                  "gradient output"));
            }
        P.status = status;
        BW_CUDA(moe::launch_bwd_gemm(epi, P, sms, s), what);
        return MOE_OK;
    };
    cudaEvent_t ev[MOE_NUM_BWD_STAGES + 1] = {};
    if (stage_events)
        for (int i = 0; i <= MOE_NUM_BWD_STAGES; ++i) ev[i] = static_cast<cudaEvent_t>(stage_events[i]);
    auto mark = [&](int i) -> moe_status_t {
        if (ev[i]) BW_CUDA(cudaEventRecord(ev[i], s), "event record");
        return MOE_OK;
    };
    BW_TRY(mark(0));

    // 1. expert segments
    moe::PermuteArgs pa;
    pa.idx = topk_idx;
    pa.offsets = offsets;
    pa.rows = at<int32_t>(ws, L.rows);
    pa.pos = pos;
    pa.chunk_base = at<int32_t>(ws, L.chunk);
    pa.T = T;
    pa.k = k;
    pa.E = E;
    BW_CUDA(moe::launch_permute(pa, s), "permute launch");
    // 2. padded segments
    PlanArgs pl{offsets, pstart, tstart, ttab, E};
    bwd_plan_kernel<<<1, 1024, 0, s>>>(pl);
    BW_CUDA(cudaGetLastError(), "plan launch");
    // 3. gather
    BGatherArgs ga{static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(dout), topk_idx,
                   topk_w, pos, offsets, pstart, prow, wpad, xpad, dypad, T, k, H, E};
    bwd_gather_kernel<<<(unsigned)((n + E + 7) / 8), 256, 0, s>>>(ga);
    BW_CUDA(cudaGetLastError(), "gather launch");

    BW_TRY(mark(1));
    // 4. G|U = X W13^T (routed, padded rows) and x W13s^T (shared)
    {
        moe::BwdParams P;
        memset(&P, 0, sizeof(P));
        moe::BwdProblem& p = P.p[0];
        BW_TRY(kmap(&p.ta, w13, (size_t)E * 2 * I, H, "w13"));
        BW_TRY(kB(p, xpad, R, H, "padded x"));
        p.seg = pstart;
        p.tstart = tstart;
        p.ttab = ttab;
        p.n_grp = E;
        p.M = 2 * I;
        p.K = H;
        p.a_grp_rows = 2 * I;
        p.out = gu;
        p.ld_out = 2 * I;
        p.out_f32 = 1;
        P.n_problems = 1;
        if (Is > 0) {
            moe::BwdProblem& q = P.p[1];
            BW_TRY(kmap(&q.ta, w13s, (size_t)2 * Is, H, "w13s"));
            BW_TRY(kB(q, x, T, H, "x"));
            q.n_grp = 1;
            q.n_rows = T;
            q.M = 2 * Is;
            q.K = H;
            q.out = gus;
            q.ld_out = 2 * Is;
            q.out_f32 = 1;
            P.n_problems = 2;
        }
        BW_TRY(gemm(moe::BEPI_STORE, P, "gate/up recompute GEMM launch"));
    }
    BW_TRY(mark(2));
    // 5. dA' = dY W2_e with the SwiGLU backward in the epilogue
    {
        moe::BwdParams P;
        memset(&P, 0, sizeof(P));
        moe::BwdProblem& p = P.p[0];
        BW_TRY(mnmap(&p.ta, w2, (size_t)E * H, I, "w2"));
        BW_TRY(kB(p, dypad, R, H, "padded dout"));
        p.a_mn = 1;
        p.seg = pstart;
        p.tstart = tstart;
        p.ttab = ttab;
        p.n_grp = E;
        p.M = I;
        p.K = H;
        p.a_grp_rows = H;
        p.gu = gu;
        p.ld_gu = 2 * I;
        p.half = I;
        p.row_w = wpad;
        p.dgu = dgu;
        p.ld_dgu = 2 * I;
        p.aw = aw;
        p.ld_aw = I;
        p.dw_part = dwpart;
        p.ld_dw = I / 32;
        P.n_problems = 1;
        if (Is > 0) {
            moe::BwdProblem& q = P.p[1];
            BW_TRY(mnmap(&q.ta, w2s, H, Is, "w2s"));
            BW_TRY(kB(q, dout, T, H, "dout"));
            q.a_mn = 1;
            q.n_grp = 1;
            q.n_rows = T;
            q.M = Is;
            q.K = H;
            q.gu = gus;
            q.ld_gu = 2 * Is;
            q.half = Is;
            q.dgu = dgus;
            q.ld_dgu = 2 * Is;
            q.aw = as;
            q.ld_aw = Is;
            P.n_problems = 2;
        }
        BW_TRY(gemm(moe::BEPI_DSWIGLU, P, "down backward GEMM launch"));
    }
    BW_TRY(mark(3));
    // 6. router gradient
    {
        BRouterArgs ra{logits, topk_idx, prow, dwpart, I / 32, dl, ld_dl, dlogits, T, E, k,
                       cfg->norm_topk_prob != 0, cfg->routed_scaling_factor};
        bwd_router_kernel<<<(unsigned)((T + 7) / 8), 256, 0, s>>>(ra);
        BW_CUDA(cudaGetLastError(), "router gradient launch");
    }
    BW_TRY(mark(4));
    // 7. dX = dG|dU W13_e (routed), dG|dU W13s (shared), dL W_g (router)
    {
        moe::BwdParams P;
        memset(&P, 0, sizeof(P));
        int np = 0;
        moe::BwdProblem& p = P.p[np++];
        BW_TRY(mnmap(&p.ta, w13, (size_t)E * 2 * I, H, "w13"));
        BW_TRY(kB(p, dgu, R, 2 * I, "padded dgate/dup"));
        p.a_mn = 1;
        p.seg = pstart;
        p.tstart = tstart;
        p.ttab = ttab;
        p.n_grp = E;
        p.M = H;
        p.K = 2 * I;
        p.a_grp_rows = 2 * I;
        p.out = dxpad;
        p.ld_out = H;
        if (Is > 0) {
            moe::BwdProblem& q = P.p[np++];
            BW_TRY(mnmap(&q.ta, w13s, (size_t)2 * Is, H, "w13s"));
            BW_TRY(kB(q, dgus, T, 2 * Is, "shared dgate/dup"));
            q.a_mn = 1;
            q.n_grp = 1;
            q.n_rows = T;
            q.M = H;
            q.K = 2 * Is;
            q.out = dxsh;
            q.ld_out = H;
            q.out_f32 = 1;
        }
        moe::BwdProblem& r = P.p[np++];
        BW_TRY(mnmap(&r.ta, w_router, E, H, "w_router"));
        BW_TRY(kB(r, dl, T, ld_dl, "router dlogits"));
        r.a_mn = 1;
        r.n_grp = 1;
        r.n_rows = T;
        r.M = H;
        r.K = E;
        r.out = dxr;
        r.ld_out = H;
        r.out_f32 = 1;
        P.n_problems = np;
        BW_TRY(gemm(moe::BEPI_STORE, P, "input gradient GEMM launch"));
    }
    BW_TRY(mark(5));
    // 8. weight gradients: K = the expert's padded rows (or the T tokens)
    {
        moe::BwdParams P;
        memset(&P, 0, sizeof(P));
        int np = 0;
        moe::BwdProblem& p = P.p[np++];  // dW2_e[h][i] = sum_r dY[r][h] (w a)[r][i]
        BW_TRY(mnmap(&p.ta, aw, R, I, "padded w*a"));
        BW_TRY(mnmap(&p.tb, dypad, R, H, "padded dout"));
        p.a_mn = p.b_mn = 1;
        p.rows_as_k = 1;
        p.seg = pstart;
        p.n_grp = E;
        p.M = I;
        p.N = H;
        p.out = dw2;
        p.ld_out = I;
        p.out_grp = (long long)H * I;
        p.out_f32 = 1;
        moe::BwdProblem& q = P.p[np++];  // dW13_e[j][h] = sum_r dGU[r][j] X[r][h]
        BW_TRY(mnmap(&q.ta, xpad, R, H, "padded x"));
        BW_TRY(mnmap(&q.tb, dgu, R, 2 * I, "padded dgate/dup"));
        q.a_mn = q.b_mn = 1;
        q.rows_as_k = 1;
        q.seg = pstart;
        q.n_grp = E;
        q.M = H;
        q.N = 2 * I;
        q.out = dw13;
        q.ld_out = H;
        q.out_grp = (long long)2 * I * H;
        q.out_f32 = 1;
        if (Is > 0) {
            moe::BwdProblem& a2 = P.p[np++];  // dW2s[h][i]
            BW_TRY(mnmap(&a2.ta, as, T, Is, "shared a"));
            BW_TRY(mnmap(&a2.tb, dout, T, H, "dout"));
            a2.a_mn = a2.b_mn = 1;
            a2.rows_as_k = 1;
            a2.n_grp = 1;
            a2.n_rows = T;
            a2.M = Is;
            a2.N = H;
            a2.out = dw2s;
            a2.ld_out = Is;
            a2.out_f32 = 1;
            moe::BwdProblem& a3 = P.p[np++];  // dW13s[j][h]
            BW_TRY(mnmap(&a3.ta, x, T, H, "x"));
            BW_TRY(mnmap(&a3.tb, dgus, T, 2 * Is, "shared dgate/dup"));
            a3.a_mn = a3.b_mn = 1;
            a3.rows_as_k = 1;
            a3.n_grp = 1;
            a3.n_rows = T;
            a3.M = H;
            a3.N = 2 * Is;
            a3.out = dw13s;
            a3.ld_out = H;
            a3.out_f32 = 1;
        }
        moe::BwdProblem& g = P.p[np++];  // dW_g[e][h] = sum_t dL[t][e] x[t][h]
        BW_TRY(mnmap(&g.ta, x, T, H, "x"));
        BW_TRY(mnmap(&g.tb, dl, T, ld_dl, "router dlogits"));
        g.a_mn = g.b_mn = 1;
        g.rows_as_k = 1;
        g.n_grp = 1;
        g.n_rows = T;
        g.M = H;
        g.N = E;
        g.out = dw_router;
        g.ld_out = H;
        g.out_f32 = 1;
        P.n_problems = np;
        BW_TRY(gemm(moe::BEPI_STORE, P, "weight gradient GEMM launch"));
    }
    BW_TRY(mark(6));
    // 9. dx
    {
        BCombineArgs ca{dxpad, prow, Is > 0 ? dxsh : nullptr, dxr, static_cast<uint16_t*>(dx), T, k, H};
        const long long nthreads = (long long)T * (H / 8);
        bwd_combine_kernel<<<(unsigned)((nthreads + 255) / 256), 256, 0, s>>>(ca);
        BW_CUDA(cudaGetLastError(), "input gradient combine launch");
    }
    return mark(7);
}

}  // extern "C"
