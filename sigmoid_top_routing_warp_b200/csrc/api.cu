// api.cu -- the C ABI declared in include/moe.h: argument checks, workspace
// layout, TMA tensor maps and the launch sequence of the MoE FFN layer.
// The library never allocates device memory; every buffer is the caller's.
#include "moe.h"
#include "kernels.cuh"

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>

namespace {

thread_local char g_err[512] = "";

moe_status_t fail(moe_status_t st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return st;
}

moe_status_t cuda_fail(cudaError_t e, const char* what) {
    return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define MOE_CUDA(call, what)                            \
    do {                                                \
        cudaError_t e_ = (call);                        \
        if (e_ != cudaSuccess) return cuda_fail(e_, what); \
    } while (0)

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------ config
moe_status_t check_config(const moe_config_t* c) {
    if (!c) return fail(MOE_ERR_INVALID_ARG, "config is NULL");
    if (c->T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d must be >= 0", c->T);
    if (c->dtype != MOE_DTYPE_BF16 && c->dtype != MOE_DTYPE_FP8_E4M3_BLOCK128)
        return fail(MOE_ERR_UNSUPPORTED, "dtype %d not supported", c->dtype);
    if (c->H <= 0 || c->H % 128)
        return fail(MOE_ERR_UNSUPPORTED, "H=%d must be a positive multiple of 128", c->H);
    if (c->E < 32 || c->E > 1024 || c->E % 32)
        return fail(MOE_ERR_UNSUPPORTED, "E=%d must be a multiple of 32 in [32, 1024]", c->E);
    switch (c->E / 32) {
        case 1: case 2: case 3: case 4: case 5: case 6: case 8: case 10: case 12: case 16:
        case 24: case 32: break;
        default: return fail(MOE_ERR_UNSUPPORTED, "E=%d: E/32 must be one of 1-6,8,10,12,16,24,32", c->E);
    }
    if (c->flags & ~(uint32_t)MOE_FLAG_TEST_STALL)
        return fail(MOE_ERR_INVALID_ARG, "unknown flags 0x%x", c->flags);
    if (c->k < 1 || c->k > 32 || c->k > c->E)
        return fail(MOE_ERR_INVALID_ARG, "k=%d must be in [1, min(E, 32)]", c->k);
    if (c->I <= 0 || c->I % 128)
        return fail(MOE_ERR_UNSUPPORTED, "I=%d must be a positive multiple of 128", c->I);
    if (c->n_shared < 0 || (long long)c->n_shared * c->I > (1 << 20))
        return fail(MOE_ERR_INVALID_ARG, "n_shared=%d out of range", c->n_shared);
    const int G = c->n_group, tg = c->topk_group;
    if (G < 1 || G > 32 || c->E % G)
        return fail(MOE_ERR_INVALID_ARG, "n_group=%d must divide E and be in [1, 32]", G);
    if (tg < 1 || tg > G)
        return fail(MOE_ERR_INVALID_ARG, "topk_group=%d must be in [1, n_group]", tg);
    if (G > 1 && (c->group_topn < 1 || c->group_topn > c->E / G))
        return fail(MOE_ERR_INVALID_ARG, "group_topn=%d must be in [1, E/n_group]", c->group_topn);
    if (c->k > tg * (c->E / G))
        return fail(MOE_ERR_INVALID_ARG, "k=%d exceeds the experts of topk_group groups", c->k);
    if ((long long)c->T * c->k > (1ll << 30) / 8)
        return fail(MOE_ERR_UNSUPPORTED, "T*k=%lld too large", (long long)c->T * c->k);
    return MOE_OK;
}

// Token-tile width of the expert GEMMs: the MMA N operand.  Decode-sized
// batches (a few tokens per expert) use 16 on single CTAs; prefill-sized
// batches use 256-token tiles on CTA pairs.
int expert_bn(const moe_config_t* c) {
    const double avg = c->E ? (double)c->T * c->k / c->E : 0.0;
    return avg <= 24.0 ? 16 : avg <= 96.0 ? 64 : moe::kPairTokens;
}
inline bool is_fp8(const moe_config_t* c) { return c->dtype == MOE_DTYPE_FP8_E4M3_BLOCK128; }

// Token tile of the FP8 expert GEMMs (register accumulators: 16, 32 or 64
// tokens; 64-token tiles use eight epilogue warps).
// Token tile of the fp8 expert GEMMs: 16 / 32 / 64 rows for the weight-major
// kernel, or the token-major kernel's 128 when experts average more than 48
// rows and both contractions have K a multiple of 512.
// Token tile of the fp8 expert GEMMs.  The token-major kernel (128) wherever
// its shape rules hold: with 256 weight rows on the MMA's N side, each
// K-block partial handed to the promotion warps covers twice the weight
// bytes of a weight-major tile (128 weight rows on M), whatever the number of
// tokens per expert; at decode-sized batches that made the down GEMM ~27 %
// faster.  Otherwise weight-major tiles sized to the mean rows per expert.
int fp8_bn(const moe_config_t* c) {
    if (c->H % 512 == 0 && c->I % 512 == 0) return moe::kFp8TokTile;
    const double avg = c->E ? (double)c->T * c->k / c->E : 0.0;
    if (avg <= 24.0) return 16;
    if (avg <= 48.0) return 32;
    return 64;
}

int router_bn(const moe_config_t* c) { return c->T <= 16 ? 16 : c->T <= 64 ? 64 : 128; }

// K slices of the router GEMM: small batches have too few output tiles to
// keep the GPU busy, so the K loop is split (the selection kernel sums the
// slices in order).  The largest split of H/64 k-blocks into at most 16
// slices that keeps the tile count within 148 CTAs.
int router_split(const moe_config_t* c) {
    const int bn = router_bn(c);
    const int tiles = ((c->E + 127) / 128) * ((c->T + bn - 1) / bn);
    const int nk = c->H / 64;
    if (tiles >= 32) return 1;
    for (int s = 16; s > 1; --s)
        if (nk % s == 0 && tiles * s <= 148) return s;
    return 1;
}

struct Layout {
    size_t status, logits, rpart, idx, w, offsets, rows, pos, wperm, tokstart, chunk, xperm, a, ash,
        y, ysh, xq, sx, xpq, sxp, aq, sa, ashq, sash, toktiles, u, total;
};

Layout layout(const moe_config_t* c) {
    Layout L{};
    const size_t T = c->T, E = c->E, k = c->k, H = c->H, I = c->I, Is = (size_t)c->n_shared * c->I;
    const size_t n = T * k;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + bytes, 256);
        return at;
    };
    L.status = take(256);
    L.logits = take(T * E * 4);
    const int rs = router_split(c);
    L.rpart = take(rs > 1 ? (size_t)rs * T * E * 4 : 0);
    L.idx = take(n * 4);
    L.w = take(n * 4);
    L.offsets = take((E + 1) * 4);
    L.rows = take(n * 4);
    L.pos = take(n * 4);
    L.wperm = take(n * 4);
    L.tokstart = take((E + 1) * 4);
    L.toktiles = take((n / 16 + E + 1) * 16);  // token tiles of at least 16 rows
    L.chunk = take((size_t)moe::permute_chunks((int)n) * E * 4);
    L.xperm = take(n * H * 2);
    L.a = take(n * I * 2);
    L.ash = take(T * Is * 2);
    L.y = take(n * H * (c->k == 1 ? 4 : 2));  // routed outputs: fp32 when k = 1
    L.ysh = take(T * H * 4);
    const bool q = is_fp8(c);
    L.xq = take(q ? T * H : 0);
    L.sx = take(q ? T * (H / 128) * 4 : 0);
    L.xpq = take(q ? n * H : 0);
    L.sxp = take(q ? n * (H / 128) * 4 : 0);
    L.aq = take(q ? n * I : 0);
    L.sa = take(q ? n * (I / 128) * 4 : 0);
    L.ashq = take(q ? T * Is : 0);
    L.sash = take(q ? T * (Is / 128) * 4 : 0);
    L.u = take(T * H * 2);  // normalised block input (moe_forward_block)
    L.total = off;
    return L;
}

template <typename Tp>
Tp* at(void* ws, size_t off) {
    return reinterpret_cast<Tp*>(static_cast<char*>(ws) + off);
}

moe_status_t check_ws(const moe_config_t* c, void* ws, size_t ws_bytes) {
    if (!ws) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
    if (reinterpret_cast<uintptr_t>(ws) & 255u)
        return fail(MOE_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const size_t need = layout(c).total;
    if (ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
    return MOE_OK;
}

// ------------------------------------------------------------------ TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// bf16 row-major [rows, cols] as a 2-D tensor, box {64 columns, box_rows},
// 128-byte swizzle (the K-major layout the tensor-core descriptors expect).
moe_status_t make_map(CUtensorMap* m, const void* ptr, size_t rows, size_t cols, int box_rows,
                      const char* what) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    if (!aligned16(ptr)) return fail(MOE_ERR_INVALID_ARG, "%s must be 16-byte aligned", what);
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map for %s failed (%d)", what, (int)r);
    return MOE_OK;
}

// Packed gate/up matrix [n_exp][2 n_feat][K] (bf16) as the 5-D view
// {K, 8, 2, n_feat/8, n_exp}: a box {64, 8, 2, 8, 1} brings 64 features as
// alternating 8-row gate and up blocks (128 rows of 128 bytes, 128-byte swizzle).
moe_status_t make_map_gate_up_interleaved(CUtensorMap* m, const void* ptr, size_t n_exp,
                                          size_t n_feat, size_t K, const char* what) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    if (!aligned16(ptr)) return fail(MOE_ERR_INVALID_ARG, "%s must be 16-byte aligned", what);
    cuuint64_t dims[5] = {K, 8, 2, n_feat / 8, n_exp};
    cuuint64_t strides[4] = {K * 2, n_feat * K * 2, 8 * K * 2, 2 * n_feat * K * 2};
    cuuint32_t box[5] = {64, 8, 2, 8, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map for %s failed (%d)", what, (int)r);
    return MOE_OK;
}

moe_status_t sm_count(int* n) {
    int dev = 0;
    MOE_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    MOE_CUDA(cudaDeviceGetAttribute(n, cudaDevAttrMultiProcessorCount, dev), "SM count");
    return MOE_OK;
}

moe_status_t reset_claims(void* ws, cudaStream_t s) {
    MOE_CUDA(moe::reset_claim_counters(static_cast<int*>(ws), s), "claim-counter reset");
    return MOE_OK;
}

#define MOE_TRY(x)                          \
    do {                                    \
        moe_status_t st_ = (x);             \
        if (st_ != MOE_OK) return st_;      \
    } while (0)

// e4m3 codes (1 byte) row-major [rows, cols] as a 2-D tensor, box {128
// columns, box_rows}, 128-byte swizzle (K-major rows of 128 bytes).
moe_status_t make_map_u8(CUtensorMap* m, const void* ptr, size_t rows, size_t cols, int box_rows,
                         const char* what) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    if (!aligned16(ptr)) return fail(MOE_ERR_INVALID_ARG, "%s must be 16-byte aligned", what);
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map for %s failed (%d)", what, (int)r);
    return MOE_OK;
}

// fp32 block scales [rows][kbs] for the token-major fp8 kernel: box {4, box_rows}
// (the scales of four K blocks of box_rows rows); kbs must be a multiple of 4.
moe_status_t make_map_scales(CUtensorMap* m, const float* ptr, size_t rows, size_t kbs,
                             int box_rows, const char* what) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    if (!aligned16(ptr)) return fail(MOE_ERR_INVALID_ARG, "%s must be 16-byte aligned", what);
    cuuint64_t dims[2] = {kbs, rows};
    cuuint64_t strides[1] = {kbs * 4};
    cuuint32_t box[2] = {4, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map for %s failed (%d)", what, (int)r);
    return MOE_OK;
}

// The token boxes of the CTA-pair kernels: 16, 32, 64 and 128 rows.
moe_status_t make_pair_boxes(CUtensorMap* maps, const void* ptr, size_t rows, size_t cols,
                             const char* what) {
    for (int b = 0; b < moe::kPairBoxes; ++b) MOE_TRY(make_map(&maps[b], ptr, rows, cols, 16 << b, what));
    return MOE_OK;
}

// ------------------------------------------------------------------ stages
moe_status_t run_router_gemm(const moe_config_t* c, const void* x, const void* wg, float* logits,
                             int* status, cudaStream_t s) {
    const int split = router_split(c);
    moe::GemmParams P;
    memset(&P, 0, sizeof(P));
    const int bn = router_bn(c);
    moe::GemmProblem& p = P.p[0];
    MOE_TRY(make_map(&p.tw, wg, c->E, c->H, 128, "w_router"));
    MOE_TRY(make_map(&p.tx, x, c->T, c->H, bn, "x"));
    p.seg = nullptr;
    p.tok_start = nullptr;
    p.n_exp = 1;
    p.n_rows = c->T;
    p.K = c->H;
    p.n_feat = c->E;
    p.w_rows = c->E;
    p.out = logits;
    p.ld_out = c->E;
    p.row_w = nullptr;
    p.k_split = split;
    p.split_stride = (long long)c->T * c->E;
    P.n_problems = 1;
    P.status = status;
    P.test_stall = (c->flags & MOE_FLAG_TEST_STALL) ? 1 : 0;
    int sms = 0;
    MOE_TRY(sm_count(&sms));
    const int tiles = ((c->E + 127) / 128) * ((c->T + bn - 1) / bn) * split;
    const int grid = tiles < sms ? tiles : sms;
    MOE_CUDA(moe::launch_grouped_gemm(moe::EPI_F32, bn, P, grid, s), "router GEMM launch");
    return MOE_OK;
}

moe_status_t run_select(const moe_config_t* c, const float* logits, const float* bias,
                        int32_t* idx, float* w, cudaStream_t s, int n_split = 1,
                        float* logits_out = nullptr) {
    moe::RouteArgs a;
    a.logits = logits;
    a.n_split = n_split;
    a.logits_out = logits_out;
    a.bias = bias;
    a.idx = idx;
    a.w = w;
    a.T = c->T;
    a.E = c->E;
    a.k = c->k;
    a.n_group = c->n_group;
    a.topk_group = c->topk_group;
    a.group_topn = c->group_topn;
    a.norm = c->norm_topk_prob != 0;
    a.rsf = c->routed_scaling_factor;
    MOE_CUDA(moe::launch_route_select(a, s), "router selection launch");
    return MOE_OK;
}

moe_status_t run_permute(const moe_config_t* c, const int32_t* idx, int32_t* offsets,
                         int32_t* rows, int32_t* pos, void* ws, cudaStream_t s) {
    moe::PermuteArgs a;
    a.idx = idx;
    a.offsets = offsets;
    a.rows = rows;
    a.pos = pos;
    a.chunk_base = at<int32_t>(ws, layout(c).chunk);
    a.T = c->T;
    a.k = c->k;
    a.E = c->E;
    MOE_CUDA(moe::launch_permute(a, s), "permute launch");
    return MOE_OK;
}

struct Weights {
    const void *w13, *w2, *w13s, *w2s;
    const float *s13, *s2, *s13s, *s2s;  // fp8 block scales (null for bf16)
};

// FP8 layer: a0 quantisation of x, gather of codes and scales, then both
// expert GEMMs on e4m3 operands with scale promotion (gemm_fp8.cu).
// One fp8 expert GEMM launch: the weight-major kernel, or (bn = 128) the
// token-major kernel with its scale tensor maps (problem 0 has `rows0`
// activation rows, problem 1 `rows1`).
moe_status_t launch_fp8(int epi, int bn, moe::GemmParams& P, int rows0, int rows1, int sms,
                        cudaStream_t s, const char* what) {
    if (bn == moe::kFp8TokTile) {
        for (int pi = 0; pi < P.n_problems; ++pi) {
            moe::GemmProblem& p = P.p[pi];
            const size_t kbs = (size_t)p.K / 128;
            MOE_TRY(make_map_scales(&p.tsx, p.x_scale, pi == 0 ? rows0 : rows1, kbs,
                                    moe::kFp8TokTile, "activation scales"));
            MOE_TRY(make_map_scales(&p.tsw, p.w_scale, (size_t)p.n_exp * p.w_rows / 128, kbs, 1,
                                    "weight scales"));
        }
        MOE_CUDA(moe::launch_fp8_tm_gemm(epi, P, sms, s), what);
        return MOE_OK;
    }
    MOE_CUDA(moe::launch_fp8_gemm(epi, bn, P, sms, s), what);
    return MOE_OK;
}

moe_status_t run_expert_ffn_fp8(const moe_config_t* c, const void* x, const int32_t* offsets,
                                const int32_t* pos, const float* topk_w, const Weights& W,
                                void* y, void* y_shared, void* ws, cudaStream_t s,
                                cudaEvent_t ev_mid, cudaEvent_t ev_gemm2) {
    const Layout L = layout(c);
    const int bn = fp8_bn(c);
    const int n = c->T * c->k;
    const int Is = c->n_shared * c->I;
    moe::QuantArgs qa;
    qa.x = static_cast<const uint16_t*>(x);
    qa.q = at<uint8_t>(ws, L.xq);
    qa.scale = at<float>(ws, L.sx);
    qa.rows = c->T;
    qa.cols = c->H;
    MOE_CUDA(moe::launch_quant_act(qa, s), "activation quantisation launch");
    moe::GatherQArgs g;
    g.xq = qa.q;
    g.sx = qa.scale;
    g.pos = pos;
    g.topk_w = topk_w;
    g.offsets = offsets;
    g.xq_perm = at<uint8_t>(ws, L.xpq);
    g.sx_perm = at<float>(ws, L.sxp);
    g.w_perm = at<float>(ws, L.wperm);
    g.tok_start = at<int32_t>(ws, L.tokstart);
    g.T = c->T;
    g.k = c->k;
    g.H = c->H;
    g.E = c->E;
    g.bn = bn;
    MOE_CUDA(moe::launch_gather_q(g, s), "fp8 gather launch");
    if (ev_mid) MOE_CUDA(cudaEventRecord(ev_mid, s), "event record");
    int sms = 0;
    MOE_TRY(sm_count(&sms));
    int* status = at<int>(ws, L.status);

    moe::GemmParams P1;
    memset(&P1, 0, sizeof(P1));
    {
        moe::GemmProblem& p = P1.p[0];
        MOE_TRY(make_map_u8(&p.tw, W.w13, (size_t)c->E * 2 * c->I, c->H, 128, "w13"));
        MOE_TRY(make_map_u8(&p.tx, g.xq_perm, n, c->H, bn, "gathered x codes"));
        p.seg = offsets;
        p.tok_start = g.tok_start;
        p.n_exp = c->E;
        p.K = c->H;
        p.n_feat = c->I;
        p.w_rows = 2 * c->I;
        p.ld_out = c->I;
        p.w_scale = W.s13;
        p.x_scale = g.sx_perm;
        p.out_q = at<uint8_t>(ws, L.aq);
        p.out_scale = at<float>(ws, L.sa);
        P1.n_problems = 1;
        if (Is > 0) {
            moe::GemmProblem& q = P1.p[1];
            MOE_TRY(make_map_u8(&q.tw, W.w13s, (size_t)2 * Is, c->H, 128, "w13s"));
            MOE_TRY(make_map_u8(&q.tx, qa.q, c->T, c->H, bn, "x codes"));
            q.n_exp = 1;
            q.n_rows = c->T;
            q.K = c->H;
            q.n_feat = Is;
            q.w_rows = 2 * Is;
            q.ld_out = Is;
            q.w_scale = W.s13s;
            q.x_scale = qa.scale;
            q.out_q = at<uint8_t>(ws, L.ashq);
            q.out_scale = at<float>(ws, L.sash);
            P1.n_problems = 2;
        }
        P1.status = status;
    }
    MOE_TRY(launch_fp8(moe::EPI_SWIGLU, bn, P1, n, c->T, sms, s, "fp8 gate/up GEMM launch"));
    if (ev_gemm2) MOE_CUDA(cudaEventRecord(ev_gemm2, s), "event record");

    moe::GemmParams P2;
    memset(&P2, 0, sizeof(P2));
    {
        moe::GemmProblem& p = P2.p[0];
        MOE_TRY(make_map_u8(&p.tw, W.w2, (size_t)c->E * c->H, c->I, 128, "w2"));
        MOE_TRY(make_map_u8(&p.tx, at<void>(ws, L.aq), n, c->I, bn, "expert activation codes"));
        p.seg = offsets;
        p.tok_start = g.tok_start;
        p.n_exp = c->E;
        p.K = c->I;
        p.n_feat = c->H;
        p.w_rows = c->H;
        p.out = y;
        p.ld_out = c->H;
        p.row_w = g.w_perm;
        p.out_f32 = c->k == 1;
        p.w_scale = W.s2;
        p.x_scale = at<float>(ws, L.sa);
        P2.n_problems = 1;
        if (Is > 0) {
            moe::GemmProblem& q = P2.p[1];
            MOE_TRY(make_map_u8(&q.tw, W.w2s, c->H, Is, 128, "w2s"));
            MOE_TRY(make_map_u8(&q.tx, at<void>(ws, L.ashq), c->T, Is, bn, "shared activation codes"));
            q.n_exp = 1;
            q.n_rows = c->T;
            q.K = Is;
            q.n_feat = c->H;
            q.w_rows = c->H;
            q.out = y_shared;
            q.ld_out = c->H;
            q.out_f32 = 1;
            q.w_scale = W.s2s;
            q.x_scale = at<float>(ws, L.sash);
            P2.n_problems = 2;
        }
        P2.status = status;
    }
    MOE_TRY(launch_fp8(moe::EPI_SCALE, bn, P2, n, c->T, sms, s, "fp8 down GEMM launch"));
    return MOE_OK;
}

// Prefill-sized batches: both expert GEMMs on CTA pairs (256 x 256 tiles).
moe_status_t run_expert_ffn_pairs(const moe_config_t* c, const void* x, const int32_t* offsets,
                                  const Weights& W, void* y, void* y_shared, void* ws,
                                  cudaStream_t s, cudaEvent_t ev_gemm2, const moe::GatherArgs& g,
                                  int sms, int* status) {
    const Layout L = layout(c);
    const int n = c->T * c->k;
    const int Is = c->n_shared * c->I;
    moe::PairParams P1;
    memset(&P1, 0, sizeof(P1));
    {
        moe::PairProblem& p = P1.p[0];
        MOE_TRY(make_map_gate_up_interleaved(&p.tw, W.w13, c->E, c->I, c->H, "w13"));
        MOE_TRY(make_pair_boxes(p.tx, g.x_perm, n, c->H, "gathered x"));
        p.seg = offsets;
        p.tok_start = g.tok_start;
        p.tok_tiles = g.tok_tiles;
        p.n_exp = c->E;
        p.K = c->H;
        p.n_feat = c->I;
        p.out = at<void>(ws, L.a);
        p.ld_out = c->I;
        P1.n_problems = 1;
        if (Is > 0) {
            moe::PairProblem& q = P1.p[1];
            MOE_TRY(make_map_gate_up_interleaved(&q.tw, W.w13s, 1, Is, c->H, "w13s"));
            MOE_TRY(make_pair_boxes(q.tx, x, c->T, c->H, "x"));
            q.n_exp = 1;
            q.n_rows = c->T;
            q.K = c->H;
            q.n_feat = Is;
            q.out = at<void>(ws, L.ash);
            q.ld_out = Is;
            P1.n_problems = 2;
        }
        P1.status = status;
    }
    MOE_CUDA(moe::launch_pair_gemm(moe::EPI_SWIGLU, P1, sms, s), "gate/up pair GEMM launch");
    if (ev_gemm2) MOE_CUDA(cudaEventRecord(ev_gemm2, s), "event record");

    moe::PairParams P2;
    memset(&P2, 0, sizeof(P2));
    {
        moe::PairProblem& p = P2.p[0];
        MOE_TRY(make_map(&p.tw, W.w2, (size_t)c->E * c->H, c->I, 128, "w2"));
        MOE_TRY(make_pair_boxes(p.tx, at<void>(ws, L.a), n, c->I, "expert activations"));
        p.seg = offsets;
        p.tok_start = g.tok_start;
        p.tok_tiles = g.tok_tiles;
        p.n_exp = c->E;
        p.K = c->I;
        p.n_feat = c->H;
        p.out = y;
        p.ld_out = c->H;
        p.row_w = g.w_perm;
        p.out_f32 = c->k == 1;
        P2.n_problems = 1;
        if (Is > 0) {
            moe::PairProblem& q = P2.p[1];
            MOE_TRY(make_map(&q.tw, W.w2s, c->H, Is, 128, "w2s"));
            MOE_TRY(make_pair_boxes(q.tx, at<void>(ws, L.ash), c->T, Is, "shared activations"));
            q.n_exp = 1;
            q.n_rows = c->T;
            q.K = Is;
            q.n_feat = c->H;
            q.out = y_shared;
            q.ld_out = c->H;
            q.out_f32 = 1;
            P2.n_problems = 2;
        }
        P2.status = status;
    }
    MOE_CUDA(moe::launch_pair_gemm(moe::EPI_SCALE, P2, sms, s), "down pair GEMM launch");
    return MOE_OK;
}

moe_status_t run_expert_ffn(const moe_config_t* c, const void* x, const int32_t* offsets,
                            const int32_t* pos, const float* topk_w, const Weights& W, void* y,
                            void* y_shared, void* ws, cudaStream_t s, cudaEvent_t ev_mid,
                            cudaEvent_t ev_gemm2) {
    if (is_fp8(c))
        return run_expert_ffn_fp8(c, x, offsets, pos, topk_w, W, y, y_shared, ws, s, ev_mid, ev_gemm2);
    const Layout L = layout(c);
    const int bn = expert_bn(c);
    const int n = c->T * c->k;
    const int Is = c->n_shared * c->I;

    moe::GatherArgs g;
    g.x = static_cast<const uint16_t*>(x);
    g.pos = pos;
    g.topk_w = topk_w;
    g.offsets = offsets;
    g.x_perm = at<uint16_t>(ws, L.xperm);
    g.w_perm = at<float>(ws, L.wperm);
    g.tok_start = at<int32_t>(ws, L.tokstart);
    g.tok_tiles = at<int4>(ws, L.toktiles);
    g.T = c->T;
    g.k = c->k;
    g.H = c->H;
    g.E = c->E;
    g.bn = bn;
    MOE_CUDA(moe::launch_gather(g, s), "gather launch");
    if (ev_mid) MOE_CUDA(cudaEventRecord(ev_mid, s), "event record");

    int sms = 0;
    MOE_TRY(sm_count(&sms));
    int* status = at<int>(ws, L.status);
    if (bn == moe::kPairTokens)
        return run_expert_ffn_pairs(c, x, offsets, W, y, y_shared, ws, s, ev_gemm2, g, sms,
                                    status);

    // gate/up GEMM + SwiGLU: routed experts, then the shared expert
    moe::GemmParams P1;
    memset(&P1, 0, sizeof(P1));
    {
        moe::GemmProblem& p = P1.p[0];
        MOE_TRY(make_map(&p.tw, W.w13, (size_t)c->E * 2 * c->I, c->H, 128, "w13"));
        MOE_TRY(make_map(&p.tx, g.x_perm, n, c->H, bn, "gathered x"));
        p.seg = offsets;
        p.tok_start = g.tok_start;
        p.n_exp = c->E;
        p.K = c->H;
        p.n_feat = c->I;
        p.w_rows = 2 * c->I;
        p.out = at<void>(ws, L.a);
        p.ld_out = c->I;
        P1.n_problems = 1;
        if (Is > 0) {
            moe::GemmProblem& q = P1.p[1];
            MOE_TRY(make_map(&q.tw, W.w13s, (size_t)2 * Is, c->H, 128, "w13s"));
            MOE_TRY(make_map(&q.tx, x, c->T, c->H, bn, "x"));
            q.seg = nullptr;
            q.tok_start = nullptr;
            q.n_exp = 1;
            q.n_rows = c->T;
            q.K = c->H;
            q.n_feat = Is;
            q.w_rows = 2 * Is;
            q.out = at<void>(ws, L.ash);
            q.ld_out = Is;
            P1.n_problems = 2;
        }
        P1.status = status;
    }
    MOE_CUDA(moe::launch_grouped_gemm(moe::EPI_SWIGLU, bn, P1, sms, s), "gate/up GEMM launch");
    if (ev_gemm2) MOE_CUDA(cudaEventRecord(ev_gemm2, s), "event record");

    // down GEMM x routing weight: routed experts, then the shared expert
    moe::GemmParams P2;
    memset(&P2, 0, sizeof(P2));
    {
        moe::GemmProblem& p = P2.p[0];
        MOE_TRY(make_map(&p.tw, W.w2, (size_t)c->E * c->H, c->I, 128, "w2"));
        MOE_TRY(make_map(&p.tx, at<void>(ws, L.a), n, c->I, bn, "expert activations"));
        p.seg = offsets;
        p.tok_start = g.tok_start;
        p.n_exp = c->E;
        p.K = c->I;
        p.n_feat = c->H;
        p.w_rows = c->H;
        p.out = y;
        p.ld_out = c->H;
        p.row_w = g.w_perm;
        p.out_f32 = c->k == 1;
        P2.n_problems = 1;
        if (Is > 0) {
            moe::GemmProblem& q = P2.p[1];
            MOE_TRY(make_map(&q.tw, W.w2s, c->H, Is, 128, "w2s"));
            MOE_TRY(make_map(&q.tx, at<void>(ws, L.ash), c->T, Is, bn, "shared activations"));
            q.seg = nullptr;
            q.tok_start = nullptr;
            q.n_exp = 1;
            q.n_rows = c->T;
            q.K = Is;
            q.n_feat = c->H;
            q.w_rows = c->H;
            q.out = y_shared;
            q.ld_out = c->H;
            q.row_w = nullptr;
            q.out_f32 = 1;
            P2.n_problems = 2;
        }
        P2.status = status;
    }
    MOE_CUDA(moe::launch_grouped_gemm(moe::EPI_SCALE, bn, P2, sms, s), "down GEMM launch");
    return MOE_OK;
}

// The shared expert alone (bf16): y_shared = SwiGLU_shared(x) in fp32, on CTA
// pairs for prefill-sized batches, single CTAs otherwise.
moe_status_t run_shared_only(const moe_config_t* c, const void* x, const void* w13s,
                             const void* w2s, float* y_shared, void* ws, cudaStream_t s) {
    const Layout L = layout(c);
    const int Is = c->n_shared * c->I;
    int sms = 0;
    MOE_TRY(sm_count(&sms));
    int* status = at<int>(ws, L.status);
    void* ash = at<void>(ws, L.ash);
    if (c->T >= 512) {
        moe::PairParams P1;
        memset(&P1, 0, sizeof(P1));
        moe::PairProblem& q = P1.p[0];
        MOE_TRY(make_map_gate_up_interleaved(&q.tw, w13s, 1, Is, c->H, "w13s"));
        MOE_TRY(make_pair_boxes(q.tx, x, c->T, c->H, "x"));
        q.n_exp = 1;
        q.n_rows = c->T;
        q.K = c->H;
        q.n_feat = Is;
        q.out = ash;
        q.ld_out = Is;
        P1.n_problems = 1;
        P1.status = status;
        MOE_CUDA(moe::launch_pair_gemm(moe::EPI_SWIGLU, P1, sms, s), "shared gate/up launch");
        moe::PairParams P2;
        memset(&P2, 0, sizeof(P2));
        moe::PairProblem& r = P2.p[0];
        MOE_TRY(make_map(&r.tw, w2s, c->H, Is, 128, "w2s"));
        MOE_TRY(make_pair_boxes(r.tx, ash, c->T, Is, "shared activations"));
        r.n_exp = 1;
        r.n_rows = c->T;
        r.K = Is;
        r.n_feat = c->H;
        r.out = y_shared;
        r.ld_out = c->H;
        r.out_f32 = 1;
        P2.n_problems = 1;
        P2.status = status;
        MOE_CUDA(moe::launch_pair_gemm(moe::EPI_SCALE, P2, sms, s), "shared down launch");
        return MOE_OK;
    }
    const int bn = c->T <= 16 ? 16 : c->T <= 64 ? 64 : 128;
    moe::GemmParams P1;
    memset(&P1, 0, sizeof(P1));
    moe::GemmProblem& q = P1.p[0];
    MOE_TRY(make_map(&q.tw, w13s, (size_t)2 * Is, c->H, 128, "w13s"));
    MOE_TRY(make_map(&q.tx, x, c->T, c->H, bn, "x"));
    q.n_exp = 1;
    q.n_rows = c->T;
    q.K = c->H;
    q.n_feat = Is;
    q.w_rows = 2 * Is;
    q.out = ash;
    q.ld_out = Is;
    P1.n_problems = 1;
    P1.status = status;
    MOE_CUDA(moe::launch_grouped_gemm(moe::EPI_SWIGLU, bn, P1, sms, s), "shared gate/up launch");
    moe::GemmParams P2;
    memset(&P2, 0, sizeof(P2));
    moe::GemmProblem& r = P2.p[0];
    MOE_TRY(make_map(&r.tw, w2s, c->H, Is, 128, "w2s"));
    MOE_TRY(make_map(&r.tx, ash, c->T, Is, bn, "shared activations"));
    r.n_exp = 1;
    r.n_rows = c->T;
    r.K = Is;
    r.n_feat = c->H;
    r.w_rows = c->H;
    r.out = y_shared;
    r.ld_out = c->H;
    r.out_f32 = 1;
    P2.n_problems = 1;
    P2.status = status;
    MOE_CUDA(moe::launch_grouped_gemm(moe::EPI_SCALE, bn, P2, sms, s), "shared down launch");
    return MOE_OK;
}

moe_status_t check_eps(float eps) {
    if (!(eps >= 0.0f) || !(eps < 1e30f))
        return fail(MOE_ERR_INVALID_ARG, "eps must be finite and >= 0 (got %g)", (double)eps);
    return MOE_OK;
}

moe_status_t run_rmsnorm(const moe_config_t* c, const void* h, const void* gamma, float eps,
                         void* u, cudaStream_t s) {
    moe::NormArgs a;
    a.h = static_cast<const uint16_t*>(h);
    a.gamma = static_cast<const uint16_t*>(gamma);
    a.u = static_cast<uint16_t*>(u);
    a.T = c->T;
    a.H = c->H;
    a.eps = eps;
    MOE_CUDA(moe::launch_rmsnorm(a, s), "rmsnorm launch");
    return MOE_OK;
}

moe_status_t run_combine(const moe_config_t* c, const void* y, const int32_t* pos,
                         const void* y_shared, void* out, cudaStream_t s,
                         const void* residual = nullptr) {
    moe::CombineArgs a;
    a.y = y;
    a.y_f32 = c->k == 1;
    a.pos = pos;
    a.y_shared = static_cast<const float*>(y_shared);
    a.residual = static_cast<const uint16_t*>(residual);
    a.out = static_cast<uint16_t*>(out);
    a.T = c->T;
    a.k = c->k;
    a.H = c->H;
    MOE_CUDA(moe::launch_combine(a, s), "combine launch");
    return MOE_OK;
}

moe_status_t need(const void* p, const char* name) {
    return p ? MOE_OK : fail(MOE_ERR_INVALID_ARG, "%s is NULL", name);
}

moe_status_t need16(const void* p, const char* name) {
    MOE_TRY(need(p, name));
    return aligned16(p) ? MOE_OK : fail(MOE_ERR_INVALID_ARG, "%s must be 16-byte aligned", name);
}

moe_status_t check_scales(const moe_config_t* cfg, const float* a, const float* b, const float* c2,
                          const float* d) {
    if (!is_fp8(cfg)) {
        if (a || b || c2 || d)
            return fail(MOE_ERR_INVALID_ARG, "weight scales must be NULL for bf16 weights");
        return MOE_OK;
    }
    if (!a || !b) return fail(MOE_ERR_INVALID_ARG, "fp8 weights need w13_scale and w2_scale");
    if (cfg->n_shared > 0 && (!c2 || !d))
        return fail(MOE_ERR_INVALID_ARG, "fp8 shared weights need w13s_scale and w2s_scale");
    return MOE_OK;
}

}  // namespace

// ====================================================================== ABI
extern "C" {

const char* moe_get_last_error(void) { return g_err; }

size_t moe_workspace_size(const moe_config_t* cfg) {
    if (check_config(cfg) != MOE_OK) return 0;
    return layout(cfg).total;
}

size_t moe_workspace_offset(const moe_config_t* cfg, int32_t which) {
    if (check_config(cfg) != MOE_OK) return (size_t)-1;
    const Layout L = layout(cfg);
    switch (which) {
        case 0: return L.logits;
        case 1: return L.idx;
        case 2: return L.w;
        case 3: return L.offsets;
        case 4: return L.rows;
        case 5: return L.pos;
        case 6: return L.y;
        case 7: return L.ysh;
        case 8: return L.u;
        default: fail(MOE_ERR_INVALID_ARG, "unknown workspace item %d", which); return (size_t)-1;
    }
}

moe_status_t moe_route(const moe_config_t* cfg, const void* x, const void* w_router,
                       const float* bias, float* logits, int32_t* topk_idx, float* topk_w,
                       void* ws, size_t ws_bytes, moe_stream_t stream) {
    g_err[0] = 0;
    MOE_TRY(check_config(cfg));
    MOE_TRY(check_ws(cfg, ws, ws_bytes));
    MOE_TRY(need16(x, "x"));
    MOE_TRY(need16(w_router, "w_router"));
    MOE_TRY(need(bias, "bias"));
    MOE_TRY(need(logits, "logits"));
    MOE_TRY(need(topk_idx, "topk_idx"));
    MOE_TRY(need(topk_w, "topk_w"));
    if (cfg->T == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    MOE_TRY(reset_claims(ws, s));
    const Layout L = layout(cfg);
    const int split = router_split(cfg);
    float* gemm_out = split > 1 ? at<float>(ws, L.rpart) : logits;
    MOE_TRY(run_router_gemm(cfg, x, w_router, gemm_out, at<int>(ws, L.status), s));
    return run_select(cfg, gemm_out, bias, topk_idx, topk_w, s, split, logits);
}

moe_status_t moe_route_from_logits(const moe_config_t* cfg, const float* logits,
                                   const float* bias, int32_t* topk_idx, float* topk_w,
                                   moe_stream_t stream) {
    g_err[0] = 0;
    MOE_TRY(check_config(cfg));
    MOE_TRY(need(logits, "logits"));
    MOE_TRY(need(bias, "bias"));
    MOE_TRY(need(topk_idx, "topk_idx"));
    MOE_TRY(need(topk_w, "topk_w"));
    if (cfg->T == 0) return MOE_OK;
    return run_select(cfg, logits, bias, topk_idx, topk_w, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_permute(const moe_config_t* cfg, const int32_t* topk_idx, int32_t* offsets,
                         int32_t* rows, int32_t* pos, void* ws, size_t ws_bytes,
                         moe_stream_t stream) {
    g_err[0] = 0;
    MOE_TRY(check_config(cfg));
    MOE_TRY(check_ws(cfg, ws, ws_bytes));
    MOE_TRY(need(topk_idx, "topk_idx"));
    MOE_TRY(need(offsets, "offsets"));
    MOE_TRY(need(rows, "rows"));
    MOE_TRY(need(pos, "pos"));
    return run_permute(cfg, topk_idx, offsets, rows, pos, ws, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_expert_ffn(const moe_config_t* cfg, const void* x, const int32_t* offsets,
                            const int32_t* rows, const int32_t* pos, const float* topk_w,
                            const void* w13, const float* w13_scale, const void* w2,
                            const float* w2_scale, const void* w13s, const float* w13s_scale,
                            const void* w2s, const float* w2s_scale, void* y, void* y_shared,
                            void* ws, size_t ws_bytes, moe_stream_t stream) {
    g_err[0] = 0;
    MOE_TRY(check_config(cfg));
    MOE_TRY(check_ws(cfg, ws, ws_bytes));
    MOE_TRY(check_scales(cfg, w13_scale, w2_scale, w13s_scale, w2s_scale));
    MOE_TRY(need16(x, "x"));
    MOE_TRY(need(offsets, "offsets"));
    MOE_TRY(need(rows, "rows"));
    MOE_TRY(need(pos, "pos"));
    MOE_TRY(need(topk_w, "topk_w"));
    MOE_TRY(need16(w13, "w13"));
    MOE_TRY(need16(w2, "w2"));
    MOE_TRY(need16(y, "y"));
    if (cfg->n_shared > 0) {
        MOE_TRY(need16(w13s, "w13s"));
        MOE_TRY(need16(w2s, "w2s"));
        MOE_TRY(need16(y_shared, "y_shared"));
    }
    if (cfg->T == 0) return MOE_OK;
    MOE_TRY(reset_claims(ws, static_cast<cudaStream_t>(stream)));
    Weights W{w13, w2, w13s, w2s, w13_scale, w2_scale, w13s_scale, w2s_scale};
    return run_expert_ffn(cfg, x, offsets, pos, topk_w, W, y, y_shared, ws,
                          static_cast<cudaStream_t>(stream), nullptr, nullptr);
}

moe_status_t moe_shared_expert(const moe_config_t* cfg, const void* x, const void* w13s,
                               const void* w2s, float* y_shared, void* ws, size_t ws_bytes,
                               moe_stream_t stream) {
    g_err[0] = 0;
    MOE_TRY(check_config(cfg));
    if (is_fp8(cfg)) return fail(MOE_ERR_UNSUPPORTED, "moe_shared_expert: bf16 layers only");
    if (cfg->n_shared < 1) return fail(MOE_ERR_INVALID_ARG, "moe_shared_expert: n_shared is 0");
    MOE_TRY(check_ws(cfg, ws, ws_bytes));
    MOE_TRY(need16(x, "x"));
    MOE_TRY(need16(w13s, "w13s"));
    MOE_TRY(need16(w2s, "w2s"));
    MOE_TRY(need16(y_shared, "y_shared"));
    if (cfg->T == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    MOE_TRY(reset_claims(ws, s));
    return run_shared_only(cfg, x, w13s, w2s, y_shared, ws, s);
}

moe_status_t moe_combine(const moe_config_t* cfg, const void* y, const int32_t* pos,
                         const void* y_shared, void* out, moe_stream_t stream) {
    g_err[0] = 0;
    MOE_TRY(check_config(cfg));
    MOE_TRY(need16(y, "y"));
    MOE_TRY(need(pos, "pos"));
    MOE_TRY(need16(out, "out"));
    if (y_shared && !aligned16(y_shared))
        return fail(MOE_ERR_INVALID_ARG, "y_shared must be 16-byte aligned");
    if (cfg->T == 0) return MOE_OK;
    return run_combine(cfg, y, pos, y_shared, out, static_cast<cudaStream_t>(stream));
}

// The layer (steps a1-a9) on one stream.  With gamma: the pre-norm block,
// x is the residual stream h, the layer runs on u = RMSNorm(h) (kept in the
// workspace) and the combine adds h.
moe_status_t forward_impl(const moe_config_t* cfg, const void* x, const void* gamma, float eps,
                          const void* w_router, const float* bias, const void* w13,
                          const float* w13_scale, const void* w2, const float* w2_scale,
                          const void* w13s, const float* w13s_scale, const void* w2s,
                          const float* w2s_scale, void* out, void* ws, size_t ws_bytes,
                          void* const* stage_events, moe_stream_t stream) {
    MOE_TRY(check_config(cfg));
    MOE_TRY(check_ws(cfg, ws, ws_bytes));
    MOE_TRY(check_scales(cfg, w13_scale, w2_scale, w13s_scale, w2s_scale));
    MOE_TRY(need16(x, gamma ? "h" : "x"));
    MOE_TRY(need16(w_router, "w_router"));
    MOE_TRY(need(bias, "bias"));
    MOE_TRY(need16(w13, "w13"));
    MOE_TRY(need16(w2, "w2"));
    MOE_TRY(need16(out, "out"));
    if (cfg->n_shared > 0) {
        MOE_TRY(need16(w13s, "w13s"));
        MOE_TRY(need16(w2s, "w2s"));
    }
    if (gamma) {
        MOE_TRY(need16(gamma, "gamma"));
        MOE_TRY(check_eps(eps));
    }
    if (cfg->T == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaEvent_t ev[MOE_NUM_STAGES + 1] = {};
    if (stage_events)
        for (int i = 0; i <= MOE_NUM_STAGES; ++i) ev[i] = static_cast<cudaEvent_t>(stage_events[i]);
    auto mark = [&](int i) -> moe_status_t {
        if (ev[i]) MOE_CUDA(cudaEventRecord(ev[i], s), "event record");
        return MOE_OK;
    };
    const Layout L = layout(cfg);
    float* logits = at<float>(ws, L.logits);
    int32_t* idx = at<int32_t>(ws, L.idx);
    float* w = at<float>(ws, L.w);
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* pos = at<int32_t>(ws, L.pos);
    void* y = at<void>(ws, L.y);
    void* ysh = cfg->n_shared > 0 ? at<void>(ws, L.ysh) : nullptr;

    const int split = router_split(cfg);
    float* gemm_out = split > 1 ? at<float>(ws, L.rpart) : logits;
    MOE_TRY(mark(0));
    MOE_TRY(reset_claims(ws, s));
    const void* xin = x;
    if (gamma) {
        void* u = at<void>(ws, L.u);
        MOE_TRY(run_rmsnorm(cfg, x, gamma, eps, u, s));
        xin = u;
    }
    MOE_TRY(run_router_gemm(cfg, xin, w_router, gemm_out, at<int>(ws, L.status), s));
    MOE_TRY(mark(1));
    MOE_TRY(run_select(cfg, gemm_out, bias, idx, w, s, split, logits));
    MOE_TRY(mark(2));
    MOE_TRY(run_permute(cfg, idx, offsets, at<int32_t>(ws, L.rows), pos, ws, s));
    Weights W{w13, w2, w13s, w2s, w13_scale, w2_scale, w13s_scale, w2s_scale};
    MOE_TRY(run_expert_ffn(cfg, xin, offsets, pos, w, W, y, ysh, ws, s, ev[3], ev[4]));
    MOE_TRY(mark(5));
    MOE_TRY(run_combine(cfg, y, pos, ysh, out, s, gamma ? x : nullptr));
    return mark(6);
}

moe_status_t moe_forward(const moe_config_t* cfg, const void* x, const void* w_router,
                         const float* bias, const void* w13, const float* w13_scale,
                         const void* w2, const float* w2_scale, const void* w13s,
                         const float* w13s_scale, const void* w2s, const float* w2s_scale,
                         void* out, void* ws, size_t ws_bytes, void* const* stage_events,
                         moe_stream_t stream) {
    g_err[0] = 0;
    return forward_impl(cfg, x, nullptr, 0.0f, w_router, bias, w13, w13_scale, w2, w2_scale, w13s,
                        w13s_scale, w2s, w2s_scale, out, ws, ws_bytes, stage_events, stream);
}

moe_status_t moe_forward_block(const moe_config_t* cfg, const void* h, const void* gamma,
                               float eps, const void* w_router, const float* bias,
                               const void* w13, const float* w13_scale, const void* w2,
                               const float* w2_scale, const void* w13s, const float* w13s_scale,
                               const void* w2s, const float* w2s_scale, void* out, void* ws,
                               size_t ws_bytes, void* const* stage_events, moe_stream_t stream) {
    g_err[0] = 0;
    MOE_TRY(need(gamma, "gamma"));
    if (cfg && h && out && out != h) {
        const size_t bytes = (size_t)cfg->T * cfg->H * 2;
        const char* hp = static_cast<const char*>(h);
        const char* op = static_cast<const char*>(out);
        if (op < hp + bytes && hp < op + bytes)
            return fail(MOE_ERR_INVALID_ARG, "out must be h or not overlap it");
    }
    return forward_impl(cfg, h, gamma, eps, w_router, bias, w13, w13_scale, w2, w2_scale, w13s,
                        w13s_scale, w2s, w2s_scale, out, ws, ws_bytes, stage_events, stream);
}

moe_status_t moe_rmsnorm(const moe_config_t* cfg, const void* h, const void* gamma, float eps,
                         void* u, moe_stream_t stream) {
    g_err[0] = 0;
    if (!cfg) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
    if (cfg->T < 0 || cfg->H <= 0 || cfg->H % 8)
        return fail(MOE_ERR_INVALID_ARG, "T=%d H=%d: need T >= 0 and H a positive multiple of 8",
                    cfg->T, cfg->H);
    MOE_TRY(need16(h, "h"));
    MOE_TRY(need16(gamma, "gamma"));
    MOE_TRY(need16(u, "u"));
    MOE_TRY(check_eps(eps));
    const size_t bytes = (size_t)cfg->T * cfg->H * 2;
    const char* hp = static_cast<const char*>(h);
    const char* up = static_cast<const char*>(u);
    if (up < hp + bytes && hp < up + bytes) return fail(MOE_ERR_INVALID_ARG, "u must not overlap h");
    return run_rmsnorm(cfg, h, gamma, eps, u, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_quantize_act(const void* x, int32_t rows, int32_t cols, uint8_t* q, float* scale,
                              moe_stream_t stream) {
    g_err[0] = 0;
    if (rows < 0 || cols <= 0 || cols % 128)
        return fail(MOE_ERR_INVALID_ARG, "rows=%d cols=%d: cols must be a positive multiple of 128",
                    rows, cols);
    MOE_TRY(need16(x, "x"));
    MOE_TRY(need16(q, "q"));
    MOE_TRY(need(scale, "scale"));
    if (rows == 0) return MOE_OK;
    moe::QuantArgs a;
    a.x = static_cast<const uint16_t*>(x);
    a.q = q;
    a.scale = scale;
    a.rows = rows;
    a.cols = cols;
    MOE_CUDA(moe::launch_quant_act(a, static_cast<cudaStream_t>(stream)), "quantisation launch");
    return MOE_OK;
}

moe_status_t moe_check_device_status(void* ws, moe_stream_t stream) {
    g_err[0] = 0;
    if (!ws) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    MOE_CUDA(cudaStreamSynchronize(s), "stream synchronize");
    int words[moe::kStatusWords];
    MOE_CUDA(cudaMemcpy(words, ws, sizeof(words), cudaMemcpyDeviceToHost), "status read");
    int dirty = -1;
    for (int i = moe::kSchedFirstWord; i < moe::kStatusWords; ++i)
        if (words[i] != 0) {
            dirty = i;
            break;
        }
    const int zero[moe::kStatusWords] = {};
    MOE_CUDA(cudaMemcpy(ws, zero, sizeof(zero), cudaMemcpyHostToDevice), "status clear");
    if (words[0] & moe::DEV_STATUS_TIMEOUT)
        return fail(MOE_ERR_TIMEOUT, "a kernel gave up a bounded wait (status 0x%x)", words[0]);
    if (words[0] & moe::DEV_STATUS_CAPACITY)
        return fail(MOE_ERR_WORKSPACE,
                    "an expert-parallel receive buffer was smaller than the rows sent to it "
                    "(status 0x%x): the rows beyond it were dropped",
                    words[0]);
    if (dirty >= 0)
        return fail(MOE_ERR_WORKSPACE,
                    "tile-claim counter word %d was %d after the stream drained: a launch "
                    "stopped part-way (the counters are now cleared)",
                    dirty, words[dirty]);
    return MOE_OK;
}

}  // extern "C"

// Argument checks and the last-error message, shared with entry points that
// live in other translation units of the library.
namespace moe {
moe_status_t api_check_config(const moe_config_t* c) { return check_config(c); }
moe_status_t api_fail(moe_status_t st, const char* msg) { return fail(st, "%s", msg); }
void api_clear_error() { g_err[0] = 0; }
moe_status_t api_sm_count(int* n) { return sm_count(n); }

// bf16 row-major [rows, cols] as a 2-D tensor, box {box_cols, box_rows}, 128-byte swizzle.
moe_status_t api_make_map_2d_bf16(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols,
                                  uint32_t box_cols, uint32_t box_rows, const char* what) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    if (!aligned16(ptr)) return fail(MOE_ERR_INVALID_ARG, "%s must be 16-byte aligned", what);
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map for %s failed (%d)", what, (int)r);
    return MOE_OK;
}

// bf16 3-D tensor map {d0, d1, d2} (d0 contiguous; byte strides of d1 and d2),
// box {b0, b1, b2}, 128-byte swizzle.
moe_status_t api_make_map_3d_bf16(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1,
                                  uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t b0,
                                  uint32_t b1, uint32_t b2, const char* what) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    if (!aligned16(ptr)) return fail(MOE_ERR_INVALID_ARG, "%s must be 16-byte aligned", what);
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1, stride2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map for %s failed (%d)", what, (int)r);
    return MOE_OK;
}

// Store map of an fp32 or bf16 3-D tensor {d0, d1, d2} (d0 contiguous; byte
// strides of d1 and d2), box {b0, b1, 1}, no swizzle: a staged row-major
// [b1][b0] tile in shared memory goes out in one bulk tensor store, clipped
// at the tensor's edges.
moe_status_t api_make_map_store_3d(CUtensorMap* m, const void* ptr, int f32, uint64_t d0,
                                   uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2,
                                   uint32_t b0, uint32_t b1, const char* what) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    if (!aligned16(ptr)) return fail(MOE_ERR_INVALID_ARG, "%s must be 16-byte aligned", what);
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1, stride2};
    cuuint32_t box[3] = {b0, b1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                    const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "tensor map for %s failed (%d)", what, (int)r);
    return MOE_OK;
}
}  // namespace moe
