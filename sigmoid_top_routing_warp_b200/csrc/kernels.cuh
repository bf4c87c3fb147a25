// kernels.cuh -- launch interface between the C-ABI layer (api.cu) and the
// CUDA kernels of the MoE FFN layer.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Device status word bits (stored in the workspace).
enum : int { DEV_STATUS_TIMEOUT = 1, DEV_STATUS_CAPACITY = 4 };

// The workspace's first 256 bytes: word 0 is the status word; words
// kSchedFirstWord .. kStatusWords - 1 hold the persistent GEMMs' tile-claim
// counters (a claim counter and a finished-CTA count per kernel and
// epilogue kind).  Every entry point that launches a claiming kernel zeroes
// those words on its stream first, and the last CTA of each launch zeroes
// its own pair again; a non-zero word after the stream has drained means a
// launch stopped part-way.
constexpr int kStatusWords = 64;
constexpr int kSchedFirstWord = 16;
cudaError_t reset_claim_counters(int* status, cudaStream_t s);

// ---------------------------------------------------------------- router
struct RouteArgs {
    const float* logits;  // [n_split, T, E]: logits, or K-slice partials summed in order
    int n_split;          // 1: logits as given; > 1: sum the slices, write logits_out
    float* logits_out;    // [T, E] summed logits (n_split > 1)
    const float* bias;    // [E]
    int32_t* idx;         // [T, k]
    float* w;             // [T, k]
    int T, E, k, n_group, topk_group, group_topn, norm;
    float rsf;
};
cudaError_t launch_route_select(const RouteArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- dispatch
struct PermuteArgs {
    const int32_t* idx;   // [T, k]
    int32_t* offsets;     // [E + 1]
    int32_t* rows;        // [T*k]
    int32_t* pos;         // [T*k]
    int32_t* chunk_base;  // [n_chunks, E] scratch (large path)
    int T, k, E;
};
int permute_chunks(int n_slots);  // chunks of the multi-block path (0: single block)
cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s);

struct GatherArgs {
    const uint16_t* x;        // bf16 [T, H]
    const int32_t* pos;       // [T*k]
    const float* topk_w;      // [T*k]
    const int32_t* offsets;   // [E + 1]
    uint16_t* x_perm;         // bf16 [T*k, H]
    float* w_perm;            // [T*k]
    int32_t* tok_start;       // [E + 1] token-tile prefix, tiles of bn rows
    int4* tok_tiles;          // [T*k/bn + E] per token tile: {expert, first row, rows, 0}
    int T, k, H, E, bn;
};
cudaError_t launch_gather(const GatherArgs& a, cudaStream_t s);

struct CombineArgs {
    const void* y;            // [T*k, H]: bf16, or fp32 with y_f32
    const int32_t* pos;       // [T*k]
    const float* y_shared;    // fp32 [T, H] or null
    const uint16_t* residual; // bf16 [T, H] added in the same fp32 sum, or null
    uint16_t* out;            // bf16 [T, H]
    int T, k, H;
    int y_f32;                // routed outputs stored fp32 (k = 1)
};
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- pre-norm
struct NormArgs {
    const uint16_t* h;        // bf16 [T, H]
    const uint16_t* gamma;    // bf16 [H]
    uint16_t* u;              // bf16 [T, H]
    int T, H;                 // H a multiple of 8
    float eps;
};
cudaError_t launch_rmsnorm(const NormArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- FP8 (e4m3, 128-blocks)
// Activation quantisation: per row, per 128 columns, scale = amax / 448,
// codes = RNE-satfinite e4m3(x / scale); an all-zero block gets scale 1.
struct QuantArgs {
    const uint16_t* x;   // bf16 [rows, cols]
    uint8_t* q;          // e4m3 [rows, cols]
    float* scale;        // [rows, cols / 128]
    int rows, cols;      // cols multiple of 128
};
cudaError_t launch_quant_act(const QuantArgs& a, cudaStream_t s);

// Row gather of e4m3 codes and their scales, plus the routing weight per
// sorted row and the token-tile prefix (as launch_gather).
struct GatherQArgs {
    const uint8_t* xq;        // [T, H]
    const float* sx;          // [T, H/128]
    const int32_t* pos;       // [T*k]
    const float* topk_w;      // [T*k]
    const int32_t* offsets;   // [E + 1]
    uint8_t* xq_perm;         // [T*k, H]
    float* sx_perm;           // [T*k, H/128]
    float* w_perm;            // [T*k]
    int32_t* tok_start;       // [E + 1]
    int T, k, H, E, bn;
};
cudaError_t launch_gather_q(const GatherQArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- grouped GEMM
enum Epilogue : int { EPI_F32 = 0, EPI_SWIGLU = 1, EPI_SCALE = 2 };

// One problem of a grouped GEMM launch, in "weights x tokens" orientation:
// for every expert e and every 128-row tile of its weight matrix,
//   D[f, r] = sum_k W_e[f, k] * X[r, k]  over the token rows r of expert e,
// written transposed to out[r, f].
struct GemmProblem {
    CUtensorMap tw;           // weights, bf16 2-D [rows, K], box {64, 128}
    CUtensorMap tx;           // activations, bf16 2-D [rows, K], box {64, bn}
    const int32_t* seg;       // [n_exp + 1] token-row offsets, or null: rows [0, n_rows)
    const int32_t* tok_start; // [n_exp + 1] token-tile prefix, or null with seg
    int n_exp;
    int n_rows;               // used when seg is null
    int K;                    // multiple of 64
    int n_feat;               // output features per expert
    int w_rows;               // weight rows per expert
    void* out;                // [rows, ld_out] (fp32 for EPI_F32, bf16 otherwise)
    int ld_out;
    const float* row_w;       // EPI_SCALE: per-row factor, or null (1.0)
    int out_f32;              // EPI_SCALE: store fp32 instead of bf16
    int k_split;              // EPI_F32: K slices (>= 1); slice s writes out + s * split_stride
    long long split_stride;   // elements between the slices' outputs
    // FP8 (e4m3 operands with fp32 scales per 128-block, see gemm_fp8.cu):
    const float* w_scale;     // [n_exp][w_rows/128][K/128] weight block scales
    const float* x_scale;     // [rows][K/128] activation scales
    uint8_t* out_q;           // EPI_SWIGLU: e4m3 codes [rows, ld_out]
    float* out_scale;         // EPI_SWIGLU: scales [rows, ld_out/128]
    // token-major fp8 kernel: the same scales as fp32 2-D tensor maps,
    // x_scale box {4, 128} and w_scale box {4, 1}
    CUtensorMap tsx;
    CUtensorMap tsw;
};

struct GemmParams {
    GemmProblem p[2];
    int n_problems;
    int* status;
    int test_stall;  // test only: CTA 0 never fills its first pipeline stage
};

// bn: token tile (16, 64 or 128).  grid: persistent CTAs.
cudaError_t launch_grouped_gemm(int epi, int bn, const GemmParams& params, int grid,
                                cudaStream_t s);

// ---------------------------------------------------------------- CTA-pair grouped GEMM
// Prefill-sized version of the grouped GEMM: clusters of two CTAs run one
// M = 256 MMA per K step (128 weight rows per CTA) over a 256-token tile
// (128 token rows loaded per CTA).
constexpr int kPairTokens = 256;
constexpr int kPairBoxes = 4;  // token boxes of 16, 32, 64, 128 rows per CTA

struct PairProblem {
    // EPI_SWIGLU: 5-D view {K, 8, 2, n_feat/8, n_exp} of the packed gate/up
    // matrix [n_exp][2 n_feat][K] (box {64, 8, 2, 8, 1}: 64 features as
    // 8-row gate / up blocks).  EPI_SCALE: 2-D [n_exp * n_feat, K], box {64, 128}.
    CUtensorMap tw;
    // activations, bf16 2-D [rows, K], box {64, 16 << i}: a tile loads only
    // the rows it uses (its MMA width / 2 per CTA, rounded up to a box)
    CUtensorMap tx[kPairBoxes];
    const int32_t* seg;       // [n_exp + 1] token-row offsets, or null: rows [0, n_rows)
    const int32_t* tok_start; // [n_exp + 1] prefix of 256-token tiles, or null with seg
    const int4* tok_tiles;    // with seg: token tile j = {expert, first row, rows, 0}
    int n_exp;
    int n_rows;
    int K;                    // multiple of 64
    int n_feat;               // output features per expert (multiple of 8)
    void* out;                // bf16 [rows, ld_out] (fp32 if out_f32)
    int ld_out;
    const float* row_w;       // EPI_SCALE: per-row factor, or null (1.0)
    int out_f32;              // EPI_SCALE: store fp32 instead of bf16
};

struct PairParams {
    PairProblem p[2];
    int n_problems;
    int* status;
};

cudaError_t launch_pair_gemm(int epi, const PairParams& params, int grid, cudaStream_t s);

// FP8 grouped GEMM (single CTA, weights as the M operand): EPI_SWIGLU
// (writes e4m3 codes + scales of A) or EPI_SCALE (bf16 / fp32 out).  bn 16, 32, 64.
cudaError_t launch_fp8_gemm(int epi, int bn, const GemmParams& params, int grid, cudaStream_t s);

// Token-major FP8 grouped GEMM (tokens as the M operand, 128-row token tiles;
// features per tile: 128 for EPI_SWIGLU, 256 for EPI_SCALE).  Needs K a
// multiple of 512, n_feat a multiple of 128, and the tsx / tsw maps.
constexpr int kFp8TokTile = 128;
cudaError_t launch_fp8_tm_gemm(int epi, const GemmParams& params, int grid, cudaStream_t s);

// ---------------------------------------------------------------- backward GEMMs
// One problem of a backward grouped GEMM launch (gemm_bwd.cu).  The tensor-
// memory accumulator of a tile is D[m, n] = sum_k A(m, k) B(n, k) over a
// 256 x 256 tile of a CTA pair (128 rows m per CTA, lane = m, column = n);
// each operand is K-major (a 2-D map [rows, K], box {64, 128}; K-major B also
// {64, 16 << i}) or MN-major (a 3-D view {64, K rows, MN / 64} of the
// row-major [K, MN] matrix, strides {MN * 2, 128} bytes, box {64, 64, 2}).
// Each CTA of the pair stages 128 of the tile's m and half of its n.
//   rows_as_k = 0: the N dimension runs over token rows, grouped by `seg`
//     (per group: tiles of 256 rows, prefix `tstart`), K = [0, K); A's row
//     coordinate is offset by group * a_grp_rows (the group's weights).
//     Output out[row * ld_out + m].
//   rows_as_k = 1: K runs over the token rows of a group, [seg[g], seg[g+1])
//     (or [0, n_rows) without seg); tiles cover M x N per group.  Output
//     out[g * out_grp + n * ld_out + m] (a group's weight gradient).
enum BwdEpilogue : int { BEPI_STORE = 0, BEPI_DSWIGLU = 1 };
struct BwdProblem {
    CUtensorMap ta, tb;
    CUtensorMap tbs[3];       // K-major B: the same operand with boxes {64, 16 << i} rows
                              // (tb: {64, 128}); MN-major B: tb only, box {64, 64, 2}
    CUtensorMap to;           // BEPI_STORE: store map of out, 3-D {M, rows, groups}, box
                              // {32, 16 or 32, 1}
    int a_mn, b_mn;
    int rows_as_k;
    const int32_t* seg;       // [n_grp + 1] group row offsets, or null: one group [0, n_rows)
    const int32_t* tstart;    // rows_as_k = 0 with seg: [n_grp + 1] prefix of 256-row tiles
    const int32_t* ttab;      // with tstart, or null: [tstart[n_grp]] the group of each row tile
    int n_grp, n_rows;
    int M, N, K;
    int a_grp_rows;
    void* out;
    int ld_out;
    long long out_grp;
    int out_f32;
    // BEPI_DSWIGLU (rows_as_k = 0, M = half): D[i, r] = dL/da'_r[i] before the
    // routing weight; gu [rows, 2 half] (fp32) holds the gate (cols < half) and
    // up pre-activations of each row
    const float* gu;
    int ld_gu, half;
    const float* row_w;       // routing weight per row, or null (1)
    uint16_t* dgu;            // [rows, ld_dgu]: dgate | dup (bf16)
    int ld_dgu;
    uint16_t* aw;             // [rows, ld_aw]: w * SiLU(g) * u (bf16)
    int ld_aw;
    float* dw_part;           // [rows, ld_dw]: sum over 32 features of a' * da, or null
    int ld_dw;
};
constexpr int kBwdMaxProblems = 5;
struct BwdParams {
    BwdProblem p[kBwdMaxProblems];
    int n_problems;
    int* status;
};
cudaError_t launch_bwd_gemm(int epi, const BwdParams& params, int grid, cudaStream_t s);

}  // namespace moe
