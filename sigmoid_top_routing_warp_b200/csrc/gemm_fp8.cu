// gemm_fp8.cu -- grouped expert GEMMs on e4m3 operands with fp32 block
// scales (steps a6-a8 of the FP8 layer), tcgen05 kind::f8f6f4 + TMEM.
//
// Source of the operation: "Xiaohongshu dots3 note Open Source Deep Dive",
// §8.2 (gmm1 -> swiglu -> gmm2) and §3.2 (FP8 weights fit one 8xH100 node);
// "dots3-note 架构深度解析" (mlqm.cn), 部署实战 (FP8 weights, dots3-note-prev-fp8).
// Recipe: weights e4m3 with one fp32 scale per 128x128 block; activations e4m3
// with one fp32 scale per row and 128 columns (see quant.cu).
//
// The fp32 scales are not powers of two, so the tensor core's block-scaled
// modes cannot apply them.  Each 128-wide K block is therefore one MMA group
// (4 x K=32 f8f6f4 MMAs) into a tensor-memory partial; the epilogue warps
// read the partial and promote it into fp32 register accumulators:
//   acc[f, r] += s_w(tile, kb) * s_x(r, kb) * partial[f, r].
// Two partial buffers let the MMAs of block kb+1 run while block kb is
// promoted.  Weights are the MMA's M operand (128 rows of one 128x128 scale
// block); tokens are N (bn = 16 or 32).
//
// EPI_SWIGLU: after the last block, a = SiLU(acc_gate) * acc_up is quantised
// per token over the tile's 128 features (one e4m3 block of A): the four
// epilogue warps exchange per-token maxima through shared memory under a
// bounded mbarrier, then write codes and the block scale.
// EPI_SCALE: y = acc * routing weight, stored bf16 (or fp32 for the shared
// expert).
//
// Waits are bounded as in gemm.cu (DEV_STATUS_TIMEOUT, abort flag, drain).
#include "kernels.cuh"
#include "ptx.cuh"
#include "tiles.cuh"

#include <cuda_bf16.h>
#include <cuda_fp8.h>

namespace moe {

namespace {

constexpr int kQBK = 128;                      // K per stage (one scale block), 128 B rows
constexpr int kQWTile = 128 * kQBK;            // 16 KB of weights

template <int EPI, int BN>
struct QCfg {
    // epilogue warps: 4 (one per TMEM lane quadrant), or 8 for 64-token tiles
    // (two warps per quadrant, each promoting half of the token columns)
    static constexpr int EW = BN >= 64 ? 8 : 4;
    static constexpr int THREADS = 64 + 32 * EW;
    static constexpr int CW = BN * 4 / EW;     // token columns per epilogue warp
    static constexpr int NW = (EPI == EPI_SWIGLU) ? 2 : 1;
    static constexpr int STAGE_BYTES = NW * kQWTile + BN * kQBK;
    static constexpr int STAGES_RAW = (216 * 1024) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_RAW > 12 ? 12 : STAGES_RAW;
    static constexpr int PART_COLS = NW * BN;  // one partial buffer
    // partial buffers: the MMAs may run this many K blocks ahead of promotion
    static constexpr int NP = (512 / PART_COLS) > 8 ? 8 : (512 / PART_COLS);
    static constexpr int TMEM_NEED = NP * PART_COLS;
    static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64
                                   : TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
    static constexpr int AMAX_BYTES = 2 * 4 * BN * 4;  // [2 parities][4 warps][BN] floats
    static constexpr int BAR_BYTES = 512;
    static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + AMAX_BYTES + BAR_BYTES;
    // kind::f8f6f4: fp32 accumulator, e4m3 A and B (format 0), K-major, M=128, N=BN
    static constexpr uint32_t IDESC = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(STAGES >= 3, "pipeline too shallow");
};

__device__ __forceinline__ void tc_mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

}  // namespace

template <int EPI, int BN>
__global__ void __launch_bounds__(QCfg<EPI, BN>::THREADS, 1)
    fp8_gemm_kernel(const __grid_constant__ GemmParams P) {
    using C = QCfg<EPI, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* amax_sm = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::AMAX_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* pfull = empty + C::STAGES;   // partial buffer ready (MMA -> epilogue)
    uint64_t* pempty = pfull + C::NP;      // partial buffer read (epilogue -> MMA)
    uint64_t* amax_bar = pempty + C::NP;   // per-token maxima of the 4 warps written [2]
    uint64_t* mma_done = amax_bar + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < C::NP; ++b) {
            mbar_init(&pfull[b], 1);
            mbar_init(&pempty[b], C::EW);
        }
        for (int b = 0; b < 2; ++b) mbar_init(&amax_bar[b], C::EW);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        for (int pi = 0; pi < P.n_problems; ++pi) {
            tma_prefetch_desc(&P.p[pi].tw);
            tma_prefetch_desc(&P.p[pi].tx);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int ntiles = total_tiles(P, BN);

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0, issued = 0;
            uint32_t last_ph[12] = {0};
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                Tile tl;
                tile_at(P, BN, t, tl);
                const GemmProblem& p = P.p[tl.prob];
                const int wrow = tl.exp * p.w_rows + tl.f0;
                const int nk = p.K / kQBK;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!wait_bar(&empty[s], ph ^ 1, abort_flag, P.status)) { ok = false; break; }
                    uint8_t* st = smem + s * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
                    tma_load_2d(st, &p.tw, &full[s], kb * kQBK, wrow);
                    if (C::NW == 2) tma_load_2d(st + kQWTile, &p.tw, &full[s], kb * kQBK, wrow + p.n_feat);
                    tma_load_2d(st + C::NW * kQWTile, &p.tx, &full[s], kb * kQBK, tl.row0);
                    issued |= 1u << s;
                    last_ph[s] = ph;
                    if (++s == C::STAGES) { s = 0; ph ^= 1; }
                }
            }
            for (int i = 0; i < C::STAGES; ++i)
                if (issued >> i & 1u) wait_bar(&full[i], last_ph[i], abort_flag, P.status, true);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer: one group per K block
        if (lane == 0) {
            int s = 0, pb = 0;
            uint32_t ph = 0, pph = 0;
            bool ok = true, any = false;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                Tile tl;
                tile_at(P, BN, t, tl);
                const int nk = P.p[tl.prob].K / kQBK;
                for (int kb = 0; kb < nk && ok; ++kb) {
                    if (!wait_bar(&pempty[pb], pph ^ 1, abort_flag, P.status)) { ok = false; break; }
                    if (!wait_bar(&full[s], ph, abort_flag, P.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_addr(smem + s * C::STAGE_BYTES);
                    const uint32_t xt = st + C::NW * kQWTile;
                    const uint32_t d = tmem_base + pb * C::PART_COLS;
#pragma unroll
                    for (int kk = 0; kk < kQBK / 32; ++kk) {
                        const uint64_t bdesc = smem_desc_k_sw128(xt + kk * 32);
#pragma unroll
                        for (int w = 0; w < C::NW; ++w)
                            tc_mma_f8(d + w * BN, smem_desc_k_sw128(st + w * kQWTile + kk * 32), bdesc,
                                      C::IDESC, kk != 0);
                    }
                    tc_commit(&empty[s]);
                    tc_commit(&pfull[pb]);
                    any = true;
                    if (++s == C::STAGES) { s = 0; ph ^= 1; }
                    if (++pb == C::NP) { pb = 0; pph ^= 1; }
                }
            }
            if (any) {
                tc_commit(mma_done);
                wait_bar(mma_done, 0, abort_flag, P.status, true);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue: promote, then finish the tile
        const int q = warp & 3;                   // TMEM lane quadrant
        const int cb = ((warp - 2) >> 2) * C::CW; // first token column of this warp
        int pb = 0, tile_no = 0;
        uint32_t pph = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tile_no) {
            Tile tl;
            tile_at(P, BN, t, tl);
            const GemmProblem& p = P.p[tl.prob];
            const int nk = p.K / kQBK;
            const int f = tl.f0 + q * 32 + lane;
            const int kbs = p.K / kQBK;  // scale blocks along K
            float acc[C::NW][C::CW];
#pragma unroll
            for (int w = 0; w < C::NW; ++w)
#pragma unroll
                for (int j = 0; j < C::CW; ++j) acc[w][j] = 0.0f;
            // Scales, fetched SC K blocks at a time one chunk ahead so that their
            // global-load latency overlaps the promotion of the previous chunk:
            // weight blocks (one per 128-row tile) and lane j's token cb + j.
            constexpr int SC = C::EW == 8 ? 2 : 4;  // 8-warp variants have fewer registers
            const int jl = cb + lane;
            const bool jv = lane < C::CW && jl < tl.nvalid;
            const float* xs = p.x_scale + (size_t)(tl.row0 + (jv ? jl : 0)) * kbs;
            const float* wsp[C::NW];
#pragma unroll
            for (int w = 0; w < C::NW; ++w)
                wsp[w] = p.w_scale + (size_t)((tl.exp * p.w_rows + tl.f0 + w * p.n_feat) / 128) * kbs;
            float nx[SC], nw[C::NW][SC];
#pragma unroll
            for (int i = 0; i < SC; ++i) {
                nx[i] = (jv && i < nk) ? __ldg(xs + i) : 0.0f;
#pragma unroll
                for (int w = 0; w < C::NW; ++w) nw[w][i] = i < nk ? __ldg(wsp[w] + i) : 0.0f;
            }
            for (int k0 = 0; k0 < nk && ok; k0 += SC) {
                float cx[SC], cw[C::NW][SC];
#pragma unroll
                for (int i = 0; i < SC; ++i) {
                    cx[i] = nx[i];
#pragma unroll
                    for (int w = 0; w < C::NW; ++w) cw[w][i] = nw[w][i];
                    const int kn = k0 + SC + i;
                    nx[i] = (jv && kn < nk) ? __ldg(xs + kn) : 0.0f;
#pragma unroll
                    for (int w = 0; w < C::NW; ++w) nw[w][i] = kn < nk ? __ldg(wsp[w] + kn) : 0.0f;
                }
#pragma unroll
                for (int i = 0; i < SC; ++i) {
                    if (k0 + i >= nk) break;
                    if (!wait_bar(&pfull[pb], pph, abort_flag, P.status)) { ok = false; break; }
                    tc_fence_after();
                    uint32_t r[C::NW][C::CW];
                    const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + pb * C::PART_COLS + cb;
#pragma unroll
                    for (int w = 0; w < C::NW; ++w)
#pragma unroll
                        for (int c0 = 0; c0 < C::CW; c0 += 16)
                            tmem_ld_16(tb + w * BN + c0, *reinterpret_cast<uint32_t(*)[16]>(&r[w][c0]));
                    tmem_wait_ld();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pempty[pb]);
                    if (++pb == C::NP) { pb = 0; pph ^= 1; }
#pragma unroll
                    for (int j = 0; j < C::CW; ++j) {
                        const float sxj = __shfl_sync(0xffffffffu, cx[i], j);
#pragma unroll
                        for (int w = 0; w < C::NW; ++w)
                            acc[w][j] = fmaf(cw[w][i] * sxj, __uint_as_float(r[w][j]), acc[w][j]);
                    }
                }
            }
            if (!ok) break;
            const bool fok = f < p.n_feat;
            if (EPI == EPI_SWIGLU) {
                // a = SiLU(gate) * up; e4m3 block of 128 features per token
                float a[C::CW];
                float m[C::CW];
#pragma unroll
                for (int j = 0; j < C::CW; ++j) {
                    a[j] = acc[0][j] / (1.0f + __expf(-acc[0][j])) * acc[1][j];
                    m[j] = fok ? fabsf(a[j]) : 0.0f;
                }
#pragma unroll
                for (int j = 0; j < C::CW; ++j)
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1)
                        m[j] = fmaxf(m[j], __shfl_xor_sync(0xffffffffu, m[j], off));
                const int par = tile_no & 1;
                float* mine = amax_sm + (par * 4 + q) * BN + cb;
#pragma unroll
                for (int j = 0; j < C::CW; ++j)
                    if (lane == j) mine[j] = m[j];
                __syncwarp();
                if (lane == 0) mbar_arrive(&amax_bar[par]);
                if (!wait_bar(&amax_bar[par], (tile_no >> 1) & 1, abort_flag, P.status)) break;
                uint8_t* outq = p.out_q;
#pragma unroll
                for (int jj = 0; jj < C::CW; ++jj) {
                    const int j = cb + jj;
                    const float* all = amax_sm + par * 4 * BN;
                    const float amax = fmaxf(fmaxf(all[j], all[BN + j]), fmaxf(all[2 * BN + j], all[3 * BN + j]));
                    const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
                    if (j < tl.nvalid) {
                        const int row = tl.row0 + j;
                        if (fok)
                            outq[(size_t)row * p.ld_out + f] =
                                __nv_cvt_float_to_fp8(__fdiv_rn(a[jj], sc), __NV_SATFINITE, __NV_E4M3);
                        if (q == 0 && lane == 0) p.out_scale[(size_t)row * (p.ld_out / 128) + tl.f0 / 128] = sc;
                    }
                }
            } else {
                __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
                float* outf = reinterpret_cast<float*>(p.out);
#pragma unroll
                for (int jj = 0; jj < C::CW; ++jj) {
                    const int j = cb + jj;
                    if (j < tl.nvalid && fok) {
                        const int row = tl.row0 + j;
                        const float wr = p.row_w ? __ldg(p.row_w + row) : 1.0f;
                        const float v = acc[0][jj] * wr;
                        if (p.out_f32) outf[(size_t)row * p.ld_out + f] = v;
                        else out[(size_t)row * p.ld_out + f] = __float2bfloat16_rn(v);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

template <int EPI, int BN>
static cudaError_t launch_q(const GemmParams& params, int grid, cudaStream_t s) {
    using C = QCfg<EPI, BN>;
    cudaError_t e = cudaFuncSetAttribute(fp8_gemm_kernel<EPI, BN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    fp8_gemm_kernel<EPI, BN><<<grid, C::THREADS, C::SMEM, s>>>(params);
    return cudaGetLastError();
}

cudaError_t launch_fp8_gemm(int epi, int bn, const GemmParams& params, int grid, cudaStream_t s) {
    if (epi == EPI_SWIGLU && bn == 16) return launch_q<EPI_SWIGLU, 16>(params, grid, s);
    if (epi == EPI_SWIGLU && bn == 32) return launch_q<EPI_SWIGLU, 32>(params, grid, s);
    if (epi == EPI_SCALE && bn == 16) return launch_q<EPI_SCALE, 16>(params, grid, s);
    if (epi == EPI_SCALE && bn == 32) return launch_q<EPI_SCALE, 32>(params, grid, s);
    if (epi == EPI_SWIGLU && bn == 64) return launch_q<EPI_SWIGLU, 64>(params, grid, s);
    if (epi == EPI_SCALE && bn == 64) return launch_q<EPI_SCALE, 64>(params, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace moe
