// gemm.cu -- persistent grouped GEMM on the 5th-generation tensor cores
// (tcgen05 + tensor memory), fed by TMA.  Steps a1 (router logits), a6
// (gate/up GEMM with the SwiGLU epilogue), a7 (down GEMM with the routing
// weight epilogue) and a8 (the shared expert, as a second problem of the same
// launch).
//
// Source of the operation: "Xiaohongshu dots3 note Open Source Deep Dive",
// §8.2 (FUSED_MC2: gmm1 -> swiglu -> gmm2) and §3.1 (the sketch notes the
// real implementation runs the experts as a grouped GEMM);
// "Transformers 中的 dots.llm1（Dots1）模型" (blog.gitcode.com), parallel-plan
// paragraph (packed gate_up_proj; experts as grouped_gemm).
//
// Orientation: the weight matrix is the MMA's M operand (128 weight rows per
// tile) and the tokens of one expert are the N operand (bn = 16, 64 or 128
// rows).  A decode-sized expert with two tokens therefore still runs full
// 128-row MMAs and streams its weights at full width, while a prefill-sized
// expert uses bn = 128 token tiles.  The accumulator D[f, r] sits in tensor
// memory with lane = weight row f and column = token r.
//
// Roles (192 threads, one CTA per SM, persistent):
//   warp 0      tile claims and TMA producer: weight tile(s) + token tile per
//               64-wide K step
//   warp 1      TMEM allocator and single-thread MMA issuer
//   warps 2..5  epilogue: tcgen05.ld, SiLU*up / x weight / fp32, stores
// Shared-memory ring of STAGES {weights, tokens} slots with full/empty
// mbarriers; two TMEM accumulator buffers with full/empty mbarriers so the
// epilogue of one tile overlaps the main loop of the next.
//
// Tiles are claimed at run time: the producer takes the next tile index from
// a counter in the workspace status block and hands it to the MMA thread and
// the epilogue through a 4-slot ring.  Claims follow the tile order (expert,
// feature tile, token tile), so the CTAs working at the same time still
// share weight tiles in L2, and no CTA sits idle while another has two tiles
// left: at decode sizes a static round-robin left the CTAs' end times ≈65 µs
// apart.  The last CTA to finish resets the counter (the workspace starts
// zero-filled).
//
// Every mbarrier wait is bounded: when a wait runs past kWaitLimit cycles the
// CTA records DEV_STATUS_TIMEOUT in the status word, raises a shared abort
// flag that ends every role's loop, waits for its own copies and MMAs in
// flight (again bounded), frees its tensor memory and returns.
#include "kernels.cuh"
#include "ptx.cuh"
#include "tiles.cuh"

#include <cuda_bf16.h>

namespace moe {

constexpr int kThreads = 192;
constexpr int kBK = 64;                        // K elements per stage (128 B rows)
constexpr int kWTileBytes = 128 * kBK * 2;     // one 128-row weight tile
constexpr int kRing = 4;                       // claimed tile ids in flight (producer -> MMA, epilogue)
constexpr int kSchedWord = 16;                 // first scheduling word in the status block

template <int BN>
struct TokTile {
    static constexpr int bytes = BN * kBK * 2;
};

template <int EPI, int BN>
struct Cfg {
    static constexpr int NW = (EPI == EPI_SWIGLU) ? 2 : 1;  // weight tiles per stage
    static constexpr int STAGE_BYTES = NW * kWTileBytes + TokTile<BN>::bytes;
    static constexpr int STAGES_RAW = (220 * 1024) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_RAW > 12 ? 12 : STAGES_RAW;
    static constexpr int ACC_COLS = NW * BN;      // columns of one accumulator buffer
    static constexpr int TMEM_NEED = 2 * ACC_COLS;
    static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64
                                   : TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
    static constexpr int BAR_BYTES = 512;
    static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
    static constexpr uint32_t IDESC = idesc_bf16_f32(128, BN);
    static_assert(TMEM_NEED <= 512, "accumulators exceed tensor memory");
    static_assert(STAGES >= 2, "pipeline too shallow");
    static_assert(SMEM <= 232448, "shared memory budget");
};



template <int EPI, int BN>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_kernel(const __grid_constant__ GemmParams P) {
    using C = Cfg<EPI, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* tfull = empty + C::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint64_t* rfull = mma_done + 1;          // [kRing] a claimed tile id is in the ring
    uint64_t* rempty = rfull + kRing;        // [kRing] read by the MMA thread and 4 epilogue warps
    int* ring = reinterpret_cast<int*>(rempty + kRing);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(ring + kRing);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        mbar_init(mma_done, 1);
        for (int r = 0; r < kRing; ++r) {
            mbar_init(&rfull[r], 1);
            mbar_init(&rempty[r], 5);
        }
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
    // tile claim counter and finished-CTA count of this epilogue kind, in the
    // workspace status block (word 0 is the status word)
    int* sched = P.status + kSchedWord + 2 * EPI;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued = 0;          // stages ever filled
            uint32_t last_ph[12] = {0};   // parity of the last fill of each stage
            bool ok = true;
            int rs = 0;
            uint32_t rph = 0;
            while (ok) {
                // claim the next tile and hand its id to the MMA thread and the epilogue
                int t = atomicAdd(&sched[0], 1);
                if (t >= ntiles) t = -1;
                if (!wait_bar(&rempty[rs], rph ^ 1, abort_flag, P.status)) { ok = false; break; }
                ring[rs] = t;
                mbar_arrive(&rfull[rs]);
                if (++rs == kRing) { rs = 0; rph ^= 1; }
                if (t < 0) break;
                Tile tl;
                tile_at(P, BN, t, tl);
                const GemmProblem& p = P.p[tl.prob];
                const int wrow = tl.exp * p.w_rows + tl.f0;
                const int nk = p.K / kBK / max(p.k_split, 1);
                const int kb0 = tl.kslice * nk;
                for (int kb = kb0; kb < kb0 + nk; ++kb) {
                    if (!wait_bar(&empty[s], ph ^ 1, abort_flag, P.status)) { ok = false; break; }
                    if (P.test_stall && blockIdx.x == 0 && issued == 0 && s == 0 && ph == 0) {
                        // test of the bounded waits: this stage is never filled, so the
                        // MMA's wait on it runs out; the stage is not marked issued
                        if (++s == C::STAGES) { s = 0; ph ^= 1; }
                        continue;
                    }
                    uint8_t* st = smem + s * C::STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
                    tma_load_2d(st, &p.tw, &full[s], kb * kBK, wrow);
                    if (C::NW == 2) tma_load_2d(st + kWTileBytes, &p.tw, &full[s], kb * kBK, wrow + p.n_feat);
                    tma_load_2d(st + C::NW * kWTileBytes, &p.tx, &full[s], kb * kBK, tl.row0);
                    issued |= 1u << s;
                    last_ph[s] = ph;
                    if (++s == C::STAGES) { s = 0; ph ^= 1; }
                }
            }
            // Leave no copy in flight: wait for the last fill of every stage.
            for (int i = 0; i < C::STAGES; ++i)
                if (issued >> i & 1u) wait_bar(&full[i], last_ph[i], abort_flag, P.status, true);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int s = 0, buf = 0;
            uint32_t ph = 0, aph = 0;
            bool ok = true, any = false;
            int rs = 0;
            uint32_t rph = 0;
            while (ok) {
                if (!wait_bar(&rfull[rs], rph, abort_flag, P.status)) break;
                const int t = ring[rs];
                mbar_arrive(&rempty[rs]);
                if (++rs == kRing) { rs = 0; rph ^= 1; }
                if (t < 0) break;
                Tile tl;
                tile_at(P, BN, t, tl);
                const int nk = P.p[tl.prob].K / kBK / max(P.p[tl.prob].k_split, 1);
                if (!wait_bar(&tempty[buf], aph ^ 1, abort_flag, P.status)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + buf * C::ACC_COLS;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!wait_bar(&full[s], ph, abort_flag, P.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_addr(smem + s * C::STAGE_BYTES);
                    const uint32_t xt = st + C::NW * kWTileBytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t bdesc = smem_desc_k_sw128(xt + kk * 32);
#pragma unroll
                        for (int w = 0; w < C::NW; ++w) {
                            const uint64_t adesc = smem_desc_k_sw128(st + w * kWTileBytes + kk * 32);
                            tc_mma_f16(d + w * BN, adesc, bdesc, C::IDESC, (kb | kk) != 0);
                        }
                    }
                    tc_commit(&empty[s]);
                    any = true;
                    if (++s == C::STAGES) { s = 0; ph ^= 1; }
                }
                if (!ok) break;
                tc_commit(&tfull[buf]);
                if (++buf == 2) { buf = 0; aph ^= 1; }
            }
            // Leave no MMA in flight before the tensor memory is freed.
            if (any) {
                tc_commit(mma_done);
                wait_bar(mma_done, 0, abort_flag, P.status, true);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;  // tensor-memory lane quadrant of this warp
        int buf = 0;
        uint32_t aph = 0;
        int rs = 0;
        uint32_t rph = 0;
        while (true) {
            if (!wait_bar(&rfull[rs], rph, abort_flag, P.status)) break;
            const int t = ring[rs];
            __syncwarp();
            if (lane == 0) mbar_arrive(&rempty[rs]);
            if (++rs == kRing) { rs = 0; rph ^= 1; }
            if (t < 0) break;
            Tile tl;
            tile_at(P, BN, t, tl);
            const GemmProblem& p = P.p[tl.prob];
            if (!wait_bar(&tfull[buf], aph, abort_flag, P.status)) break;
            tc_fence_after();
            const int f = tl.f0 + q * 32 + lane;
            const bool fok = f < p.n_feat;
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + buf * C::ACC_COLS;
            for (int c0 = 0; c0 < tl.nvalid; c0 += 16) {
                uint32_t r[16];
                tmem_ld_16(tbase + c0, r);
                if (EPI == EPI_SWIGLU) {
                    uint32_t u[16];
                    tmem_ld_16(tbase + BN + c0, u);
                    tmem_wait_ld();
                    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        if (c0 + j < tl.nvalid && fok) {
                            const float g = __uint_as_float(r[j]);
                            const float a = silu(g) * __uint_as_float(u[j]);
                            out[(size_t)(tl.row0 + c0 + j) * p.ld_out + f] = __float2bfloat16_rn(a);
                        }
                    }
                } else if (EPI == EPI_SCALE) {
                    tmem_wait_ld();
                    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
                    float* outf = reinterpret_cast<float*>(p.out);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        if (c0 + j < tl.nvalid && fok) {
                            const int row = tl.row0 + c0 + j;
                            const float wr = p.row_w ? __ldg(p.row_w + row) : 1.0f;
                            const float v = __uint_as_float(r[j]) * wr;
                            if (p.out_f32)
                                outf[(size_t)row * p.ld_out + f] = v;
                            else
                                out[(size_t)row * p.ld_out + f] = __float2bfloat16_rn(v);
                        }
                    }
                } else {
                    tmem_wait_ld();
                    float* out = reinterpret_cast<float*>(p.out) + tl.kslice * p.split_stride;
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (c0 + j < tl.nvalid && fok)
                            out[(size_t)(tl.row0 + c0 + j) * p.ld_out + f] = __uint_as_float(r[j]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);
            if (++buf == 2) { buf = 0; aph ^= 1; }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
    // the last CTA to finish leaves the claim counters at zero for the next launch
    // (every CTA's claims came from thread 0 before this point)
    if (threadIdx.x == 0 && atomicAdd(&sched[1], 1) == (int)gridDim.x - 1) {
        atomicExch(&sched[0], 0);
        atomicExch(&sched[1], 0);
    }
}

template <int EPI, int BN>
static cudaError_t launch_t(const GemmParams& params, int grid, cudaStream_t s) {
    using C = Cfg<EPI, BN>;
    // The attribute is per device; setting it again is cheap.
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<EPI, BN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    grouped_gemm_kernel<EPI, BN><<<grid, kThreads, C::SMEM, s>>>(params);
    return cudaGetLastError();
}

cudaError_t launch_grouped_gemm(int epi, int bn, const GemmParams& params, int grid, cudaStream_t s) {
    if (params.status == nullptr) return cudaErrorInvalidValue;  // holds the tile claim counters
#define MOE_GEMM_CASE(E_, B_) \
    if (epi == E_ && bn == B_) return launch_t<E_, B_>(params, grid, s);
    MOE_GEMM_CASE(EPI_F32, 16)
    MOE_GEMM_CASE(EPI_F32, 64)
    MOE_GEMM_CASE(EPI_F32, 128)
    MOE_GEMM_CASE(EPI_SWIGLU, 16)
    MOE_GEMM_CASE(EPI_SWIGLU, 64)
    MOE_GEMM_CASE(EPI_SWIGLU, 128)
    MOE_GEMM_CASE(EPI_SCALE, 16)
    MOE_GEMM_CASE(EPI_SCALE, 64)
    MOE_GEMM_CASE(EPI_SCALE, 128)
#undef MOE_GEMM_CASE
    return cudaErrorInvalidValue;
}

}  // namespace moe
