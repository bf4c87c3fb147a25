// gemm_bwd.cu -- the grouped GEMMs of the layer's backward pass on the
// 5th-generation tensor cores (tcgen05 + tensor memory), fed by TMA.
//
// The backward pass is the chain rule through the forward pass that
// "Xiaohongshu dots3 note Open Source Deep Dive" describes (§3.1: gate ->
// scores -> top-k -> renormalise -> shared + weighted routed sum; §8.2:
// gmm1 -> swiglu -> gmm2), with the expert choice held fixed.  Its GEMMs
// contract along three different axes:
//   - recomputed gate/up pre-activations  G|U = X W13^T        (K = hidden)
//   - the down projection's input grad    dA  = dY W2_e        (K = hidden,
//                                           W2_e read with I contiguous)
//   - the input grad                      dX  = dG|dU W13_e    (K = 2I,
//                                           W13_e read with H contiguous)
//   - the weight grads                    dW2_e = dY_e^T (w A)_e,
//                                          dW13_e = dG|dU_e^T X_e
//                                           (K = the expert's token rows)
// so, unlike the forward kernels, operands come K-major or MN-major (the
// tensor core reads either from shared memory; the instruction descriptor
// says which), and K may run over an expert's row segment.
//
// Tile: 128 x 256 (M = output features in tensor-memory lanes, N = token
// rows or output columns), K step 64; the MMA's N is the tile's valid
// columns rounded up to 16.  Roles (352 threads, one CTA per SM,
// persistent, static round-robin over the tile list):
//   warp 0      TMA producer of the A operand (one 16 KB box per stage: K-major
//               {64, 128}, or MN-major {64, 64, 2} of a 3-D view that brings
//               two 64-wide chunks), warp 10 of the B operand (32 KB: {64, 256}
//               or {64, 64, 4}); two issuing threads, because one thread's
//               tensor copies top out well below the SM's L2 bandwidth
//   warp 1      TMEM allocator and single-thread MMA issuer
//   warps 2..9  epilogue (tcgen05.ld 32x32b: lane = feature m): two warps per
//               tensor-memory lane quadrant, each taking half of the tile's
//               columns; stores go through a per-warp shared-memory transpose
//               so that each thread writes 16 bytes of one output row
// Two 256-column accumulators (all of tensor memory) let the epilogue of one
// tile overlap the main loop of the next.  Row segments are padded to 16 rows by the caller, so a
// segment ends on an MMA boundary: a K step whose 64 rows run past the
// segment issues only the MMAs inside it.
//
// Every mbarrier wait is bounded (see wait_bar): on timeout the CTA records
// DEV_STATUS_TIMEOUT, stops, waits for its copies and MMAs in flight
// (bounded), frees tensor memory and returns.
#include "kernels.cuh"
#include "ptx.cuh"
#include "tiles.cuh"

#include <cuda_bf16.h>

namespace moe {

namespace {

constexpr int kBEpiWarps = 8;
constexpr int kBThreads = 32 * (3 + kBEpiWarps);
constexpr int kBProdB = 2 + kBEpiWarps;           // producer warp of the B operand
constexpr int kBBK = 64;                          // K per stage
constexpr int kBT = 128;                          // tile M (tensor-memory lanes)
constexpr int kBN = 256;                          // tile N (columns)
constexpr int kBABytes = kBT * kBBK * 2;          // 16 KB of A per stage
constexpr int kBBBytes = kBN * kBBK * 2;          // 32 KB of B per stage
constexpr int kBStage = kBABytes + kBBBytes;
constexpr int kBStages = 4;
constexpr uint32_t kBChunk = kBBK * 128;          // one 64-wide MN chunk: 64 K rows x 128 B
constexpr int kBBarBytes = 256;
constexpr int kBEpiBytes = kBEpiWarps * 32 * 32 * 4;  // per-warp [32 columns][32 features] fp32
constexpr int kBSmem = 1024 + kBStages * kBStage + kBEpiBytes + kBBarBytes;
constexpr int kBTmemCols = 2 * kBN;
static_assert(kBSmem <= 232448, "shared memory budget");

struct BTile {
    int prob, grp, m0, n0, nvalid, k0, k1;
};

__device__ __forceinline__ int bprob_tiles(const BwdProblem& p) {
    const int mt = (p.M + kBT - 1) / kBT;
    if (p.rows_as_k) return p.n_grp * mt * ((p.N + kBN - 1) / kBN);
    if (p.seg == nullptr) return mt * ((p.n_rows + kBN - 1) / kBN);
    return mt * __ldg(p.tstart + p.n_grp);
}

__device__ __forceinline__ int btotal(const BwdParams& P) {
    int n = 0;
    for (int i = 0; i < P.n_problems; ++i) n += bprob_tiles(P.p[i]);
    return n;
}

// Tile t of the launch.  Order inside a problem: group, feature tile, then
// row (or column) tile, so that CTAs working at once share operand tiles in L2.
__device__ __forceinline__ bool btile_at(const BwdParams& P, int t, BTile& o) {
    for (int pi = 0; pi < P.n_problems; ++pi) {
        const BwdProblem& p = P.p[pi];
        const int n = bprob_tiles(p);
        if (t >= n) {
            t -= n;
            continue;
        }
        const int mt = (p.M + kBT - 1) / kBT;
        o.prob = pi;
        if (p.rows_as_k) {
            const int nt = (p.N + kBN - 1) / kBN;
            const int g = t / (mt * nt);
            const int l = t - g * mt * nt;
            o.grp = g;
            o.m0 = (l / nt) * kBT;
            o.n0 = (l % nt) * kBN;
            o.nvalid = min(kBN, p.N - o.n0);
            o.k0 = p.seg ? __ldg(p.seg + g) : 0;
            o.k1 = p.seg ? __ldg(p.seg + g + 1) : p.n_rows;
        } else if (p.seg == nullptr) {
            const int nt = (p.n_rows + kBN - 1) / kBN;
            o.grp = 0;
            o.m0 = (t / nt) * kBT;
            o.n0 = (t % nt) * kBN;
            o.nvalid = min(kBN, p.n_rows - o.n0);
            o.k0 = 0;
            o.k1 = p.K;
        } else {
            // largest group g with mt * tstart[g] <= t (a group with no rows has no tiles)
            int lo = 0, hi = p.n_grp - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (mt * __ldg(p.tstart + mid) <= t) lo = mid; else hi = mid - 1;
            }
            const int g = lo;
            const int l = t - mt * __ldg(p.tstart + g);
            const int ntg = __ldg(p.tstart + g + 1) - __ldg(p.tstart + g);
            o.grp = g;
            o.m0 = (l / ntg) * kBT;
            o.n0 = __ldg(p.seg + g) + (l % ntg) * kBN;
            o.nvalid = min(kBN, __ldg(p.seg + g + 1) - o.n0);
            o.k0 = 0;
            o.k1 = p.K;
        }
        return true;
    }
    return false;
}

__device__ __forceinline__ int bk_blocks(const BTile& t) {
    return t.k1 > t.k0 ? (t.k1 - t.k0 + kBBK - 1) / kBBK : 0;
}

// One operand of one stage: a K-major box {64 K, 128 rows} at (k, row0 + mn0)
// of a 2-D map, or an MN-major box {64, 64 K, 2 chunks} at (0, row0 + k,
// mn0 / 64) of the 3-D view {64, rows, MN / 64} (chunk c lands kBChunk bytes
// after chunk c - 1).
__device__ __forceinline__ void load_operand(uint8_t* dst, const CUtensorMap* m, int mn_major,
                                             int mn0, int k, int row0, uint64_t* bar) {
    if (!mn_major)
        tma_load_2d(dst, m, bar, k, row0 + mn0);
    else
        tma_load_3d(dst, m, bar, 0, row0 + k, mn0 >> 6);
}

// Descriptor of the 16-deep K slice kk of an operand stage.
__device__ __forceinline__ uint64_t op_desc(uint32_t base, int mn_major, int kk) {
    return mn_major ? smem_desc_mn_sw128(base + kk * 16 * 128, kBChunk, 1024)
                    : smem_desc_k_sw128(base + kk * 32);
}

__device__ __forceinline__ uint16_t f2bf(float v) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

}  // namespace

template <int EPI>
__global__ void __launch_bounds__(kBThreads, 1) bwd_gemm_kernel(const __grid_constant__ BwdParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    float* epi_smem = reinterpret_cast<float*>(smem + kBStages * kBStage);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBStages * kBStage + kBEpiBytes);
    uint64_t* empty = full + kBStages;
    uint64_t* tfull = empty + kBStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kBStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kBEpiWarps);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        for (int pi = 0; pi < P.n_problems; ++pi) {
            tma_prefetch_desc(&P.p[pi].ta);
            tma_prefetch_desc(&P.p[pi].tb);
            if (!P.p[pi].rows_as_k && !P.p[pi].b_mn) tma_prefetch_desc(&P.p[pi].tb_half);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kBTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int ntiles = btotal(P);

    if (warp == 0 || warp == kBProdB) {
        // ------------------------------------------------ TMA producers
        // Warp 0 loads A and sets the stage's expected bytes (both operands);
        // warp kBProdB loads B.  A copy that lands before the expectation is
        // set leaves the barrier's phase open: warp 0's arrival is pending.
        if (lane == 0) {
            const bool pa = warp == 0;
            int s = 0;
            uint32_t ph = 0, issued = 0, last_ph = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
                BTile tl;
                btile_at(P, t, tl);
                const BwdProblem& p = P.p[tl.prob];
                const int nkb = bk_blocks(tl);
                const int arow = p.rows_as_k ? 0 : tl.grp * p.a_grp_rows;
                // a row tile with at most 128 valid rows loads a 128-row B box
                const bool bhalf = !p.rows_as_k && !p.b_mn && tl.nvalid <= kBN / 2;
                const uint32_t stage_bytes = kBABytes + (bhalf ? kBBBytes / 2 : kBBBytes);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!wait_bar(&empty[s], ph ^ 1, abort_flag, P.status)) { ok = false; break; }
                    uint8_t* st = smem + s * kBStage;
                    const int k = tl.k0 + kb * kBBK;
                    if (pa) {
                        mbar_arrive_expect_tx(&full[s], stage_bytes);
                        load_operand(st, &p.ta, p.a_mn, tl.m0, k, arow, &full[s]);
                    } else {
                        load_operand(st + kBABytes, bhalf ? &p.tb_half : &p.tb, p.b_mn, tl.n0, k, 0,
                                     &full[s]);
                    }
                    issued |= 1u << s;
                    last_ph = (last_ph & ~(1u << s)) | (ph << s);
                    if (++s == kBStages) { s = 0; ph ^= 1; }
                }
            }
            // leave no copy in flight: warp 0 waits for the last fill of every
            // stage, which counts both producers' copies
            if (pa)
                for (int i = 0; i < kBStages; ++i)
                    if (issued >> i & 1u) wait_bar(&full[i], last_ph >> i & 1u, abort_flag, P.status, true);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int s = 0, buf = 0;
            uint32_t ph = 0, aph = 0;
            bool ok = true, any = false;
            for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
                BTile tl;
                btile_at(P, t, tl);
                const BwdProblem& p = P.p[tl.prob];
                const int nkb = bk_blocks(tl);
                // N: the tile's valid columns rounded up to 16 (an M = 128 MMA
                // takes N in steps of 16), so a ragged row tile pays only for its rows
                const uint32_t idesc = idesc_bf16_f32_major(kBT, min(kBN, (tl.nvalid + 15) & ~15),
                                                            p.a_mn, p.b_mn);
                if (!wait_bar(&tempty[buf], aph ^ 1, abort_flag, P.status)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + buf * kBN;
                bool first = true;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!wait_bar(&full[s], ph, abort_flag, P.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_addr(smem + s * kBStage);
                    const int krem = tl.k1 - (tl.k0 + kb * kBBK);  // rows of K left in the range
#pragma unroll
                    for (int kk = 0; kk < kBBK / 16; ++kk) {
                        if (16 * kk < krem) {
                            tc_mma_f16(d, op_desc(st, p.a_mn, kk), op_desc(st + kBABytes, p.b_mn, kk),
                                       idesc, first ? 0u : 1u);
                            first = false;
                        }
                    }
                    tc_commit(&empty[s]);
                    any = true;
                    if (++s == kBStages) { s = 0; ph ^= 1; }
                }
                if (!ok) break;
                // a tile with an empty K range issues no MMA: the commit then
                // only orders it after the earlier tiles, and the epilogue
                // writes zeros without reading tensor memory
                tc_commit(&tfull[buf]);
                any = true;
                if (++buf == 2) { buf = 0; aph ^= 1; }
            }
            if (any) {
                tc_commit(mma_done);
                wait_bar(mma_done, 0, abort_flag, P.status, true);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;           // tensor-memory lane quadrant of this warp
        const int half = (warp - 2) >> 2;  // columns [64 half, 64 half + 64) of a tile
        float* stg = epi_smem + (warp - 2) * 32 * 32;
        int buf = 0;
        uint32_t aph = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
            BTile tl;
            btile_at(P, t, tl);
            const BwdProblem& p = P.p[tl.prob];
            if (!wait_bar(&tfull[buf], aph, abort_flag, P.status)) break;
            tc_fence_after();
            const bool has_k = bk_blocks(tl) > 0;
            const int m = tl.m0 + q * 32 + lane;
            const bool mok = m < p.M;
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + buf * kBN;
            const int cend = min(tl.nvalid, (kBN / 2) * half + kBN / 2);
            if (EPI == BEPI_STORE) {
                const size_t obase = (size_t)tl.grp * (size_t)p.out_grp;
                const int mq = tl.m0 + q * 32;  // first feature of this warp's 32
                for (int c0 = (kBN / 2) * half; c0 < cend; c0 += 32) {
                    uint32_t r[32];
                    if (has_k) {
                        tmem_ld_32(tbase + c0, r);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) r[j] = 0u;
                    }
                    // transpose: stg[column j][feature lane]
#pragma unroll
                    for (int j = 0; j < 32; ++j) stg[j * 32 + lane] = __uint_as_float(r[j]);
                    __syncwarp();
                    if (p.out_f32) {
                        // 8 lanes write one column's 32 features (128 B) as 16-byte chunks
                        float* out = reinterpret_cast<float*>(p.out) + obase;
#pragma unroll
                        for (int it = 0; it < 8; ++it) {
                            const int row = 4 * it + (lane >> 3), ch = lane & 7;
                            if (c0 + row < tl.nvalid && mq + 4 * ch < p.M)
                                *reinterpret_cast<float4*>(out + (size_t)(tl.n0 + c0 + row) * p.ld_out +
                                                           mq + 4 * ch) =
                                    *reinterpret_cast<const float4*>(stg + row * 32 + 4 * ch);
                        }
                    } else {
                        // 4 lanes write one column's 32 features (64 B) as 8 bf16 each
                        uint16_t* out = reinterpret_cast<uint16_t*>(p.out) + obase;
#pragma unroll
                        for (int it = 0; it < 4; ++it) {
                            const int row = 8 * it + (lane >> 2), ch = lane & 3;
                            if (c0 + row < tl.nvalid && mq + 8 * ch < p.M) {
                                const float* v = stg + row * 32 + 8 * ch;
                                uint32_t w4[4];
#pragma unroll
                                for (int h = 0; h < 4; ++h)
                                    w4[h] = (uint32_t)f2bf(v[2 * h]) | ((uint32_t)f2bf(v[2 * h + 1]) << 16);
                                *reinterpret_cast<uint4*>(out + (size_t)(tl.n0 + c0 + row) * p.ld_out +
                                                          mq + 8 * ch) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                            }
                        }
                    }
                    __syncwarp();
                }
            } else {
                // SwiGLU backward for 128 features i (lanes) of 32 rows at a
                // time: with da' = D[i, r] (before the routing weight w),
                //   a = SiLU(g) u,  da = w da',
                //   dg = da u sigma(g) (1 + g (1 - sigma(g))),  du = da SiLU(g),
                // and the routing-weight gradient's partial sum over this
                // warp's 32 features, sum_i a_i da'_i.
                for (int c0 = (kBN / 2) * half; c0 < cend; c0 += 32) {
                    uint32_t r[32];
                    if (has_k) {
                        tmem_ld_32(tbase + c0, r);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) r[j] = 0u;
                    }
                    float part[32];
                    // eight rows at a time: their pre-activations and weights are
                    // loaded (read-only path) before any of the eight rows' stores
#pragma unroll
                    for (int j0 = 0; j0 < 32; j0 += 8) {
                        float gv[8], uv[8], wv[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int row = tl.n0 + c0 + j0 + j;
                            const bool ok_rc = c0 + j0 + j < tl.nvalid && mok;
                            gv[j] = ok_rc ? __ldg(p.gu + (size_t)row * p.ld_gu + m) : 0.0f;
                            uv[j] = ok_rc ? __ldg(p.gu + (size_t)row * p.ld_gu + p.half + m) : 0.0f;
                            wv[j] = (ok_rc && p.row_w) ? __ldg(p.row_w + row) : 1.0f;
                        }
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int row = tl.n0 + c0 + j0 + j;
                            part[j0 + j] = 0.0f;
                            if (c0 + j0 + j < tl.nvalid && mok) {
                                const float da1 = __uint_as_float(r[j0 + j]);
                                const float g = gv[j], u = uv[j], w = wv[j];
                                const float sg = __fdividef(1.0f, 1.0f + __expf(-g));
                                const float sl = g * sg;
                                const float a = sl * u;
                                const float da = w * da1;
                                const float dg = da * u * sg * (1.0f + g * (1.0f - sg));
                                const float du = da * sl;
                                p.dgu[(size_t)row * p.ld_dgu + m] = f2bf(dg);
                                p.dgu[(size_t)row * p.ld_dgu + p.half + m] = f2bf(du);
                                p.aw[(size_t)row * p.ld_aw + m] = f2bf(w * a);
                                part[j0 + j] = a * da1;
                            }
                        }
                    }
                    if (p.dw_part) {
                        // butterfly reduce-scatter over the warp: afterwards lane L
                        // holds the sum over the 32 lanes of row c0 + L (fixed order)
#pragma unroll
                        for (int off = 16; off >= 1; off >>= 1) {
                            const bool hi = (lane & off) != 0;
#pragma unroll
                            for (int i = 0; i < off; ++i) {
                                const float send = hi ? part[i] : part[i + off];
                                const float keep = hi ? part[i + off] : part[i];
                                part[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                            }
                        }
                        if (c0 + lane < tl.nvalid)
                            p.dw_part[(size_t)(tl.n0 + c0 + lane) * p.ld_dw + (tl.m0 >> 5) + q] = part[0];
                    }
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
    if (warp == 1) tmem_dealloc(tmem_base, kBTmemCols);
}

template <int EPI>
static cudaError_t launch_bwd_t(const BwdParams& params, int grid, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(bwd_gemm_kernel<EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kBSmem);
    if (e != cudaSuccess) return e;
    bwd_gemm_kernel<EPI><<<grid, kBThreads, kBSmem, s>>>(params);
    return cudaGetLastError();
}

cudaError_t launch_bwd_gemm(int epi, const BwdParams& params, int grid, cudaStream_t s) {
    if (params.n_problems < 1 || params.n_problems > kBwdMaxProblems) return cudaErrorInvalidValue;
    if (grid < 1) grid = 1;
    if (epi == BEPI_STORE) return launch_bwd_t<BEPI_STORE>(params, grid, s);
    if (epi == BEPI_DSWIGLU) return launch_bwd_t<BEPI_DSWIGLU>(params, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace moe
