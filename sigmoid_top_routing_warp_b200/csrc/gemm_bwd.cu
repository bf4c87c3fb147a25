// gemm_bwd.cu -- the grouped GEMMs of the layer's backward pass on CTA pairs
// (tcgen05 cta_group::2): K- or MN-major operands, token rows along N or K
// over an expert's row segment, a 256 x 256 tile over two SMs.
//
// Source of the operation: the chain rule through the forward pass of
// "Xiaohongshu dots3 note Open Source Deep Dive" §3.1 / §8.2 (see
// backward.cu), the expert choice held fixed.
//
// Why pairs.  A CTA of the pair stages its own 128 rows of A and half of the
// tile's N columns of B: 32 KB per 64-deep K step for 2 M MACs, where a
// single-CTA 128 x 256 tile needs 48 KB for the same work, and five or six
// stages fit in shared memory instead of four.  The leader issues one
// M = 256 MMA per 16-deep K slice; its commits arrive on both CTAs' barriers.
// D[m, n] sits in the tensor memory of the CTA that owns row m: each CTA's
// epilogue writes its 128 rows.
//
// N per tile: token rows (K-major B) use the tile's valid rows rounded up to
// 16, each CTA supplying half of them from the smallest of its 16-, 32-, 64-
// or 128-row boxes that holds them; output columns (MN-major B) use 256.
//
// Roles per CTA (352 threads): warp 0 loads A and (leader) sets the stage's
// expected bytes for both CTAs, warp 1 loads B, warp 2 holds the tensor
// memory and (leader, one thread) issues the MMAs, warps 3..10 are the
// epilogue (two per lane quadrant, half the columns each; staged tiles leave
// in bulk tensor stores, or the SwiGLU backward in registers).  Static
// round-robin of tiles over pairs.
// Every wait is bounded; on timeout a CTA records DEV_STATUS_TIMEOUT, stops,
// drains what it issued, meets its peer at the last cluster barrier and
// frees its tensor memory.
#include "kernels.cuh"
#include "ptx.cuh"

#include <cuda_bf16.h>

namespace moe {

namespace {

constexpr int kQEpiWarps = 8;
constexpr int kQThreads = 32 * (3 + kQEpiWarps);
constexpr int kQMmaWarp = 2;                       // warps 0, 1 load; 2 issues; 3..10 drain
constexpr int kQEpi0 = kQMmaWarp + 1;
constexpr int kQBK = 64;
constexpr int kQM = 256;                           // pair tile M (128 rows per CTA)
constexpr int kQN = 256;                           // tile N (128 per CTA staged)
constexpr int kQOpBytes = 128 * kQBK * 2;          // 16 KB: A or the CTA's half of B
constexpr int kQStage = 2 * kQOpBytes;
constexpr uint32_t kQChunk = kQBK * 128;           // one 64-wide MN chunk: 64 K rows x 128 B
constexpr int kQBarBytes = 256;
constexpr int kQTmemCols = 2 * kQN;
constexpr long long kQWaitLimit = 1ll << 31;
// the launch passes every problem's tensor maps by value (4.75 KB for
// five problems): within the 32,764-byte kernel parameter limit of sm_70+
// with CUDA 12.1 and later
static_assert(sizeof(BwdParams) <= 32764, "kernel parameter size");
// Shared memory per epilogue: stores keep five operand stages and two 4 KB
// staging tiles per epilogue warp; the SwiGLU backward needs no staging and
// takes six stages.
template <int EPI>
struct QCfg {
    static constexpr int STAGES = EPI == BEPI_DSWIGLU ? 6 : 5;
    static constexpr int SBUF = EPI == BEPI_DSWIGLU ? 0 : 2;
    static constexpr int EPI_BYTES = kQEpiWarps * SBUF * 4096;
    static constexpr int SMEM = 1024 + STAGES * kQStage + EPI_BYTES + kQBarBytes;
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct QTile {
    int prob, grp, m0, n0, nvalid, k0, k1;
};

__device__ __forceinline__ int qprob_tiles(const BwdProblem& p) {
    const int mt = (p.M + kQM - 1) / kQM;
    if (p.rows_as_k) return p.n_grp * mt * ((p.N + kQN - 1) / kQN);
    if (p.seg == nullptr) return mt * ((p.n_rows + kQN - 1) / kQN);
    return mt * __ldg(p.tstart + p.n_grp);
}

__device__ __forceinline__ int qtotal(const BwdParams& P) {
    int n = 0;
    for (int i = 0; i < P.n_problems; ++i) n += qprob_tiles(P.p[i]);
    return n;
}

// Tile t: group, N tile, then M tile innermost.  With token rows along N the
// pairs running together share a tile of token rows while the group's
// weights (at most a few tens of MB) stay in L2 across its row tiles.  With
// rows as K (weight gradients, out[n][m], m contiguous) the pairs running
// together write adjacent column ranges of the same output rows, so the
// fp32 gradients reach DRAM as runs of whole rows rather than 1 KB pieces.
__device__ __forceinline__ void qtile_at(const BwdParams& P, int t, QTile& o) {
    for (int pi = 0; pi < P.n_problems; ++pi) {
        const BwdProblem& p = P.p[pi];
        const int n = qprob_tiles(p);
        if (t >= n) {
            t -= n;
            continue;
        }
        const int mt = (p.M + kQM - 1) / kQM;
        o.prob = pi;
        if (p.rows_as_k) {
            const int nt = (p.N + kQN - 1) / kQN;
            const int g = t / (mt * nt);
            const int l = t - g * mt * nt;
            o.grp = g;
            o.m0 = (l % mt) * kQM;
            o.n0 = (l / mt) * kQN;
            o.nvalid = min(kQN, p.N - o.n0);
            o.k0 = p.seg ? __ldg(p.seg + g) : 0;
            o.k1 = p.seg ? __ldg(p.seg + g + 1) : p.n_rows;
        } else if (p.seg == nullptr) {
            o.grp = 0;
            o.m0 = (t % mt) * kQM;
            o.n0 = (t / mt) * kQN;
            o.nvalid = min(kQN, p.n_rows - o.n0);
            o.k0 = 0;
            o.k1 = p.K;
        } else {
            int g;
            if (p.ttab != nullptr) {
                g = __ldg(p.ttab + t / mt);
            } else {
                int lo = 0, hi = p.n_grp - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (mt * __ldg(p.tstart + mid) <= t) lo = mid; else hi = mid - 1;
                }
                g = lo;
            }
            const int l = t - mt * __ldg(p.tstart + g);
            o.grp = g;
            o.m0 = (l % mt) * kQM;
            o.n0 = __ldg(p.seg + g) + (l / mt) * kQN;
            o.nvalid = min(kQN, __ldg(p.seg + g + 1) - o.n0);
            o.k0 = 0;
            o.k1 = p.K;
        }
        return;
    }
}

__device__ __forceinline__ int qk_blocks(const QTile& t) {
    return t.k1 > t.k0 ? (t.k1 - t.k0 + kQBK - 1) / kQBK : 0;
}

// MMA N of a tile: token rows (K-major B) trimmed to the valid rows rounded
// up to 16; output columns (MN-major B, whose halves must start on a 64-wide
// chunk) the full 256.
__device__ __forceinline__ int qtile_n(const BwdProblem& p, const QTile& t) {
    return p.b_mn ? kQN : min(kQN, (t.nvalid + 15) & ~15);
}

__device__ __forceinline__ bool qwait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                      int* status, bool drain = false) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait_cluster(bar, parity)) return true;
        if (!drain && *abort_flag) return false;
        if (clock64() - t0 > kQWaitLimit) {
            *abort_flag = 1;
            if (status) atomicOr(status, DEV_STATUS_TIMEOUT);
            return false;
        }
    }
}

// One operand half of one stage into this CTA's shared memory, counted on
// the leader's barrier: K-major box {64 K, 128 rows} at (k, row0 + mn0), or
// MN-major box {64, 64 K, 2 chunks} at (0, row0 + k, mn0 / 64).
__device__ __forceinline__ void qload(uint8_t* dst, const CUtensorMap* m, int mn_major, int mn0,
                                      int k, int row0, uint32_t bar_cluster) {
    if (!mn_major)
        tma_load_2d_pair(dst, m, bar_cluster, k, row0 + mn0);
    else
        tma_load_3d_pair(dst, m, bar_cluster, 0, row0 + k, mn0 >> 6);
}

__device__ __forceinline__ uint64_t qdesc(uint32_t base, int mn_major, int kk) {
    return mn_major ? smem_desc_mn_sw128(base + kk * 16 * 128, kQChunk, 1024)
                    : smem_desc_k_sw128(base + kk * 32);
}

__device__ __forceinline__ uint16_t qbf(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }

}  // namespace

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kQThreads, 1)
    bwd_pair_gemm_kernel(const __grid_constant__ BwdParams P) {
    using C = QCfg<EPI>;
    constexpr int kQStages = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    float* epi_smem = reinterpret_cast<float*>(smem + kQStages * kQStage);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kQStages * kQStage + C::EPI_BYTES);
    uint64_t* empty = full + kQStages;
    uint64_t* tfull = empty + kQStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t cta = cluster_ctarank();
    const bool leader = cta == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(&full[s], 1);    // the leader's A producer (expected bytes of both CTAs)
            mbar_init(&empty[s], 1);   // one multicast commit per phase
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);                 // one multicast commit per tile
            mbar_init(&tempty[b], 2 * kQEpiWarps);   // both CTAs' epilogue warps (leader's copy)
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        for (int pi = 0; pi < P.n_problems; ++pi) {
            tma_prefetch_desc(&P.p[pi].ta);
            tma_prefetch_desc(&P.p[pi].tb);
        }
    }
    if (warp == kQMmaWarp) {
        tmem_alloc_pair(tmem_holder, kQTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int ntiles = qtotal(P);

    if (warp < kQMmaWarp) {
        // ------------------------------------------------ TMA producers (both CTAs)
        if (lane == 0) {
            const bool pa = warp == 0;
            const uint32_t full_leader = mapa_shared(smem_addr(&full[0]), 0);
            uint32_t it = 0;  // k-blocks of this CTA so far
            bool ok = true;
            for (int t = pair; ok && t < ntiles; t += npairs) {
                QTile tl;
                qtile_at(P, t, tl);
                const BwdProblem& p = P.p[tl.prob];
                const int nkb = qk_blocks(tl);
                const int arow = p.rows_as_k ? 0 : tl.grp * p.a_grp_rows;
                const int half = qtile_n(p, tl) >> 1;  // B columns each CTA supplies
                // K-major B: the smallest box of 16 << b rows that holds them
                int box = 3;
                if (!p.b_mn) {
                    box = 0;
                    while ((16 << box) < half) ++box;
                }
                const CUtensorMap* bmap = box == 3 ? &p.tb : &p.tbs[box];
                const uint32_t stage_bytes = kQOpBytes + (p.b_mn ? kQOpBytes : (16u << box) * 128u);
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = (int)(it % kQStages);
                    const uint32_t ph = (it / kQStages) & 1u;
                    if (!qwait(&empty[s], ph ^ 1, abort_flag, P.status)) { ok = false; break; }
                    uint8_t* st = smem + s * kQStage;
                    const int k = tl.k0 + kb * kQBK;
                    const uint32_t fb = full_leader + 8u * s;
                    if (pa) {
                        if (leader) mbar_arrive_expect_tx(&full[s], 2 * stage_bytes);
                        qload(st, &p.ta, p.a_mn, tl.m0 + 128 * (int)cta, k, arow, fb);
                    } else {
                        qload(st + kQOpBytes, bmap, p.b_mn, tl.n0 + half * (int)cta, k, 0, fb);
                    }
                }
            }
            // The leader's full barriers count both CTAs' copies: its A
            // producer waits for the last phase of every stage in use.
            if (leader && pa)
                for (uint32_t j = it > (uint32_t)kQStages ? it - kQStages : 0u; j < it; ++j)
                    qwait(&full[j % kQStages], (j / kQStages) & 1u, abort_flag, P.status, true);
        }
        __syncwarp();
    } else if (warp == kQMmaWarp) {
        // ------------------------------------------------ MMA issuer (leader only)
        if (leader && lane == 0) {
            int s = 0, buf = 0;
            uint32_t ph = 0, aph = 0;
            bool ok = true, any = false;
            for (int t = pair; ok && t < ntiles; t += npairs) {
                QTile tl;
                qtile_at(P, t, tl);
                const BwdProblem& p = P.p[tl.prob];
                const int nkb = qk_blocks(tl);
                const uint32_t idesc = idesc_bf16_f32_major(kQM, qtile_n(p, tl), p.a_mn, p.b_mn);
                if (!qwait(&tempty[buf], aph ^ 1, abort_flag, P.status)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + buf * kQN;
                bool first = true;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!qwait(&full[s], ph, abort_flag, P.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_addr(smem + s * kQStage);
                    const int krem = tl.k1 - (tl.k0 + kb * kQBK);
#pragma unroll
                    for (int kk = 0; kk < kQBK / 16; ++kk) {
                        if (16 * kk < krem) {
                            tc_mma_f16_pair(d, qdesc(st, p.a_mn, kk), qdesc(st + kQOpBytes, p.b_mn, kk),
                                            idesc, first ? 0u : 1u);
                            first = false;
                        }
                    }
                    tc_commit_pair(&empty[s], 0x3);
                    any = true;
                    if (++s == kQStages) { s = 0; ph ^= 1; }
                }
                if (!ok) break;
                // a tile with an empty K range issues no MMA; its epilogue writes zeros
                tc_commit_pair(&tfull[buf], 0x3);
                any = true;
                if (++buf == 2) { buf = 0; aph ^= 1; }
            }
            if (any) {
                tc_commit_pair(mma_done, 0x1);
                qwait(mma_done, 0, abort_flag, P.status, true);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        const int hw = (warp - kQEpi0) >> 2;  // columns [128 hw, 128 hw + 128)
        float* stgs = epi_smem + (warp - kQEpi0) * C::SBUF * 32 * 32;
        int sb = 0;  // staging tile of the next step
        const uint32_t tempty_leader = mapa_shared(smem_addr(&tempty[0]), 0);
        int buf = 0;
        uint32_t aph = 0;
        for (int t = pair; t < ntiles; t += npairs) {
            QTile tl;
            qtile_at(P, t, tl);
            const BwdProblem& p = P.p[tl.prob];
            if (!qwait(&tfull[buf], aph, abort_flag, P.status)) break;
            tc_fence_after();
            const bool has_k = qk_blocks(tl) > 0;
            const int mrow = tl.m0 + 128 * (int)cta;       // this CTA's first row of D
            const int m = mrow + q * 32 + lane;
            const bool mok = m < p.M;
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + buf * kQN;
            const int cend = min(tl.nvalid, 128 * hw + 128);
            if constexpr (EPI == BEPI_STORE) {
                // staged [rows][32 features] boxes leave in bulk tensor stores
                // from two alternating staging tiles.  Token-row tiles of a
                // padded segment store 16-row boxes that start below the
                // tile's valid rows (a multiple of 16); elsewhere one 32-row
                // box, which the map clips at the tensor's edge.
                const int mq = mrow + q * 32;
                const int g3 = p.rows_as_k ? tl.grp : 0;
                const bool rows16 = !p.rows_as_k && p.seg != nullptr;
                for (int c0 = 128 * hw; c0 < cend; c0 += 32) {
                    uint32_t r[32];
                    if (has_k) {
                        tmem_ld_32(tbase + c0, r);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) r[j] = 0u;
                    }
                    float* stg = stgs + sb * 1024;
                    uint16_t* stg16 = reinterpret_cast<uint16_t*>(stg);
                    if (lane == 0) bulk_wait_read<C::SBUF - 1>();  // this tile's last stores have read it
                    __syncwarp();
                    if (p.out_f32) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) stg[j * 32 + lane] = __uint_as_float(r[j]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) stg16[j * 32 + lane] = qbf(__uint_as_float(r[j]));
                    }
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        if (mq < p.M) {
                            if (!rows16) {
                                tma_store_3d(&p.to, stg, mq, tl.n0 + c0, g3);
                            } else {
#pragma unroll
                                for (int h = 0; h < 2; ++h)
                                    if (c0 + 16 * h < tl.nvalid)
                                        tma_store_3d(&p.to,
                                                     p.out_f32 ? static_cast<const void*>(stg + h * 512)
                                                               : static_cast<const void*>(stg16 + h * 512),
                                                     mq, tl.n0 + c0 + 16 * h, g3);
                            }
                        }
                        bulk_commit();  // one group per step, empty or not
                    }
                    if (++sb == C::SBUF) sb = 0;
                }
            } else {
                // SwiGLU backward: D[i, r] = da'_r[i] (the row's output gradient
                // times W2's column i, before the routing weight w_r) for this
                // CTA's 128 features i, 32 rows at a time.  With s = sigmoid(g),
                // a = SiLU(g) u and da = w_r da':
                //   dg = da u s (1 + g (1 - s)),  du = da SiLU(g),
                // stored bf16 with w_r a (the down weights' gradient operand);
                // the routing weight's gradient sum_i a_i da'_i goes out as
                // per-warp partials over 32 features
                for (int c0 = 128 * hw; c0 < cend; c0 += 32) {
                    uint32_t r[32];
                    if (has_k) {
                        tmem_ld_32(tbase + c0, r);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) r[j] = 0u;
                    }
                    float part[32];
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
                                p.dgu[(size_t)row * p.ld_dgu + m] = qbf(dg);
                                p.dgu[(size_t)row * p.ld_dgu + p.half + m] = qbf(du);
                                p.aw[(size_t)row * p.ld_aw + m] = qbf(w * a);
                                part[j0 + j] = a * da1;
                            }
                        }
                    }
                    // a quadrant past the problem's features (M not a multiple of
                    // 256) writes no partial: I is a multiple of 32
                    if (p.dw_part && mrow + 32 * q < p.M) {
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
                            p.dw_part[(size_t)(tl.n0 + c0 + lane) * p.ld_dw + (mrow >> 5) + q] = part[0];
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_leader + 8u * buf);
            if (++buf == 2) { buf = 0; aph ^= 1; }
        }
        if (EPI == BEPI_STORE && lane == 0) bulk_wait_all();
        __syncwarp();
    }

    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == kQMmaWarp) tmem_dealloc_pair(tmem_base, kQTmemCols);
}

template <int EPI>
static cudaError_t launch_bwd_pair_t(const BwdParams& params, int grid, cudaStream_t s) {
    constexpr int kQSmem = QCfg<EPI>::SMEM;
    cudaError_t e = cudaFuncSetAttribute(bwd_pair_gemm_kernel<EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kQThreads);
    cfg.dynamicSmemBytes = kQSmem;
    cfg.stream = s;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, bwd_pair_gemm_kernel<EPI>, &cfg) == cudaSuccess &&
        clusters > 0 && 2 * clusters < grid)
        grid = 2 * clusters;
    cudaGetLastError();
    bwd_pair_gemm_kernel<EPI><<<grid, kQThreads, kQSmem, s>>>(params);
    return cudaGetLastError();
}

cudaError_t launch_bwd_gemm(int epi, const BwdParams& params, int grid, cudaStream_t s) {
    if (params.n_problems < 1 || params.n_problems > kBwdMaxProblems) return cudaErrorInvalidValue;
    grid &= ~1;
    if (grid < 2) grid = 2;
    if (epi == BEPI_STORE) return launch_bwd_pair_t<BEPI_STORE>(params, grid, s);
    if (epi == BEPI_DSWIGLU) return launch_bwd_pair_t<BEPI_DSWIGLU>(params, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace moe
