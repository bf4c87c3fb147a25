// gemm_pair.cu -- the grouped expert GEMMs for prefill-sized batches on CTA
// pairs (tcgen05 cta_group::2).  Steps a6 (gate/up + SwiGLU), a7 (down x
// routing weight) and a8 (the shared expert as a second problem).
//
// Source of the operation: "Xiaohongshu dots3 note Open Source Deep Dive",
// §8.2 (FUSED_MC2: gmm1 -> swiglu -> gmm2); "Transformers 中的 dots.llm1
// （Dots1）模型" (blog.gitcode.com), parallel-plan paragraph (packed
// gate_up_proj; experts as grouped_gemm).
//
// A cluster of two CTAs computes one 256 x 256 tile: 256 weight rows (128 in
// each CTA's shared memory and tensor memory) by 256 tokens (128 token rows
// staged by each CTA), one M = 256 MMA per 16-wide K step issued by the
// leader CTA.  Per CTA and K step that is 32 KB of operands for 2 M MACs,
// twice the reuse of a single-CTA 128 x 128 tile.
//
// Gate/up layout: a 5-D TMA view loads the packed [gate; up] matrix so that
// the 128 weight rows of a CTA alternate 8 gate rows and the 8 up rows of the
// same features.  tcgen05.ld.16x256b then hands every epilogue thread the gate
// value (lane r) and the up value (lane r + 8) of one feature, and SwiGLU is
// computed in registers.
//
// Epilogue: tensor memory -> registers -> global stores.  The gate/up GEMM
// stores its SwiGLU outputs straight from registers, which frees the shared
// memory of a seventh operand stage (2.41-2.47 -> 2.34 ms at prefill); the
// down GEMM, whose output is four times larger, goes through per-warp
// shared-memory transposes for 16-byte stores of whole token rows (stored
// straight from registers it took twice as long).  Two accumulator buffers
// (2 x 256 columns) let the epilogue of one tile overlap the main loop of the
// next.
//
// Gate/up tiles are claimed at run time: the leader's weight producer takes the next
// tile index from a counter in the workspace status block and posts it to
// both CTAs' 4-slot rings (a remote store and a remote arrive); every role of
// both CTAs reads it there and releases the slot on the leader.  The last CTA
// to finish resets the counter (the workspace starts zero-filled).  The down
// GEMM keeps a static round-robin over the pairs.
//
// Every wait is bounded (see wait_cl); on timeout the CTA records
// DEV_STATUS_TIMEOUT, stops, drains its in-flight copies and MMAs (bounded),
// meets its peer at the final cluster barrier and frees tensor memory.
#include "kernels.cuh"
#include "ptx.cuh"

#include <cuda_bf16.h>

namespace moe {

namespace {

constexpr int kPThreads = 224;                     // 7 warps
constexpr int kPTokWarp = 6;                       // token-tile producer
constexpr int kPBK = 64;
constexpr int kPHalf = kPairTokens / 2;            // token rows per CTA
constexpr int kPWBytes = 128 * kPBK * 2;           // 16 KB of weights per CTA
constexpr int kPXBytes = kPHalf * kPBK * 2;        // 16 KB of tokens per CTA
constexpr int kPStage = kPWBytes + kPXBytes;       // 32 KB
constexpr int kPBarBytes = 256;
// The gate/up GEMM stores its SwiGLU outputs straight from registers and
// gives the operand ring a seventh stage; the down GEMM's larger output goes
// through per-warp shared-memory transposes (16-byte stores), six stages.
template <int EPI>
struct PCfg {
    static constexpr int STAGES = EPI == EPI_SWIGLU ? 7 : 6;
    static constexpr int EPI_BYTES = EPI == EPI_SWIGLU ? 0 : 4 * 4096;
    static constexpr int SMEM = 1024 + STAGES * kPStage + EPI_BYTES + kPBarBytes;
    static_assert(SMEM <= 232448, "shared memory budget");
};
constexpr int kPTmemCols = 2 * kPairTokens;        // two 256-column accumulators
constexpr long long kPWaitLimit = 1ll << 31;
constexpr int kPRing = 4;                          // claimed tile ids in flight
constexpr int kPSchedWord = 32;                    // first scheduling word in the status block
// consumers of a ring slot: both CTAs' two producers and 4 epilogue warps, and
// the leader's MMA thread
constexpr int kPRingReaders = 2 * (2 + 4) + 1;

struct PTile {
    int prob, exp, row0, nvalid, f0;
};

// MMA width of a tile: its valid tokens rounded up to 16 (the M = 256 MMA
// takes N in steps of 16); each CTA of the pair supplies N/2 token rows.
__device__ __forceinline__ int tile_n(int nvalid) {
    return min(kPairTokens, (nvalid + 15) & ~15);
}

template <int EPI>
__device__ __forceinline__ int feat_tile() { return EPI == EPI_SWIGLU ? 128 : 256; }

template <int EPI>
__device__ __forceinline__ int ptiles(const PairProblem& p) {
    const int nf = (p.n_feat + feat_tile<EPI>() - 1) / feat_tile<EPI>();
    if (p.seg == nullptr) return nf * ((p.n_rows + kPairTokens - 1) / kPairTokens);
    return nf * __ldg(p.tok_start + p.n_exp);
}

template <int EPI>
__device__ __forceinline__ bool ptile_at(const PairParams& P, int t, PTile& o) {
    for (int pi = 0; pi < P.n_problems; ++pi) {
        const PairProblem& p = P.p[pi];
        const int n = ptiles<EPI>(p);
        if (t >= n) {
            t -= n;
            continue;
        }
        const int nf = (p.n_feat + feat_tile<EPI>() - 1) / feat_tile<EPI>();
        int e = 0, first = 0, ntok, seg0, seg1;
        if (p.seg != nullptr && p.tok_tiles != nullptr) {
            // feature tile innermost: t = token tile * nf + feature tile
            const int j = t / nf;
            const int4 info = __ldg(p.tok_tiles + j);
            o.prob = pi;
            o.exp = info.x;
            o.f0 = (t - j * nf) * feat_tile<EPI>();
            o.row0 = info.y;
            o.nvalid = info.z;
            return true;
        }
        if (p.seg == nullptr) {
            ntok = (p.n_rows + kPairTokens - 1) / kPairTokens;
            seg0 = 0;
            seg1 = p.n_rows;
        } else {
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
        // feature tile innermost: the tiles running together share one token
        // tile, and the expert's weights stay in L2 across its token tiles
        const int local = t - first;
        const int tt = local / nf, ft = local - tt * nf;
        (void)ntok;
        o.prob = pi;
        o.exp = e;
        o.f0 = ft * feat_tile<EPI>();
        o.row0 = seg0 + tt * kPairTokens;
        o.nvalid = min(kPairTokens, seg1 - o.row0);
        return true;
    }
    return false;
}

template <int EPI>
__device__ __forceinline__ int ptotal(const PairParams& P) {
    int n = 0;
    for (int pi = 0; pi < P.n_problems; ++pi) n += ptiles<EPI>(P.p[pi]);
    return n;
}

// Bounded wait with cluster-scope acquire (arrivals come from the peer CTA
// and from the pair's tensor-core commits).
__device__ __forceinline__ bool wait_cl(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                        int* status, bool drain = false) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait_cluster(bar, parity)) return true;
        if (!drain && *abort_flag) return false;
        if (clock64() - t0 > kPWaitLimit) {
            *abort_flag = 1;
            if (status) atomicOr(status, DEV_STATUS_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

// Store a word into the shared memory of a CTA of the cluster (shared::cluster address).
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

}  // namespace

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPThreads, 1)
    pair_gemm_kernel(const __grid_constant__ PairParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    constexpr int kPStages = PCfg<EPI>::STAGES;
    uint8_t* epi_buf = smem + kPStages * kPStage;
    uint64_t* full = reinterpret_cast<uint64_t*>(epi_buf + PCfg<EPI>::EPI_BYTES);
    uint64_t* empty = full + kPStages;
    uint64_t* tfull = empty + kPStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* mma_done = tempty + 2;
    uint64_t* rfull = mma_done + 1;          // [kPRing] a claimed tile id is in this CTA's ring
    uint64_t* rempty = rfull + kPRing;       // [kPRing] read by every reader of both CTAs (leader's copy used)
    int* ring = reinterpret_cast<int*>(rempty + kPRing);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(ring + kPRing);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t cta = cluster_ctarank();
    const bool leader = cta == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    // gate/up claims tiles at run time; the down GEMM keeps a static
    // round-robin over the pairs (run-time claims made it ~6 % slower)
    constexpr bool kClaim = EPI == EPI_SWIGLU;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&full[s], 1);    // the leader's producer (expect_tx of both CTAs)
            mbar_init(&empty[s], 1);   // one multicast commit per phase
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);   // one multicast commit per tile
            mbar_init(&tempty[b], 8);  // 4 epilogue warps x 2 CTAs (leader's copy used)
        }
        mbar_init(mma_done, 1);
        for (int r = 0; r < kPRing; ++r) {
            mbar_init(&rfull[r], 1);                // the leader's claimer
            mbar_init(&rempty[r], kPRingReaders);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        for (int pi = 0; pi < P.n_problems; ++pi) {
            tma_prefetch_desc(&P.p[pi].tw);
            for (int b = 0; b < kPairBoxes; ++b) tma_prefetch_desc(&P.p[pi].tx[b]);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, kPTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int ntiles = ptotal<EPI>(P);
    // tile claim counter and finished-CTA count (workspace status block)
    int* sched = P.status + kPSchedWord + 2 * EPI;
    const uint32_t rempty_leader = mapa_shared(smem_addr(&rempty[0]), 0);
    // the next claimed tile of the pair: waits for its slot, reads the id and
    // releases the slot on the leader
    auto next_tile = [&](int& rs, uint32_t& rph, int& t) -> bool {
        if (!kClaim) {  // rs counts this role's tiles
            t = pair + rs * npairs;
            ++rs;
            if (t >= ntiles) t = -1;
            return true;
        }
        if (!wait_cl(&rfull[rs], rph, abort_flag, P.status)) return false;
        t = ring[rs];
        __syncwarp(__activemask());  // every lane has read the id before lane 0 releases it
        if ((threadIdx.x & 31) == 0) mbar_arrive_cluster(rempty_leader + 8u * rs);
        if (++rs == kPRing) { rs = 0; rph ^= 1; }
        return true;
    };

    if (warp == 0 || warp == kPTokWarp) {
        // ---------------------------------------------------- TMA producers (both CTAs)
        // Warp 0 loads the weight tiles, warp kPTokWarp the token tiles: one
        // issuing thread tops out near 40 B/clk of 16 KB tensor copies, two
        // reach the SM's L2 bandwidth.  Both count on the leader's full
        // barrier; the leader's weight producer sets its expected bytes.
        if (lane == 0) {
            const bool wprod = warp == 0;
            const uint32_t full_leader = mapa_shared(smem_addr(&full[0]), 0);
            int s = 0;
            uint32_t ph = 0, issued = 0, last_ph = 0;
            bool ok = true;
            const bool claimer = leader && wprod;
            const uint32_t ring_peer = mapa_shared(smem_addr(&ring[0]), 1);
            const uint32_t rfull_peer = mapa_shared(smem_addr(&rfull[0]), 1);
            int rs = 0, cs = 0;
            uint32_t rph = 0, cph = 0;
            while (ok) {
                if (kClaim && claimer) {
                    // claim the next tile for the pair and post it to both CTAs
                    int c = atomicAdd(&sched[0], 1);
                    if (c >= ntiles) c = -1;
                    if (!wait_cl(&rempty[cs], cph ^ 1, abort_flag, P.status)) { ok = false; break; }
                    ring[cs] = c;
                    st_cluster_u32(ring_peer + 4u * cs, (uint32_t)c);
                    mbar_arrive(&rfull[cs]);
                    mbar_arrive_cluster(rfull_peer + 8u * cs);
                    if (++cs == kPRing) { cs = 0; cph ^= 1; }
                }
                int t;
                if (!next_tile(rs, rph, t)) { ok = false; break; }
                if (t < 0) break;
                PTile tl;
                ptile_at<EPI>(P, t, tl);
                const PairProblem& p = P.p[tl.prob];
                const int nk = p.K / kPBK;
                const int half = tile_n(tl.nvalid) >> 1;  // token rows this CTA feeds the MMA
                int box = 0;
                while ((16 << box) < half) ++box;
                const uint32_t stage_bytes = kPWBytes + (16u << box) * kPBK * 2;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!wait_cl(&empty[s], ph ^ 1, abort_flag, P.status)) { ok = false; break; }
                    uint8_t* st = smem + s * kPStage;
                    const uint32_t fb = full_leader + 8u * s;
                    if (wprod) {
                        if (leader) mbar_arrive_expect_tx(&full[s], 2 * stage_bytes);
                        if (EPI == EPI_SWIGLU)
                            tma_load_5d_pair(st, &p.tw, fb, kb * kPBK, 0, 0,
                                             (tl.f0 + 64 * (int)cta) >> 3, tl.exp);
                        else
                            tma_load_2d_pair(st, &p.tw, fb, kb * kPBK,
                                             tl.exp * p.n_feat + tl.f0 + 128 * (int)cta);
                    } else {
                        tma_load_2d_pair(st + kPWBytes, &p.tx[box], fb, kb * kPBK,
                                         tl.row0 + half * (int)cta);
                    }
                    issued |= 1u << s;
                    last_ph = (last_ph & ~(1u << s)) | (ph << s);
                    if (++s == kPStages) { s = 0; ph ^= 1; }
                }
            }
            // The leader's full barriers count both CTAs' copies (weights and
            // tokens): its weight producer drains them.
            if (leader && wprod)
                for (int i = 0; i < kPStages; ++i)
                    if (issued >> i & 1u) wait_cl(&full[i], last_ph >> i & 1u, abort_flag, P.status, true);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer (leader only)
        if (leader && lane == 0) {
            int s = 0, buf = 0;
            uint32_t ph = 0, aph = 0;
            bool ok = true, any = false;
            int rs = 0;
            uint32_t rph = 0;
            while (ok) {
                int t;
                if (!next_tile(rs, rph, t) || t < 0) break;
                PTile tl;
                ptile_at<EPI>(P, t, tl);
                const int nk = P.p[tl.prob].K / kPBK;
                const uint32_t idesc = idesc_bf16_f32(256, tile_n(tl.nvalid));
                if (!wait_cl(&tempty[buf], aph ^ 1, abort_flag, P.status)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + buf * kPairTokens;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!wait_cl(&full[s], ph, abort_flag, P.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_addr(smem + s * kPStage);
#pragma unroll
                    for (int kk = 0; kk < kPBK / 16; ++kk)
                        tc_mma_f16_pair(d, smem_desc_k_sw128(st + kk * 32),
                                        smem_desc_k_sw128(st + kPWBytes + kk * 32), idesc,
                                        (kb | kk) != 0);
                    tc_commit_pair(&empty[s], 0x3);
                    any = true;
                    if (++s == kPStages) { s = 0; ph ^= 1; }
                }
                if (!ok) break;
                tc_commit_pair(&tfull[buf], 0x3);
                if (++buf == 2) { buf = 0; aph ^= 1; }
            }
            if (any) {
                tc_commit_pair(mma_done, 0x1);
                wait_cl(mma_done, 0, abort_flag, P.status, true);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue (both CTAs)
        const int q = warp & 3;
        const uint32_t tempty_leader = mapa_shared(smem_addr(&tempty[0]), 0);
        uint8_t* stage = epi_buf + q * 4096;
        int buf = 0;
        uint32_t aph = 0;
        int rs = 0;
        uint32_t rph = 0;
        while (true) {
            int t;
            if (!next_tile(rs, rph, t) || t < 0) break;
            PTile tl;
            ptile_at<EPI>(P, t, tl);
            const PairProblem& p = P.p[tl.prob];
            if (!wait_cl(&tfull[buf], aph, abort_flag, P.status)) break;
            tc_fence_after();
            __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
            const uint32_t col0 = buf * kPairTokens;
            if (EPI == EPI_SWIGLU) {
                // this warp: features fbase .. fbase + 15 (gate lanes 32q + 16h + t/4);
                // thread t holds feature 8h + t/4 of tokens 8i + 2(t%4) + {0, 1}
                const int fbase = tl.f0 + 64 * (int)cta + 16 * q;
                for (int c0 = 0; c0 < tl.nvalid; c0 += 32) {
                    uint32_t r0[16], r1[16];
                    tmem_ld_16x256b_x4(tmem_base + ((uint32_t)(32 * q) << 16) + col0 + c0, r0);
                    tmem_ld_16x256b_x4(tmem_base + ((uint32_t)(32 * q + 16) << 16) + col0 + c0, r1);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t* r = h ? r1 : r0;
                        const int f = fbase + 8 * h + (lane >> 2);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int tok = c0 + 8 * i + 2 * (lane & 3) + e;
                                if (tok < tl.nvalid && f < p.n_feat) {
                                    const float g = __uint_as_float(r[4 * i + e]);
                                    const float u = __uint_as_float(r[4 * i + 2 + e]);
                                    out[(size_t)(tl.row0 + tok) * p.ld_out + f] =
                                        __float2bfloat16_rn(silu_f(g) * u);
                                }
                            }
                    }
                }
            } else {
                // this warp: features fbase .. fbase + 31 (lane = feature)
                const int fbase = tl.f0 + 128 * (int)cta + 32 * q;
                __nv_bfloat16* st = reinterpret_cast<__nv_bfloat16*>(stage);  // [32 tokens][32]
                float* stf = reinterpret_cast<float*>(stage);                 // [32 tokens][32]
                float* outf = reinterpret_cast<float*>(p.out);
                // routing weights of the tile's tokens, loaded once: lane l holds token c0 + l
                float wpre[kPairTokens / 32];
#pragma unroll
                for (int i = 0; i < kPairTokens / 32; ++i) {
                    const int c = 32 * i + lane;
                    wpre[i] = (p.row_w && c < tl.nvalid) ? __ldg(p.row_w + tl.row0 + c) : 1.0f;
                }
#pragma unroll 1
                for (int c0 = 0; c0 < tl.nvalid; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld_32(tmem_base + ((uint32_t)(32 * q) << 16) + col0 + c0, r);
                    tmem_wait_ld();
                    float wv = wpre[0];
#pragma unroll
                    for (int i = 1; i < kPairTokens / 32; ++i)
                        if (c0 == 32 * i) wv = wpre[i];
                    if (p.out_f32) {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            stf[j * 32 + lane] = __uint_as_float(r[j]) * __shfl_sync(0xffffffffu, wv, j);
                        __syncwarp();
#pragma unroll
                        for (int it = 0; it < 8; ++it) {
                            const int tok = 4 * it + (lane >> 3), part = lane & 7;
                            const int f = fbase + 4 * part;
                            if (c0 + tok < tl.nvalid && f < p.n_feat)
                                *reinterpret_cast<float4*>(outf + (size_t)(tl.row0 + c0 + tok) * p.ld_out + f) =
                                    *reinterpret_cast<const float4*>(stf + tok * 32 + 4 * part);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float wj = __shfl_sync(0xffffffffu, wv, j);
                            st[j * 32 + lane] = __float2bfloat16_rn(__uint_as_float(r[j]) * wj);
                        }
                        __syncwarp();
#pragma unroll
                        for (int it = 0; it < 4; ++it) {
                            const int tok = 8 * it + (lane >> 2), part = lane & 3;
                            const int f = fbase + 8 * part;
                            if (c0 + tok < tl.nvalid && f < p.n_feat)
                                *reinterpret_cast<uint4*>(out + (size_t)(tl.row0 + c0 + tok) * p.ld_out + f) =
                                    *reinterpret_cast<const uint4*>(st + tok * 32 + 8 * part);
                        }
                    }
                    __syncwarp();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_leader + 8u * buf);
            if (++buf == 2) { buf = 0; aph ^= 1; }
        }
    }

    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, kPTmemCols);
    // the last CTA to finish leaves the claim counters at zero for the next launch
    if (kClaim && threadIdx.x == 0 && atomicAdd(&sched[1], 1) == (int)gridDim.x - 1) {
        atomicExch(&sched[0], 0);
        atomicExch(&sched[1], 0);
    }
}

template <int EPI>
static cudaError_t launch_pair_t(const PairParams& params, int grid, cudaStream_t s) {
    constexpr int kPSmem = PCfg<EPI>::SMEM;
    cudaError_t e = cudaFuncSetAttribute(pair_gemm_kernel<EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem);
    if (e != cudaSuccess) return e;
    // As many clusters as can be resident at once (SM pairs of one GPC).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = kPSmem;
    cfg.stream = s;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, pair_gemm_kernel<EPI>, &cfg) == cudaSuccess &&
        clusters > 0 && 2 * clusters < grid)
        grid = 2 * clusters;
    cudaGetLastError();
    pair_gemm_kernel<EPI><<<grid, kPThreads, kPSmem, s>>>(params);
    return cudaGetLastError();
}

cudaError_t launch_pair_gemm(int epi, const PairParams& params, int grid, cudaStream_t s) {
    if (params.status == nullptr) return cudaErrorInvalidValue;  // holds the tile claim counters
    grid &= ~1;
    if (grid < 2) grid = 2;
    if (epi == EPI_SWIGLU) return launch_pair_t<EPI_SWIGLU>(params, grid, s);
    if (epi == EPI_SCALE) return launch_pair_t<EPI_SCALE>(params, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace moe
