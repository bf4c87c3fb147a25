// dsa_scores.cu -- DSA indexer scores on tcgen05:
//   I[t, s] = sum_h w[t, h] * max(0, q[t, h, :] . k[s, h, :]),  head dim 128.
//
// Source of the operation: "Xiaohongshu dots3 note Open Source Deep Dive",
// §4.2 "How DSA Works" (indexer listing: per-head q.k, ReLU, weighted by a
// per-query head weight, summed over heads); "dots3-note 架构深度解析"
// (mlqm.cn), 混合注意力 paragraph (64 index heads).
//
// A CTA computes a tile of 128 queries (the MMA's M, one per TMEM lane) by
// 256 keys (N).  The 64 heads play the role of K blocks: per head, two
// 64-wide panels of q (16 KB) and k (32 KB) go through a 4-stage ring, eight
// kind::f16 MMAs (K = 16) build the head's q.k in a TMEM partial, and 16
// epilogue warps fold w[t, h] * ReLU(partial) into fp32 register
// accumulators (each thread owns one query row and 64 key columns).  The
// ReLU sits between the heads, so the heads cannot be summed inside the
// tensor core.  Two 256-column partials let the next head's MMAs run while
// one is folded.
//
// Roles (19 warps): warp 0 loads q panels, warp 18 k panels (two issuing
// threads: one tops out near 40 B/clk of tensor copies), warp 1 allocates
// tensor memory and issues the MMAs, warps 2-17 fold and store.
//
// Causal mask (optional): query t (absolute position q_offset + t) sees keys
// s <= q_offset + t.  Tiles entirely above the diagonal skip loads and MMAs
// and only store -inf; diagonal tiles store -inf past the limit.  Tiles are
// walked in groups of 32 query tiles x 4 key tiles so that the q and k rows
// a group needs stay in L2.  CTAs claim tiles at run time in that order from
// a counter in the workspace status block (the q producer claims and hands
// the id to the other roles through a 4-slot ring; the last CTA to finish
// resets the counter): a CTA that drew masked tiles takes more computed ones,
// so no CTA ends far behind the others.
//
// Waits are bounded as in the GEMMs (DEV_STATUS_TIMEOUT, abort flag, drain).
#include "dsa_kernels.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "tiles.cuh"

#include <cuda_bf16.h>

namespace moe {

namespace {

constexpr int kSQ = 128;                       // queries per tile
constexpr int kSK = 256;                       // keys per tile
constexpr int kSPanels = kDsaHeadDim / 64;     // 64-wide panels per head
constexpr int kSABytes = kSQ * 128;            // 16 KB of q per panel
constexpr int kSBBytes = kSK * 128;            // 32 KB of k per panel
constexpr int kSStage = kSABytes + kSBBytes;
constexpr int kSStages = 4;
constexpr int kSEpiWarps = 16;
constexpr int kSBWarp = 2 + kSEpiWarps;        // k-panel producer
constexpr int kSThreads = 32 * (kSBWarp + 1);
constexpr int kSNP = 2;
constexpr int kSBarBytes = 512;
constexpr int kSRing = 4;                      // claimed tile ids in flight
constexpr int kSSchedWord = 16;                // first scheduling word in the status block
constexpr int kSSmem = 1024 + kSStages * kSStage + kSBarBytes;
constexpr int kSGroupQ = 32, kSGroupK = 4;
static_assert(kSSmem <= 232448, "shared memory budget");

struct STile {
    int i, j;      // query tile, key tile
    bool masked;   // entirely above the causal diagonal
};

__device__ __forceinline__ STile stile_at(const DsaScoreArgs& a, int t) {
    const int nqt = (a.Sq + kSQ - 1) / kSQ, nkt = (a.Sk + kSK - 1) / kSK;
    const int ngk = (nkt + kSGroupK - 1) / kSGroupK;
    STile o{0, 0, true};
    // groups in (query group, key group) order; tiles inside a group key-minor
    for (int gi = 0; gi * kSGroupQ < nqt; ++gi) {
        const int gq = min(kSGroupQ, nqt - gi * kSGroupQ);
        for (int gj = 0; gj < ngk; ++gj) {
            const int gk = min(kSGroupK, nkt - gj * kSGroupK);
            if (t < gq * gk) {
                o.i = gi * kSGroupQ + t / gk;
                o.j = gj * kSGroupK + t % gk;
                o.masked = a.causal && (long long)o.j * kSK > (long long)a.q_offset + (long long)o.i * kSQ + kSQ - 1;
                return o;
            }
            t -= gq * gk;
        }
    }
    return o;
}

}  // namespace

__global__ void __launch_bounds__(kSThreads, 1) dsa_scores_kernel(const __grid_constant__ DsaScoreArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kSStages * kSStage);
    uint64_t* empty = full + kSStages;
    uint64_t* pfull = empty + kSStages;
    uint64_t* pempty = pfull + kSNP;
    uint64_t* mma_done = pempty + kSNP;
    uint64_t* rfull = mma_done + 1;          // [kSRing] a claimed tile id is in the ring
    uint64_t* rempty = rfull + kSRing;       // [kSRing] read by the k producer, the MMA thread, 16 epilogue warps
    int* ring = reinterpret_cast<int*>(rempty + kSRing);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(ring + kSRing);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kSStages; ++s) {
            mbar_init(&full[s], 1);   // q producer's arrive with the stage's bytes
            mbar_init(&empty[s], 1);  // one MMA commit
        }
        for (int b = 0; b < kSNP; ++b) {
            mbar_init(&pfull[b], 1);
            mbar_init(&pempty[b], kSEpiWarps);
        }
        mbar_init(mma_done, 1);
        for (int r = 0; r < kSRing; ++r) {
            mbar_init(&rfull[r], 1);
            mbar_init(&rempty[r], 2 + kSEpiWarps);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&a.tq);
        tma_prefetch_desc(&a.tk);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kSNP * kSK);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int ntiles = ((a.Sq + kSQ - 1) / kSQ) * ((a.Sk + kSK - 1) / kSK);
    // tile claim counter and finished-CTA count (workspace status block; word 0
    // is the status word)
    int* sched = a.status + kSSchedWord;

    if (warp == 0 || warp == kSBWarp) {
        // ------------------------------------------------ TMA producers
        if (lane == 0) {
            const bool qprod = warp == 0;
            int s = 0;
            uint32_t ph = 0, issued = 0, last_ph = 0;
            bool ok = true;
            int rs = 0;
            uint32_t rph = 0;
            while (ok) {
                // the q producer claims the next tile (masked ones too) and hands
                // its id to the k producer, the MMA thread and the epilogue
                int t;
                if (qprod) {
                    t = atomicAdd(&sched[0], 1);
                    if (t >= ntiles) t = -1;
                    if (!wait_bar(&rempty[rs], rph ^ 1, abort_flag, a.status)) { ok = false; break; }
                    ring[rs] = t;
                    mbar_arrive(&rfull[rs]);
                } else {
                    if (!wait_bar(&rfull[rs], rph, abort_flag, a.status)) { ok = false; break; }
                    t = ring[rs];
                    mbar_arrive(&rempty[rs]);
                }
                if (++rs == kSRing) { rs = 0; rph ^= 1; }
                if (t < 0) break;
                const STile tl = stile_at(a, t);
                if (tl.masked) continue;
                for (int h = 0; h < a.nh && ok; ++h)
                    for (int p = 0; p < kSPanels; ++p) {
                        if (!wait_bar(&empty[s], ph ^ 1, abort_flag, a.status)) { ok = false; break; }
                        uint8_t* st = smem + s * kSStage;
                        if (qprod) {
                            mbar_arrive_expect_tx(&full[s], kSStage);
                            tma_load_3d(st, &a.tq, &full[s], p * 64, h, tl.i * kSQ);
                        } else {
                            tma_load_3d(st + kSABytes, &a.tk, &full[s], p * 64, h, tl.j * kSK);
                        }
                        issued |= 1u << s;
                        last_ph = (last_ph & ~(1u << s)) | (ph << s);
                        if (++s == kSStages) { s = 0; ph ^= 1; }
                    }
            }
            // a stage's full barrier completes only with both producers' bytes
            if (qprod)
                for (int i = 0; i < kSStages; ++i)
                    if (issued >> i & 1u) wait_bar(&full[i], last_ph >> i & 1u, abort_flag, a.status, true);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer: eight K=16 MMAs per head
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kSQ, kSK);
            int s = 0, pb = 0;
            uint32_t ph = 0, pph = 0;
            bool ok = true, any = false;
            int rs = 0;
            uint32_t rph = 0;
            while (ok) {
                if (!wait_bar(&rfull[rs], rph, abort_flag, a.status)) break;
                const int t = ring[rs];
                mbar_arrive(&rempty[rs]);
                if (++rs == kSRing) { rs = 0; rph ^= 1; }
                if (t < 0) break;
                const STile tl = stile_at(a, t);
                if (tl.masked) continue;
                for (int h = 0; h < a.nh && ok; ++h) {
                    if (!wait_bar(&pempty[pb], pph ^ 1, abort_flag, a.status)) { ok = false; break; }
                    const uint32_t d = tmem_base + pb * kSK;
                    for (int p = 0; p < kSPanels; ++p) {
                        if (!wait_bar(&full[s], ph, abort_flag, a.status)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t st = smem_addr(smem + s * kSStage);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc_mma_f16(d, smem_desc_k_sw128(st + kk * 32),
                                       smem_desc_k_sw128(st + kSABytes + kk * 32), idesc, (p | kk) != 0);
                        tc_commit(&empty[s]);
                        any = true;
                        if (++s == kSStages) { s = 0; ph ^= 1; }
                    }
                    if (!ok) break;
                    tc_commit(&pfull[pb]);
                    if (++pb == kSNP) { pb = 0; pph ^= 1; }
                }
            }
            if (any) {
                tc_commit(mma_done);
                wait_bar(mma_done, 0, abort_flag, a.status, true);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue: fold w * ReLU(q.k) over heads
        const int q = warp & 3;
        const int g = (warp - 2) >> 2;
        const int tok = 32 * q + lane;
        int pb = 0;
        uint32_t pph = 0;
        bool ok = true;
        int rs = 0;
        uint32_t rph = 0;
        while (ok) {
            if (!wait_bar(&rfull[rs], rph, abort_flag, a.status)) break;
            const int t = ring[rs];
            __syncwarp();
            if (lane == 0) mbar_arrive(&rempty[rs]);
            if (++rs == kSRing) { rs = 0; rph ^= 1; }
            if (t < 0) break;
            const STile tl = stile_at(a, t);
            const int row = tl.i * kSQ + tok;
            const bool rvalid = row < a.Sq;
            float acc[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) acc[c] = 0.0f;
            if (!tl.masked) {
                const uint16_t* wrow = a.w + (size_t)(rvalid ? row : 0) * a.nh;
                float wn = rvalid ? __uint_as_float((uint32_t)__ldg(wrow) << 16) : 0.0f;
                for (int h = 0; h < a.nh; ++h) {
                    const float wc = wn;
                    wn = (rvalid && h + 1 < a.nh) ? __uint_as_float((uint32_t)__ldg(wrow + h + 1) << 16) : 0.0f;
                    if (!wait_bar(&pfull[pb], pph, abort_flag, a.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t tb = tmem_base + ((uint32_t)(32 * q) << 16) + pb * kSK + 64 * g;
                    uint64_t w2;
                    asm("mov.b64 %0, {%1, %1};" : "=l"(w2) : "f"(wc));
#pragma unroll
                    for (int c0 = 0; c0 < 64; c0 += 16) {
                        uint32_t r[16];
                        tmem_ld_16(tb + c0, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; j += 2) {
                            // acc += w * ReLU(p), two columns per packed FMA (two IEEE
                            // fp32 FMAs: the same bits as fmaf)
                            const float p0 = fmaxf(__uint_as_float(r[j]), 0.0f);
                            const float p1 = fmaxf(__uint_as_float(r[j + 1]), 0.0f);
                            asm("{\n\t.reg .b64 acc, pp;\n\t"
                                "mov.b64 acc, {%0, %1};\n\t"
                                "mov.b64 pp, {%3, %4};\n\t"
                                "fma.rn.f32x2 acc, %2, pp, acc;\n\t"
                                "mov.b64 {%0, %1}, acc;\n\t}"
                                : "+f"(acc[c0 + j]), "+f"(acc[c0 + j + 1])
                                : "l"(w2), "f"(p0), "f"(p1));
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pempty[pb]);
                    if (++pb == kSNP) { pb = 0; pph ^= 1; }
                }
                if (!ok) break;
            }
            if (!rvalid) continue;
            // causal limit of this row (exclusive), then the 64 key columns of this warp
            const int col0 = tl.j * kSK + 64 * g;
            const int lim = tl.masked ? col0 : min(a.Sk, a.causal ? a.q_offset + row + 1 : a.Sk);
            float* out = a.scores + (size_t)row * a.Sk + col0;
            if (col0 + 64 <= a.Sk && (a.Sk & 3) == 0) {
#pragma unroll
                for (int v = 0; v < 16; ++v) {
                    const int c = col0 + 4 * v;
                    reinterpret_cast<float4*>(out)[v] =
                        make_float4(c < lim ? acc[4 * v] : -INFINITY, c + 1 < lim ? acc[4 * v + 1] : -INFINITY,
                                    c + 2 < lim ? acc[4 * v + 2] : -INFINITY,
                                    c + 3 < lim ? acc[4 * v + 3] : -INFINITY);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (col0 + c < a.Sk) out[c] = col0 + c < lim ? acc[c] : -INFINITY;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kSNP * kSK);
    // the last CTA to finish leaves the claim counters at zero for the next launch
    if (threadIdx.x == 0 && atomicAdd(&sched[1], 1) == (int)gridDim.x - 1) {
        atomicExch(&sched[0], 0);
        atomicExch(&sched[1], 0);
    }
}

cudaError_t launch_dsa_scores(const DsaScoreArgs& a, int grid, cudaStream_t s) {
    if (a.Sq == 0 || a.Sk == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(dsa_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSSmem);
    if (e != cudaSuccess) return e;
    dsa_scores_kernel<<<grid, kSThreads, kSSmem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
