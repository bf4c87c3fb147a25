// gemm_fp8_tm.cu -- token-major grouped expert GEMMs on e4m3 operands with
// fp32 block scales, for batches with many tokens per expert (steps a6-a8 of
// the FP8 layer), tcgen05 kind::f8f6f4 + TMEM.
//
// Source of the operation: "Xiaohongshu dots3 note Open Source Deep Dive",
// §8.2 (gmm1 -> swiglu -> gmm2) and §3.2 (FP8 weights); "dots3-note 架构深度解析"
// (mlqm.cn), 部署实战 (FP8 weights).  Recipe: weights e4m3 with one fp32 scale
// per 128x128 block; activations e4m3 with one fp32 scale per row and 128
// columns (quant.cu).
//
// The scales are arbitrary fp32 values, so every 128-wide K block is one MMA
// group into a tensor-memory partial that the epilogue promotes into fp32
// register accumulators:  acc[r, f] += s_x(r, kb) * s_w(f / 128, kb) * P_kb[r, f].
// Here the tokens are the MMA's M operand (128 rows, one per TMEM lane) and
// the weights its N operand (256 rows: 128 gate + 128 up features, or 256
// output features).  Each epilogue thread then owns one token row, so the
// scale of a K block is one product per thread and promotion is one FMA per
// element, with no cross-lane traffic.  (gemm_fp8.cu puts the weights in M,
// which suits a few tokens per expert but makes the scale vary along the
// accumulator's columns.)
//
// Roles (10 warps): warp 0 issues TMA loads (operands per K block; the
// scales of four K blocks at a time into a small ring: s_x for the tile's
// 128 rows as one {4, 128} box, s_w as two {4, 1} boxes), warp 1 allocates
// tensor memory and issues the MMAs (one thread), warps 2-9 promote and
// finish: warp w reads TMEM lane quadrant w % 4 and column group (w - 2) / 4,
// 128 of the 256 columns, into 128 fp32 register accumulators (with 320
// threads, three warps on a sub-partition, a thread may hold 168 registers).
// Each K block is promoted in 8-column (gate/up) or 16-column (down) chunks
// whose TMEM loads run one chunk ahead of the FMAs.  Two 256-column partial buffers let the MMAs
// of block kb+1 run while block kb is promoted.
//
// EPI_SWIGLU: a = SiLU(gate) * up, quantised per token over the tile's 128
// features (one e4m3 block of A); the four column groups exchange their
// maxima through shared memory under a bounded mbarrier.
// EPI_SCALE: y = acc * routing weight, bf16 (or fp32 for the shared expert).
//
// Tiles are claimed at run time from a counter in the workspace status block
// and handed to the MMA thread and the epilogue through a 4-slot ring, as in
// gemm.cu (with a static round-robin the CTAs' end times spread over 3.5-7.8 %
// of a launch).
//
// Waits are bounded as in gemm.cu (DEV_STATUS_TIMEOUT, abort flag, drain).
#include "kernels.cuh"
#include "ptx.cuh"
#include "tiles.cuh"

#include <cuda_bf16.h>
#include <cuda_fp8.h>

namespace moe {

namespace {

constexpr int kTMTok = 128;                    // token rows per tile (MMA M)
constexpr int kTMN = 256;                      // weight rows per tile (MMA N)
constexpr int kTMBK = 128;                     // K per stage: one scale block, 128 B rows
constexpr int kTMABytes = kTMTok * kTMBK;      // 16 KB of token codes
constexpr int kTMBBytes = kTMN * kTMBK;        // 32 KB of weight codes
constexpr int kTMStage = kTMABytes + kTMBBytes;
constexpr int kTMStages = 4;
constexpr int kTMGroup = 4;                    // K blocks per scale fetch
constexpr int kTMSSlots = 3;                   // scale ring depth
constexpr int kTMSSlot = 2304;                 // s_x [128][4] at 0, s_w rows at 2048 and 2176
constexpr int kTMEpiWarps = 8;
constexpr int kTMThreads = 64 + 32 * kTMEpiWarps;
constexpr int kTMNP = 2;                       // partial buffers of kTMN columns
constexpr int kTMAmaxBytes = 2 * 2 * kTMTok * 4;  // [2 parities][2 column groups][128 rows]
constexpr int kTMBarBytes = 512;
constexpr int kTMRing = 4;                     // claimed tile ids in flight (producer -> MMA, epilogue)
constexpr int kTMSchedWord = 24;               // first scheduling word in the status block
constexpr int kTMSmem = 1024 + kTMStages * kTMStage + kTMSSlots * kTMSSlot + kTMAmaxBytes +
                        kTMBarBytes;
// kind::f8f6f4: fp32 accumulator, e4m3 A and B (format 0), K-major, M = 128, N = 256
constexpr uint32_t kTMIdesc = (1u << 4) | ((uint32_t)(kTMN >> 3) << 17) | ((uint32_t)(kTMTok >> 4) << 24);
static_assert(kTMSmem <= 232448, "shared memory budget");
static_assert(kTMStage % 1024 == 0 && kTMSSlot % 128 == 0, "TMA destinations stay aligned");

__device__ __forceinline__ void tm_mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(kTMIdesc), "r"(accumulate)
        : "memory");
}

// {s, s} as one 64-bit operand of the packed fp32 instructions.
__device__ __forceinline__ uint64_t tm_splat2(float s) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(s));
    return r;
}

// a0 += s * b0, a1 += s * b1 in one packed instruction (two fp32 FMAs, each
// rounded to nearest: the same bits as two fmaf calls).
__device__ __forceinline__ void tm_ffma2(float& a0, float& a1, uint64_t ss, uint32_t b0, uint32_t b1) {
    asm("{\n\t.reg .b64 acc, bb;\n\t"
        "mov.b64 acc, {%0, %1};\n\t"
        "mov.b64 bb, {%3, %4};\n\t"
        "fma.rn.f32x2 acc, %2, bb, acc;\n\t"
        "mov.b64 {%0, %1}, acc;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "l"(ss), "r"(b0), "r"(b1));
}

// SiLU of the SwiGLU output that is requantised to e4m3 right after: the
// quotient by the fast reciprocal (within 2 ulp of the correctly rounded
// one; 0 for a gate below about -88, where exp overflows).
__device__ __forceinline__ float silu_q(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// A chunk of CH (8 or 16) tensor-memory columns of this thread's lane.
template <int CH>
__device__ __forceinline__ void tm_ld_chunk(uint32_t taddr, uint32_t (&r)[CH]) {
    if constexpr (CH == 16)
        tmem_ld_16(taddr, r);
    else
        tmem_ld_8(taddr, r);
}

}  // namespace

template <int EPI>
__global__ void __launch_bounds__(kTMThreads, 1)
    fp8_tm_gemm_kernel(const __grid_constant__ GemmParams P) {
    constexpr int FSZ = EPI == EPI_SWIGLU ? 128 : 256;  // output features per tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sring = smem + kTMStages * kTMStage;
    float* amax_sm = reinterpret_cast<float*>(sring + kTMSSlots * kTMSSlot);
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(amax_sm) + kTMAmaxBytes);
    uint64_t* empty = full + kTMStages;
    uint64_t* sfull = empty + kTMStages;     // scale slot loaded (TMA)
    uint64_t* sempty = sfull + kTMSSlots;    // scale slot read (16 epilogue warps)
    uint64_t* pfull = sempty + kTMSSlots;    // partial ready (MMA -> epilogue)
    uint64_t* pempty = pfull + kTMNP;        // partial read (16 epilogue warps)
    uint64_t* amax_bar = pempty + kTMNP;     // [2] row maxima of all column groups written
    uint64_t* mma_done = amax_bar + 2;
    uint64_t* rfull = mma_done + 1;          // [kTMRing] a claimed tile id is in the ring
    uint64_t* rempty = rfull + kTMRing;      // [kTMRing] read by the MMA thread and the 16 epilogue warps
    int* ring = reinterpret_cast<int*>(rempty + kTMRing);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(ring + kTMRing);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kTMStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < kTMSSlots; ++s) {
            mbar_init(&sfull[s], 1);
            mbar_init(&sempty[s], kTMEpiWarps);
        }
        for (int b = 0; b < kTMNP; ++b) {
            mbar_init(&pfull[b], 1);
            mbar_init(&pempty[b], kTMEpiWarps);
        }
        for (int b = 0; b < 2; ++b) mbar_init(&amax_bar[b], kTMEpiWarps);
        mbar_init(mma_done, 1);
        for (int r = 0; r < kTMRing; ++r) {
            mbar_init(&rfull[r], 1);
            mbar_init(&rempty[r], 1 + kTMEpiWarps);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        for (int pi = 0; pi < P.n_problems; ++pi) {
            tma_prefetch_desc(&P.p[pi].tw);
            tma_prefetch_desc(&P.p[pi].tx);
            tma_prefetch_desc(&P.p[pi].tsx);
            tma_prefetch_desc(&P.p[pi].tsw);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTMNP * kTMN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int ntiles = total_tiles(P, kTMTok, FSZ);
    // tile claim counter and finished-CTA count of this epilogue kind (the
    // workspace status block; word 0 is the status word)
    int* sched = P.status + kTMSchedWord + 2 * EPI;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int s = 0, ss = 0;
            uint32_t ph = 0, sph = 0, issued = 0, sissued = 0, last_ph = 0, slast_ph = 0;
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
                if (++rs == kTMRing) { rs = 0; rph ^= 1; }
                if (t < 0) break;
                Tile tl;
                tile_at(P, kTMTok, t, tl, FSZ);
                const GemmProblem& p = P.p[tl.prob];
                const int nk = p.K / kTMBK;
                // weight rows of the tile's two 128-row halves and their scale-block rows
                const int w0 = tl.exp * p.w_rows + tl.f0;
                const int w1 = EPI == EPI_SWIGLU ? w0 + p.n_feat : w0 + 128;
                for (int kb = 0; kb < nk; ++kb) {
                    if (kb % kTMGroup == 0) {
                        if (!wait_bar(&sempty[ss], sph ^ 1, abort_flag, P.status)) { ok = false; break; }
                        uint8_t* sl = sring + ss * kTMSSlot;
                        mbar_arrive_expect_tx(&sfull[ss], kTMTok * 16 + 2 * 16);
                        tma_load_2d(sl, &p.tsx, &sfull[ss], kb, tl.row0);
                        tma_load_2d(sl + 2048, &p.tsw, &sfull[ss], kb, w0 / 128);
                        tma_load_2d(sl + 2176, &p.tsw, &sfull[ss], kb, w1 / 128);
                        sissued |= 1u << ss;
                        slast_ph = (slast_ph & ~(1u << ss)) | (sph << ss);
                        if (++ss == kTMSSlots) { ss = 0; sph ^= 1; }
                    }
                    if (!wait_bar(&empty[s], ph ^ 1, abort_flag, P.status)) { ok = false; break; }
                    uint8_t* st = smem + s * kTMStage;
                    mbar_arrive_expect_tx(&full[s], kTMStage);
                    tma_load_2d(st, &p.tx, &full[s], kb * kTMBK, tl.row0);
                    tma_load_2d(st + kTMABytes, &p.tw, &full[s], kb * kTMBK, w0);
                    tma_load_2d(st + kTMABytes + kTMBBytes / 2, &p.tw, &full[s], kb * kTMBK, w1);
                    issued |= 1u << s;
                    last_ph = (last_ph & ~(1u << s)) | (ph << s);
                    if (++s == kTMStages) { s = 0; ph ^= 1; }
                }
            }
            // drain: every issued copy lands before the CTA exits
            for (int i = 0; i < kTMStages; ++i)
                if (issued >> i & 1u) wait_bar(&full[i], last_ph >> i & 1u, abort_flag, P.status, true);
            for (int i = 0; i < kTMSSlots; ++i)
                if (sissued >> i & 1u) wait_bar(&sfull[i], slast_ph >> i & 1u, abort_flag, P.status, true);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer: one group per K block
        if (lane == 0) {
            int s = 0, pb = 0;
            uint32_t ph = 0, pph = 0;
            bool ok = true, any = false;
            int rs = 0;
            uint32_t rph = 0;
            while (ok) {
                if (!wait_bar(&rfull[rs], rph, abort_flag, P.status)) break;
                const int t = ring[rs];
                mbar_arrive(&rempty[rs]);
                if (++rs == kTMRing) { rs = 0; rph ^= 1; }
                if (t < 0) break;
                Tile tl;
                tile_at(P, kTMTok, t, tl, FSZ);
                const int nk = P.p[tl.prob].K / kTMBK;
                for (int kb = 0; kb < nk && ok; ++kb) {
                    if (!wait_bar(&pempty[pb], pph ^ 1, abort_flag, P.status)) { ok = false; break; }
                    if (!wait_bar(&full[s], ph, abort_flag, P.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_addr(smem + s * kTMStage);
                    const uint32_t d = tmem_base + pb * kTMN;
#pragma unroll
                    for (int kk = 0; kk < kTMBK / 32; ++kk)
                        tm_mma_f8(d, smem_desc_k_sw128(st + kk * 32),
                                  smem_desc_k_sw128(st + kTMABytes + kk * 32), kk != 0);
                    tc_commit(&empty[s]);
                    tc_commit(&pfull[pb]);
                    any = true;
                    if (++s == kTMStages) { s = 0; ph ^= 1; }
                    if (++pb == kTMNP) { pb = 0; pph ^= 1; }
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
        const int q = warp & 3;              // TMEM lane quadrant: rows 32q .. 32q + 31
        const int g = (warp - 2) >> 2;       // column group 0 or 1
        const int tok = 32 * q + lane;       // this thread's row of the tile
        // accumulator columns: SWIGLU gate [64g, 64g+64) and up [128+64g, ...);
        // SCALE [128g, 128g+128), all in weight-scale block g
        const uint32_t ca = EPI == EPI_SWIGLU ? 64 * g : 128 * g;
        const uint32_t cb = EPI == EPI_SWIGLU ? 128 + 64 * g : 128 * g + 64;
        const int swa = EPI == EPI_SWIGLU ? 0 : g;
        const int swb = EPI == EPI_SWIGLU ? 1 : g;
        int pb = 0, ss = 0, tile_no = 0;
        uint32_t pph = 0, sph = 0;
        bool ok = true;
        int rs = 0;
        uint32_t rph = 0;
        for (; ok; ++tile_no) {
            if (!wait_bar(&rfull[rs], rph, abort_flag, P.status)) break;
            const int t = ring[rs];
            __syncwarp();
            if (lane == 0) mbar_arrive(&rempty[rs]);
            if (++rs == kTMRing) { rs = 0; rph ^= 1; }
            if (t < 0) break;
            Tile tl;
            tile_at(P, kTMTok, t, tl, FSZ);
            const GemmProblem& p = P.p[tl.prob];
            const int nk = p.K / kTMBK;
            const bool valid = tok < tl.nvalid;
            const int row = tl.row0 + tok;
            float acc[128];
#pragma unroll
            for (int j = 0; j < 128; ++j) acc[j] = 0.0f;
            for (int kb0 = 0; kb0 < nk && ok; kb0 += kTMGroup) {
                if (!wait_bar(&sfull[ss], sph, abort_flag, P.status)) { ok = false; break; }
                const float* sl = reinterpret_cast<const float*>(sring + ss * kTMSSlot);
#pragma unroll 1
                for (int i = 0; i < kTMGroup; ++i) {
                    // this K block's scales: the row's s_x and the column halves' s_w
                    const float sx = sl[4 * tok + i];
                    const uint64_t sa = tm_splat2(sx * sl[512 + 32 * swa + i]);
                    const uint64_t sb = tm_splat2(sx * sl[512 + 32 * swb + i]);
                    if (!wait_bar(&pfull[pb], pph, abort_flag, P.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t tb = tmem_base + ((uint32_t)(32 * q) << 16) + pb * kTMN;
                    // NCH chunks of CH columns (half at ca, half at cb): 8-column
                    // chunks for the gate/up GEMM, 16 for the down GEMM (measured
                    // best for each); chunk c + 1 is loaded while chunk c is
                    // accumulated, and the partial is released once the last chunk
                    // is in registers
                    constexpr int CH = EPI == EPI_SWIGLU ? 8 : 16;
                    constexpr int NCH = 128 / CH;
                    uint32_t r[2][CH];
                    tm_ld_chunk<CH>(tb + ca, r[0]);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < NCH; ++c) {
                        if (c + 1 < NCH) {
                            const int c1 = c + 1;
                            const uint32_t col = c1 < NCH / 2 ? ca + CH * c1 : cb + CH * (c1 - NCH / 2);
                            tm_ld_chunk<CH>(tb + col, r[c1 & 1]);
                        }
                        const uint64_t sc2 = c < NCH / 2 ? sa : sb;
#pragma unroll
                        for (int j = 0; j < CH; j += 2)
                            tm_ffma2(acc[CH * c + j], acc[CH * c + j + 1], sc2, r[c & 1][j], r[c & 1][j + 1]);
                        if (c + 1 < NCH) {
                            tmem_wait_ld();
                            if (c + 1 == NCH - 1) {
                                tc_fence_before();
                                __syncwarp();
                                if (lane == 0) mbar_arrive(&pempty[pb]);
                            }
                        }
                    }
                    if (++pb == kTMNP) { pb = 0; pph ^= 1; }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sempty[ss]);
                if (++ss == kTMSSlots) { ss = 0; sph ^= 1; }
            }
            if (!ok) break;
            if (EPI == EPI_SWIGLU) {
                // a = SiLU(gate) * up for features f0 + 64g .. + 63 of this row
                float m = 0.0f;
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    acc[j] = silu_q(acc[j]) * acc[64 + j];
                    m = fmaxf(m, fabsf(acc[j]));
                }
                const int par = tile_no & 1;
                amax_sm[(par * 2 + g) * kTMTok + tok] = m;
                __syncwarp();
                if (lane == 0) mbar_arrive(&amax_bar[par]);
                if (!wait_bar(&amax_bar[par], (tile_no >> 1) & 1, abort_flag, P.status)) break;
                const float* all = amax_sm + par * 2 * kTMTok + tok;
                const float amax = fmaxf(all[0], all[kTMTok]);
                const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
                // codes: a * (1 / sc), the reciprocal rounded once (within one fp32
                // ulp of a / sc before the e4m3 rounding), two per conversion
                const float inv = __frcp_rn(sc);
                if (valid) {
                    uint4* dst = reinterpret_cast<uint4*>(p.out_q + (size_t)row * p.ld_out + tl.f0 + 64 * g);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint32_t packed[4];
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            const int j = 16 * v + 4 * w;
                            const uint32_t lo = __nv_cvt_float2_to_fp8x2(
                                make_float2(acc[j] * inv, acc[j + 1] * inv), __NV_SATFINITE, __NV_E4M3);
                            const uint32_t hi = __nv_cvt_float2_to_fp8x2(
                                make_float2(acc[j + 2] * inv, acc[j + 3] * inv), __NV_SATFINITE, __NV_E4M3);
                            packed[w] = lo | (hi << 16);
                        }
                        dst[v] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                    }
                    if (g == 0) p.out_scale[(size_t)row * (p.ld_out / 128) + tl.f0 / 128] = sc;
                }
            } else {
                const int f = tl.f0 + 128 * g;
                if (valid && f < p.n_feat) {
                    const float wr = p.row_w ? __ldg(p.row_w + row) : 1.0f;
                    if (p.out_f32) {
                        float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) +
                                                                (size_t)row * p.ld_out + f);
#pragma unroll
                        for (int v = 0; v < 32; ++v)
                            dst[v] = make_float4(acc[4 * v] * wr, acc[4 * v + 1] * wr,
                                                 acc[4 * v + 2] * wr, acc[4 * v + 3] * wr);
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) +
                                                              (size_t)row * p.ld_out + f);
#pragma unroll
                        for (int v = 0; v < 16; ++v) {
                            uint32_t w4[4];
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                const __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[8 * v + 2 * h] * wr,
                                                                                acc[8 * v + 2 * h + 1] * wr);
                                w4[h] = *reinterpret_cast<const uint32_t*>(&b2);
                            }
                            dst[v] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTMNP * kTMN);
    // the last CTA to finish leaves the claim counters at zero for the next launch
    // (every CTA's claims came from thread 0 before this point)
    if (threadIdx.x == 0 && atomicAdd(&sched[1], 1) == (int)gridDim.x - 1) {
        atomicExch(&sched[0], 0);
        atomicExch(&sched[1], 0);
    }
}

template <int EPI>
static cudaError_t launch_tm(const GemmParams& params, int grid, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(fp8_tm_gemm_kernel<EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kTMSmem);
    if (e != cudaSuccess) return e;
    fp8_tm_gemm_kernel<EPI><<<grid, kTMThreads, kTMSmem, s>>>(params);
    return cudaGetLastError();
}

cudaError_t launch_fp8_tm_gemm(int epi, const GemmParams& params, int grid, cudaStream_t s) {
    if (params.status == nullptr) return cudaErrorInvalidValue;  // holds the tile claim counters
    if (epi == EPI_SWIGLU) return launch_tm<EPI_SWIGLU>(params, grid, s);
    if (epi == EPI_SCALE) return launch_tm<EPI_SCALE>(params, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace moe
