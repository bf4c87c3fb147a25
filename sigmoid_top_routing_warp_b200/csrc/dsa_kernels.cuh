// dsa_kernels.cuh -- launch interface between the DSA indexer's C-ABI layer
// (dsa_api.cu) and its two kernels (dsa_scores.cu, dsa_topk.cu).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kDsaMaxTopk = 2048;
constexpr int kDsaHeadDim = 128;

// scores: fp32 [Sq, ld], masked entries -inf (never selected)
struct DsaTopkArgs {
    const float* scores;
    int ld;
    int32_t* idx;             // [Sq, topk]
    int Sq, Sk, topk;         // topk <= kDsaMaxTopk
    int sorted;               // 1: score descending; 0: key index ascending
    int causal, q_offset;     // 1: row t reads only keys s <= q_offset + t (the
                              //    rest are the score kernel's -inf)
};
size_t dsa_topk_smem(int Sk);
cudaError_t launch_dsa_topk(const DsaTopkArgs& a, cudaStream_t s);

// I[t, s] = sum_h w[t, h] * max(0, q[t, h, :] . k[s, h, :]), fp32 [Sq, Sk]
struct DsaScoreArgs {
    CUtensorMap tq;           // bf16 3-D {D, nh, Sq}, box {64, 1, 128}
    CUtensorMap tk;           // bf16 3-D {D, nh, Sk}, box {64, 1, 256}
    const uint16_t* w;        // bf16 [Sq, nh]
    float* scores;            // [Sq, Sk]
    int Sq, Sk, nh;
    int causal, q_offset;
    int* status;
};
cudaError_t launch_dsa_scores(const DsaScoreArgs& a, int grid, cudaStream_t s);

}  // namespace moe
