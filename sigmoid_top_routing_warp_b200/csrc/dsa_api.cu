// dsa_api.cu -- the C ABI of the DSA indexer (include/dsa.h): argument
// checks, tensor maps and launches.  Shares the last-error message and the
// tensor-map helper with api.cu.
#include "dsa.h"
#include "dsa_kernels.cuh"
#include "kernels.cuh"

#include <cuda_runtime.h>

#include <cstdio>

namespace moe {
moe_status_t api_fail(moe_status_t st, const char* msg);
void api_clear_error();
moe_status_t api_sm_count(int* n);
moe_status_t api_make_map_3d_bf16(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1,
                                  uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t b0,
                                  uint32_t b1, uint32_t b2, const char* what);
}  // namespace moe

namespace {

constexpr size_t kDsaStatusBytes = 256;

moe_status_t dfail(moe_status_t st, const char* fmt, long long a = 0, long long b = 0) {
    char msg[256];
    snprintf(msg, sizeof(msg), fmt, a, b);
    return moe::api_fail(st, msg);
}

bool aligned(const void* p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

moe_status_t check_cfg(const dsa_config_t* c) {
    if (!c) return dfail(MOE_ERR_INVALID_ARG, "cfg is NULL");
    if (c->Sq < 0 || c->Sk < 0) return dfail(MOE_ERR_INVALID_ARG, "Sq=%lld Sk=%lld must be >= 0", c->Sq, c->Sk);
    if (c->n_heads < 1 || c->n_heads > 1024)
        return dfail(MOE_ERR_INVALID_ARG, "n_heads=%lld must be in [1, 1024]", c->n_heads);
    if (c->head_dim != moe::kDsaHeadDim)
        return dfail(MOE_ERR_UNSUPPORTED, "head_dim=%lld: only %lld is supported", c->head_dim,
                     moe::kDsaHeadDim);
    if (c->topk < 1 || c->topk > moe::kDsaMaxTopk)
        return dfail(MOE_ERR_INVALID_ARG, "topk=%lld must be in [1, %lld]", c->topk, moe::kDsaMaxTopk);
    if (c->causal != 0 && c->causal != 1) return dfail(MOE_ERR_INVALID_ARG, "causal must be 0 or 1");
    if (c->q_offset < 0) return dfail(MOE_ERR_INVALID_ARG, "q_offset=%lld must be >= 0", c->q_offset);
    if (c->sorted != 0 && c->sorted != 1) return dfail(MOE_ERR_INVALID_ARG, "sorted must be 0 or 1");
    return MOE_OK;
}

moe_status_t need(const void* p, const char* name, size_t align) {
    char msg[128];
    if (!p) {
        snprintf(msg, sizeof(msg), "%s is NULL", name);
        return moe::api_fail(MOE_ERR_INVALID_ARG, msg);
    }
    if (!aligned(p, align)) {
        snprintf(msg, sizeof(msg), "%s must be %zu-byte aligned", name, align);
        return moe::api_fail(MOE_ERR_INVALID_ARG, msg);
    }
    return MOE_OK;
}

#define DSA_TRY(x)                         \
    do {                                   \
        moe_status_t st_ = (x);            \
        if (st_ != MOE_OK) return st_;     \
    } while (0)

moe_status_t cuda_fail(cudaError_t e, const char* what) {
    char msg[256];
    snprintf(msg, sizeof(msg), "%s: %s", what, cudaGetErrorString(e));
    return moe::api_fail(MOE_ERR_CUDA, msg);
}

moe_status_t run_scores(const dsa_config_t* c, const void* q, const void* k, const void* w,
                        float* scores, void* ws, cudaStream_t s) {
    moe::DsaScoreArgs a;
    const uint64_t D = moe::kDsaHeadDim, nh = (uint64_t)c->n_heads;
    DSA_TRY(moe::api_make_map_3d_bf16(&a.tq, q, D, nh, (uint64_t)c->Sq, D * 2, nh * D * 2, 64, 1, 128,
                                      "q"));
    DSA_TRY(moe::api_make_map_3d_bf16(&a.tk, k, D, nh, (uint64_t)c->Sk, D * 2, nh * D * 2, 64, 1, 256,
                                      "k"));
    a.w = static_cast<const uint16_t*>(w);
    a.scores = scores;
    a.Sq = c->Sq;
    a.Sk = c->Sk;
    a.nh = c->n_heads;
    a.causal = c->causal;
    a.q_offset = c->q_offset;
    a.status = static_cast<int*>(ws);
    int sms = 0;
    DSA_TRY(moe::api_sm_count(&sms));
    cudaError_t e = moe::reset_claim_counters(a.status, s);
    if (e != cudaSuccess) return cuda_fail(e, "claim-counter reset");
    e = moe::launch_dsa_scores(a, sms, s);
    if (e != cudaSuccess) return cuda_fail(e, "DSA score kernel launch");
    return MOE_OK;
}

// causal_rows: the scores come from the score kernel, whose causal mask
// makes keys past q_offset + t -inf in row t, so those are not read.
moe_status_t run_topk(const dsa_config_t* c, const float* scores, int32_t* idx, bool causal_rows,
                      cudaStream_t s) {
    moe::DsaTopkArgs a;
    a.scores = scores;
    a.ld = c->Sk;
    a.idx = idx;
    a.Sq = c->Sq;
    a.Sk = c->Sk;
    a.topk = c->topk;
    a.sorted = c->sorted;
    a.causal = causal_rows && c->causal ? 1 : 0;
    a.q_offset = c->q_offset;
    cudaError_t e = moe::launch_dsa_topk(a, s);
    if (e != cudaSuccess) return cuda_fail(e, "DSA top-k kernel launch");
    return MOE_OK;
}

size_t scores_bytes(const dsa_config_t* c) { return (size_t)c->Sq * (size_t)c->Sk * 4; }

}  // namespace

extern "C" {

size_t dsa_workspace_size(const dsa_config_t* cfg) {
    moe::api_clear_error();
    if (check_cfg(cfg) != MOE_OK) return 0;
    return kDsaStatusBytes + ((scores_bytes(cfg) + 255) & ~(size_t)255);
}

size_t dsa_workspace_scores_offset(void) { return kDsaStatusBytes; }

moe_status_t dsa_index_scores(const dsa_config_t* cfg, const void* q, const void* k,
                              const void* w, float* scores, void* ws, size_t ws_bytes,
                              moe_stream_t stream) {
    moe::api_clear_error();
    DSA_TRY(check_cfg(cfg));
    DSA_TRY(need(q, "q", 16));
    DSA_TRY(need(k, "k", 16));
    DSA_TRY(need(w, "w", 2));
    DSA_TRY(need(scores, "scores", 16));
    DSA_TRY(need(ws, "workspace", 256));
    if (ws_bytes < kDsaStatusBytes)
        return dfail(MOE_ERR_WORKSPACE, "workspace has %lld bytes, needs %lld", (long long)ws_bytes,
                     (long long)kDsaStatusBytes);
    if (cfg->Sq == 0 || cfg->Sk == 0) return MOE_OK;
    return run_scores(cfg, q, k, w, scores, ws, static_cast<cudaStream_t>(stream));
}

moe_status_t dsa_index_topk(const dsa_config_t* cfg, const float* scores, int32_t* idx,
                            moe_stream_t stream) {
    moe::api_clear_error();
    DSA_TRY(check_cfg(cfg));
    DSA_TRY(need(scores, "scores", 4));
    DSA_TRY(need(idx, "idx", 4));
    if (cfg->Sq == 0) return MOE_OK;
    return run_topk(cfg, scores, idx, false, static_cast<cudaStream_t>(stream));
}

moe_status_t dsa_indexer(const dsa_config_t* cfg, const void* q, const void* k, const void* w,
                         int32_t* idx, void* ws, size_t ws_bytes, moe_stream_t stream) {
    moe::api_clear_error();
    DSA_TRY(check_cfg(cfg));
    DSA_TRY(need(q, "q", 16));
    DSA_TRY(need(k, "k", 16));
    DSA_TRY(need(w, "w", 2));
    DSA_TRY(need(idx, "idx", 4));
    DSA_TRY(need(ws, "workspace", 256));
    const size_t need_bytes = kDsaStatusBytes + scores_bytes(cfg);
    if (ws_bytes < need_bytes)
        return dfail(MOE_ERR_WORKSPACE, "workspace has %lld bytes, needs %lld", (long long)ws_bytes,
                     (long long)need_bytes);
    if (cfg->Sq == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float* scores = reinterpret_cast<float*>(static_cast<char*>(ws) + kDsaStatusBytes);
    if (cfg->Sk > 0) DSA_TRY(run_scores(cfg, q, k, w, scores, ws, s));
    return run_topk(cfg, scores, idx, true, s);
}

}  // extern "C"
