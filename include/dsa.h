/*
 * dsa.h -- C ABI of the DSA indexer: the lightweight scorer that picks, for
 * every query, the keys its sparse attention will read.  A second top-k
 * workload of this library next to the MoE router (include/moe.h).
 *
 * Pages: "Xiaohongshu dots3 note Open Source Deep Dive", §4.2 "How DSA Works"
 * (indexer listing: per index head h, q_h . k_h passed through ReLU,
 * weighted by a per-query head weight, summed over heads; top-k keys per
 * query); "dots3-note 架构深度解析" (mlqm.cn), 混合注意力 paragraph
 * (index_topk = 2048, 64 index heads).
 *
 *   I[t, s] = sum_h w[t, h] * max(0, q[t, h, :] . k[s, h, :])
 *   idx[t, :] = the topk keys s of row t with the largest I[t, s], by I
 *               descending (or, with sorted = 0, by s ascending), equal
 *               scores by lower s first; -1 pads rows with fewer valid keys.
 *
 * The projections that make q, k and w (and the key LayerNorm of the
 * listing) are plain per-token GEMMs and norms outside this path.  No 1/sqrt(d)
 * scale (the listing has none).
 *
 * Conventions are those of moe.h: caller-owned device memory, asynchronous
 * on `stream`, argument errors returned before any launch, device-side
 * bounded-wait timeouts recorded in the workspace status word (read with
 * moe_check_device_status).
 */
#ifndef DSA_B200_H
#define DSA_B200_H

#include "moe.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int32_t Sq;        /* queries                                              */
    int32_t Sk;        /* keys                                                 */
    int32_t n_heads;   /* index heads (64 on the pages), 1..1024               */
    int32_t head_dim;  /* must be 128 (the pages' value)                       */
    int32_t topk;      /* keys kept per query (2048 on the pages), 1..2048     */
    int32_t causal;    /* 1: query t sees keys s <= q_offset + t; 0: all keys  */
    int32_t q_offset;  /* absolute position of query 0 (causal only), >= 0     */
    int32_t sorted;    /* 1: indices by score descending (the listing's        */
                       /*    torch.topk order); 0: the same set by key index   */
                       /*    ascending (what a sparse-attention gather needs;  */
                       /*    skips the sort)                                   */
} dsa_config_t;

/* Bytes of workspace dsa_index_scores / dsa_indexer need: a 256-byte status
 * block, then (dsa_indexer) the fp32 score matrix [Sq, Sk].  0 if invalid.
 * The status block holds the status word (word 0, which must start at zero)
 * and the score kernel's tile-claim counters, which every score launch
 * zeroes on its stream first. */
size_t dsa_workspace_size(const dsa_config_t* cfg);

/* Scores.  q bf16 [Sq, n_heads, 128], k bf16 [Sk, n_heads, 128] (16-byte
 * aligned), w bf16 [Sq, n_heads]; scores fp32 [Sq, Sk] (16-byte aligned),
 * every entry written, masked ones -inf.  fp32 accumulation of exact bf16
 * products; ws: at least the status block. */
moe_status_t dsa_index_scores(const dsa_config_t* cfg, const void* q, const void* k,
                              const void* w, float* scores, void* ws, size_t ws_bytes,
                              moe_stream_t stream);

/* Top-k of each row of fp32 scores [Sq, Sk] -> idx int32 [Sq, topk]: exact
 * selection by score (-inf and NaN never chosen), order as above.  Only Sq,
 * Sk and topk of cfg are read. */
moe_status_t dsa_index_topk(const dsa_config_t* cfg, const float* scores, int32_t* idx,
                            moe_stream_t stream);

/* Both: scores into the workspace, then the top-k. */
moe_status_t dsa_indexer(const dsa_config_t* cfg, const void* q, const void* k, const void* w,
                         int32_t* idx, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Byte offset of the score matrix inside a dsa_indexer workspace. */
size_t dsa_workspace_scores_offset(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_B200_H */
