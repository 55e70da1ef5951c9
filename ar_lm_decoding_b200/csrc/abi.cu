// extern "C" entry points of libtidar: host-side argument validation and
// launch of the device kernels.  Nothing here allocates device memory.
#include <cmath>

#include "attn.cuh"
#include "../../include/tidar_testing.h"

namespace tidar {
size_t verify_workspace_bytes(int B, int k, int V);
cudaError_t verify_launch(const void *, const void *, int, const int32_t *, const uint8_t *, const float *,
                          const float *, int, int, int, float, int32_t *, int32_t *, int32_t *, int32_t *, float *,
                          float *, void *, int32_t *, cudaStream_t);
size_t commit_workspace_bytes(int B, int k, int V);
cudaError_t commit_launch(void *const *, void *const *, const void *const *, const void *const *, int, int, int, int,
                          int, int, int32_t *, const int32_t *, const int32_t *, const void *, int, int, const float *,
                          int32_t *, uint8_t *, int32_t *, void *, int32_t *, cudaStream_t, const int32_t *, int, int);
size_t verify_commit_workspace_bytes(int B, int k, int V);
cudaError_t verify_commit_launch(const void *, const void *, int, const int32_t *, const uint8_t *, const float *,
                                 const float *, float, void *const *, void *const *, const void *const *,
                                 const void *const *, const int32_t *, int, int, int, int, int, int, int, int, int,
                                 int32_t *, const void *, const float *, int32_t *, int32_t *, int32_t *, int32_t *,
                                 float *, float *, int32_t *, uint8_t *, int32_t *, void *, int32_t *, cudaStream_t);

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
bool aligned256(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 255) == 0; }

struct AttnPlan {
    tidar_status status;
    int R, G, M, Mpad, n_splits, mtiles, max_tiles;
    size_t ws_bytes;
};

AttnPlan plan_attn(int B, int Hq, int Hkv, int D, int k, int P_max) {
    AttnPlan pl{};
    if (B < 1 || Hq < 1 || Hkv < 1 || k < 1 || P_max < 0) { pl.status = TIDAR_ERR_INVALID_ARG; return pl; }
    if (Hq % Hkv != 0 || (D != 64 && D != 128) || k > kMaxDraft) { pl.status = TIDAR_ERR_UNSUPPORTED; return pl; }
    pl.R = k * (k + 2);
    pl.G = Hq / Hkv;
    pl.M = pl.R * pl.G;
    const int rows = attn_sm100_rows_per_tile();
    const int keys = attn_sm100_keys_per_tile();
    const int mtiles = ceil_div(pl.M, rows);
    pl.Mpad = mtiles * rows;
    pl.mtiles = mtiles;
    pl.max_tiles = ceil_div(P_max, keys) + ceil_div(pl.R, keys);
    pl.n_splits = 0;  // chosen at launch (needs the device's cluster occupancy)
    pl.ws_bytes = 0;  // split-KV partials move through the cluster's distributed shared memory
    pl.status = TIDAR_OK;
    return pl;
}

tidar_status launched(cudaError_t e) { return e == cudaSuccess ? TIDAR_OK : TIDAR_ERR_CUDA; }

}  // namespace
}  // namespace tidar

using namespace tidar;

extern "C" {

size_t tidar_attn_workspace_size(int B, int Hq, int Hkv, int D, int k, int P_max) {
    const AttnPlan pl = plan_attn(B, Hq, Hkv, D, k, P_max);
    return pl.status == TIDAR_OK ? pl.ws_bytes : 0;
}

namespace {

struct PagedKV {  // a paged cache (block_table null: contiguous caches)
    const int32_t *block_table;
    int max_pages, num_pages;
};

tidar_status attn_step(const void *q, const void *k_new, const void *v_new, const void *k_cache, const void *v_cache,
                       const int32_t *prefix_len, int B, int Hq, int Hkv, int D, int k, int P_max,
                       float softmax_scale, int mask_mode, void *out, float *lse, void *workspace, size_t ws_bytes,
                       int32_t *dev_status, void *stream, long long wait_cycles, int stall_test,
                       PagedKV paged = PagedKV{nullptr, 0, 0}) {
    const AttnPlan pl = plan_attn(B, Hq, Hkv, D, k, P_max);
    if (pl.status != TIDAR_OK) return pl.status;
    if (!q || !k_new || !v_new || !k_cache || !v_cache || !prefix_len || !out || !dev_status)
        return TIDAR_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned16(out) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
        return TIDAR_ERR_INVALID_ARG;
    if (mask_mode != TIDAR_MASK_HYBRID && mask_mode != TIDAR_MASK_CAUSAL) return TIDAR_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale) || !(softmax_scale > 0.f)) return TIDAR_ERR_INVALID_ARG;
    if (pl.ws_bytes > 0) {
        if (!workspace || !aligned256(workspace)) return TIDAR_ERR_INVALID_ARG;
        if (ws_bytes < pl.ws_bytes) return TIDAR_ERR_WORKSPACE;
    }
    AttnParams p;
    p.q = static_cast<const bf16 *>(q);
    p.k_new = static_cast<const bf16 *>(k_new);
    p.v_new = static_cast<const bf16 *>(v_new);
    p.k_cache = static_cast<const bf16 *>(k_cache);
    p.v_cache = static_cast<const bf16 *>(v_cache);
    p.prefix_len = prefix_len;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.D = D;
    p.k = k;
    p.R = pl.R;
    p.G = pl.G;
    p.M = pl.M;
    p.P_max = P_max;
    p.scale_log2 = softmax_scale * kLog2e;
    p.mask_mode = mask_mode;
    // one CTA per SM: every row tile's key tiles are split over a cluster of CTAs so that the whole
    // grid is resident in one wave
    p.n_splits = attn_sm100_pick_splits(D, (long)B * Hkv * pl.mtiles, pl.max_tiles);
    p.Mpad = pl.Mpad;
    p.out = static_cast<bf16 *>(out);
    p.lse = lse;
    p.dev_status = dev_status;
    p.wait_cycles = wait_cycles;
    p.stall_test = stall_test;
    p.block_table = paged.block_table;
    p.max_pages = paged.max_pages;
    p.num_pages = paged.num_pages;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return launched(attn_sm100_launch(p, s));
}

}  // namespace

tidar_status tidar_attn_step(const void *q, const void *k_new, const void *v_new, const void *k_cache,
                             const void *v_cache, const int32_t *prefix_len, int B, int Hq, int Hkv, int D, int k,
                             int P_max, float softmax_scale, int mask_mode, void *out, float *lse, void *workspace,
                             size_t ws_bytes, int32_t *dev_status, void *stream) {
    return attn_step(q, k_new, v_new, k_cache, v_cache, prefix_len, B, Hq, Hkv, D, k, P_max, softmax_scale, mask_mode,
                     out, lse, workspace, ws_bytes, dev_status, stream, kAttnWaitCycles, 0);
}

tidar_status tidar_attn_step_paged(const void *q, const void *k_new, const void *v_new, const void *k_pool,
                                   const void *v_pool, const int32_t *block_table, int max_pages, int num_pages,
                                   const int32_t *prefix_len, int B, int Hq, int Hkv, int D, int k,
                                   float softmax_scale, int mask_mode, void *out, float *lse, int32_t *dev_status,
                                   void *stream) {
    if (!block_table || max_pages < 1 || num_pages < 1) return TIDAR_ERR_INVALID_ARG;
    if (max_pages > kMaxPagesPerSeq) return TIDAR_ERR_UNSUPPORTED;
    if ((long long)num_pages * Hkv * kPageRows >= (1LL << 31)) return TIDAR_ERR_UNSUPPORTED;
    return attn_step(q, k_new, v_new, k_pool, v_pool, prefix_len, B, Hq, Hkv, D, k, max_pages * kPageRows,
                     softmax_scale, mask_mode, out, lse, nullptr, 0, dev_status, stream, kAttnWaitCycles, 0,
                     PagedKV{block_table, max_pages, num_pages});
}

tidar_status tidar_testing_attn_step_stalled(const void *q, const void *k_new, const void *v_new,
                                             const void *k_cache, const void *v_cache, const int32_t *prefix_len,
                                             int B, int Hq, int Hkv, int D, int k, int P_max, float softmax_scale,
                                             int mask_mode, void *out, float *lse, int32_t *dev_status,
                                             long long wait_cycles, void *stream) {
    if (wait_cycles < 1) return TIDAR_ERR_INVALID_ARG;
    return attn_step(q, k_new, v_new, k_cache, v_cache, prefix_len, B, Hq, Hkv, D, k, P_max, softmax_scale, mask_mode,
                     out, lse, nullptr, 0, dev_status, stream, wait_cycles, 1);
}

int tidar_testing_attn_splits(int B, int Hq, int Hkv, int D, int k, int P_max) {
    const AttnPlan pl = plan_attn(B, Hq, Hkv, D, k, P_max);
    if (pl.status != TIDAR_OK) return 0;
    return attn_sm100_pick_splits(D, (long)B * Hkv * pl.mtiles, pl.max_tiles);
}

size_t tidar_verify_workspace_size(int B, int k, int V) {
    if (B < 1 || k < 1 || k > kMaxDraft || V < 1 || V > kMaxVocab) return 0;
    return verify_workspace_bytes(B, k, V);
}

tidar_status tidar_verify_trust_mix(const void *p_logits, const void *q_logits, int logits_dtype,
                                    const int32_t *drafts, const uint8_t *preaccepted, const float *u_acc,
                                    const float *u_res, int B, int k, int V, float trust_ar, int32_t *accept_len,
                                    int32_t *resampled, int32_t *tokens, int32_t *n_emitted, float *logp_d,
                                    float *logq_d, void *workspace, size_t ws_bytes, int32_t *dev_status,
                                    void *stream) {
    if (B < 1 || k < 1 || V < 1) return TIDAR_ERR_INVALID_ARG;
    if (!(trust_ar >= 0.f && trust_ar <= 1.f)) return TIDAR_ERR_INVALID_ARG;
    if (k > kMaxDraft || V > kMaxVocab) return TIDAR_ERR_UNSUPPORTED;
    if (logits_dtype != TIDAR_DT_BF16 && logits_dtype != TIDAR_DT_F32) return TIDAR_ERR_INVALID_ARG;
    if (!p_logits || !q_logits || !drafts || !preaccepted || !u_acc || !u_res || !accept_len || !resampled ||
        !tokens || !n_emitted || !workspace || !dev_status)
        return TIDAR_ERR_INVALID_ARG;
    if (!aligned256(workspace)) return TIDAR_ERR_INVALID_ARG;
    if (ws_bytes < verify_workspace_bytes(B, k, V)) return TIDAR_ERR_WORKSPACE;
    return launched(verify_launch(p_logits, q_logits, logits_dtype, drafts, preaccepted, u_acc, u_res, B, k, V,
                                  trust_ar, accept_len, resampled, tokens, n_emitted, logp_d, logq_d, workspace,
                                  dev_status, static_cast<cudaStream_t>(stream)));
}

tidar_status tidar_verify(const void *p_logits, const void *q_logits, int logits_dtype, const int32_t *drafts,
                          const uint8_t *preaccepted, const float *u_acc, const float *u_res, int B, int k, int V,
                          int32_t *accept_len, int32_t *resampled, int32_t *tokens, int32_t *n_emitted,
                          float *logp_d, float *logq_d, void *workspace, size_t ws_bytes, int32_t *dev_status,
                          void *stream) {
    return tidar_verify_trust_mix(p_logits, q_logits, logits_dtype, drafts, preaccepted, u_acc, u_res, B, k, V, 1.f,
                                  accept_len, resampled, tokens, n_emitted, logp_d, logq_d, workspace, ws_bytes,
                                  dev_status, stream);
}

size_t tidar_kv_commit_workspace_size(int B, int k, int V) {
    if (B < 1 || k < 1 || k > kMaxDraft || V < 1 || V > kMaxVocab) return 0;
    return commit_workspace_bytes(B, k, V);
}

tidar_status tidar_kv_commit(void *const *k_caches, void *const *v_caches, const void *const *k_news,
                             const void *const *v_news, int L, int B, int Hkv, int D, int k, int P_max,
                             int32_t *prefix_len, const int32_t *accept_len, const int32_t *resampled,
                             const void *group_logits, int logits_dtype, int V, const float *u_draft,
                             int32_t *next_drafts, uint8_t *next_preaccepted, int32_t *next_q_group, void *workspace,
                             size_t ws_bytes, int32_t *dev_status, void *stream) {
    if (L < 1 || B < 1 || Hkv < 1 || k < 1 || V < 1 || P_max < 0) return TIDAR_ERR_INVALID_ARG;
    if (k > kMaxDraft || V > kMaxVocab || (D != 64 && D != 128)) return TIDAR_ERR_UNSUPPORTED;
    if (logits_dtype != TIDAR_DT_BF16 && logits_dtype != TIDAR_DT_F32) return TIDAR_ERR_INVALID_ARG;
    if (!k_caches || !v_caches || !k_news || !v_news || !prefix_len || !accept_len || !resampled || !group_logits ||
        !u_draft || !next_drafts || !next_preaccepted || !next_q_group || !workspace || !dev_status)
        return TIDAR_ERR_INVALID_ARG;
    if (!aligned256(workspace)) return TIDAR_ERR_INVALID_ARG;
    if (ws_bytes < commit_workspace_bytes(B, k, V)) return TIDAR_ERR_WORKSPACE;
    return launched(commit_launch(k_caches, v_caches, k_news, v_news, L, B, Hkv, D, k, P_max, prefix_len, accept_len,
                                  resampled, group_logits, logits_dtype, V, u_draft, next_drafts, next_preaccepted,
                                  next_q_group, workspace, dev_status, static_cast<cudaStream_t>(stream), nullptr, 0,
                                  0));
}

tidar_status tidar_kv_commit_paged(void *const *k_pools, void *const *v_pools, const void *const *k_news,
                                   const void *const *v_news, const int32_t *block_table, int max_pages,
                                   int num_pages, int L, int B, int Hkv, int D, int k, int32_t *prefix_len,
                                   const int32_t *accept_len, const int32_t *resampled, const void *group_logits,
                                   int logits_dtype, int V, const float *u_draft, int32_t *next_drafts,
                                   uint8_t *next_preaccepted, int32_t *next_q_group, void *workspace,
                                   size_t ws_bytes, int32_t *dev_status, void *stream) {
    if (!block_table || max_pages < 1 || num_pages < 1) return TIDAR_ERR_INVALID_ARG;
    if (max_pages > kMaxPagesPerSeq) return TIDAR_ERR_UNSUPPORTED;
    if (L < 1 || B < 1 || Hkv < 1 || k < 1 || V < 1) return TIDAR_ERR_INVALID_ARG;
    if (k > kMaxDraft || V > kMaxVocab || (D != 64 && D != 128)) return TIDAR_ERR_UNSUPPORTED;
    if (logits_dtype != TIDAR_DT_BF16 && logits_dtype != TIDAR_DT_F32) return TIDAR_ERR_INVALID_ARG;
    if (!k_pools || !v_pools || !k_news || !v_news || !prefix_len || !accept_len || !resampled || !group_logits ||
        !u_draft || !next_drafts || !next_preaccepted || !next_q_group || !workspace || !dev_status)
        return TIDAR_ERR_INVALID_ARG;
    if (!aligned256(workspace)) return TIDAR_ERR_INVALID_ARG;
    if (ws_bytes < commit_workspace_bytes(B, k, V)) return TIDAR_ERR_WORKSPACE;
    return launched(commit_launch(k_pools, v_pools, k_news, v_news, L, B, Hkv, D, k, max_pages * kPageRows, prefix_len,
                                  accept_len, resampled, group_logits, logits_dtype, V, u_draft, next_drafts,
                                  next_preaccepted, next_q_group, workspace, dev_status,
                                  static_cast<cudaStream_t>(stream), block_table, max_pages, num_pages));
}

size_t tidar_verify_commit_workspace_size(int B, int k, int V) {
    if (B < 1 || k < 1 || k > kMaxDraft || V < 1 || V > kMaxVocab) return 0;
    return verify_commit_workspace_bytes(B, k, V);
}

tidar_status tidar_verify_commit(const void *p_logits, const void *q_logits, int logits_dtype, const int32_t *drafts,
                                 const uint8_t *preaccepted, const float *u_acc, const float *u_res, float trust_ar,
                                 void *const *k_caches, void *const *v_caches, const void *const *k_news,
                                 const void *const *v_news, const int32_t *block_table, int max_pages, int num_pages,
                                 int L, int B, int Hkv, int D, int k, int P_max, int V, int32_t *prefix_len,
                                 const void *group_logits, const float *u_draft, int32_t *accept_len,
                                 int32_t *resampled, int32_t *tokens, int32_t *n_emitted, float *logp_d,
                                 float *logq_d, int32_t *next_drafts, uint8_t *next_preaccepted,
                                 int32_t *next_q_group, void *workspace, size_t ws_bytes, int32_t *dev_status,
                                 void *stream) {
    if (L < 1 || B < 1 || Hkv < 1 || k < 1 || V < 1) return TIDAR_ERR_INVALID_ARG;
    if (!(trust_ar >= 0.f && trust_ar <= 1.f)) return TIDAR_ERR_INVALID_ARG;
    if (k > kMaxDraft || V > kMaxVocab || (D != 64 && D != 128)) return TIDAR_ERR_UNSUPPORTED;
    if (logits_dtype != TIDAR_DT_BF16 && logits_dtype != TIDAR_DT_F32) return TIDAR_ERR_INVALID_ARG;
    if (block_table) {
        if (max_pages < 1 || num_pages < 1) return TIDAR_ERR_INVALID_ARG;
        if (max_pages > kMaxPagesPerSeq) return TIDAR_ERR_UNSUPPORTED;
        P_max = max_pages * kPageRows;
    } else if (P_max < 0) {
        return TIDAR_ERR_INVALID_ARG;
    }
    if (!p_logits || !q_logits || !drafts || !preaccepted || !u_acc || !u_res || !k_caches || !v_caches ||
        !k_news || !v_news || !prefix_len || !group_logits || !u_draft || !accept_len || !resampled || !tokens ||
        !n_emitted || !next_drafts || !next_preaccepted || !next_q_group || !workspace || !dev_status)
        return TIDAR_ERR_INVALID_ARG;
    if (!aligned256(workspace)) return TIDAR_ERR_INVALID_ARG;
    if (ws_bytes < verify_commit_workspace_bytes(B, k, V)) return TIDAR_ERR_WORKSPACE;
    return launched(verify_commit_launch(p_logits, q_logits, logits_dtype, drafts, preaccepted, u_acc, u_res,
                                         trust_ar, k_caches, v_caches, k_news, v_news, block_table,
                                         block_table ? max_pages : 0, block_table ? num_pages : 0, L, B, Hkv, D, k,
                                         P_max, V, prefix_len, group_logits, u_draft, accept_len, resampled, tokens,
                                         n_emitted, logp_d, logq_d, next_drafts, next_preaccepted, next_q_group,
                                         workspace, dev_status, static_cast<cudaStream_t>(stream)));
}

const char *tidar_status_string(tidar_status s) {
    switch (s) {
        case TIDAR_OK: return "TIDAR_OK";
        case TIDAR_ERR_INVALID_ARG: return "TIDAR_ERR_INVALID_ARG";
        case TIDAR_ERR_UNSUPPORTED: return "TIDAR_ERR_UNSUPPORTED";
        case TIDAR_ERR_WORKSPACE: return "TIDAR_ERR_WORKSPACE";
        case TIDAR_ERR_CUDA: return "TIDAR_ERR_CUDA";
    }
    return "TIDAR_STATUS_UNKNOWN";
}

}  // extern "C"
