/*
 * CPU oracle for one TiDAR decode step.  TEST INFRASTRUCTURE ONLY: the tests,
 * the smoke check and the benchmark's CPU-baseline leg call it; the product
 * library never does.  It shares no code, header or constant with the CUDA
 * library.
 *
 * Source: "TiDAR: Think in Diffusion, Talk in Autoregression" (MLSys 2026),
 * awesome-system-papers summary, section 核心方法 -> "并行 self-speculative 生成
 * (§3.2)" (three partitions per step: cached causal prefix; the previous
 * drafts, verified by AR rejection sampling against this step's causal logits;
 * pre-drafts for every possible accept prefix; surplus KV evicted) and
 * "推理优化 (§3.3)" (fixed attention pattern, exact KV cache).  KV keep/evict
 * rules: bxzpzcl.cn "TiDAR架构设计解析", §1.3 推理过程详解.
 *
 * Everything accumulates in double precision.  bf16 inputs are uint16 bit
 * patterns; logits are bf16 bits (dtype 0) or float32 (dtype 1).
 *
 * Row order of the R = k(k+2) query rows (and of the R new keys): rows
 * 0..k-1 are drafts d_1..d_k; row k + j*k + s is slot s of pre-draft group j
 * (j = 0..k).  Group j conditions on d_1..d_j.
 */
#ifndef TIDAR_ORACLE_H
#define TIDAR_ORACLE_H
#include <stdint.h>
#ifdef __cplusplus
extern "C" {
#endif

#define ORACLE_MASK_HYBRID 0
#define ORACLE_MASK_CAUSAL 1
#define ORACLE_LOGITS_BF16 0
#define ORACLE_LOGITS_F32 1

/* Dense [R][P+R] 0/1 mask, filled partition by partition. */
int oracle_hybrid_mask(int k, int P, int mode, uint8_t *mask);

/* Attention for one layer.  q: [B,R,Hq,D]; k_new/v_new: [B,R,Hkv,D];
 * caches: [B,Hkv,P_max,D]; prefix_len: [B].  Outputs o: [B,R,Hq,D] double,
 * lse: [B,R,Hq] double (natural log of the scaled scores), o_bf16 (nullable):
 * o rounded to bf16, ties to even.  use_dense: 1 = read the materialised
 * mask, 0 = evaluate the index predicate.  Rows run in parallel with OpenMP
 * when nthreads > 1. */
int oracle_attn(const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new,
                const uint16_t *k_cache, const uint16_t *v_cache, const int32_t *prefix_len,
                int B, int Hq, int Hkv, int D, int k, int P_max, double scale, int mode,
                int use_dense, int nthreads, double *o, double *lse, uint16_t *o_bf16);

/* The same, for n selected (b, h, r) rows only; outputs are [n][D] and [n]. */
int oracle_attn_rows(const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new,
                     const uint16_t *k_cache, const uint16_t *v_cache, const int32_t *prefix_len,
                     int B, int Hq, int Hkv, int D, int k, int P_max, double scale, int mode,
                     int n, const int32_t *sel_b, const int32_t *sel_h, const int32_t *sel_r,
                     int nthreads, double *o, double *lse);

/* AR rejection-sampling verify.  p/q logits: [B,k,V]; drafts [B,k];
 * preaccepted [B]; u_acc [B,k]; u_res [B].  trust_ar in [0, 1]: the target
 * distribution is softmax(trust_ar * p_logits + (1 - trust_ar) * q_logits)
 * (1 = the AR logits alone).  forced_accept_len (nullable,
 * entries < 0 mean "not forced") overrides the accept decision (used to keep
 * comparing after an exempt near-tie).  Outputs: accept_len [B], resampled [B]
 * (-1 if every draft was accepted), tokens [B,k] (-1 padded), n_emitted [B],
 * logp_d/logq_d [B,k], ratio [B,k] (p(d)/q(d); NaN where not evaluated),
 * res_lo/res_hi [B] (the chosen token's interval of the normalised residual
 * CDF; NaN when no resample). */
int oracle_verify(const void *p_logits, const void *q_logits, int logits_dtype,
                  const int32_t *drafts, const uint8_t *preaccepted,
                  const float *u_acc, const float *u_res, int B, int k, int V, double trust_ar,
                  const int32_t *forced_accept_len, int nthreads,
                  int32_t *accept_len, int32_t *resampled, int32_t *tokens, int32_t *n_emitted,
                  double *logp_d, double *logq_d, double *ratio, double *res_lo, double *res_hi);

/* KV commit / evict plus next-draft selection.  Caches: [L,B,Hkv,P_max,D];
 * new K/V: [L,B,R,Hkv,D]; prefix_len [B] updated in place; group_logits
 * [B,k+1,k,V]; u_draft [B,k].  Outputs next_drafts [B,k], next_preaccepted
 * [B], next_q_group [B], draft_lo/draft_hi [B,k] (interval of the chosen token
 * in the normalised CDF). */
int oracle_kv_commit(uint16_t *k_caches, uint16_t *v_caches,
                     const uint16_t *k_news, const uint16_t *v_news,
                     int L, int B, int Hkv, int D, int k, int P_max,
                     int32_t *prefix_len, const int32_t *accept_len, const int32_t *resampled,
                     const void *group_logits, int logits_dtype, int V, const float *u_draft,
                     int nthreads,
                     int32_t *next_drafts, uint8_t *next_preaccepted, int32_t *next_q_group,
                     double *draft_lo, double *draft_hi);

/* Position of row r (0..R-1) of a step whose sequence has cached prefix P. */
int oracle_row_position(int k, int P, int r);

/* Rotary embedding of the fused QKV projection output qkv [B,R,Hq+2Hkv,D]
 * (bf16 bits) into q [B,R,Hq,D], k_new and v_new [B,R,Hkv,D] (bf16 bits). */
int oracle_rope_qkv(const uint16_t *qkv, const int32_t *prefix_len, int B, int Hq, int Hkv, int D, int k,
                    double theta, uint16_t *q, uint16_t *k_new, uint16_t *v_new);

#ifdef __cplusplus
}
#endif
#endif
