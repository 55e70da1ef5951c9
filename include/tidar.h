/*
 * tidar.h -- C ABI of the B200 (sm_100a) TiDAR decode-step library.
 *
 * One TiDAR decode step ("TiDAR: Think in Diffusion, Talk in Autoregression",
 * MLSys 2026; awesome-system-papers summary, section 核心方法, "并行
 * self-speculative 生成 (§3.2)") runs, per layer, a single forward over three
 * partitions -- the cached causal prefix, the k drafts of the previous step,
 * and k+1 pre-draft groups of k mask tokens -- then verifies the drafts by AR
 * rejection sampling, evicts the rejected drafts' KV and takes the next draft
 * block from the pre-draft group that matches the accept length.
 *
 * Three calls cover that hot path:
 *   tidar_attn_step   the structured hybrid-mask attention of one layer;
 *   tidar_verify      the AR rejection-sampling verify of the drafts;
 *   tidar_kv_commit   the exact-KV-cache commit/evict + next-draft selection;
 * tidar_verify_commit makes the last two in one launch.
 *
 * Conventions shared by every call
 * --------------------------------
 * - k = draft length (1..16); R = k(k+2) query rows per sequence.  Rows (and
 *   the R new keys) are ordered: rows 0..k-1 = drafts d_1..d_k; row
 *   k + j*k + s = slot s of pre-draft group j (j = 0..k).
 * - All pointers are DEVICE pointers unless stated otherwise.  The caller owns
 *   every buffer; the library allocates no device memory, keeps no pointer
 *   after a call returns and holds no per-call state.
 * - Every call is asynchronous: it validates its scalar arguments on the host,
 *   enqueues its kernels on `stream` (a cudaStream_t; NULL = legacy default
 *   stream) and returns.  Outputs are valid in stream order.
 * - Host-side argument errors return TIDAR_ERR_INVALID_ARG (bad pointer or
 *   size), TIDAR_ERR_UNSUPPORTED (a shape outside the supported set) or
 *   TIDAR_ERR_WORKSPACE (workspace too small) before anything is launched.
 *   A failed launch returns TIDAR_ERR_CUDA.
 * - Data-dependent errors are found on the device: the kernels OR a
 *   TIDAR_DEV_* bit into *dev_status (an int32 the caller zeroes and reads
 *   when it chooses) and skip the affected sequence.  No kernel traps, asserts
 *   or waits without a bound.
 */
#ifndef TIDAR_H
#define TIDAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TIDAR_OK = 0,
    TIDAR_ERR_INVALID_ARG = 1,
    TIDAR_ERR_UNSUPPORTED = 2,
    TIDAR_ERR_WORKSPACE = 3,
    TIDAR_ERR_CUDA = 4
} tidar_status;

/* bits of *dev_status */
#define TIDAR_DEV_BAD_PREFIX 1 /* prefix_len[b] < 0, or beyond the cache capacity */
#define TIDAR_DEV_BAD_TOKEN 2  /* a draft or resampled token outside [0, V) */
#define TIDAR_DEV_BAD_ACCEPT 4 /* accept_len[b] outside [0, k] */
#define TIDAR_DEV_TIMEOUT 8    /* a bounded on-chip wait expired; the outputs are not valid */
#define TIDAR_DEV_BAD_PAGE 16  /* a block-table entry outside [0, num_pages) (paged caches) */

typedef enum { TIDAR_DT_BF16 = 0, TIDAR_DT_F32 = 1 } tidar_dtype;

typedef enum {
    TIDAR_MASK_HYBRID = 0, /* the TiDAR decode mask (below) */
    TIDAR_MASK_CAUSAL = 1  /* plain causal attention over prefix + R tokens (pure AR mode) */
} tidar_mask_mode;

/* ------------------------------------------------------------------------ */
/* Attention                                                                 */
/* ------------------------------------------------------------------------ */

/* Bytes of device scratch tidar_attn_step needs for these sizes.  It is 0 for
 * every size: the partial rows of the split-KV reduction pass between the CTAs
 * of a thread-block cluster through distributed shared memory.  Invalid sizes
 * are reported by tidar_attn_step itself. */
size_t tidar_attn_workspace_size(int B, int Hq, int Hkv, int D, int k, int P_max);

/*
 * One layer of TiDAR hybrid-mask attention.
 *
 * Defined by: TiDAR summary §3.2 (three partitions in one forward; drafts are
 * verified with this step's causal logits; pre-draft group j is conditioned on
 * the accept prefix d_1..d_j) and §3.3 (fixed per-step attention pattern over
 * an exact KV cache); the bxzpzcl.cn walkthrough §1.2 (only the last block is
 * bidirectional).  Mask for query row r and key n (keys in the order
 * [cache rows 0..P_b-1 | the R new keys]): every cached key is visible; draft
 * d_i sees drafts d_1..d_i; a slot of group j sees d_1..d_j and the k slots of
 * group j; drafts never see mask tokens.  The mask is evaluated from indices.
 * TIDAR_MASK_CAUSAL instead gives row r the keys 0..P_b+r (the pages' pure
 * causal likelihood mode).
 *
 * q          bf16 [B, R, Hq, D]   post-RoPE queries
 * k_new      bf16 [B, R, Hkv, D]  post-RoPE keys of this step's R tokens
 * v_new      bf16 [B, R, Hkv, D]
 * k_cache    bf16 [B, Hkv, P_max, D]  rows 0..P_b-1 are used; whole 128-row tiles
 *            are read (with a contiguous cache also up to 15 tiles from row 0
 *            whatever P_b is), always inside the buffer, and rows past P_b are
 *            ignored, whatever they hold (NaN included)
 * v_cache    bf16 [B, Hkv, P_max, D]  (likewise)
 * prefix_len int32 [B]  P_b, 0 <= P_b <= P_max
 * Hq % Hkv == 0; query head h reads KV head h / (Hq/Hkv).  D in {64, 128}.
 * softmax_scale  score multiplier, > 0 (1/sqrt(D) for the standard scale).
 * out        bf16 [B, R, Hq, D]  softmax(scale * q k^T) v over the visible keys
 * lse        f32  [B, R, Hq] or NULL: natural-log log-sum-exp of the scaled scores
 * workspace  >= tidar_attn_workspace_size(...) bytes of device memory, 256-byte
 *            aligned; may be NULL (with ws_bytes 0) when that size is 0.
 * dev_status int32*; TIDAR_DEV_BAD_PREFIX set (and that sequence skipped) when
 *            a prefix length is out of range.
 * All tensor pointers must be 16-byte aligned.
 */
tidar_status tidar_attn_step(const void *q, const void *k_new, const void *v_new,
                             const void *k_cache, const void *v_cache, const int32_t *prefix_len,
                             int B, int Hq, int Hkv, int D, int k, int P_max, float softmax_scale,
                             int mask_mode, void *out, float *lse, void *workspace, size_t ws_bytes,
                             int32_t *dev_status, void *stream);

/*
 * tidar_attn_step over a paged KV cache.
 *
 * Defined by: as tidar_attn_step; the paging is the serving layout the TiDAR
 * summary names as the next step beyond its batch-1 runs ("局限与 Future Work":
 * batch > 1, continuous batching and PagedAttention left untested).  Cache row
 * n of sequence b is row n % 64 of page block_table[b * max_pages + n / 64] of
 * the pools:
 *
 * k_pool, v_pool  bf16 [num_pages, Hkv, 64, D]: pages shared by all sequences;
 *                 a sequence's pages need not be contiguous or ordered
 * block_table     int32 [B, max_pages] (device): page ids of each sequence's
 *                 cache rows, in row order; entries past ceil(P_b / 64) are
 *                 not read.  1 <= max_pages <= 1024 (P_b <= 64 * max_pages).
 * Everything else as tidar_attn_step (no workspace).  A page id outside
 * [0, num_pages) sets TIDAR_DEV_BAD_PAGE and that sequence is skipped.  The
 * results equal tidar_attn_step's on the same rows laid out contiguously.
 */
tidar_status tidar_attn_step_paged(const void *q, const void *k_new, const void *v_new,
                                   const void *k_pool, const void *v_pool, const int32_t *block_table,
                                   int max_pages, int num_pages, const int32_t *prefix_len,
                                   int B, int Hq, int Hkv, int D, int k, float softmax_scale,
                                   int mask_mode, void *out, float *lse, int32_t *dev_status, void *stream);

/*
 * Rotary position embedding of one step's rows, fused with the re-layout of the
 * QKV projection output into tidar_attn_step's inputs (q, k_new, v_new).
 *
 * Defined by: the Qwen backbones the TiDAR pages start from (summary, 核心方法 /
 * initialisation: Qwen2.5-1.5B, Qwen3-8B; rotary embedding, base theta = 1e6
 * for both) and the step layout of summary §3.2.  Row positions (the pages
 * give the partitions, not the positions): draft d_i at P_b + i - 1; slot s of
 * pre-draft group j at P_b + j + s.  Pair (x_i, x_{i+D/2}), i < D/2, of every
 * query and key head is rotated by pos * theta^(-2i/D); value heads are copied.
 * The rotation is computed in double precision and rounded once to bf16.
 *
 * qkv        bf16 [B, R, Hq + 2 Hkv, D]: Q heads, then K heads, then V heads
 * prefix_len int32 [B] (device)
 * theta      rotary base, > 1
 * q          bf16 [B, R, Hq, D]; k_new, v_new bf16 [B, R, Hkv, D]
 * D in {64, 128}, Hq % Hkv == 0, k in 1..16; all tensors 4-byte aligned.
 * dev_status TIDAR_DEV_BAD_PREFIX (and that sequence's Q/K left unwritten) for
 *            a negative prefix length.
 */
tidar_status tidar_rope_qkv(const void *qkv, const int32_t *prefix_len, int B, int Hq, int Hkv, int D, int k,
                            double theta, void *q, void *k_new, void *v_new, int32_t *dev_status, void *stream);

/* ------------------------------------------------------------------------ */
/* Verify                                                                    */
/* ------------------------------------------------------------------------ */

size_t tidar_verify_workspace_size(int B, int k, int V);

/*
 * AR rejection-sampling verify of the previous step's drafts.
 *
 * Defined by: TiDAR summary §3.2 ("Talk": the previous drafts, proposed from
 * the diffusion marginals, are verified by AR rejection sampling against this
 * step's causal logits); the speculative-sampling rule it names: draft d_i is
 * accepted with probability min(1, p_i(d_i)/q_i(d_i)), the scan stops at the
 * first rejection, and a replacement is drawn from norm(max(0, p - q)) at the
 * rejected slot.
 *
 * p_logits   [B, k, V] (bf16 or f32 per logits_dtype): AR logits for slots
 *            1..k (slot 1's row is carried from the previous forward; slot i>1
 *            is the causal output of draft row i-1).  p = softmax(row).
 * q_logits   [B, k, V]: the stored diffusion logits that proposed the drafts.
 * drafts     int32 [B, k]; preaccepted uint8 [B]: 1 = slot 1 is the previous
 *            step's resampled token and is accepted unconditionally.
 * u_acc      f32 [B, k] uniforms in [0,1): slot i accepted iff u < p(d)/q(d).
 * u_res      f32 [B]: the residual draw picks the smallest v with
 *            sum_{w<=v} r(w) > u * sum r, r = max(0, p - q).
 * accept_len int32 [B]    j* = number of leading accepted slots
 * resampled  int32 [B]    the residual draw, or -1 when j* = k
 * tokens     int32 [B, k] tokens emitted this step (accepted drafts that were
 *            not pre-accepted, then the resampled token), -1 padded
 * n_emitted  int32 [B]
 * logp_d, logq_d  f32 [B, k] or NULL: log p_i(d_i), log q_i(d_i)
 * dev_status TIDAR_DEV_BAD_TOKEN when a draft is outside [0, V).
 * V <= 524288 (else TIDAR_ERR_UNSUPPORTED).
 */
tidar_status tidar_verify(const void *p_logits, const void *q_logits, int logits_dtype,
                          const int32_t *drafts, const uint8_t *preaccepted,
                          const float *u_acc, const float *u_res, int B, int k, int V,
                          int32_t *accept_len, int32_t *resampled, int32_t *tokens, int32_t *n_emitted,
                          float *logp_d, float *logq_d, void *workspace, size_t ws_bytes,
                          int32_t *dev_status, void *stream);

/*
 * tidar_verify with a trust-mixed target.
 *
 * Defined by: TiDAR summary, "Trust AR vs trust diffusion logits (验证时混合)"
 * (Fig. 6: the AR and diffusion logits are mixed with a weight lambda at
 * verification; quality barely moves across lambda) and the notes.yuuk.io talk
 * notes §生成評価 ("Trust Diff" mode).  The target of the rejection test of slot
 * i becomes p_i = softmax(trust_ar * p_logits_i + (1 - trust_ar) * q_logits_i)
 * (q_logits_i, the stored diffusion logits that proposed d_i, serve as the
 * diffusion logits of that position): draft d_i is accepted with probability
 * min(1, p_i(d_i)/q_i(d_i)) and a rejection draws from norm(max(0, p_i - q_i)).
 * trust_ar = 1 is tidar_verify; trust_ar = 0 accepts every draft.  The mix is
 * formed in fp32 from the stored logits; at the endpoints the stored row is
 * used as is.
 *
 * trust_ar   in [0, 1], else TIDAR_ERR_INVALID_ARG.  logp_d receives
 *            log p_i(d_i) of the mixed target.  Everything else as tidar_verify
 *            (same workspace size).
 */
tidar_status tidar_verify_trust_mix(const void *p_logits, const void *q_logits, int logits_dtype,
                                    const int32_t *drafts, const uint8_t *preaccepted,
                                    const float *u_acc, const float *u_res, int B, int k, int V, float trust_ar,
                                    int32_t *accept_len, int32_t *resampled, int32_t *tokens, int32_t *n_emitted,
                                    float *logp_d, float *logq_d, void *workspace, size_t ws_bytes,
                                    int32_t *dev_status, void *stream);

/*
 * tidar_verify without a caller workspace.  The paper has no counterpart: this
 * entry point exists for callers that cannot allocate device memory -- e.g. a
 * plug-in inside a host runtime that owns all device memory and forbids
 * cudaMalloc on its decode path, or a serving loop that must not allocate after
 * start-up -- and so cannot pass the workspace tidar_verify needs.
 *
 * Arguments, outputs, device-status bits and results are those of
 * tidar_verify.  The scratch is a fixed 2 MiB device array inside the library
 * (held by every GPU that loads it until the process exits); calls whose
 * tidar_verify_workspace_size(B, k, V) exceeds 2 MiB return
 * TIDAR_ERR_WORKSPACE without launching.  The first call on each device
 * resolves the array's device address (cudaGetSymbolAddress) with that device
 * current, so it should come before any stream capture.  All calls on a device
 * share the array: calls whose kernels may overlap on the GPU race on it and
 * must be ordered by the caller.  The library allocates nothing for this call.
 */
tidar_status tidar_verify_noalloc(const void *p_logits, const void *q_logits, int logits_dtype,
                                  const int32_t *drafts, const uint8_t *preaccepted,
                                  const float *u_acc, const float *u_res, int B, int k, int V,
                                  int32_t *accept_len, int32_t *resampled, int32_t *tokens, int32_t *n_emitted,
                                  float *logp_d, float *logq_d, int32_t *dev_status, void *stream);

/* ------------------------------------------------------------------------ */
/* Commit                                                                    */
/* ------------------------------------------------------------------------ */

size_t tidar_kv_commit_workspace_size(int B, int k, int V);

/*
 * Exact-KV-cache commit/evict plus next-draft selection.
 *
 * Defined by: TiDAR summary §3.2 (KV beyond the accept length is evicted, no
 * recompute) and §3.3 (exact KV cache); the bxzpzcl.cn walkthrough §1.3 (keep
 * the KV of causally computed accepted tokens, drop rejected tokens' KV at
 * once, pre-draft tokens never occupy the persistent cache) and §2.2; the
 * summary's 观察 2 / §3.2 on one-step drafting (each slot drawn independently
 * from its diffusion marginal) and pre-drafting for every accept outcome.
 *
 * For every layer l and sequence b the first accept_len[b] new-key rows (the
 * accepted drafts, which attended causally, so their K/V equal plain AR K/V)
 * are copied from k_news[l]/v_news[l] ([B, R, Hkv, D]) into cache rows
 * P_b .. P_b+j*-1 of k_caches[l]/v_caches[l] ([B, Hkv, P_max, D]); then
 * prefix_len[b] += j*.  Nothing else in the caches is written.
 * Next drafts: slot s is the smallest v with sum_{w<=v} softmax(g)(w) > u_draft
 * [b,s] for g = group_logits[b, j*, s, :]; when j* < k slot 0 is replaced by
 * resampled[b] and next_preaccepted[b] = 1, else 0.  next_q_group[b] = j*: the
 * caller's next q_logits are rows group_logits[b, j*, :, :].
 *
 * k_caches, v_caches   device array of L device pointers (bf16 caches)
 * k_news, v_news       device array of L device pointers (bf16 new K/V)
 * prefix_len           int32 [B], read and updated in place
 * accept_len, resampled  int32 [B] from tidar_verify
 * group_logits         [B, k+1, k, V] (bf16 or f32); u_draft f32 [B, k]
 * next_drafts int32 [B, k]; next_preaccepted uint8 [B]; next_q_group int32 [B]
 * dev_status  TIDAR_DEV_BAD_ACCEPT / TIDAR_DEV_BAD_PREFIX / TIDAR_DEV_BAD_TOKEN
 *             when accept_len, P_b + j* or resampled is out of range; that
 *             sequence is then left untouched.
 * V <= 524288 (else TIDAR_ERR_UNSUPPORTED).
 */
tidar_status tidar_kv_commit(void *const *k_caches, void *const *v_caches,
                             const void *const *k_news, const void *const *v_news,
                             int L, int B, int Hkv, int D, int k, int P_max,
                             int32_t *prefix_len, const int32_t *accept_len, const int32_t *resampled,
                             const void *group_logits, int logits_dtype, int V, const float *u_draft,
                             int32_t *next_drafts, uint8_t *next_preaccepted, int32_t *next_q_group,
                             void *workspace, size_t ws_bytes, int32_t *dev_status, void *stream);

/* ------------------------------------------------------------------------ */
/* Draft length (host functions, no device work)                             */
/* ------------------------------------------------------------------------ */

/*
 * Expected number of tokens one decode step emits in steady state when every
 * draft is accepted independently with probability alpha, at draft length k.
 *
 * Defined by: the decode step of this library (summary §3.2: a rejected draft
 * is replaced by a draw from the residual; the pre-drafts of group j* become
 * the next drafts), read as a two-state chain: a step with a pre-accepted slot
 * 1 (the previous step's resampled token, already emitted) tests k - 1 drafts,
 * one without tests k.  Testing m drafts emits sum_{i=1..m} alpha^i + (1 -
 * alpha^m) new tokens on average (the accepted drafts, then the resampled
 * token unless all m were accepted).  Returns E, or -1 for k outside 1..16 or
 * alpha outside [0, 1].
 */
double tidar_expected_tokens_per_step(int k, double alpha);

/*
 * Draft length that maximises expected tokens per microsecond.
 *
 * Defined by: the summary's "局限与 Future Work" (Future work 2: choose the
 * draft block to fit the GPU's free token slots) and the zero-shot draft
 * length of §3.3 (the draft length can change at inference time).
 * step_us[k-1] (host array of n <= 16 doubles) is the latency of one decode
 * step at draft length k -- measured (bench.py --k-sweep) or from a roofline
 * model; entries <= 0 or non-finite are skipped.  Returns the k in 1..n with
 * the largest tidar_expected_tokens_per_step(k, alpha) / step_us[k-1] (the
 * shorter k on a tie) and writes that rate to *tokens_per_us (nullable); 0 on
 * invalid arguments or when no entry is usable.
 */
int tidar_pick_draft_length(const double *step_us, int n, double alpha, double *tokens_per_us);

/*
 * tidar_kv_commit over paged KV caches (see tidar_attn_step_paged for the
 * layout).  k_pools / v_pools: device arrays of L device pointers, one pool
 * [num_pages, Hkv, 64, D] per layer; block_table [B, max_pages] as for the
 * attention.  The pages that receive rows P_b .. P_b + j* - 1 must already be
 * in the block table (the caller allocates pages before the step); an invalid
 * id there sets TIDAR_DEV_BAD_PAGE and leaves the sequence untouched.
 * Everything else as tidar_kv_commit (same workspace size).
 */
tidar_status tidar_kv_commit_paged(void *const *k_pools, void *const *v_pools,
                                   const void *const *k_news, const void *const *v_news,
                                   const int32_t *block_table, int max_pages, int num_pages,
                                   int L, int B, int Hkv, int D, int k,
                                   int32_t *prefix_len, const int32_t *accept_len, const int32_t *resampled,
                                   const void *group_logits, int logits_dtype, int V, const float *u_draft,
                                   int32_t *next_drafts, uint8_t *next_preaccepted, int32_t *next_q_group,
                                   void *workspace, size_t ws_bytes, int32_t *dev_status, void *stream);

/* ------------------------------------------------------------------------ */
/* Verify + commit in one launch                                             */
/* ------------------------------------------------------------------------ */

size_t tidar_verify_commit_workspace_size(int B, int k, int V);

/*
 * tidar_verify_trust_mix followed by tidar_kv_commit (tidar_kv_commit_paged
 * when block_table is not NULL) as one launch: the verify's accept length j*
 * and replacement token feed the commit directly.
 *
 * Defined by: the same passages as the two calls it replaces (TiDAR summary
 * §3.2 "Talk" / "Think": the drafts are verified, the KV of the accepted ones
 * is kept, and the pre-drafts of the group matching the accept outcome become
 * the next drafts -- all within one decode step).  The results are those of
 * the two calls made in turn on the same arguments, with these differences:
 *  - the commit's P_b is prefix_len[b] as it was when the call started (the
 *    commit never reads its own update);
 *  - a sequence with a draft outside [0, V) (TIDAR_DEV_BAD_TOKEN) is left
 *    untouched by the commit, since it has no accept length;
 *  - with a block table, P_max is ignored (the capacity is max_pages * 64);
 *    block_table, max_pages and num_pages are as for tidar_kv_commit_paged;
 *  - if the replacement draw finds no token (every weight zero, which only an
 *    all -inf row allows), TIDAR_DEV_BAD_TOKEN is set and the sequence's
 *    state (prefix_len, next_q_group, next_preaccepted, next_drafts[b][0]) is
 *    not advanced; cache rows P_b .. P_b + j* - 1 may have been written.
 * The verify outputs (accept_len, resampled, tokens, n_emitted, logp_d,
 * logq_d) are written as tidar_verify writes them, also for a sequence whose
 * commit inputs are invalid (prefix or page; that sequence's commit is
 * skipped with the matching TIDAR_DEV_* bit).  trust_ar = 1 is the plain AR
 * verify.  V <= 524288.  The workspace is tidar_verify_commit_workspace_size
 * bytes, 256-byte aligned.
 */
tidar_status tidar_verify_commit(const void *p_logits, const void *q_logits, int logits_dtype,
                                 const int32_t *drafts, const uint8_t *preaccepted,
                                 const float *u_acc, const float *u_res, float trust_ar,
                                 void *const *k_caches, void *const *v_caches,
                                 const void *const *k_news, const void *const *v_news,
                                 const int32_t *block_table, int max_pages, int num_pages,
                                 int L, int B, int Hkv, int D, int k, int P_max, int V,
                                 int32_t *prefix_len, const void *group_logits, const float *u_draft,
                                 int32_t *accept_len, int32_t *resampled, int32_t *tokens, int32_t *n_emitted,
                                 float *logp_d, float *logq_d, int32_t *next_drafts, uint8_t *next_preaccepted,
                                 int32_t *next_q_group, void *workspace, size_t ws_bytes, int32_t *dev_status,
                                 void *stream);

/* Human-readable name of a status code (static storage). */
const char *tidar_status_string(tidar_status s);

#ifdef __cplusplus
}
#endif
#endif /* TIDAR_H */
