// Exact-KV-cache commit / evict and next-draft selection (one kernel).
//
// Two kinds of CTAs in one grid:
//   - copy CTAs (one per layer x sequence x KV head): the first j* new-key
//     rows (accepted drafts) of K/V are copied into cache rows P..P+j*-1, 16
//     bytes per thread.  Rejected drafts and mask tokens are never written:
//     eviction is simply not committing them.
//   - draft CTAs (chunks x k slots x B): per-chunk max / sum-exp of slot s of
//     pre-draft group j*.  The last CTA of a (sequence, slot) row to finish
//     (an atomic counter; nobody waits) merges the row's statistics, finds the
//     chunk that holds u_draft * Z and rescans it with a block prefix scan:
//     slot s of the next draft block.  After a rejection slot 0 is the
//     resampled token instead.
// The last CTA of a sequence (over both kinds) writes next_q_group and
// next_preaccepted and advances prefix_len by j*, after every copy CTA of that
// sequence has read the old prefix length.  The counters are zeroed in stream
// order before the launch.
#include "vocab.cuh"

namespace tidar {

namespace {

struct CommitParams {
    void *const *k_caches;
    void *const *v_caches;
    const void *const *k_news;
    const void *const *v_news;
    int L, B, Hkv, D, k, R, P_max;
    int32_t *prefix_len;
    const int32_t *accept_len, *resampled;
    const void *group_logits;
    int dtype, V, nchunk;
    const float *u_draft;
    int32_t *next_drafts;
    uint8_t *next_preaccepted;
    int32_t *next_q_group;
    ChunkStat *stats;     // [B][k][nchunk]
    int32_t *row_count;   // [B][k] draft CTAs done per row
    int32_t *seq_count;   // [B] CTAs done per sequence
    int32_t *dev_status;
    int n_copy_ctas;
};

// Validates the commit inputs of sequence b; returns j* or -1.
__device__ __forceinline__ int checked_accept(const CommitParams &p, int b, bool report) {
    const int j = p.accept_len[b];
    const int P = p.prefix_len[b];
    int bits = 0;
    if (j < 0 || j > p.k) bits |= TIDAR_DEV_BAD_ACCEPT;
    if (P < 0 || (bits == 0 && P + j > p.P_max)) bits |= TIDAR_DEV_BAD_PREFIX;
    if (bits == 0 && j < p.k && (p.resampled[b] < 0 || p.resampled[b] >= p.V)) bits |= TIDAR_DEV_BAD_TOKEN;
    if (bits) {
        if (report) atomicOr(p.dev_status, bits);
        return -1;
    }
    return j;
}

__device__ __forceinline__ const void *group_row(const CommitParams &p, int b, int j, int s) {
    const size_t es = p.dtype == TIDAR_DT_BF16 ? 2 : 4;
    const size_t row = ((size_t)b * (p.k + 1) + j) * p.k + s;
    return reinterpret_cast<const uint8_t *>(p.group_logits) + row * p.V * es;
}

__global__ void __launch_bounds__(kStatThreads) commit_kernel(const CommitParams p) {
    __shared__ float redf[8];
    __shared__ double redd[8], scan_buf[8];
    __shared__ int s_flag, s_pick[2], s_chunk;
    __shared__ double s_target;
    __shared__ float s_m;
    const int cta = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int b, j;
    if (cta < p.n_copy_ctas) {
        // ---- accepted K/V rows into the cache ----
        const int kvh = cta % p.Hkv;
        b = (cta / p.Hkv) % p.B;
        const int l = cta / (p.Hkv * p.B);
        j = checked_accept(p, b, l == 0 && kvh == 0 && tid == 0);
        if (j > 0) {
            const int P = p.prefix_len[b];
            const int vec = p.D / 8;  // 16-byte vectors per row
            const bf16 *kn = reinterpret_cast<const bf16 *>(p.k_news[l]);
            const bf16 *vn = reinterpret_cast<const bf16 *>(p.v_news[l]);
            bf16 *kc = reinterpret_cast<bf16 *>(p.k_caches[l]);
            bf16 *vc = reinterpret_cast<bf16 *>(p.v_caches[l]);
            for (int idx = tid; idx < j * vec; idx += blockDim.x) {
                const int i = idx / vec, c = idx % vec;
                const size_t src = ((size_t)(b * p.R + i) * p.Hkv + kvh) * p.D + c * 8;
                const size_t dst = ((size_t)(b * p.Hkv + kvh) * p.P_max + P + i) * p.D + c * 8;
                *reinterpret_cast<uint4 *>(kc + dst) = *reinterpret_cast<const uint4 *>(kn + src);
                *reinterpret_cast<uint4 *>(vc + dst) = *reinterpret_cast<const uint4 *>(vn + src);
            }
        }
    } else {
        // ---- one chunk of slot s of pre-draft group j* ----
        const int t = cta - p.n_copy_ctas;
        const int c = t % p.nchunk;
        const int s = (t / p.nchunk) % p.k;
        b = t / (p.nchunk * p.k);
        j = checked_accept(p, b, false);
        if (j >= 0 && s == 0 && j < p.k) {  // slot 0 is the resampled token
            if (c == 0 && tid == 0) p.next_drafts[(size_t)b * p.k] = p.resampled[b];
        } else if (j >= 0) {
            const void *row = group_row(p, b, j, s);
            const ChunkStat st = chunk_stat(row, p.dtype, p.V, c, redf, redd);
            if (tid == 0) p.stats[((size_t)b * p.k + s) * p.nchunk + c] = st;
            __threadfence();
            __syncthreads();
            if (tid == 0) s_flag = atomicAdd(&p.row_count[b * p.k + s], 1) == p.nchunk - 1;
            __syncthreads();
            if (s_flag) {  // the last chunk of this row: draw slot s
                __threadfence();
                if (warp == 0) {
                    const ChunkStat *rs = p.stats + ((size_t)b * p.k + s) * p.nchunk;
                    float m = -INFINITY;
                    for (int cc = lane; cc < p.nchunk; cc += 32) m = fmaxf(m, __ldcg(&rs[cc].m));
                    m = warp_max(m);
                    double tot = 0.0;
                    for (int cc = lane; cc < p.nchunk; cc += 32) {
                        const float mc = __ldcg(&rs[cc].m);
                        if (mc != -INFINITY) tot += __ldcg(&rs[cc].z) * (double)exp2f((mc - m) * kLog2e);
                    }
                    tot = warp_sum_d(tot);
                    const double target = (double)p.u_draft[(size_t)b * p.k + s] * tot;
                    double run = 0.0, before = 0.0;
                    int ch = -1, last_pos = -1;
                    for (int c0 = 0; c0 < p.nchunk && ch < 0; c0 += 32) {
                        const int cc = c0 + lane;
                        double wc = 0.0;
                        if (cc < p.nchunk) {
                            const float mc = __ldcg(&rs[cc].m);
                            if (mc != -INFINITY) wc = __ldcg(&rs[cc].z) * (double)exp2f((mc - m) * kLog2e);
                        }
                        double incl = wc;
#pragma unroll
                        for (int o = 1; o < 32; o <<= 1) {
                            const double y = __shfl_up_sync(0xffffffffu, incl, o);
                            if (lane >= o) incl += y;
                        }
                        const unsigned hit = __ballot_sync(0xffffffffu, wc > 0.0 && run + incl > target);
                        const unsigned pos = __ballot_sync(0xffffffffu, wc > 0.0);
                        if (pos) last_pos = c0 + 31 - __clz(pos);
                        if (hit) {
                            const int hl = __ffs(hit) - 1;
                            ch = c0 + hl;
                            before = run + __shfl_sync(0xffffffffu, incl - wc, hl);
                        }
                        run += __shfl_sync(0xffffffffu, incl, 31);
                    }
                    if (lane == 0) {
                        s_chunk = ch >= 0 ? ch : last_pos;
                        s_target = ch >= 0 ? target - before : INFINITY;  // not found only through rounding
                        s_m = m;
                    }
                }
                __syncthreads();
                if (s_chunk < 0) {  // every logit of the row is -inf: no distribution to draw from
                    if (tid == 0) p.next_drafts[(size_t)b * p.k + s] = -1;
                } else {
                    float z[32];
                    load_chunk32_contig(row, p.dtype, p.V, s_chunk, z);
                    const float ms = s_m * kLog2e;
                    double w[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        w[e] = z[e] == -INFINITY ? 0.0 : (double)fast_exp2(fmaf(z[e], kLog2e, -ms));
                    const int loc = chunk_search256(w, s_target, scan_buf, s_pick);
                    if (tid == 0) p.next_drafts[(size_t)b * p.k + s] = s_chunk * kChunk + loc;
                }
            }
        }
    }
    // ---- the last CTA of sequence b publishes the new state ----
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const int total = p.L * p.Hkv + p.nchunk * p.k;
        if (atomicAdd(&p.seq_count[b], 1) == total - 1 && j >= 0) {
            __threadfence();
            p.next_q_group[b] = j;
            p.next_preaccepted[b] = j < p.k ? 1 : 0;
            p.prefix_len[b] += j;
        }
    }
}

}  // namespace

size_t commit_workspace_bytes(int B, int k, int V) {
    return align256(sizeof(ChunkStat) * (size_t)B * k * vocab_chunks(V)) + align256(sizeof(int32_t) * B * (k + 1));
}

cudaError_t commit_launch(void *const *k_caches, void *const *v_caches, const void *const *k_news,
                          const void *const *v_news, int L, int B, int Hkv, int D, int k, int P_max,
                          int32_t *prefix_len, const int32_t *accept_len, const int32_t *resampled,
                          const void *group_logits, int dtype, int V, const float *u_draft, int32_t *next_drafts,
                          uint8_t *next_preaccepted, int32_t *next_q_group, void *ws, int32_t *dev_status,
                          cudaStream_t s) {
    CommitParams p;
    p.k_caches = k_caches;
    p.v_caches = v_caches;
    p.k_news = k_news;
    p.v_news = v_news;
    p.L = L;
    p.B = B;
    p.Hkv = Hkv;
    p.D = D;
    p.k = k;
    p.R = k * (k + 2);
    p.P_max = P_max;
    p.prefix_len = prefix_len;
    p.accept_len = accept_len;
    p.resampled = resampled;
    p.group_logits = group_logits;
    p.dtype = dtype;
    p.V = V;
    p.nchunk = vocab_chunks(V);
    p.u_draft = u_draft;
    p.next_drafts = next_drafts;
    p.next_preaccepted = next_preaccepted;
    p.next_q_group = next_q_group;
    p.stats = reinterpret_cast<ChunkStat *>(ws);
    uint8_t *cnt = reinterpret_cast<uint8_t *>(ws) + align256(sizeof(ChunkStat) * (size_t)B * k * p.nchunk);
    p.row_count = reinterpret_cast<int32_t *>(cnt);
    p.seq_count = p.row_count + B * k;
    p.dev_status = dev_status;
    p.n_copy_ctas = L * B * Hkv;
    cudaError_t e = cudaMemsetAsync(cnt, 0, sizeof(int32_t) * B * (k + 1), s);
    if (e != cudaSuccess) return e;
    const long ctas = (long)p.n_copy_ctas + (long)p.nchunk * k * B;
    commit_kernel<<<(unsigned)ctas, kStatThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace tidar
