// Exact-KV-cache commit / evict and next-draft selection.
//
//  1. commit_copy_stats: one grid with two roles.
//     - copy CTAs (one per layer x sequence x KV head): the first j* new-key
//       rows (accepted drafts) of K/V are copied into cache rows P..P+j*-1,
//       16 bytes per thread.  Rejected drafts and mask tokens are never
//       written: eviction is simply not committing them.
//     - stats CTAs (chunks x k slots x B): per-chunk max / sum-exp of the k
//       logit rows of pre-draft group j*.
//  2. commit_select (k x B CTAs): draws slot s of the next draft block from
//     softmax(group_logits[b, j*, s]) by inverse CDF (chunk search + block
//     scan), replaces slot 0 by the resampled token after a rejection, and
//     advances prefix_len by j*.
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
    ChunkStat *stats;  // [B][k][nchunk]
    int32_t *jv;       // [B] validated j* (-1 = invalid), for the select kernel
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

__global__ void __launch_bounds__(kStatThreads) commit_copy_stats_kernel(const CommitParams p) {
    __shared__ float redf[8];
    __shared__ double redd[8];
    const int cta = blockIdx.x;
    if (cta < p.n_copy_ctas) {
        const int kvh = cta % p.Hkv;
        const int b = (cta / p.Hkv) % p.B;
        const int l = cta / (p.Hkv * p.B);
        const bool first = l == 0 && kvh == 0;
        const int j = checked_accept(p, b, first);
        if (first && threadIdx.x == 0) p.jv[b] = j;
        if (j <= 0) return;
        const int P = p.prefix_len[b];
        const int vec = p.D / 8;  // 16-byte vectors per row
        const bf16 *kn = reinterpret_cast<const bf16 *>(p.k_news[l]);
        const bf16 *vn = reinterpret_cast<const bf16 *>(p.v_news[l]);
        bf16 *kc = reinterpret_cast<bf16 *>(p.k_caches[l]);
        bf16 *vc = reinterpret_cast<bf16 *>(p.v_caches[l]);
        for (int idx = threadIdx.x; idx < j * vec; idx += blockDim.x) {
            const int i = idx / vec, c = idx % vec;
            const size_t src = ((size_t)(b * p.R + i) * p.Hkv + kvh) * p.D + c * 8;
            const size_t dst = ((size_t)(b * p.Hkv + kvh) * p.P_max + P + i) * p.D + c * 8;
            *reinterpret_cast<uint4 *>(kc + dst) = *reinterpret_cast<const uint4 *>(kn + src);
            *reinterpret_cast<uint4 *>(vc + dst) = *reinterpret_cast<const uint4 *>(vn + src);
        }
        return;
    }
    const int t = cta - p.n_copy_ctas;
    const int c = t % p.nchunk;
    const int s = (t / p.nchunk) % p.k;
    const int b = t / (p.nchunk * p.k);
    const int j = checked_accept(p, b, false);
    if (j < 0 || (s == 0 && j < p.k)) return;  // slot 0 is the resampled token then
    const ChunkStat st = chunk_stat(group_row(p, b, j, s), p.dtype, p.V, c, redf, redd);
    if (threadIdx.x == 0) p.stats[((size_t)b * p.k + s) * p.nchunk + c] = st;
}

__global__ void __launch_bounds__(kScanThreads) commit_select_kernel(const CommitParams p) {
    __shared__ double scan_buf[32];
    __shared__ int pick[2];
    __shared__ int s_chunk;
    __shared__ double s_target;
    __shared__ float s_m;
    const int s = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const int j = p.jv[b];  // prefix_len is advanced below, so it is not re-validated here
    if (j < 0) return;
    if (s == 0 && tid == 0) {
        p.next_q_group[b] = j;
        p.next_preaccepted[b] = j < p.k ? 1 : 0;
        p.prefix_len[b] += j;
    }
    if (s == 0 && j < p.k) {
        if (tid == 0) p.next_drafts[(size_t)b * p.k] = p.resampled[b];
    } else {
        const ChunkStat *st = p.stats + ((size_t)b * p.k + s) * p.nchunk;
        if (tid == 0) {
            float m;
            double z;
            merge_stats(st, p.nchunk, m, z);
            const double target = (double)p.u_draft[(size_t)b * p.k + s] * z;
            double cum = 0.0;
            int ch = -1;
            bool found = false;
            for (int c = 0; c < p.nchunk; ++c) {
                if (st[c].m == -INFINITY) continue;
                const double wc = st[c].z * exp2((double)(st[c].m - m) * 1.4426950408889634);
                ch = c;
                if (cum + wc > target) { found = true; break; }
                cum += wc;
            }
            s_chunk = ch;
            s_target = found ? target - cum : INFINITY;
            s_m = m;
        }
        __syncthreads();
        if (s_chunk < 0) {  // every logit of the row is -inf: no distribution to draw from
            if (tid == 0) p.next_drafts[(size_t)b * p.k + s] = -1;
            return;
        }
        float z[8];
        load_chunk8(group_row(p, b, j, s), p.dtype, p.V, s_chunk, z);
        const float ms = s_m * kLog2e;
        double w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = z[e] == -INFINITY ? 0.0 : (double)fast_exp2(fmaf(z[e], kLog2e, -ms));
        const int loc = chunk_search(w, s_target, scan_buf, pick);
        if (tid == 0) p.next_drafts[(size_t)b * p.k + s] = s_chunk * kChunk + loc;
    }
}

}  // namespace

size_t commit_workspace_bytes(int B, int k, int V) {
    return align256(sizeof(ChunkStat) * (size_t)B * k * vocab_chunks(V)) + align256(sizeof(int32_t) * B);
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
    p.jv = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(ws) +
                                       align256(sizeof(ChunkStat) * (size_t)B * k * p.nchunk));
    p.dev_status = dev_status;
    p.n_copy_ctas = L * B * Hkv;
    const long ctas = (long)p.n_copy_ctas + (long)p.nchunk * k * B;
    commit_copy_stats_kernel<<<(unsigned)ctas, kStatThreads, 0, s>>>(p);
    commit_select_kernel<<<dim3(k, B), kScanThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace tidar
