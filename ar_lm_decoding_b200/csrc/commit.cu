// Exact-KV-cache commit / evict and next-draft selection: one cooperative
// kernel in two phases separated by a grid barrier.
//
//  A. work items of two kinds, spread over the grid:
//     - copies (one per layer x sequence x KV head): the first j* new-key rows
//       (accepted drafts) of K/V into cache rows P..P+j*-1, 16 bytes per
//       thread.  Rejected drafts and mask tokens are never written: eviction is
//       simply not committing them.
//     - statistics (chunks x k slots x B): per-chunk max / sum-exp of slot s of
//       pre-draft group j*.
//  B. per (sequence, slot): merge the row's statistics, find the chunk that
//     holds u_draft * Z (a warp scan) and rescan it with a block prefix scan:
//     slot s of the next draft block.  After a rejection slot 0 is the
//     resampled token instead.  The (sequence, slot 0) item also writes
//     next_q_group and next_preaccepted and advances prefix_len by j* -- after
//     the barrier, so every copy has read the old prefix length.
// The grid is resident at once (a cooperative launch); the barrier's wait is
// bounded and raises TIDAR_DEV_TIMEOUT when it expires.
#include "vocab.cuh"

namespace tidar {

namespace {

constexpr long long kBarrierCycles = 4000000000LL;  // bound of the grid-barrier wait (~2 s)

struct CommitParams {
    void *const *k_caches;
    void *const *v_caches;
    const void *const *k_news;
    const void *const *v_news;
    int L, B, Hkv, D, k, R, P_max;
    // paged caches (null: contiguous [B, Hkv, P_max, D]): cache row n of sequence b is row n % 64 of page
    // block_table[b * max_pages + n / 64] of the pool [num_pages, Hkv, 64, D]
    const int32_t *block_table;
    int max_pages, num_pages;
    int32_t *prefix_len;
    const int32_t *accept_len, *resampled;
    const void *group_logits;
    int dtype, V, nchunk;
    const float *u_draft;
    int32_t *next_drafts;
    uint8_t *next_preaccepted;
    int32_t *next_q_group;
    ChunkStat *stats;   // [B][k][nchunk]
    int32_t *seq_j;     // [B] j* as phase A validated it (-1: sequence skipped)
    unsigned *barrier;  // grid-barrier counter (zeroed before the launch)
    int32_t *dev_status;
};

// Validates the commit inputs of sequence b; returns j* or -1.
__device__ __forceinline__ int checked_accept(const CommitParams &p, int b, bool report) {
    const int j = p.accept_len[b];
    const int P = p.prefix_len[b];
    int bits = 0;
    if (j < 0 || j > p.k) bits |= TIDAR_DEV_BAD_ACCEPT;
    if (P < 0 || (bits == 0 && P + j > p.P_max)) bits |= TIDAR_DEV_BAD_PREFIX;
    if (bits == 0 && j < p.k && (p.resampled[b] < 0 || p.resampled[b] >= p.V)) bits |= TIDAR_DEV_BAD_TOKEN;
    if (bits == 0 && p.block_table && j > 0) {  // the pages that receive rows P .. P+j-1
        for (int pi = P / kPageRows; pi <= (P + j - 1) / kPageRows; ++pi) {
            const int pg = p.block_table[(size_t)b * p.max_pages + pi];
            if (pg < 0 || pg >= p.num_pages) bits |= TIDAR_DEV_BAD_PAGE;
        }
    }
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
    __shared__ int s_pick[2], s_chunk;
    __shared__ double s_target;
    __shared__ float s_m;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned G = gridDim.x;
    const int n_copy = p.L * p.B * p.Hkv;

    // ---- A: accepted K/V rows into the caches; statistics of group j*'s slot rows ----
    const long itemsA = (long)n_copy + (long)p.B * p.k * p.nchunk;
    for (long it = blockIdx.x; it < itemsA; it += G) {
        if (it < n_copy) {
            const int kvh = (int)(it % p.Hkv);
            const int b = (int)((it / p.Hkv) % p.B);
            const int l = (int)(it / (p.Hkv * p.B));
            const int j = checked_accept(p, b, l == 0 && kvh == 0 && tid == 0);
            if (l == 0 && kvh == 0 && tid == 0) p.seq_j[b] = j;
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
                    size_t drow;
                    if (p.block_table) {
                        const int n = P + i;
                        const int pg = p.block_table[(size_t)b * p.max_pages + n / kPageRows];
                        drow = ((size_t)pg * p.Hkv + kvh) * kPageRows + n % kPageRows;
                    } else {
                        drow = (size_t)(b * p.Hkv + kvh) * p.P_max + P + i;
                    }
                    const size_t dst = drow * p.D + c * 8;
                    *reinterpret_cast<uint4 *>(kc + dst) = *reinterpret_cast<const uint4 *>(kn + src);
                    *reinterpret_cast<uint4 *>(vc + dst) = *reinterpret_cast<const uint4 *>(vn + src);
                }
            }
        } else {
            const long t = it - n_copy;
            const int c = (int)(t % p.nchunk);
            const int s = (int)((t / p.nchunk) % p.k);
            const int b = (int)(t / ((long)p.nchunk * p.k));
            const int j = checked_accept(p, b, false);
            if (j >= 0 && !(s == 0 && j < p.k)) {  // slot 0 after a rejection is the resampled token
                const ChunkStat st = chunk_stat(group_row(p, b, j, s), p.dtype, p.V, c, redf, redd);
                if (tid == 0) p.stats[((size_t)b * p.k + s) * p.nchunk + c] = st;
            }
        }
        __syncthreads();  // redf / redd are reused by the next item
    }
    if (!grid_barrier(p.barrier, G, p.dev_status, kBarrierCycles)) return;

    // ---- B: draw slot s of the next draft block of sequence b; (b, 0) also publishes the new state ----
    for (int it = blockIdx.x; it < p.B * p.k; it += G) {
        const int s = it % p.k, b = it / p.k;
        const int j = __ldcg(p.seq_j + b);  // phase A's verdict: prefix_len may already have been advanced
        if (j < 0) continue;
        if (s == 0 && j < p.k) {
            if (tid == 0) p.next_drafts[(size_t)b * p.k] = p.resampled[b];
        } else {
            if (warp == 0) {
                const ChunkStat *rs = p.stats + ((size_t)b * p.k + s) * p.nchunk;
                float m;
                double tot;
                merge_stats_warp(rs, p.nchunk, m, tot);
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
                load_chunk32_contig(group_row(p, b, j, s), p.dtype, p.V, s_chunk, z);
                const float ms = s_m * kLog2e;
                double w[32];
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    w[e] = z[e] == -INFINITY ? 0.0 : (double)fast_exp2(fmaf(z[e], kLog2e, -ms));
                const int loc = chunk_search256(w, s_target, scan_buf, s_pick);
                if (tid == 0) p.next_drafts[(size_t)b * p.k + s] = s_chunk * kChunk + loc;
            }
        }
        if (s == 0 && tid == 0) {
            p.next_q_group[b] = j;
            p.next_preaccepted[b] = j < p.k ? 1 : 0;
            p.prefix_len[b] += j;
        }
        __syncthreads();
    }
}

// CTAs of commit_kernel that fit on the device at once (0 if the query fails).
int resident_ctas() {
    static int n = -1;
    if (n >= 0) return n;
    int dev = 0, sms = 0, per = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, commit_kernel, kStatThreads, 0) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    n = sms * per;
    return n;
}

}  // namespace

size_t commit_workspace_bytes(int B, int k, int V) {
    return align256(sizeof(ChunkStat) * (size_t)B * k * vocab_chunks(V)) + align256(sizeof(int32_t) * B) + 256;
}

cudaError_t commit_launch(void *const *k_caches, void *const *v_caches, const void *const *k_news,
                          const void *const *v_news, int L, int B, int Hkv, int D, int k, int P_max,
                          int32_t *prefix_len, const int32_t *accept_len, const int32_t *resampled,
                          const void *group_logits, int dtype, int V, const float *u_draft, int32_t *next_drafts,
                          uint8_t *next_preaccepted, int32_t *next_q_group, void *ws, int32_t *dev_status,
                          cudaStream_t s, const int32_t *block_table, int max_pages, int num_pages) {
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
    p.block_table = block_table;
    p.max_pages = max_pages;
    p.num_pages = num_pages;
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
    uint8_t *w = reinterpret_cast<uint8_t *>(ws);
    p.stats = reinterpret_cast<ChunkStat *>(w);
    w += align256(sizeof(ChunkStat) * (size_t)B * k * p.nchunk);
    p.seq_j = reinterpret_cast<int32_t *>(w);
    w += align256(sizeof(int32_t) * B);
    p.barrier = reinterpret_cast<unsigned *>(w);
    p.dev_status = dev_status;
    const int cap = resident_ctas();
    if (cap <= 0) return cudaErrorLaunchFailure;
    const long itemsA = (long)L * B * Hkv + (long)p.nchunk * k * B;
    const int grid = (int)std::min<long>(itemsA, std::min(cap, 2 * kNumSMs));
    cudaError_t e = cudaMemsetAsync(p.barrier, 0, sizeof(unsigned), s);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kStatThreads, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident at once: the grid barrier can complete
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, commit_kernel, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace tidar
