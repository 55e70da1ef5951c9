// AR rejection-sampling verify of the previous step's drafts (two kernels).
//
//  1. verify_stats   (chunks x 2k rows x B CTAs): per-chunk max and sum-exp of
//                    every p row and q row -- one coalesced 16-byte sweep of
//                    the 2k vocabulary rows (the HBM-bound part).  CTA (0,0,b)
//                    also zeroes sequence b's completion counter.
//  2. verify_decide  (chunks x B CTAs): every CTA merges the row statistics
//                    (one warp per row), runs the k ratio tests
//                    a_i = [u_i < p_i(d_i)/q_i(d_i)] in parallel (double
//                    precision; slot 1 forced when pre-accepted) and takes j*
//                    as the first rejection (a warp ballot), then sums the
//                    residual weights max(0, p - q) of its chunk of slot j*+1
//                    (L2-hot).  The last CTA of the sequence to finish (an
//                    atomic counter; nobody waits) finds the chunk that holds
//                    u_res * Z_r, rescans it with a block prefix scan and
//                    writes the resampled token, the emitted tokens and n.
#include "vocab.cuh"

namespace tidar {

namespace {

struct VerifyParams {
    const void *p_logits, *q_logits;
    int dtype;
    const int32_t *drafts;
    const uint8_t *preaccepted;
    const float *u_acc, *u_res;
    int B, k, V, nchunk;
    int32_t *accept_len, *resampled, *tokens, *n_emitted;
    float *logp_d, *logq_d;
    ChunkStat *stats;  // [B][2k][nchunk]: p rows then q rows
    double *res_part;  // [B][nchunk] residual weight per chunk
    double *p_part;    // [B][nchunk] p weight per chunk (fallback when p == q)
    int32_t *counter;  // [B] CTAs of verify_decide done (zeroed by verify_stats)
    int32_t *dev_status;
};

__device__ __forceinline__ const void *row_ptr(const void *base, int dtype, size_t row, int V) {
    const size_t es = dtype == TIDAR_DT_BF16 ? 2 : 4;
    return reinterpret_cast<const uint8_t *>(base) + row * V * es;
}

__global__ void __launch_bounds__(kStatThreads) verify_stats_kernel(const VerifyParams p) {
    __shared__ float redf[8];
    __shared__ double redd[8];
    const int c = blockIdx.x, row = blockIdx.y, b = blockIdx.z;
    if (c == 0 && row == 0 && threadIdx.x == 0) p.counter[b] = 0;
    const int slot = row % p.k;
    const void *base = row < p.k ? p.p_logits : p.q_logits;
    const void *r = row_ptr(base, p.dtype, (size_t)b * p.k + slot, p.V);
    const ChunkStat st = chunk_stat(r, p.dtype, p.V, c, redf, redd);
    if (threadIdx.x == 0) p.stats[((size_t)b * 2 * p.k + row) * p.nchunk + c] = st;
}

// Residual and p weights of one vocabulary entry given the slot constants.
__device__ __forceinline__ void slot_weights(float zp, float zq, float mp, float lzp, float mq, float lzq,
                                             float &res, float &pw) {
    const float pv = fast_exp2(fmaf(zp, kLog2e, -mp * kLog2e) - lzp);
    const float qv = fast_exp2(fmaf(zq, kLog2e, -mq * kLog2e) - lzq);
    pw = zp == -INFINITY ? 0.f : pv;
    res = zp == -INFINITY ? 0.f : fmaxf(pv - qv, 0.f);
}

__global__ void __launch_bounds__(kStatThreads) verify_decide_kernel(const VerifyParams p) {
    __shared__ float m_row[32];
    __shared__ double lz_row[32];
    __shared__ int s_j, s_last, s_pick[2];
    __shared__ double redd[8], scan_buf[8];
    __shared__ double s_target;
    __shared__ int s_chunk, s_use_p;
    const int c = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = p.k;
    // row statistics: one warp per row
    for (int row = warp; row < 2 * k; row += kStatThreads / 32) {
        float m;
        double z;
        merge_stats_warp(p.stats + ((size_t)b * 2 * k + row) * p.nchunk, p.nchunk, m, z);
        if (lane == 0) {
            m_row[row] = m;
            lz_row[row] = log2(z);
        }
    }
    __syncthreads();
    // the k ratio tests in parallel, then j* = first rejection
    if (warp == 0) {
        bool accept = true, bad = false;
        if (lane < k) {
            const int d = p.drafts[b * k + lane];
            bad = d < 0 || d >= p.V;
            if (!bad) {
                const size_t row = (size_t)b * k + lane;
                const double zp = load_logit(p.p_logits, p.dtype, row * p.V + d);
                const double zq = load_logit(p.q_logits, p.dtype, row * p.V + d);
                const double lp = (zp - m_row[lane]) * 1.4426950408889634 - lz_row[lane];          // log2 p_i(d_i)
                const double lq = (zq - m_row[k + lane]) * 1.4426950408889634 - lz_row[k + lane];  // log2 q_i(d_i)
                if (c == 0) {
                    if (p.logp_d) p.logp_d[row] = (float)(lp * 0.6931471805599453);
                    if (p.logq_d) p.logq_d[row] = (float)(lq * 0.6931471805599453);
                }
                accept = (lane == 0 && p.preaccepted[b]) || (double)p.u_acc[row] < exp2(lp - lq);
            }
        }
        const unsigned badm = __ballot_sync(0xffffffffu, bad);
        const unsigned rejm = __ballot_sync(0xffffffffu, !accept);
        if (lane == 0) {
            const int j = badm ? -1 : (rejm ? __ffs(rejm) - 1 : k);
            s_j = j;
            if (c == 0) {
                if (j < 0)
                    atomicOr(p.dev_status, TIDAR_DEV_BAD_TOKEN);
                else
                    p.accept_len[b] = j;
            }
        }
    }
    __syncthreads();
    const int j = s_j;
    const bool resample = j >= 0 && j < k;
    const size_t srow = (size_t)b * k + (resample ? j : 0);
    const float mp = resample ? m_row[j] : 0.f, mq = resample ? m_row[k + j] : 0.f;
    const float lzp = resample ? (float)lz_row[j] : 0.f, lzq = resample ? (float)lz_row[k + j] : 0.f;
    if (resample) {  // residual weights of this chunk of slot j+1
        float zp[32], zq[32];
        load_chunk32(row_ptr(p.p_logits, p.dtype, srow, p.V), p.dtype, p.V, c, zp);
        load_chunk32(row_ptr(p.q_logits, p.dtype, srow, p.V), p.dtype, p.V, c, zq);
        double rs = 0.0, ps = 0.0;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            float res, pw;
            slot_weights(zp[e], zq[e], mp, lzp, mq, lzq, res, pw);
            rs += res;
            ps += pw;
        }
        rs = block_sum_d<kStatThreads>(rs, redd);
        ps = block_sum_d<kStatThreads>(ps, redd);
        if (tid == 0) {
            p.res_part[(size_t)b * p.nchunk + c] = rs;
            p.p_part[(size_t)b * p.nchunk + c] = ps;
        }
    }
    // ---- the last CTA of this sequence draws the replacement and writes the emitted tokens ----
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&p.counter[b], 1) == p.nchunk - 1;
    __syncthreads();
    if (!s_last || j < 0) return;
    __threadfence();
    int t = -1;
    if (resample) {
        if (warp == 0) {  // chunk totals, then the chunk whose cumulative weight first exceeds u * Z
            double zr = 0.0;
            for (int cc = lane; cc < p.nchunk; cc += 32) zr += __ldcg(p.res_part + (size_t)b * p.nchunk + cc);
            zr = warp_sum_d(zr);
            const int use_p = !(zr > 0.0);  // p == q: the residual is empty
            const double *w = (use_p ? p.p_part : p.res_part) + (size_t)b * p.nchunk;
            double tot = 0.0;
            for (int cc = lane; cc < p.nchunk; cc += 32) tot += __ldcg(w + cc);
            tot = warp_sum_d(tot);
            const double target = (double)p.u_res[b] * tot;
            double run = 0.0, before = 0.0;
            int ch = -1, last_pos = -1;
            for (int c0 = 0; c0 < p.nchunk && ch < 0; c0 += 32) {
                const int cc = c0 + lane;
                const double wc = cc < p.nchunk ? __ldcg(w + cc) : 0.0;
                double incl = wc;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const double y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                const unsigned hit = __ballot_sync(0xffffffffu, cc < p.nchunk && wc > 0.0 && run + incl > target);
                const unsigned pos = __ballot_sync(0xffffffffu, cc < p.nchunk && wc > 0.0);
                if (pos) last_pos = c0 + 31 - __clz(pos);
                if (hit) {
                    const int l = __ffs(hit) - 1;
                    ch = c0 + l;
                    before = run + __shfl_sync(0xffffffffu, incl - wc, l);
                }
                run += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) {
                s_chunk = ch >= 0 ? ch : last_pos;
                // not found only through rounding: the last positive entry is then taken
                s_target = ch >= 0 ? target - before : INFINITY;
                s_use_p = use_p;
            }
        }
        __syncthreads();
        const int ch = s_chunk;
        if (ch >= 0) {
            float zp[32], zq[32];
            load_chunk32_contig(row_ptr(p.p_logits, p.dtype, srow, p.V), p.dtype, p.V, ch, zp);
            load_chunk32_contig(row_ptr(p.q_logits, p.dtype, srow, p.V), p.dtype, p.V, ch, zq);
            double w[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                float res, pw;
                slot_weights(zp[e], zq[e], mp, lzp, mq, lzq, res, pw);
                w[e] = s_use_p ? (double)pw : (double)res;
            }
            const int loc = chunk_search256(w, s_target, scan_buf, s_pick);
            t = loc < 0 ? -1 : ch * kChunk + loc;
        }
    }
    if (tid == 0) {
        const int pre = p.preaccepted[b] ? 1 : 0;
        int n = 0;
        int32_t *tok = p.tokens + (size_t)b * k;
        for (int i = pre; i < j; ++i) tok[n++] = p.drafts[b * k + i];
        if (j < k) tok[n++] = t;
        p.n_emitted[b] = n;
        for (int i = n; i < k; ++i) tok[i] = -1;
        p.resampled[b] = j < k ? t : -1;
    }
}

}  // namespace

size_t verify_workspace_bytes(int B, int k, int V) {
    const size_t nc = vocab_chunks(V);
    return align256(sizeof(ChunkStat) * B * 2 * k * nc) + align256(sizeof(double) * B * nc) * 2 +
           align256(sizeof(int32_t) * B);
}

cudaError_t verify_launch(const void *p_logits, const void *q_logits, int dtype, const int32_t *drafts,
                          const uint8_t *preaccepted, const float *u_acc, const float *u_res, int B, int k, int V,
                          int32_t *accept_len, int32_t *resampled, int32_t *tokens, int32_t *n_emitted,
                          float *logp_d, float *logq_d, void *ws, int32_t *dev_status, cudaStream_t s) {
    VerifyParams p;
    p.p_logits = p_logits;
    p.q_logits = q_logits;
    p.dtype = dtype;
    p.drafts = drafts;
    p.preaccepted = preaccepted;
    p.u_acc = u_acc;
    p.u_res = u_res;
    p.B = B;
    p.k = k;
    p.V = V;
    p.nchunk = vocab_chunks(V);
    p.accept_len = accept_len;
    p.resampled = resampled;
    p.tokens = tokens;
    p.n_emitted = n_emitted;
    p.logp_d = logp_d;
    p.logq_d = logq_d;
    uint8_t *w = reinterpret_cast<uint8_t *>(ws);
    const size_t nc = p.nchunk;
    p.stats = reinterpret_cast<ChunkStat *>(w);
    w += align256(sizeof(ChunkStat) * B * 2 * k * nc);
    p.res_part = reinterpret_cast<double *>(w);
    w += align256(sizeof(double) * B * nc);
    p.p_part = reinterpret_cast<double *>(w);
    w += align256(sizeof(double) * B * nc);
    p.counter = reinterpret_cast<int32_t *>(w);
    p.dev_status = dev_status;
    verify_stats_kernel<<<dim3(p.nchunk, 2 * k, B), kStatThreads, 0, s>>>(p);
    verify_decide_kernel<<<dim3(p.nchunk, B), kStatThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace tidar
