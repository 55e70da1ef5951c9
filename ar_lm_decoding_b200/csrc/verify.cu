// AR rejection-sampling verify of the previous step's drafts.
//
//  1. verify_stats   (chunks x 2k rows x B CTAs): per-chunk max and sum-exp of
//                    every p row and q row -- one coalesced 16-byte sweep of
//                    the 2k vocabulary rows (the HBM-bound part).
//  2. verify_decide  (chunks x B CTAs): each CTA merges the row statistics,
//                    runs the ratio test a_i = [u_i < p_i(d_i)/q_i(d_i)] in
//                    double precision (slot 1 forced when pre-accepted) to
//                    find j*, then sums the residual weights
//                    max(0, p - q) of its chunk of slot j*+1 (L2-resident).
//  3. verify_final   (B CTAs): locates the chunk holding u_res * Z_r, rescans
//                    it with a block prefix scan and writes the resampled token,
//                    the emitted tokens and their count.
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
    ChunkStat *stats;    // [B][2k][nchunk]: p rows then q rows
    double *res_part;    // [B][nchunk] residual weight per chunk
    double *p_part;      // [B][nchunk] p weight per chunk (fallback when p == q)
    double *slot_const;  // [B][4]: m_p, log2 Z_p, m_q, log2 Z_q of slot j*+1
    int32_t *jstar;      // [B] (-1 = invalid input)
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
    __shared__ int s_j;
    __shared__ double redd[8];
    const int c = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x;
    const int k = p.k;
    if (tid < 2 * k) {
        float m;
        double z;
        merge_stats(p.stats + ((size_t)b * 2 * k + tid) * p.nchunk, p.nchunk, m, z);
        m_row[tid] = m;
        lz_row[tid] = log2(z);
    }
    __syncthreads();
    if (tid == 0) {
        int j = 0;
        bool stop = false, bad = false;
        for (int i = 0; i < k; ++i) {
            const int d = p.drafts[b * k + i];
            if (d < 0 || d >= p.V) { bad = true; break; }
            const size_t row = (size_t)b * k + i;
            const double zp = load_logit(p.p_logits, p.dtype, row * p.V + d);
            const double zq = load_logit(p.q_logits, p.dtype, row * p.V + d);
            const double lp = (zp - m_row[i]) * 1.4426950408889634 - lz_row[i];      // log2 p_i(d_i)
            const double lq = (zq - m_row[k + i]) * 1.4426950408889634 - lz_row[k + i];  // log2 q_i(d_i)
            if (c == 0) {
                if (p.logp_d) p.logp_d[row] = (float)(lp * 0.6931471805599453);
                if (p.logq_d) p.logq_d[row] = (float)(lq * 0.6931471805599453);
            }
            if (stop) continue;
            if (i == 0 && p.preaccepted[b]) { j = 1; continue; }
            if ((double)p.u_acc[row] < exp2(lp - lq))
                j = i + 1;
            else
                stop = true;
        }
        if (bad) {
            j = -1;
            if (c == 0) atomicOr(p.dev_status, TIDAR_DEV_BAD_TOKEN);
        }
        s_j = j;
        if (c == 0) {
            p.jstar[b] = j;
            if (j >= 0) p.accept_len[b] = j;
            if (j >= 0 && j < k) {
                double *sc = p.slot_const + 4 * b;
                sc[0] = m_row[j];
                sc[1] = lz_row[j];
                sc[2] = m_row[k + j];
                sc[3] = lz_row[k + j];
            }
        }
    }
    __syncthreads();
    const int j = s_j;
    if (j < 0 || j >= k) return;
    const float mp = m_row[j], lzp = (float)lz_row[j], mq = m_row[k + j], lzq = (float)lz_row[k + j];
    const size_t row = (size_t)b * k + j;
    float zp[32], zq[32];
    load_chunk32(row_ptr(p.p_logits, p.dtype, row, p.V), p.dtype, p.V, c, zp);
    load_chunk32(row_ptr(p.q_logits, p.dtype, row, p.V), p.dtype, p.V, c, zq);
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

__global__ void __launch_bounds__(kScanThreads) verify_final_kernel(const VerifyParams p) {
    __shared__ double scan_buf[32];
    __shared__ int pick[2];
    __shared__ int s_chunk;
    __shared__ double s_target;
    __shared__ int s_use_p;
    const int b = blockIdx.x, tid = threadIdx.x, k = p.k;
    const int j = p.jstar[b];
    if (j < 0) return;
    const int pre = p.preaccepted[b] ? 1 : 0;
    int t = -1;
    if (j < k) {
        if (tid == 0) {
            const double *res = p.res_part + (size_t)b * p.nchunk;
            const double *pp = p.p_part + (size_t)b * p.nchunk;
            double zr = 0.0;
            for (int c = 0; c < p.nchunk; ++c) zr += res[c];
            const int use_p = !(zr > 0.0);  // p == q: the residual is empty
            const double *w = use_p ? pp : res;
            double tot = 0.0;
            for (int c = 0; c < p.nchunk; ++c) tot += w[c];
            const double target = (double)p.u_res[b] * tot;
            double cum = 0.0;
            int ch = -1;
            bool found = false;
            for (int c = 0; c < p.nchunk; ++c) {
                if (w[c] > 0.0) ch = c;
                if (cum + w[c] > target && w[c] > 0.0) { found = true; break; }
                cum += w[c];
            }
            s_chunk = ch;
            // not found only through rounding: the last positive entry is then taken
            s_target = found ? target - cum : INFINITY;
            s_use_p = use_p;
        }
        __syncthreads();
        const int ch = s_chunk < 0 ? 0 : s_chunk;  // < 0 only if every p logit is -inf
        const double *sc = p.slot_const + 4 * b;
        const float mp = (float)sc[0], lzp = (float)sc[1], mq = (float)sc[2], lzq = (float)sc[3];
        const size_t row = (size_t)b * k + j;
        float zp[8], zq[8];
        load_chunk8(row_ptr(p.p_logits, p.dtype, row, p.V), p.dtype, p.V, ch, zp);
        load_chunk8(row_ptr(p.q_logits, p.dtype, row, p.V), p.dtype, p.V, ch, zq);
        double w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float res, pw;
            slot_weights(zp[e], zq[e], mp, lzp, mq, lzq, res, pw);
            w[e] = s_use_p ? (double)pw : (double)res;
        }
        const int loc = chunk_search(w, s_target, scan_buf, pick);
        t = s_chunk < 0 || loc < 0 ? -1 : ch * kChunk + loc;
    }
    if (tid == 0) {
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
           align256(sizeof(double) * 4 * B) + align256(sizeof(int32_t) * B);
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
    p.slot_const = reinterpret_cast<double *>(w);
    w += align256(sizeof(double) * 4 * B);
    p.jstar = reinterpret_cast<int32_t *>(w);
    p.dev_status = dev_status;
    verify_stats_kernel<<<dim3(p.nchunk, 2 * k, B), kStatThreads, 0, s>>>(p);
    verify_decide_kernel<<<dim3(p.nchunk, B), kStatThreads, 0, s>>>(p);
    verify_final_kernel<<<B, kScanThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace tidar
