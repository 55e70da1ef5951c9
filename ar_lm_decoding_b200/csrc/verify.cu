// AR rejection-sampling verify of the previous step's drafts: one cooperative
// kernel in three phases separated by grid barriers.
//
//  A. vocabulary statistics: per-chunk max and sum-exp of every target row
//     and every q row -- one coalesced 16-byte sweep of the 2k vocabulary rows
//     (the HBM-bound part).  The target row of slot i is the AR row, or with
//     trust-mix the logits lambda * z_AR + (1 - lambda) * z_diff.
//  B. per (sequence, chunk): merge the 2k rows' statistics (one warp per
//     row), run the k ratio tests a_i = [u_i < p_i(d_i)/q_i(d_i)] in double
//     precision (slot 1 forced when pre-accepted), j* = first rejection (a warp
//     ballot); then the residual weights max(0, p - q) of this chunk of slot
//     j*+1 (the rows are L2-hot) and their sum.
//  C. per sequence: the chunk that holds u_res * Z_r (a warp scan of the chunk
//     sums), a rescan of that chunk with a block prefix scan, and the emitted
//     tokens.
// The grid is small enough to be resident at once (a cooperative launch), so
// the barriers cannot wait for a CTA that never runs; each wait is bounded
// anyway and raises TIDAR_DEV_TIMEOUT when it expires.
#include "vocab.cuh"

namespace tidar {

namespace {

constexpr long long kBarrierCycles = 4000000000LL;  // bound of a grid-barrier wait (~2 s)

struct SlotState {  // what phase C needs of sequence b: j* and the statistics of slot j*+1's rows
    int j;
    float mp, mq;
    float lzp, lzq;  // log2 of the row sums
};

struct VerifyParams {
    const void *p_logits, *q_logits;
    int dtype;
    const int32_t *drafts;
    const uint8_t *preaccepted;
    const float *u_acc, *u_res;
    int B, k, V, nchunk;
    float lambda;  // trust-mix weight of the AR logits (1: the AR logits alone)
    int32_t *accept_len, *resampled, *tokens, *n_emitted;
    float *logp_d, *logq_d;
    ChunkStat *stats;   // [B][2k][nchunk]: target rows then q rows
    double *res_part;   // [B][nchunk] residual weight per chunk
    double *p_part;     // [B][nchunk] target weight per chunk (fallback when p == q)
    SlotState *slot;    // [B]
    unsigned *barrier;  // grid-barrier counter (zeroed before the launch)
    int32_t *dev_status;
};

__device__ __forceinline__ const void *row_ptr(const void *base, int dtype, size_t row, int V) {
    const size_t es = dtype == TIDAR_DT_BF16 ? 2 : 4;
    return reinterpret_cast<const uint8_t *>(base) + row * V * es;
}

// Residual and target weights of one vocabulary entry given the slot constants (target logit zt).
__device__ __forceinline__ void slot_weights(float zt, float zq, float mp, float lzp, float mq, float lzq,
                                             float &res, float &pw) {
    const float pv = fast_exp2(fmaf(zt, kLog2e, -mp * kLog2e) - lzp);
    const float qv = fast_exp2(fmaf(zq, kLog2e, -mq * kLog2e) - lzq);
    pw = zt == -INFINITY ? 0.f : pv;
    res = zt == -INFINITY ? 0.f : fmaxf(pv - qv, 0.f);
}

// This thread's 32 target logits and 32 q logits of chunk c of slot row `row` (strided or contiguous layout).
template <bool CONTIG>
__device__ __forceinline__ void load_slot_chunk(const VerifyParams &p, size_t row, int c, float (&zt)[32],
                                                float (&zq)[32]) {
    const void *pr = row_ptr(p.p_logits, p.dtype, row, p.V), *qr = row_ptr(p.q_logits, p.dtype, row, p.V);
    if (CONTIG)
        load_chunk32_contig(qr, p.dtype, p.V, c, zq);
    else
        load_chunk32(qr, p.dtype, p.V, c, zq);
    if (p.lambda == 0.f) {
#pragma unroll
        for (int e = 0; e < 32; ++e) zt[e] = zq[e];
        return;
    }
    if (CONTIG)
        load_chunk32_contig(pr, p.dtype, p.V, c, zt);
    else
        load_chunk32(pr, p.dtype, p.V, c, zt);
    if (p.lambda != 1.f) {
#pragma unroll
        for (int e = 0; e < 32; ++e) zt[e] = mix_logit(zt[e], zq[e], p.lambda);
    }
}

__global__ void __launch_bounds__(kStatThreads) verify_kernel(const VerifyParams p) {
    __shared__ float redf[8];
    __shared__ double redd[8], scan_buf[8];
    __shared__ float m_row[2 * kMaxDraft];
    __shared__ double lz_row[2 * kMaxDraft];
    __shared__ int s_pick[2], s_chunk, s_use_p;
    __shared__ double s_target;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = p.k, nchunk = p.nchunk;
    const unsigned G = gridDim.x;

    // ---- A: chunk statistics of the 2k rows of every sequence ----
    const int itemsA = p.B * 2 * k * nchunk;
    for (int it = blockIdx.x; it < itemsA; it += G) {
        const int c = it % nchunk, row = (it / nchunk) % (2 * k), b = it / (nchunk * 2 * k);
        const size_t srow = (size_t)b * k + row % k;
        float v[32];
        if (row < k) {  // target row of slot `row`
            float zq[32];
            load_slot_chunk<false>(p, srow, c, v, zq);
        } else {
            load_chunk32(row_ptr(p.q_logits, p.dtype, srow, p.V), p.dtype, p.V, c, v);
        }
        const ChunkStat st = stat_of(v, redf, redd);
        if (tid == 0) p.stats[((size_t)b * 2 * k + row) * nchunk + c] = st;
    }
    if (!grid_barrier(p.barrier, G, p.dev_status, kBarrierCycles)) return;

    // ---- B: ratio tests and j* per sequence, residual weights of slot j*+1 per chunk ----
    const int itemsB = p.B * nchunk;
    for (int it = blockIdx.x; it < itemsB; it += G) {
        const int c = it % nchunk, b = it / nchunk;
        for (int row = warp; row < 2 * k; row += kStatThreads / 32) {
            float m;
            double z;
            merge_stats_warp(p.stats + ((size_t)b * 2 * k + row) * nchunk, nchunk, m, z);
            if (lane == 0) {
                m_row[row] = m;
                lz_row[row] = log2(z);
            }
        }
        __syncthreads();
        if (warp == 0) {
            bool accept = true, bad = false;
            if (lane < k) {
                const int d = p.drafts[b * k + lane];
                bad = d < 0 || d >= p.V;
                if (!bad) {
                    const size_t row = (size_t)b * k + lane;
                    const float zq = load_logit(p.q_logits, p.dtype, row * p.V + d);
                    const float zt = mix_logit(load_logit(p.p_logits, p.dtype, row * p.V + d), zq, p.lambda);
                    const double lp = ((double)zt - m_row[lane]) * 1.4426950408889634 - lz_row[lane];  // log2 p_i(d_i)
                    const double lq = ((double)zq - m_row[k + lane]) * 1.4426950408889634 - lz_row[k + lane];
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
                s_pick[0] = j;
                if (c == 0) {
                    if (j < 0) atomicOr(p.dev_status, TIDAR_DEV_BAD_TOKEN);
                    else p.accept_len[b] = j;
                    SlotState ss;
                    ss.j = j;
                    const int sj = (j >= 0 && j < k) ? j : 0;
                    ss.mp = m_row[sj];
                    ss.mq = m_row[k + sj];
                    ss.lzp = (float)lz_row[sj];
                    ss.lzq = (float)lz_row[k + sj];
                    p.slot[b] = ss;
                }
            }
        }
        __syncthreads();
        const int j = s_pick[0];
        if (j >= 0 && j < k) {  // residual weights of this chunk of slot j+1
            const float mp = m_row[j], mq = m_row[k + j];
            const float lzp = (float)lz_row[j], lzq = (float)lz_row[k + j];
            float zt[32], zq[32];
            load_slot_chunk<false>(p, (size_t)b * k + j, c, zt, zq);
            double rs = 0.0, ps = 0.0;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                float res, pw;
                slot_weights(zt[e], zq[e], mp, lzp, mq, lzq, res, pw);
                rs += res;
                ps += pw;
            }
            rs = block_sum_d<kStatThreads>(rs, redd);
            ps = block_sum_d<kStatThreads>(ps, redd);
            if (tid == 0) {
                p.res_part[(size_t)b * nchunk + c] = rs;
                p.p_part[(size_t)b * nchunk + c] = ps;
            }
        }
        __syncthreads();  // m_row / s_pick are reused by the next item
    }
    if (!grid_barrier(p.barrier, 2 * G, p.dev_status, kBarrierCycles)) return;

    // ---- C: the replacement draw and the emitted tokens, one sequence per CTA ----
    for (int b = blockIdx.x; b < p.B; b += G) {
        SlotState ss;
        {
            const int *src = reinterpret_cast<const int *>(p.slot + b);
            int w[5];
#pragma unroll
            for (int e = 0; e < 5; ++e) w[e] = __ldcg(src + e);
            ss.j = w[0];
            ss.mp = __int_as_float(w[1]);
            ss.mq = __int_as_float(w[2]);
            ss.lzp = __int_as_float(w[3]);
            ss.lzq = __int_as_float(w[4]);
        }
        const int j = ss.j;
        if (j < 0) continue;  // a draft outside the vocabulary: reported in phase B, sequence skipped
        int t = -1;
        if (j < k) {
            if (warp == 0) {  // chunk totals, then the chunk whose cumulative weight first exceeds u * Z
                double zr = 0.0;
                for (int cc = lane; cc < nchunk; cc += 32) zr += __ldcg(p.res_part + (size_t)b * nchunk + cc);
                zr = warp_sum_d(zr);
                const int use_p = !(zr > 0.0);  // p == q: the residual is empty
                const double *w = (use_p ? p.p_part : p.res_part) + (size_t)b * nchunk;
                double tot = 0.0;
                for (int cc = lane; cc < nchunk; cc += 32) tot += __ldcg(w + cc);
                tot = warp_sum_d(tot);
                const double target = (double)p.u_res[b] * tot;
                double run = 0.0, before = 0.0;
                int ch = -1, last_pos = -1;
                for (int c0 = 0; c0 < nchunk && ch < 0; c0 += 32) {
                    const int cc = c0 + lane;
                    const double wc = cc < nchunk ? __ldcg(w + cc) : 0.0;
                    double incl = wc;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const double y = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += y;
                    }
                    const unsigned hit = __ballot_sync(0xffffffffu, cc < nchunk && wc > 0.0 && run + incl > target);
                    const unsigned pos = __ballot_sync(0xffffffffu, cc < nchunk && wc > 0.0);
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
                float zt[32], zq[32];
                load_slot_chunk<true>(p, (size_t)b * k + j, ch, zt, zq);
                double w[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    float res, pw;
                    slot_weights(zt[e], zq[e], ss.mp, ss.lzp, ss.mq, ss.lzq, res, pw);
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
        __syncthreads();
    }
}

// CTAs of verify_kernel that fit on the device at once (0 if the query fails).
int resident_ctas() {
    static int n = -1;
    if (n >= 0) return n;
    int dev = 0, sms = 0, per = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, verify_kernel, kStatThreads, 0) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    n = sms * per;
    return n;
}

}  // namespace

size_t verify_workspace_bytes(int B, int k, int V) {
    const size_t nc = vocab_chunks(V);
    return align256(sizeof(ChunkStat) * B * 2 * k * nc) + align256(sizeof(double) * B * nc) * 2 +
           align256(sizeof(SlotState) * B) + 256;
}

cudaError_t verify_launch(const void *p_logits, const void *q_logits, int dtype, const int32_t *drafts,
                          const uint8_t *preaccepted, const float *u_acc, const float *u_res, int B, int k, int V,
                          float lambda, int32_t *accept_len, int32_t *resampled, int32_t *tokens, int32_t *n_emitted,
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
    p.lambda = lambda;
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
    p.slot = reinterpret_cast<SlotState *>(w);
    w += align256(sizeof(SlotState) * B);
    p.barrier = reinterpret_cast<unsigned *>(w);
    p.dev_status = dev_status;
    const int cap = resident_ctas();
    if (cap <= 0) return cudaErrorLaunchFailure;
    const long itemsA = (long)B * 2 * k * p.nchunk;
    const int grid = (int)std::min<long>(itemsA, std::min(cap, 2 * kNumSMs));
    cudaError_t e = cudaMemsetAsync(p.barrier, 0, sizeof(unsigned), s);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kStatThreads, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident at once: the grid barriers can complete
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, verify_kernel, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace tidar
