// The end of a TiDAR decode step: the AR rejection-sampling verify of the
// previous step's drafts, the exact-KV-cache commit of the accepted rows and
// the next-draft selection.  One cooperative kernel in three modes: the
// verify alone, the commit alone, or both fused into one launch.
//
// The vocabulary is cut into chunks of 8192 entries (a CTA of 256 threads, 32
// entries per thread).  Every step is latency-bound (a few MB per call), so
// the kernel is laid out to keep the chain of dependent memory round trips
// short: loads that do not depend on each other are issued together, and a
// result that one CTA needs next is handed over by an arrival counter (the
// CTA that completes a set of chunks carries on with their merge) instead of
// a grid barrier wherever the dependency allows.
//
//  A  (verify) per-chunk max and sum-exp of the 2k target rows and q rows of
//     every sequence -- the HBM-bound sweep; a CTA takes its items two at a
//     time (bf16) with both sets of loads in flight, and the thread holding
//     entry d_i of a row keeps that logit.  The CTA that completes the last
//     chunk of a sequence merges the sequence's row statistics, runs the k
//     ratio tests a_i = [u_i < p_i(d_i)/q_i(d_i)] in double precision (slot 1
//     forced when pre-accepted), takes j* = first rejection and publishes it
//     with the statistics of slot j*+1's rows (and, fused, the prefix length
//     and the commit's validity).
//  -- grid barrier (bounded) --
//  B  block items, each ending with an arrival on a per-sequence or
//     per-slot counter; the CTA that completes the last chunk draws at once:
//     - residual chunk (verify): sums of max(0, p - q) and of p over chunk c
//       of slot j*+1; the last one draws the replacement token (the chunk
//       holding u_res * Z, then a rescan of that chunk) and writes the
//       emitted tokens;
//     - group chunk (commit): statistics of chunk c of slot s of pre-draft
//       group j*; the last one draws slot s of the next draft block.
//     warp items (commit): the j* accepted K/V rows of one (layer, sequence,
//     KV head) copied into the cache, 16 bytes per lane.
//     The (sequence, slot 0) draw also publishes the sequence's new state:
//     next_q_group, next_preaccepted and prefix_len = P + j* (P as phase A
//     read it, so no copy can see the new value).
// The commit alone (accept lengths and replacement tokens given) has no phase
// A; its copies read prefix_len themselves, so its draws and state update
// follow a grid barrier instead:  B' copies + group chunks -- barrier -- C'
// draws.
// Every CTA is resident (cooperative launch), so no barrier waits for a CTA
// that never runs; each wait is bounded anyway and raises TIDAR_DEV_TIMEOUT.
#include "vocab.cuh"

namespace tidar {

namespace {

constexpr long long kBarrierCycles = 4000000000LL;  // bound of a grid-barrier wait (~2 s)
constexpr int kModeVerify = 1, kModeCommit = 2, kModeFused = 3;
constexpr int kWarps = kStatThreads / 32;
constexpr double kLog2eD = 1.4426950408889634;
constexpr double kLn2D = 0.6931471805599453;

struct SeqState {  // one sequence's verdict, published by phase A (or, commit alone, by its copies)
    int j;    // j*: leading accepted drafts; -1: the sequence is skipped
    int jc;   // fused: j* when the commit may proceed, else -1
    int P;    // fused: prefix length before the commit
    int pad;
    float mp, mq;    // max of slot j*+1's target and q rows
    float lzp, lzq;  // log2 of their sums of exp(x - max)
};

struct TailParams {
    // verify
    const void *p_logits, *q_logits;
    const int32_t *drafts;
    const uint8_t *preaccepted;
    const float *u_acc, *u_res;
    float lambda;  // trust-mix weight of the AR logits (1: the AR logits alone)
    int32_t *accept_len, *resampled, *tokens, *n_emitted;
    float *logp_d, *logq_d;
    // commit
    void *const *k_caches;
    void *const *v_caches;
    const void *const *k_news;
    const void *const *v_news;
    int L, Hkv, D, R, P_max;
    // paged caches (null: contiguous [B, Hkv, P_max, D]): cache row n of sequence b is row n % 64 of page
    // block_table[b * max_pages + n / 64] of the pool [num_pages, Hkv, 64, D]
    const int32_t *block_table;
    int max_pages, num_pages;
    int32_t *prefix_len;
    const int32_t *accept_in, *resampled_in;  // commit alone: the verify's outputs
    const void *group_logits;
    const float *u_draft;
    int32_t *next_drafts;
    uint8_t *next_preaccepted;
    int32_t *next_q_group;
    // both
    int dtype, B, k, V, nchunk;
    ChunkStat *vstats;          // [B][2k][nchunk]: target rows, then q rows
    float *dlogit;              // [B][2k]: target and q logit of each row's draft
    ChunkStat *gstats;          // [B][k][nchunk]: slot rows of group j*
    double *res_part, *p_part;  // [B][nchunk]: residual and target weight per chunk of slot j*+1
    SeqState *seq;              // [B]
    unsigned *barrier;          // grid-barrier counter
    unsigned *cnt_rows;         // [B]   phase-A chunks done per sequence
    unsigned *cnt_res;          // [B]   residual chunks done per sequence
    unsigned *cnt_grp;          // [B*k] group chunks done per (sequence, slot)
    int32_t *dev_status;
};

struct TailSmem {
    float redf[2 * kWarps];
    double redd[2 * kWarps];
    double scan_buf[kWarps];
    float m_row[2 * kMaxDraft];
    double lz_row[2 * kMaxDraft];
    int pick[2];
    int chunk, use_p, last[2];
    double target;
    float m;
    int drafts[kMaxDraft];
    int pre;
};

// ---------------------------------------------------------------------------------------------------------
// A thread's 32 entries of one chunk as loaded (strided layout: entry e of thread t is at chunk offset
// (e/8)*2048 + t*8 + e%8, so that a warp reads 512 contiguous bytes per bf16 load).  Entries beyond V hold
// -inf.

template <int DT>
struct Raw;

template <>
struct Raw<TIDAR_DT_BF16> {
    uint4 u[4];
    __device__ __forceinline__ float get(int e) const {
        const uint4 &x = u[e >> 3];
        const int h = (e & 7) >> 1;
        const uint32_t w = h == 0 ? x.x : h == 1 ? x.y : h == 2 ? x.z : x.w;
        return (e & 1) ? __uint_as_float(w & 0xffff0000u) : __uint_as_float(w << 16);
    }
};

template <>
struct Raw<TIDAR_DT_F32> {
    float4 f[8];
    __device__ __forceinline__ float get(int e) const {
        const float4 &x = f[e >> 2];
        const int h = e & 3;
        return h == 0 ? x.x : h == 1 ? x.y : h == 2 ? x.z : x.w;
    }
};

__device__ __forceinline__ uint32_t bf16_bits_or_ninf(const bf16 *r, int i, int V) {
    return i < V ? (uint32_t)__bfloat16_as_ushort(r[i]) : 0xff80u;
}

template <int DT>
__device__ __forceinline__ void load_raw(const void *row, int V, int c, Raw<DT> &x) {
    const int base = c * kChunk, tid = threadIdx.x;
    if constexpr (DT == TIDAR_DT_BF16) {
        const bf16 *r = reinterpret_cast<const bf16 *>(row);
        const bool fast = base + kChunk <= V && (reinterpret_cast<uintptr_t>(r) & 15) == 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i0 = base + j * 2048 + tid * 8;
            if (fast) {
                x.u[j] = __ldg(reinterpret_cast<const uint4 *>(r + i0));
            } else {
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    w[e] = bf16_bits_or_ninf(r, i0 + 2 * e, V) | (bf16_bits_or_ninf(r, i0 + 2 * e + 1, V) << 16);
                x.u[j] = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    } else {
        const float *r = reinterpret_cast<const float *>(row);
        const bool fast = base + kChunk <= V && (reinterpret_cast<uintptr_t>(r) & 15) == 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i0 = base + j * 2048 + tid * 8;
            if (fast) {
                x.f[2 * j] = __ldg(reinterpret_cast<const float4 *>(r + i0));
                x.f[2 * j + 1] = __ldg(reinterpret_cast<const float4 *>(r + i0 + 4));
            } else {
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = i0 + e < V ? r[i0 + e] : -INFINITY;
                x.f[2 * j] = make_float4(v[0], v[1], v[2], v[3]);
                x.f[2 * j + 1] = make_float4(v[4], v[5], v[6], v[7]);
            }
        }
    }
}

// Entry e of the row an item reads: the stored row, or (trust mix) lambda * p + (1 - lambda) * q.
template <int DT>
__device__ __forceinline__ float item_val(const Raw<DT> &t, const Raw<DT> &q, bool mix, float lambda, int e) {
    return mix ? mix_logit(t.get(e), q.get(e), lambda) : t.get(e);
}

__device__ __forceinline__ const void *logit_row(const void *base, int dtype, size_t row, int V) {
    const size_t es = dtype == TIDAR_DT_BF16 ? 2 : 4;
    return reinterpret_cast<const uint8_t *>(base) + row * V * es;
}

__device__ __forceinline__ const void *group_row(const TailParams &p, int b, int j, int s) {
    return logit_row(p.group_logits, p.dtype, ((size_t)b * (p.k + 1) + j) * p.k + s, p.V);
}

// Block-wide max / double sum of N values per thread at once (one pair of __syncthreads for all N).  The
// order of every reduction is fixed: lanes by butterfly, then warps 0..7 in turn.
template <int N>
__device__ __forceinline__ void block_max_n(float (&v)[N], float *red) {
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = warp_max(v[i]);
    __syncthreads();
    if (l == 0) {
#pragma unroll
        for (int i = 0; i < N; ++i) red[i * kWarps + w] = v[i];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < N; ++i) {
        float r = red[i * kWarps];
#pragma unroll
        for (int x = 1; x < kWarps; ++x) r = fmaxf(r, red[i * kWarps + x]);
        v[i] = r;
    }
}

template <int N>
__device__ __forceinline__ void block_sum_n(double (&v)[N], double *red) {
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = warp_sum_d(v[i]);
    __syncthreads();
    if (l == 0) {
#pragma unroll
        for (int i = 0; i < N; ++i) red[i * kWarps + w] = v[i];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < N; ++i) {
        double r = 0.0;
#pragma unroll
        for (int x = 0; x < kWarps; ++x) r += red[i * kWarps + x];
        v[i] = r;
    }
}

// Arrival of this CTA on `counter` after its writes (thread 0; the caller has passed a __syncthreads since
// they were made): true for the CTA that brings it to `total`, which may then read every arrival's writes.
__device__ __forceinline__ bool arrive_last(unsigned *counter, unsigned total) {
    __threadfence();
    const unsigned old = atomicAdd(counter, 1u);
    if (old + 1 == total) {
        __threadfence();
        return true;
    }
    return false;
}

__device__ __forceinline__ SeqState load_seq(const SeqState *s) {
    const int4 a = __ldcg(reinterpret_cast<const int4 *>(s));
    const int4 c = __ldcg(reinterpret_cast<const int4 *>(s) + 1);
    SeqState r;
    r.j = a.x;
    r.jc = a.y;
    r.P = a.z;
    r.pad = a.w;
    r.mp = __int_as_float(c.x);
    r.mq = __int_as_float(c.y);
    r.lzp = __int_as_float(c.z);
    r.lzq = __int_as_float(c.w);
    return r;
}

__device__ __forceinline__ void store_seq(SeqState *s, const SeqState &v) {
    reinterpret_cast<int4 *>(s)[0] = make_int4(v.j, v.jc, v.P, v.pad);
    reinterpret_cast<int4 *>(s)[1] =
        make_int4(__float_as_int(v.mp), __float_as_int(v.mq), __float_as_int(v.lzp), __float_as_int(v.lzq));
}

__device__ __forceinline__ void load_stat(const ChunkStat *st, float &m, double &z) {
    const double2 v = __ldcg(reinterpret_cast<const double2 *>(st));
    m = __int_as_float(__double2loint(v.x));
    z = v.y;
}

// Residual and target weights of one vocabulary entry given slot j*+1's constants (target logit zt).
__device__ __forceinline__ void slot_weights(float zt, float zq, const SeqState &ss, float &res, float &pw) {
    const float pv = fast_exp2(fmaf(zt, kLog2e, -ss.mp * kLog2e) - ss.lzp);
    const float qv = fast_exp2(fmaf(zq, kLog2e, -ss.mq * kLog2e) - ss.lzq);
    pw = zt == -INFINITY ? 0.f : pv;
    res = zt == -INFINITY ? 0.f : fmaxf(pv - qv, 0.f);
}

// Commit inputs of sequence b when the commit runs alone: j* if valid, else -1 (bits reported if asked).
__device__ __forceinline__ int checked_accept(const TailParams &p, int b, bool report) {
    const int j = p.accept_in[b];
    const int P = p.prefix_len[b];
    int bits = 0;
    if (j < 0 || j > p.k) bits |= TIDAR_DEV_BAD_ACCEPT;
    if (P < 0 || (bits == 0 && P + j > p.P_max)) bits |= TIDAR_DEV_BAD_PREFIX;
    if (bits == 0 && j < p.k && (p.resampled_in[b] < 0 || p.resampled_in[b] >= p.V)) bits |= TIDAR_DEV_BAD_TOKEN;
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

// Warp 0: the chunk whose cumulative weight first exceeds `target` among chunks c = lane + 32h (weights
// w[h], zero for missing chunks), and the weight before it; the last chunk with positive weight when
// rounding leaves none (target = INFINITY then).  Results in sm.chunk / sm.target.
__device__ __forceinline__ void find_chunk(const double (&w)[2], double target, int nchunk, TailSmem &sm) {
    const int lane = threadIdx.x & 31;
    double run = 0.0, before = 0.0;
    int ch = -1, last_pos = -1;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int c0 = 32 * h;
        if (c0 >= nchunk || ch >= 0) break;
        const int cc = c0 + lane;
        const double wc = cc < nchunk ? w[h] : 0.0;
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
        sm.chunk = ch >= 0 ? ch : last_pos;
        sm.target = ch >= 0 ? target - before : INFINITY;
    }
}

// ---------------------------------------------------------------------------------------------------------
// Phase A's last CTA of sequence b: merge of the 2k row statistics, the ratio tests, j*.

template <int MODE>
__device__ void finalize_seq(const TailParams &p, TailSmem &sm, int b) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = p.k, nc = p.nchunk;
    // one round trip: the statistics of every row (rows warp + 8i, chunks lane + 32h), the draft logits, the
    // drafts, uniforms, pre-accepted flag and prefix length
    float mc[4][2];
    double zc[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = warp + kWarps * i;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = lane + 32 * h;
            mc[i][h] = -INFINITY;
            zc[i][h] = 0.0;
            if (r < 2 * k && c < nc) load_stat(p.vstats + ((size_t)b * 2 * k + r) * nc + c, mc[i][h], zc[i][h]);
        }
    }
    int d = 0, pre = 0, P = 0;
    float ua = 0.f, zt_d = 0.f, zq_d = 0.f;
    if (warp == 0) {
        pre = p.preaccepted[b];
        if (MODE == kModeFused) P = p.prefix_len[b];
        if (lane < k) {
            d = p.drafts[b * k + lane];
            ua = p.u_acc[b * k + lane];
            zt_d = __ldcg(p.dlogit + (size_t)b * 2 * k + lane);
            zq_d = __ldcg(p.dlogit + (size_t)b * 2 * k + k + lane);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = warp + kWarps * i;
        if (r < 2 * k) {  // warp-uniform
            const float m = warp_max(fmaxf(mc[i][0], mc[i][1]));
            double s = 0.0;
#pragma unroll
            for (int h = 0; h < 2; ++h)
                if (mc[i][h] != -INFINITY) s += zc[i][h] * (double)exp2f((mc[i][h] - m) * kLog2e);
            s = warp_sum_d(s);
            if (lane == 0) {
                sm.m_row[r] = m;
                sm.lz_row[r] = log2(s);
            }
        }
    }
    __syncthreads();
    if (warp == 0) {
        bool accept = true, bad = false;
        if (lane < k) {
            bad = d < 0 || d >= p.V;
            if (!bad) {
                const double lp = ((double)zt_d - sm.m_row[lane]) * kLog2eD - sm.lz_row[lane];  // log2 p_i(d_i)
                const double lq = ((double)zq_d - sm.m_row[k + lane]) * kLog2eD - sm.lz_row[k + lane];
                const size_t row = (size_t)b * k + lane;
                if (p.logp_d) p.logp_d[row] = (float)(lp * kLn2D);
                if (p.logq_d) p.logq_d[row] = (float)(lq * kLn2D);
                accept = (lane == 0 && pre) || (double)ua < exp2(lp - lq);
            }
        }
        const unsigned badm = __ballot_sync(0xffffffffu, bad);
        const unsigned rejm = __ballot_sync(0xffffffffu, !accept);
        const int j = badm ? -1 : (rejm ? __ffs(rejm) - 1 : k);
        // every draft accepted: the emitted tokens (drafts pre .. k-1) need no draw
        const int src = lane + pre;
        const int dv = __shfl_sync(0xffffffffu, d, src < 32 ? src : 0);
        if (j == k && lane < k) p.tokens[(size_t)b * k + lane] = src < k ? dv : -1;
        if (lane == 0) {
            SeqState ss;
            ss.j = j;
            ss.jc = -1;
            ss.P = P;
            ss.pad = 0;
            const int sj = (j >= 0 && j < k) ? j : 0;
            ss.mp = sm.m_row[sj];
            ss.mq = sm.m_row[k + sj];
            ss.lzp = (float)sm.lz_row[sj];
            ss.lzq = (float)sm.lz_row[k + sj];
            if (j < 0) {
                atomicOr(p.dev_status, TIDAR_DEV_BAD_TOKEN);
            } else {
                p.accept_len[b] = j;
                if (j == k) {
                    p.n_emitted[b] = k - pre;
                    p.resampled[b] = -1;
                }
                if (MODE == kModeFused) {  // the commit's own checks of sequence b
                    int bits = 0;
                    if (P < 0 || P + j > p.P_max) bits |= TIDAR_DEV_BAD_PREFIX;
                    if (bits == 0 && p.block_table && j > 0) {
                        for (int pi = P / kPageRows; pi <= (P + j - 1) / kPageRows; ++pi) {
                            const int pg = p.block_table[(size_t)b * p.max_pages + pi];
                            if (pg < 0 || pg >= p.num_pages) bits |= TIDAR_DEV_BAD_PAGE;
                        }
                    }
                    if (bits) atomicOr(p.dev_status, bits);
                    else ss.jc = j;
                }
            }
            store_seq(p.seq + b, ss);
        }
    }
    __syncthreads();  // m_row / lz_row are reused
}

// ---------------------------------------------------------------------------------------------------------
// Draws.  `publish`: also write sequence b's new state (fused: P and j* from phase A).

__device__ __forceinline__ void publish_state(const TailParams &p, int b, int j, int new_prefix) {
    p.next_q_group[b] = j;
    p.next_preaccepted[b] = j < p.k ? 1 : 0;
    p.prefix_len[b] = new_prefix;
}

// Replacement token of sequence b (0 <= j* < k) from norm(max(0, p - q)) of slot j*+1, then the emitted
// tokens.  Fused: the token is also slot 0 of the next draft block, and the state is published.
template <int MODE>
__device__ void residual_draw(const TailParams &p, TailSmem &sm, int b, const SeqState &ss) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = p.k, nc = p.nchunk, j = ss.j;
    if (warp == 0) {
        double rp[2], pp[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = lane + 32 * h;
            rp[h] = c < nc ? __ldcg(p.res_part + (size_t)b * nc + c) : 0.0;
            pp[h] = c < nc ? __ldcg(p.p_part + (size_t)b * nc + c) : 0.0;
        }
        const float u = p.u_res[b];
        const double zr = warp_sum_d(rp[0] + rp[1]);
        const int use_p = !(zr > 0.0);  // p == q: the residual is empty, draw from p
        const double w[2] = {use_p ? pp[0] : rp[0], use_p ? pp[1] : rp[1]};
        const double tot = use_p ? warp_sum_d(w[0] + w[1]) : zr;
        find_chunk(w, (double)u * tot, nc, sm);
        if (lane == 0) sm.use_p = use_p;
    } else if (warp == 1) {
        if (lane < k) sm.drafts[lane] = p.drafts[b * k + lane];
        if (lane == 0) sm.pre = p.preaccepted[b];
    }
    __syncthreads();
    const int ch = sm.chunk;
    int t = -1;
    if (ch >= 0) {
        const size_t row = (size_t)b * k + j;
        float zt[32], zq[32];
        load_chunk32_contig(logit_row(p.q_logits, p.dtype, row, p.V), p.dtype, p.V, ch, zq);
        load_chunk32_contig(logit_row(p.p_logits, p.dtype, row, p.V), p.dtype, p.V, ch, zt);
        const bool use_p = sm.use_p;
        double w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            float res, pw;
            slot_weights(mix_logit(zt[e], zq[e], p.lambda), zq[e], ss, res, pw);
            w[e] = use_p ? (double)pw : (double)res;
        }
        const int loc = chunk_search256(w, sm.target, sm.scan_buf, sm.pick);
        t = loc < 0 ? -1 : ch * kChunk + loc;
    }
    if (tid == 0) {
        const int pre = sm.pre;
        int n = 0;
        int32_t *tok = p.tokens + (size_t)b * k;
        for (int i = pre; i < j; ++i) tok[n++] = sm.drafts[i];
        tok[n++] = t;
        p.n_emitted[b] = n;
        for (int i = n; i < k; ++i) tok[i] = -1;
        p.resampled[b] = t;
        if (MODE == kModeFused && ss.jc >= 0) {
            if (t < 0) {  // no replacement token: the commit of this sequence is abandoned
                atomicOr(p.dev_status, TIDAR_DEV_BAD_TOKEN);
            } else {
                p.next_drafts[(size_t)b * k] = t;
                publish_state(p, b, j, ss.P + j);
            }
        }
    }
    __syncthreads();
}

// Slot s of the next draft block of sequence b from softmax(group_logits[b, j, s]).
__device__ void group_draw(const TailParams &p, TailSmem &sm, int b, int j, int s) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nc = p.nchunk;
    if (warp == 0) {
        const ChunkStat *rs = p.gstats + ((size_t)b * p.k + s) * nc;
        float mc[2];
        double zc[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = lane + 32 * h;
            mc[h] = -INFINITY;
            zc[h] = 0.0;
            if (c < nc) load_stat(rs + c, mc[h], zc[h]);
        }
        const float u = p.u_draft[(size_t)b * p.k + s];
        const float m = warp_max(fmaxf(mc[0], mc[1]));
        double w[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) w[h] = mc[h] != -INFINITY ? zc[h] * (double)exp2f((mc[h] - m) * kLog2e) : 0.0;
        const double tot = warp_sum_d(w[0] + w[1]);
        find_chunk(w, (double)u * tot, nc, sm);
        if (lane == 0) sm.m = m;
    }
    __syncthreads();
    const int ch = sm.chunk;
    int t = -1;
    if (ch >= 0) {
        float z[32];
        load_chunk32_contig(group_row(p, b, j, s), p.dtype, p.V, ch, z);
        const float ms = sm.m * kLog2e;
        double w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) w[e] = z[e] == -INFINITY ? 0.0 : (double)fast_exp2(fmaf(z[e], kLog2e, -ms));
        const int loc = chunk_search256(w, sm.target, sm.scan_buf, sm.pick);
        t = loc < 0 ? -1 : ch * kChunk + loc;
    }
    if (tid == 0) p.next_drafts[(size_t)b * p.k + s] = t;
    __syncthreads();
}

// ---------------------------------------------------------------------------------------------------------
// Copy of the j accepted K/V rows of (layer l, sequence b, KV head kvh) into cache rows P .. P+j-1 by one
// warp (16 bytes per lane, four rows' vectors in flight).
__device__ __forceinline__ void copy_rows(const TailParams &p, int l, int b, int kvh, int j, int P) {
    const int lane = threadIdx.x & 31;
    const int vec = p.D / 8;
    const int n = j * vec;
    const bf16 *kn = reinterpret_cast<const bf16 *>(p.k_news[l]);
    const bf16 *vn = reinterpret_cast<const bf16 *>(p.v_news[l]);
    bf16 *kc = reinterpret_cast<bf16 *>(p.k_caches[l]);
    bf16 *vc = reinterpret_cast<bf16 *>(p.v_caches[l]);
    for (int base = 0; base < n; base += 4 * 32) {
        uint4 kv[4], vv[4];
        size_t dst[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int idx = base + q * 32 + lane;
            if (idx < n) {
                const int i = idx / vec, c = idx % vec;
                const size_t src = ((size_t)(b * p.R + i) * p.Hkv + kvh) * p.D + c * 8;
                size_t drow;
                if (p.block_table) {
                    const int r = P + i;
                    const int pg = p.block_table[(size_t)b * p.max_pages + r / kPageRows];
                    drow = ((size_t)pg * p.Hkv + kvh) * kPageRows + r % kPageRows;
                } else {
                    drow = (size_t)(b * p.Hkv + kvh) * p.P_max + P + i;
                }
                dst[q] = drow * p.D + c * 8;
                kv[q] = *reinterpret_cast<const uint4 *>(kn + src);
                vv[q] = *reinterpret_cast<const uint4 *>(vn + src);
            }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (base + q * 32 + lane < n) {
                *reinterpret_cast<uint4 *>(kc + dst[q]) = kv[q];
                *reinterpret_cast<uint4 *>(vc + dst[q]) = vv[q];
            }
        }
    }
}

// ---------------------------------------------------------------------------------------------------------

template <int MODE, int DT>
__global__ void __launch_bounds__(kStatThreads, 2) tail_kernel(const TailParams p) {
    __shared__ TailSmem sm;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = p.k, nc = p.nchunk, B = p.B;
    const unsigned G = gridDim.x;
    constexpr bool kVerify = (MODE & kModeVerify) != 0;
    constexpr bool kCommit = (MODE & kModeCommit) != 0;

    // ---- A: chunk statistics of the 2k rows of every sequence; each sequence's last CTA finalises it ----
    if constexpr (kVerify) {
        constexpr int NP = DT == TIDAR_DT_BF16 ? 2 : 1;  // items in flight per CTA
        const int itemsA = B * 2 * k * nc;
        const bool mixing = p.lambda != 0.f && p.lambda != 1.f;
        for (int it0 = blockIdx.x; it0 < itemsA; it0 += NP * G) {
            Raw<DT> tr[NP], qr[NP];
            int ib[NP], irow[NP], ic[NP], id[NP];
            bool imix[NP];
#pragma unroll
            for (int x = 0; x < NP; ++x) {
                const int it = it0 + x * G;
                ib[x] = -1;
                if (it >= itemsA) continue;
                const int c = it % nc, row = (it / nc) % (2 * k), b = it / (nc * 2 * k);
                const int slot = row < k ? row : row - k;
                const size_t srow = (size_t)b * k + slot;
                ib[x] = b;
                irow[x] = row;
                ic[x] = c;
                id[x] = p.drafts[b * k + slot];
                // target row: the AR row, the diffusion row (lambda = 0) or both (mixed); q row: the diffusion row
                const bool tq = row >= k || p.lambda == 0.f;
                imix[x] = row < k && mixing;
                load_raw<DT>(logit_row(tq ? p.q_logits : p.p_logits, p.dtype, srow, p.V), p.V, c, tr[x]);
                if (imix[x]) load_raw<DT>(logit_row(p.q_logits, p.dtype, srow, p.V), p.V, c, qr[x]);
            }
            float mx[NP];
#pragma unroll
            for (int x = 0; x < NP; ++x) {
                mx[x] = -INFINITY;
                if (ib[x] < 0) continue;
#pragma unroll
                for (int e = 0; e < 32; ++e) mx[x] = fmaxf(mx[x], item_val(tr[x], qr[x], imix[x], p.lambda, e));
                // the thread that holds entry d of this row keeps that logit for the ratio test
                const long long off = (long long)id[x] - (long long)ic[x] * kChunk;
                if (off >= 0 && off < kChunk && (((int)off & 2047) >> 3) == tid) {
                    const int ee = ((int)off >> 11) * 8 + ((int)off & 7);
                    float zd = 0.f;
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (e == ee) zd = item_val(tr[x], qr[x], imix[x], p.lambda, e);
                    p.dlogit[(size_t)ib[x] * 2 * k + irow[x]] = zd;
                    __threadfence();  // before thread 0's arrival for this item
                }
            }
            block_max_n<NP>(mx, sm.redf);
            double sz[NP];
#pragma unroll
            for (int x = 0; x < NP; ++x) {
                const float ms = mx[x] * kLog2e;
                float s = 0.f;
                if (ib[x] >= 0) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) s += fast_exp2(fmaf(item_val(tr[x], qr[x], imix[x], p.lambda, e), kLog2e, -ms));
                }
                sz[x] = (double)s;
            }
            block_sum_n<NP>(sz, sm.redd);
            if (tid == 0) {
#pragma unroll
                for (int x = 0; x < NP; ++x) {
                    sm.last[x] = -1;
                    if (ib[x] < 0) continue;
                    ChunkStat st;
                    st.m = mx[x];
                    st.pad = 0.f;
                    st.z = sz[x];
                    p.vstats[((size_t)ib[x] * 2 * k + irow[x]) * nc + ic[x]] = st;
                }
            }
            __syncthreads();  // every thread's draft logit is written before the arrival
            if (tid == 0) {
#pragma unroll
                for (int x = 0; x < NP; ++x)
                    if (ib[x] >= 0 && arrive_last(p.cnt_rows + ib[x], 2 * k * nc)) sm.last[x] = ib[x];
            }
            __syncthreads();
#pragma unroll
            for (int x = 0; x < NP; ++x) {
                const int fb = sm.last[x];
                if (fb >= 0) finalize_seq<MODE>(p, sm, fb);
            }
        }
        if (!grid_barrier(p.barrier, G, p.dev_status, kBarrierCycles)) return;
    }

    // ---- B: block items (residual chunks, group chunks), then warp items (copies) ----
    const int n_res = kVerify ? B * nc : 0;
    const int n_grp = kCommit ? B * k * nc : 0;
    const int nb = n_res + n_grp;
    for (int it = blockIdx.x; it < nb; it += G) {
        if (it < n_res) {
            const int c = it % nc, b = it / nc;
            const SeqState ss = load_seq(p.seq + b);
            if (ss.j < 0 || ss.j >= k) continue;  // uniform: nothing to draw
            const size_t row = (size_t)b * k + ss.j;
            Raw<DT> pr, qr;
            load_raw<DT>(logit_row(p.p_logits, p.dtype, row, p.V), p.V, c, pr);
            load_raw<DT>(logit_row(p.q_logits, p.dtype, row, p.V), p.V, c, qr);
            double acc[2] = {0.0, 0.0};
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float zq = qr.get(e);
                float res, pw;
                slot_weights(mix_logit(pr.get(e), zq, p.lambda), zq, ss, res, pw);
                acc[0] += res;
                acc[1] += pw;
            }
            block_sum_n<2>(acc, sm.redd);
            if (tid == 0) {
                p.res_part[(size_t)b * nc + c] = acc[0];
                p.p_part[(size_t)b * nc + c] = acc[1];
                sm.last[0] = arrive_last(p.cnt_res + b, nc) ? 1 : 0;
            }
            __syncthreads();
            if (sm.last[0]) residual_draw<MODE>(p, sm, b, ss);
        } else {
            const int t = it - n_res;
            const int c = t % nc, s = (t / nc) % k, b = t / (nc * k);
            int j;
            SeqState ss;
            if constexpr (kVerify) {  // fused: phase A's verdict
                ss = load_seq(p.seq + b);
                j = ss.jc;
            } else {
                j = checked_accept(p, b, false);
            }
            if (j < 0 || (s == 0 && j < k)) continue;  // uniform; slot 0 after a rejection is the replacement token
            Raw<DT> gr;
            load_raw<DT>(group_row(p, b, j, s), p.V, c, gr);
            float mx[1] = {-INFINITY};
#pragma unroll
            for (int e = 0; e < 32; ++e) mx[0] = fmaxf(mx[0], gr.get(e));
            block_max_n<1>(mx, sm.redf);
            const float ms = mx[0] * kLog2e;
            float sf = 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) sf += fast_exp2(fmaf(gr.get(e), kLog2e, -ms));
            double sz[1] = {(double)sf};
            block_sum_n<1>(sz, sm.redd);
            if (tid == 0) {
                ChunkStat st;
                st.m = mx[0];
                st.pad = 0.f;
                st.z = sz[0];
                p.gstats[((size_t)b * k + s) * nc + c] = st;
                sm.last[0] = 0;
                if constexpr (kVerify) sm.last[0] = arrive_last(p.cnt_grp + b * k + s, nc) ? 1 : 0;
            }
            __syncthreads();
            if constexpr (kVerify) {
                if (sm.last[0]) {
                    group_draw(p, sm, b, j, s);
                    if (s == 0 && tid == 0) publish_state(p, b, j, ss.P + j);  // j* = k: no replacement token
                }
            }
        }
    }
    if constexpr (kCommit) {
        // copies: the warps of the CTAs without block items (of every CTA when there are more items than CTAs)
        const int cb = nb < (int)G ? nb : 0;
        if ((int)blockIdx.x >= cb) {
            const int n_copy = p.L * B * p.Hkv;
            for (int it = ((int)blockIdx.x - cb) * kWarps + warp; it < n_copy; it += ((int)G - cb) * kWarps) {
                const int kvh = it % p.Hkv, b = (it / p.Hkv) % B, l = it / (p.Hkv * B);
                int j, P;
                if constexpr (kVerify) {
                    const SeqState ss = load_seq(p.seq + b);
                    j = ss.jc;
                    P = ss.P;
                } else {
                    const bool first = l == 0 && kvh == 0;
                    j = checked_accept(p, b, first && lane == 0);
                    P = p.prefix_len[b];
                    if (first && lane == 0) {  // phase C' takes j* from here: prefix_len may be advanced by then
                        SeqState ss = {};
                        ss.j = j;
                        store_seq(p.seq + b, ss);
                    }
                }
                if (j > 0) copy_rows(p, l, b, kvh, j, P);
            }
        }
    }

    // ---- C' (commit alone): draws of the next draft block; slot 0 publishes the state ----
    if constexpr (MODE == kModeCommit) {
        if (!grid_barrier(p.barrier, G, p.dev_status, kBarrierCycles)) return;
        for (int it = blockIdx.x; it < B * k; it += G) {
            const int s = it % k, b = it / k;
            const int j = __ldcg(&p.seq[b].j);
            if (j < 0) continue;
            if (s == 0 && j < k) {
                if (tid == 0) p.next_drafts[(size_t)b * k] = p.resampled_in[b];
            } else {
                group_draw(p, sm, b, j, s);
            }
            if (s == 0 && tid == 0) publish_state(p, b, j, p.prefix_len[b] + j);
        }
    }
}

// ---------------------------------------------------------------------------------------------------------
// Workspace: [vstats | dlogit | gstats | res_part | p_part | seq | counters], each region 256-byte aligned.

struct Layout {
    size_t vstats, dlogit, gstats, res, pp, seq, counters, total;
    size_t counter_bytes;
};

Layout layout(int B, int k, int V, int mode) {
    const size_t nc = vocab_chunks(V);
    const bool v = (mode & kModeVerify) != 0, c = (mode & kModeCommit) != 0;
    Layout L;
    size_t o = 0;
    L.vstats = o;
    o += v ? align256(sizeof(ChunkStat) * B * 2 * k * nc) : 0;
    L.dlogit = o;
    o += v ? align256(sizeof(float) * B * 2 * k) : 0;
    L.gstats = o;
    o += c ? align256(sizeof(ChunkStat) * B * k * nc) : 0;
    L.res = o;
    o += v ? align256(sizeof(double) * B * nc) : 0;
    L.pp = o;
    o += v ? align256(sizeof(double) * B * nc) : 0;
    L.seq = o;
    o += align256(sizeof(SeqState) * B);
    L.counters = o;
    L.counter_bytes = sizeof(unsigned) * (1 + 2 * (size_t)B + (size_t)B * k);
    o += align256(L.counter_bytes);
    L.total = o;
    return L;
}

template <int MODE, int DT>
int resident_ctas() {
    static int n = -1;
    if (n >= 0) return n;
    int dev = 0, sms = 0, per = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, tail_kernel<MODE, DT>, kStatThreads, 0) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    n = sms * per;
    return n;
}

template <int MODE, int DT>
cudaError_t launch_mode(TailParams &p, void *ws, cudaStream_t s) {
    const Layout L = layout(p.B, p.k, p.V, MODE);
    uint8_t *w = reinterpret_cast<uint8_t *>(ws);
    p.vstats = reinterpret_cast<ChunkStat *>(w + L.vstats);
    p.dlogit = reinterpret_cast<float *>(w + L.dlogit);
    p.gstats = reinterpret_cast<ChunkStat *>(w + L.gstats);
    p.res_part = reinterpret_cast<double *>(w + L.res);
    p.p_part = reinterpret_cast<double *>(w + L.pp);
    p.seq = reinterpret_cast<SeqState *>(w + L.seq);
    unsigned *cnt = reinterpret_cast<unsigned *>(w + L.counters);
    p.barrier = cnt;
    p.cnt_rows = cnt + 1;
    p.cnt_res = cnt + 1 + p.B;
    p.cnt_grp = cnt + 1 + 2 * p.B;
    const int cap = resident_ctas<MODE, DT>();
    if (cap <= 0) return cudaErrorLaunchFailure;
    // enough CTAs for every phase's items to run at once (phase A two items per CTA), at most two per SM
    const long nc = p.nchunk;
    long want = 1;
    if (MODE & kModeVerify) want = std::max(want, ((long)p.B * 2 * p.k * nc + 1) / 2);
    long nb = (MODE & kModeVerify) ? (long)p.B * nc : 0;
    if (MODE & kModeCommit) {
        nb += (long)p.B * p.k * nc;
        want = std::max(want, nb + ((long)p.L * p.B * p.Hkv + kWarps - 1) / kWarps);
    }
    want = std::max(want, nb);
    const int grid = (int)std::min<long>(want, std::min(cap, 2 * kNumSMs));
    cudaError_t e = cudaMemsetAsync(cnt, 0, L.counter_bytes, s);
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
    e = cudaLaunchKernelEx(&cfg, tail_kernel<MODE, DT>, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int MODE>
cudaError_t launch(TailParams &p, void *ws, cudaStream_t s) {
    return p.dtype == TIDAR_DT_BF16 ? launch_mode<MODE, TIDAR_DT_BF16>(p, ws, s)
                                    : launch_mode<MODE, TIDAR_DT_F32>(p, ws, s);
}

void set_verify(TailParams &p, const void *p_logits, const void *q_logits, const int32_t *drafts,
                const uint8_t *preaccepted, const float *u_acc, const float *u_res, float lambda, int32_t *accept_len,
                int32_t *resampled, int32_t *tokens, int32_t *n_emitted, float *logp_d, float *logq_d) {
    p.p_logits = p_logits;
    p.q_logits = q_logits;
    p.drafts = drafts;
    p.preaccepted = preaccepted;
    p.u_acc = u_acc;
    p.u_res = u_res;
    p.lambda = lambda;
    p.accept_len = accept_len;
    p.resampled = resampled;
    p.tokens = tokens;
    p.n_emitted = n_emitted;
    p.logp_d = logp_d;
    p.logq_d = logq_d;
}

void set_commit(TailParams &p, void *const *k_caches, void *const *v_caches, const void *const *k_news,
                const void *const *v_news, int L, int Hkv, int D, int k, int P_max, const int32_t *block_table,
                int max_pages, int num_pages, int32_t *prefix_len, const void *group_logits, const float *u_draft,
                int32_t *next_drafts, uint8_t *next_preaccepted, int32_t *next_q_group) {
    p.k_caches = k_caches;
    p.v_caches = v_caches;
    p.k_news = k_news;
    p.v_news = v_news;
    p.L = L;
    p.Hkv = Hkv;
    p.D = D;
    p.R = k * (k + 2);
    p.P_max = P_max;
    p.block_table = block_table;
    p.max_pages = max_pages;
    p.num_pages = num_pages;
    p.prefix_len = prefix_len;
    p.group_logits = group_logits;
    p.u_draft = u_draft;
    p.next_drafts = next_drafts;
    p.next_preaccepted = next_preaccepted;
    p.next_q_group = next_q_group;
}

}  // namespace

size_t verify_workspace_bytes(int B, int k, int V) { return layout(B, k, V, kModeVerify).total; }
size_t commit_workspace_bytes(int B, int k, int V) { return layout(B, k, V, kModeCommit).total; }
size_t verify_commit_workspace_bytes(int B, int k, int V) { return layout(B, k, V, kModeFused).total; }

cudaError_t verify_launch(const void *p_logits, const void *q_logits, int dtype, const int32_t *drafts,
                          const uint8_t *preaccepted, const float *u_acc, const float *u_res, int B, int k, int V,
                          float lambda, int32_t *accept_len, int32_t *resampled, int32_t *tokens, int32_t *n_emitted,
                          float *logp_d, float *logq_d, void *ws, int32_t *dev_status, cudaStream_t s) {
    TailParams p = {};
    set_verify(p, p_logits, q_logits, drafts, preaccepted, u_acc, u_res, lambda, accept_len, resampled, tokens,
               n_emitted, logp_d, logq_d);
    p.dtype = dtype;
    p.B = B;
    p.k = k;
    p.V = V;
    p.nchunk = vocab_chunks(V);
    p.dev_status = dev_status;
    return launch<kModeVerify>(p, ws, s);
}

cudaError_t commit_launch(void *const *k_caches, void *const *v_caches, const void *const *k_news,
                          const void *const *v_news, int L, int B, int Hkv, int D, int k, int P_max,
                          int32_t *prefix_len, const int32_t *accept_len, const int32_t *resampled,
                          const void *group_logits, int dtype, int V, const float *u_draft, int32_t *next_drafts,
                          uint8_t *next_preaccepted, int32_t *next_q_group, void *ws, int32_t *dev_status,
                          cudaStream_t s, const int32_t *block_table, int max_pages, int num_pages) {
    TailParams p = {};
    set_commit(p, k_caches, v_caches, k_news, v_news, L, Hkv, D, k, P_max, block_table, max_pages, num_pages,
               prefix_len, group_logits, u_draft, next_drafts, next_preaccepted, next_q_group);
    p.accept_in = accept_len;
    p.resampled_in = resampled;
    p.dtype = dtype;
    p.B = B;
    p.k = k;
    p.V = V;
    p.nchunk = vocab_chunks(V);
    p.dev_status = dev_status;
    return launch<kModeCommit>(p, ws, s);
}

cudaError_t verify_commit_launch(const void *p_logits, const void *q_logits, int dtype, const int32_t *drafts,
                                 const uint8_t *preaccepted, const float *u_acc, const float *u_res, float lambda,
                                 void *const *k_caches, void *const *v_caches, const void *const *k_news,
                                 const void *const *v_news, const int32_t *block_table, int max_pages, int num_pages,
                                 int L, int B, int Hkv, int D, int k, int P_max, int V, int32_t *prefix_len,
                                 const void *group_logits, const float *u_draft, int32_t *accept_len,
                                 int32_t *resampled, int32_t *tokens, int32_t *n_emitted, float *logp_d,
                                 float *logq_d, int32_t *next_drafts, uint8_t *next_preaccepted,
                                 int32_t *next_q_group, void *ws, int32_t *dev_status, cudaStream_t s) {
    TailParams p = {};
    set_verify(p, p_logits, q_logits, drafts, preaccepted, u_acc, u_res, lambda, accept_len, resampled, tokens,
               n_emitted, logp_d, logq_d);
    set_commit(p, k_caches, v_caches, k_news, v_news, L, Hkv, D, k, P_max, block_table, max_pages, num_pages,
               prefix_len, group_logits, u_draft, next_drafts, next_preaccepted, next_q_group);
    p.dtype = dtype;
    p.B = B;
    p.k = k;
    p.V = V;
    p.nchunk = vocab_chunks(V);
    p.dev_status = dev_status;
    return launch<kModeFused>(p, ws, s);
}

}  // namespace tidar
