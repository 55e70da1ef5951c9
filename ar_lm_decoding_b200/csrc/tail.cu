// The end of a TiDAR decode step: the AR rejection-sampling verify of the
// previous step's drafts, the exact-KV-cache commit of the accepted rows and
// the next-draft selection.  One cooperative kernel in three modes: the
// verify alone, the commit alone, or both fused into one launch.
//
// The vocabulary is cut into chunks of 8192 entries (a CTA of 256 threads, 32
// entries per thread).  Every call moves a few MB, so its time is the chain of
// dependent memory round trips, not bandwidth; the kernel keeps that chain
// short.  There is no grid barrier and no arrival counter: every value one CTA
// hands to another goes into a slot that the launch first fills with a NaN
// bit pattern (one memset), and the consumer polls the slots themselves --
// bounded, with relaxed loads -- until none is NaN.  A value arrives together
// with the news that it is ready.
//
//  A  (verify) per-chunk max and sum-exp of the 2k target rows and q rows of
//     every sequence -- the HBM-bound sweep, two items per CTA in flight
//     (bf16); the thread holding entry d_i of a row also publishes that logit.
//  B  block items, in this order (a CTA takes items blockIdx.x, +G, ...):
//     - residual chunk (b, c) (verify): the verdict of sequence b -- every CTA
//       that needs it polls the sequence's 2k x nchunk statistics and forms it
//       itself: the merged row normalisers, the k ratio tests a_i = [u_i <
//       p_i(d_i)/q_i(d_i)] in double precision (slot 1 forced when
//       pre-accepted), j* = first rejection.  Then the sums of max(0, p - q)
//       and of p over chunk c of slot j*+1, published; the nchunk CTAs of the
//       sequence poll all sums, find the chunk that holds u_res * Z, and the
//       CTA that owns it rescans its own weights (through shared memory, in
//       vocabulary order) for the replacement token.  The c = 0 item writes
//       the verify outputs.
//     - group chunk (b, s, c) (commit): statistics of chunk c of slot s of
//       pre-draft group j*, published; the owner of the chunk that holds
//       u_draft * Z draws slot s of the next draft block.
//     - copies (b, q) (commit): 8 warps, each copying the j* accepted K/V rows
//       of one (layer, KV head) into the cache, 16 bytes per lane.
//     The (sequence, slot 0) draw -- the replacement token when j* < k --
//     also publishes the new state: next_q_group, next_preaccepted and
//     prefix_len = P + j*, where P is the prefix length captured in a slot at
//     the kernel's start (so no copy can see the new value).
// Deadlock freedom: every CTA takes its items in increasing index order; an
// item waits only for phase-A results and for the other items of its own
// group (the nchunk consecutive items of one sequence or slot), and a group
// is never larger than the grid, so the lowest unfinished item can always
// complete.  All CTAs are resident (cooperative launch) and every wait is
// bounded anyway: on expiry the CTA raises TIDAR_DEV_TIMEOUT and stops.
#include "vocab.cuh"

namespace tidar {

namespace {

constexpr long long kWaitCycles = 4000000000LL;  // bound of every poll (~2 s)
constexpr int kModeVerify = 1, kModeCommit = 2, kModeFused = 3;
constexpr int kWarps = kStatThreads / 32;
constexpr double kLog2eD = 1.4426950408889634;
constexpr double kLn2D = 0.6931471805599453;
constexpr int kPrefixUnset = -1;           // P slot before it is written (all bits set)
constexpr int kPrefixInvalid = INT32_MIN;  // P slot of a negative prefix length

struct TailParams {
    // verify
    const void *p_logits, *q_logits;
    const void *t_logits;  // the target logits when they are not mixed: p (lambda = 1) or q (lambda = 0)
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
    // slots, NaN (all bits set) until written
    double2 *vstats;  // [B][2k][nchunk] {max (float bits in the low word), sum exp}: target rows, then q rows
    float *dlogit;    // [B][2k]: the draft's logit in each row
    double2 *parts;   // [B][nchunk] {residual weight, target weight} of slot j*+1's chunks
    double2 *gstats;  // [B][k][nchunk] {max, sum exp} of group j*'s slot rows
    int32_t *pslot;   // [B] prefix length at the kernel's start
    int4 *vslot;      // [B][2] the verdict of sequence b, published by its first residual item (encoded, below)
    int32_t *dev_status;
};

struct Verdict {  // what the items of sequence b need to know
    int j;    // j* (verify, fused) or the given accept length (commit alone); -1: sequence skipped
    int jc;   // j* when the commit may proceed, else -1
    int P;    // prefix length at the kernel's start
    int pre;  // pre-accepted flag
    float mp, mq, lzp, lzq;  // max and log2 row sum of slot j*+1's target and q rows
};

struct TailSmem {
    float redf[2 * kWarps];
    double redd[2 * kWarps];
    double scan_buf[kWarps];
    float m_row[2 * kMaxDraft];
    double lz_row[2 * kMaxDraft];
    float lp[kMaxDraft], lq[kMaxDraft];
    int drafts[kMaxDraft];
    int pick[2];
    int chunk, use_p, vb, bits, expired;
    double target;
    float m;
    Verdict v;
    float w[kChunk + kChunk / 32];  // one chunk's weights in vocabulary order (one pad word per 32), for the rescan
};

// Position of chunk entry i in TailSmem::w: thread t's 32 entries t*32 .. t*32+31 then sit in 32 distinct banks.
__device__ __forceinline__ int wpos(int i) { return i + (i >> 5); }

// ---------------------------------------------------------------------------------------------------------
// Slot access: relaxed (morally strong, never cached in L1) loads and stores at GPU scope.

__device__ __forceinline__ double2 ld_slot(const double2 *a) {
    double2 v;
    asm volatile("ld.relaxed.gpu.global.v2.f64 {%0, %1}, [%2];\n" : "=d"(v.x), "=d"(v.y) : "l"(a) : "memory");
    return v;
}
__device__ __forceinline__ void st_slot(double2 *a, double x, double y) {
    asm volatile("st.relaxed.gpu.global.v2.f64 [%0], {%1, %2};\n" ::"l"(a), "d"(x), "d"(y) : "memory");
}
__device__ __forceinline__ float ld_slot(const float *a) {
    float v;
    asm volatile("ld.relaxed.gpu.global.f32 %0, [%1];\n" : "=f"(v) : "l"(a) : "memory");
    return v;
}
__device__ __forceinline__ void st_slot(float *a, float x) {
    asm volatile("st.relaxed.gpu.global.f32 [%0], %1;\n" ::"l"(a), "f"(x) : "memory");
}
__device__ __forceinline__ int ld_slot(const int32_t *a) {
    int v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];\n" : "=r"(v) : "l"(a) : "memory");
    return v;
}
__device__ __forceinline__ void st_slot(int32_t *a, int x) {
    asm volatile("st.relaxed.gpu.global.s32 [%0], %1;\n" ::"l"(a), "r"(x) : "memory");
}

// A statistics slot {max, sum}: max as float bits in the low word of x.
__device__ __forceinline__ void st_stat(double2 *a, float m, double z) {
    st_slot(a, __hiloint2double(0, __float_as_int(m)), m == -INFINITY ? 0.0 : z);
}
__device__ __forceinline__ float stat_max(const double2 &v) { return __int_as_float(__double2loint(v.x)); }
__device__ __forceinline__ bool stat_ready(const double2 &v) { return !isnan(stat_max(v)) && !isnan(v.y); }
__device__ __forceinline__ double2 empty_stat() {
    return make_double2(__hiloint2double(0, __float_as_int(-INFINITY)), 0.0);
}

// Bounded spin of one warp: repeats `round` (this lane's loads; returns whether its values are all there)
// until every lane is ready.  A hand-over between two CTAs costs about one store-to-load visibility (~0.45 us on
// B200), so the loop neither sleeps nor synchronises the CTA; the CTA joins the polling warps at one
// __syncthreads afterwards.  On expiry the warp raises TIDAR_DEV_TIMEOUT, sets sm.expired and returns false.
template <class Round>
__device__ __forceinline__ bool warp_poll(Round round, const TailParams &p, int *expired) {
    const long long t0 = clock64();
    while (true) {
        if (__all_sync(0xffffffffu, round())) return true;
        if (__shfl_sync(0xffffffffu, (int)(clock64() - t0 > kWaitCycles), 0)) {
            if ((threadIdx.x & 31) == 0) {
                *expired = 1;
                atomicOr(p.dev_status, TIDAR_DEV_TIMEOUT);
            }
            return false;
        }
    }
}

// ---------------------------------------------------------------------------------------------------------
// A thread's 32 entries of one chunk as loaded (strided layout: entry e of thread t is at chunk offset
// (e/8)*2048 + t*8 + e%8, so that a warp reads 512 contiguous bytes per bf16 load).  Entries beyond V hold
// -inf.

__host__ __device__ constexpr int entry_offset(int t, int e) { return (e >> 3) * 2048 + t * 8 + (e & 7); }

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
template <bool MIX, int DT>
__device__ __forceinline__ float item_val(const Raw<DT> &t, const Raw<DT> &q, bool mix, float lambda, int e) {
    if constexpr (MIX) return mix ? mix_logit(t.get(e), q.get(e), lambda) : t.get(e);
    return t.get(e);
}

__device__ __forceinline__ const void *logit_row(const void *base, int dtype, size_t row, int V) {
    const size_t es = dtype == TIDAR_DT_BF16 ? 2 : 4;
    return reinterpret_cast<const uint8_t *>(base) + row * V * es;
}

__device__ __forceinline__ const void *group_row(const TailParams &p, int b, int j, int s) {
    return logit_row(p.group_logits, p.dtype, ((size_t)b * (p.k + 1) + j) * p.k + s, p.V);
}

// Block-wide max / double sum of N values per thread at once.  The order of every reduction is fixed: lanes
// by butterfly, then warps 0..7 in turn.
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

// x unchanged, but opaque to the compiler: values computed from it are not merged with earlier ones.
__device__ __forceinline__ float launder(float x) {
    asm volatile("" : "+f"(x));
    return x;
}

// Residual and target weights of one vocabulary entry given slot j*+1's constants (target logit zt).
__device__ __forceinline__ void slot_weights(float zt, float zq, const Verdict &v, float &res, float &pw) {
    const float pv = fast_exp2(fmaf(zt, kLog2e, -v.mp * kLog2e) - v.lzp);
    const float qv = fast_exp2(fmaf(zq, kLog2e, -v.mq * kLog2e) - v.lzq);
    pw = zt == -INFINITY ? 0.f : pv;
    res = zt == -INFINITY ? 0.f : fmaxf(pv - qv, 0.f);
}

// Warp 0: the chunk whose cumulative weight first exceeds `target` among chunks c = lane + 32h (weights
// w[h], zero for missing chunks), and the weight before it; the last chunk with positive weight when
// rounding leaves none (target = INFINITY then), -1 when every weight is zero.  Results in sm.chunk /
// sm.target.
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

// The rescan of the chosen chunk by the CTA that owns it: every thread has written its 32 weights to sm.w
// (vocabulary order); returns the local index of the draw: the first entry whose inclusive sum (double, in
// vocabulary order) exceeds sm.target, else the last entry with positive weight, else -1.  Thread t scans
// entries t*32 .. t*32+31 after a block-wide exclusive scan of the threads' sums.
__device__ __forceinline__ int rescan(TailSmem &sm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __syncthreads();
    const float *w = sm.w + wpos(tid * 32);  // the pad word never falls inside a thread's 32 entries
    double loc = 0.0;
#pragma unroll 8
    for (int e = 0; e < 32; ++e) loc += (double)w[e];
    double incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (tid == 0) {
        sm.pick[0] = 0x7fffffff;
        sm.pick[1] = -1;
    }
    if (lane == 31) sm.scan_buf[warp] = incl;
    __syncthreads();
    double c = incl - loc;  // exclusive prefix of this thread
    for (int i = 0; i < warp; ++i) c += sm.scan_buf[i];
    const double target = sm.target;
    int first = 0x7fffffff, last = -1;
#pragma unroll 8
    for (int e = 0; e < 32; ++e) {
        const float x = w[e];
        c += (double)x;
        if (x > 0.f) {
            last = tid * 32 + e;
            if (c > target && first == 0x7fffffff) first = tid * 32 + e;
        }
    }
    if (first != 0x7fffffff) atomicMin(&sm.pick[0], first);
    if (last >= 0) atomicMax(&sm.pick[1], last);
    __syncthreads();
    return sm.pick[0] != 0x7fffffff ? sm.pick[0] : sm.pick[1];
}

// ---------------------------------------------------------------------------------------------------------
// The verdict of sequence b (every thread returns the same; false after a timeout).  Cached in sm.v for the
// next item of the same sequence.  `how`: kVerdictCompute forms it (from the phase-A statistics; the commit
// alone: from the given accept length and the checks); kVerdictPublish also publishes it (the sequence's first
// residual item, the lowest-index item of the sequence in phase B); kVerdictLookup polls the published one.

constexpr int kVerdictLookup = 0, kVerdictCompute = 1, kVerdictPublish = 2;

__device__ __forceinline__ int4 ld_slot4(const int4 *a) {
    int4 v;
    asm volatile("ld.relaxed.gpu.global.v4.s32 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(a)
                 : "memory");
    return v;
}
__device__ __forceinline__ void st_slot4(int4 *a, int4 v) {
    asm volatile("st.relaxed.gpu.global.v4.s32 [%0], {%1, %2, %3, %4};\n" ::"l"(a), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}
// Published form: {j + 2, jc + 2, P, pre}, {mp, mq, lzp, lzq}: no word is ever all ones (the unset pattern).
__device__ __forceinline__ bool vslot_ready(const int4 &a, const int4 &c) {
    return a.x != -1 && a.y != -1 && a.z != -1 && a.w != -1 && c.x != -1 && c.y != -1 && c.z != -1 && c.w != -1;
}

template <int MODE>
__device__ bool get_verdict(const TailParams &p, TailSmem &sm, int b, int how) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = p.k, nc = p.nchunk;
    constexpr bool kVerify = (MODE & kModeVerify) != 0;
    constexpr bool kCommit = (MODE & kModeCommit) != 0;
    if (sm.vb == b) {
        if (kVerify && how == kVerdictPublish && tid == 0) {
            const Verdict &v = sm.v;
            st_slot4(p.vslot + 2 * b, make_int4(v.j + 2, v.jc + 2, v.P, v.pre));
            st_slot4(p.vslot + 2 * b + 1, make_int4(__float_as_int(v.mp), __float_as_int(v.mq),
                                                    __float_as_int(v.lzp), __float_as_int(v.lzq)));
        }
        return true;
    }
    int P = 0;
    if (kVerify && how == kVerdictLookup) {
        int4 a = make_int4(0, 0, 0, 0), c = a;
        if (warp == 0) {
            if (lane < k) sm.drafts[lane] = p.drafts[b * k + lane];  // for the emitted tokens
            warp_poll([&] {
                if (lane != 0) return true;
                a = ld_slot4(p.vslot + 2 * b);
                c = ld_slot4(p.vslot + 2 * b + 1);
                return vslot_ready(a, c);
            }, p, &sm.expired);
        }
        if (tid == 0 && !sm.expired) {
            Verdict v;
            v.j = a.x - 2;
            v.jc = a.y - 2;
            v.P = a.z;
            v.pre = a.w;
            v.mp = __int_as_float(c.x);
            v.mq = __int_as_float(c.y);
            v.lzp = __int_as_float(c.z);
            v.lzq = __int_as_float(c.w);
            sm.v = v;
            sm.bits = 0;
            sm.vb = b;
        }
        __syncthreads();
        return !sm.expired;
    }
    if constexpr (kVerify) {
        int d = 0, pre = 0;
        float ua = 0.f;
        if (warp == 0) {
            pre = p.preaccepted[b];
            if (lane < k) {
                d = p.drafts[b * k + lane];
                ua = p.u_acc[b * k + lane];
            }
        }
        const bool dvalid = warp == 0 && lane < k && d >= 0 && d < p.V;
        // the statistics of every row (rows warp + 8i, chunks lane + 32h), the draft logits and (commit) the
        // prefix length, in one poll
        double2 st[4][2];
        float zt_d = 0.f, zq_d = 0.f;
        warp_poll([&] {  // every warp polls its own rows
            bool ready = true;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = warp + kWarps * i;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int c = lane + 32 * h;
                    st[i][h] = empty_stat();
                    if (r < 2 * k && c < nc) {
                        st[i][h] = ld_slot(p.vstats + ((size_t)b * 2 * k + r) * nc + c);
                        ready = ready && stat_ready(st[i][h]);
                    }
                }
            }
            if (dvalid) {
                zt_d = ld_slot(p.dlogit + (size_t)b * 2 * k + lane);
                zq_d = ld_slot(p.dlogit + (size_t)b * 2 * k + k + lane);
                ready = ready && !isnan(zt_d) && !isnan(zq_d);
            }
            if (kCommit && tid == 0) {
                P = ld_slot(p.pslot + b);
                ready = ready && P != kPrefixUnset;
            }
            return ready;
        }, p, &sm.expired);
        __syncthreads();
        if (sm.expired) return false;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = warp + kWarps * i;
            if (r < 2 * k) {  // warp-uniform
                const float m = warp_max(fmaxf(stat_max(st[i][0]), stat_max(st[i][1])));
                double s = 0.0;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float mc = stat_max(st[i][h]);
                    if (mc != -INFINITY) s += st[i][h].y * (double)exp2f((mc - m) * kLog2e);
                }
                s = warp_sum_d(s);
                if (lane == 0) {
                    sm.m_row[r] = m;
                    sm.lz_row[r] = (double)__log2f((float)s);  // the hardware log2 (rel. error ~1e-7)
                }
            }
        }
        __syncthreads();
        if (warp == 0) {
            bool accept = true;
            if (dvalid) {
                const double lp = ((double)zt_d - sm.m_row[lane]) * kLog2eD - sm.lz_row[lane];  // log2 p_i(d_i)
                const double lq = ((double)zq_d - sm.m_row[k + lane]) * kLog2eD - sm.lz_row[k + lane];
                sm.lp[lane] = (float)(lp * kLn2D);
                sm.lq[lane] = (float)(lq * kLn2D);
                accept = (lane == 0 && pre) || ua < exp2f((float)(lp - lq));
            }
            if (lane < k) sm.drafts[lane] = d;
            const unsigned badm = __ballot_sync(0xffffffffu, lane < k && !dvalid);
            const unsigned rejm = __ballot_sync(0xffffffffu, !accept);
            if (lane == 0) {
                const int j = badm ? -1 : (rejm ? __ffs(rejm) - 1 : k);
                Verdict v;
                v.j = j;
                v.jc = -1;
                v.P = 0;
                v.pre = pre;
                const int sj = (j >= 0 && j < k) ? j : 0;
                v.mp = sm.m_row[sj];
                v.mq = sm.m_row[k + sj];
                v.lzp = (float)sm.lz_row[sj];
                v.lzq = (float)sm.lz_row[k + sj];
                sm.v = v;
                sm.bits = j < 0 ? TIDAR_DEV_BAD_TOKEN : 0;
            }
        }
        __syncthreads();
    } else {
        if (tid == 0) {
            sm.v = Verdict{};
            sm.v.j = p.accept_in[b];
            sm.bits = 0;
        }
        if (warp == 0) {
            warp_poll([&] {
                if (lane != 0) return true;
                P = ld_slot(p.pslot + b);
                return P != kPrefixUnset;
            }, p, &sm.expired);
        }
        __syncthreads();
        if (sm.expired) return false;
    }
    if (tid == 0) {
        if constexpr (kCommit) {  // the commit's own checks of sequence b (P: thread 0's poll)
            const int j = sm.v.j;
            int bits = 0;
            if (!kVerify && (j < 0 || j > p.k)) bits |= TIDAR_DEV_BAD_ACCEPT;
            if (j >= 0 && bits == 0) {
                if (P < 0 || P + j > p.P_max) bits |= TIDAR_DEV_BAD_PREFIX;
                if (!kVerify && bits == 0 && j < p.k && (p.resampled_in[b] < 0 || p.resampled_in[b] >= p.V))
                    bits |= TIDAR_DEV_BAD_TOKEN;
                if (bits == 0 && p.block_table && j > 0) {  // the pages that receive rows P .. P+j-1
                    for (int pi = P / kPageRows; pi <= (P + j - 1) / kPageRows; ++pi) {
                        const int pg = p.block_table[(size_t)b * p.max_pages + pi];
                        if (pg < 0 || pg >= p.num_pages) bits |= TIDAR_DEV_BAD_PAGE;
                    }
                }
                if (bits == 0) sm.v.jc = j;
            }
            sm.v.P = P;
            sm.bits |= bits;
        }
        if (kVerify && how == kVerdictPublish) {
            const Verdict &v = sm.v;
            st_slot4(p.vslot + 2 * b, make_int4(v.j + 2, v.jc + 2, v.P, v.pre));
            st_slot4(p.vslot + 2 * b + 1, make_int4(__float_as_int(v.mp), __float_as_int(v.mq),
                                                    __float_as_int(v.lzp), __float_as_int(v.lzq)));
        }
        sm.vb = b;
    }
    __syncthreads();
    return true;
}

// The verify outputs of sequence b (one CTA per sequence writes them).
__device__ void write_verify_outputs(const TailParams &p, TailSmem &sm, int b) {
    const int tid = threadIdx.x, k = p.k;
    const Verdict &v = sm.v;
    if (tid < 32) {
        const int lane = tid;
        if (v.j >= 0 && lane < k) {
            const size_t row = (size_t)b * k + lane;
            if (p.logp_d) p.logp_d[row] = sm.lp[lane];
            if (p.logq_d) p.logq_d[row] = sm.lq[lane];
            if (v.j == k) {  // every draft accepted: the emitted tokens (drafts pre .. k-1) need no draw
                const int src = lane + v.pre;
                p.tokens[row] = src < k ? sm.drafts[src] : -1;
            }
        }
        if (lane == 0) {
            if (sm.bits) atomicOr(p.dev_status, sm.bits);
            if (v.j >= 0) {
                p.accept_len[b] = v.j;
                if (v.j == k) {
                    p.n_emitted[b] = k - v.pre;
                    p.resampled[b] = -1;
                }
            }
        }
    }
}

__device__ __forceinline__ void publish_state(const TailParams &p, int b, int j, int new_prefix) {
    p.next_q_group[b] = j;
    p.next_preaccepted[b] = j < p.k ? 1 : 0;
    p.prefix_len[b] = new_prefix;
}

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
// Block items.  Each returns false after a timeout (the CTA then stops).

// Residual chunk (b, c): partial sums of slot j*+1's residual and target weights; the owner of the chunk
// that holds the draw makes it.
template <int MODE, int DT, bool MIX>
__device__ bool residual_item(const TailParams &p, TailSmem &sm, int b, int c, int how) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = p.k, nc = p.nchunk;
    if (!get_verdict<MODE>(p, sm, b, c == 0 ? kVerdictPublish : how)) return false;
    if (c == 0) write_verify_outputs(p, sm, b);
    const Verdict v = sm.v;
    if (v.j < 0 || v.j >= k) return true;  // uniform: nothing to draw
    const size_t row = (size_t)b * k + v.j;
    Raw<DT> pr, qr;  // the target row (or, mixed, the AR row) and the q row of slot j*+1
    load_raw<DT>(logit_row(MIX ? p.p_logits : p.t_logits, p.dtype, row, p.V), p.V, c, pr);
    load_raw<DT>(logit_row(p.q_logits, p.dtype, row, p.V), p.V, c, qr);
    double acc[2] = {0.0, 0.0};
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const float zq = qr.get(e);
        float res, pw;
        slot_weights(item_val<MIX>(pr, qr, true, p.lambda, e), zq, v, res, pw);
        acc[0] += res;
        acc[1] += pw;
        sm.w[wpos(entry_offset(tid, e))] = res;  // kept for the rescan, should this CTA own the draw
    }
    block_sum_n<2>(acc, sm.redd);
    if (tid == 0) st_slot(p.parts + (size_t)b * nc + c, acc[0], acc[1]);
    // every chunk's sums, then the chunk that holds u_res * Z (warp 0)
    double2 pv[2];
    if (warp == 0) {
        warp_poll([&] {
            bool ready = true;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int cc = lane + 32 * h;
                pv[h] = make_double2(0.0, 0.0);
                if (cc < nc) {
                    pv[h] = ld_slot(p.parts + (size_t)b * nc + cc);
                    ready = ready && !isnan(pv[h].x) && !isnan(pv[h].y);
                }
            }
            return ready;
        }, p, &sm.expired);
    }
    if (warp == 0 && !__shfl_sync(0xffffffffu, sm.expired, 0)) {
        const double zr = warp_sum_d(pv[0].x + pv[1].x);
        const int use_p = !(zr > 0.0);  // p == q: the residual is empty, draw from p
        const double w[2] = {use_p ? pv[0].y : pv[0].x, use_p ? pv[1].y : pv[1].x};
        const double tot = use_p ? warp_sum_d(w[0] + w[1]) : zr;
        find_chunk(w, (double)p.u_res[b] * tot, nc, sm);
        if (lane == 0) sm.use_p = use_p;
    }
    __syncthreads();
    if (sm.expired) return false;
    const int ch = sm.chunk;
    if (ch != c && !(ch < 0 && c == 0)) return true;  // uniform: another CTA owns the draw
    int t = -1;
    if (ch >= 0) {
        if (sm.use_p) {  // p == q: the target weights replace the residual ones (rare; recomputed, not kept)
            Verdict vl = v;
            vl.mp = launder(vl.mp);
            vl.mq = launder(vl.mq);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float zq = qr.get(e);
                float res, pw;
                slot_weights(item_val<MIX>(pr, qr, true, p.lambda, e), zq, vl, res, pw);
                sm.w[wpos(entry_offset(tid, e))] = pw;
            }
        }
        const int loc = rescan(sm);
        t = loc < 0 ? -1 : ch * kChunk + loc;
    }
    if (tid == 0) {
        const int j = v.j;
        int n = 0;
        int32_t *tok = p.tokens + (size_t)b * k;
        for (int i = v.pre; i < j; ++i) tok[n++] = sm.drafts[i];
        tok[n++] = t;
        p.n_emitted[b] = n;
        for (int i = n; i < k; ++i) tok[i] = -1;
        p.resampled[b] = t;
        if (MODE == kModeFused && v.jc >= 0) {
            if (t < 0) {  // no replacement token: the commit of this sequence is abandoned
                atomicOr(p.dev_status, TIDAR_DEV_BAD_TOKEN);
            } else {
                p.next_drafts[(size_t)b * k] = t;
                publish_state(p, b, j, v.P + j);
            }
        }
    }
    __syncthreads();
    return true;
}

// Group chunk (b, s, c): statistics of chunk c of slot s of group j*; the owner of the chunk that holds the
// draw makes it (slot s of the next draft block).
template <int MODE, int DT>
__device__ bool group_item(const TailParams &p, TailSmem &sm, int b, int s, int c, int how) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = p.k, nc = p.nchunk;
    if (!get_verdict<MODE>(p, sm, b, how)) return false;
    const Verdict v = sm.v;
    if (MODE == kModeCommit && s == 0 && c == 0 && tid == 0) {
        if (sm.bits) atomicOr(p.dev_status, sm.bits);  // the commit's checks, reported once per sequence
        if (v.jc >= 0 && v.jc < k) {  // slot 0 after a rejection: the replacement token
            p.next_drafts[(size_t)b * k] = p.resampled_in[b];
            publish_state(p, b, v.jc, v.P + v.jc);
        }
    }
    const int j = v.jc;
    if (j < 0 || (s == 0 && j < k)) return true;  // uniform
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
    double2 *row_st = p.gstats + ((size_t)b * k + s) * nc;
    if (tid == 0) st_stat(row_st + c, mx[0], sz[0]);
    double2 gv[2];
    if (warp == 0) {
        warp_poll([&] {
            bool ready = true;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int cc = lane + 32 * h;
                gv[h] = empty_stat();
                if (cc < nc) {
                    gv[h] = ld_slot(row_st + cc);
                    ready = ready && stat_ready(gv[h]);
                }
            }
            return ready;
        }, p, &sm.expired);
    }
    if (warp == 0 && !__shfl_sync(0xffffffffu, sm.expired, 0)) {
        const float m = warp_max(fmaxf(stat_max(gv[0]), stat_max(gv[1])));
        double w[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float mc = stat_max(gv[h]);
            w[h] = mc != -INFINITY ? gv[h].y * (double)exp2f((mc - m) * kLog2e) : 0.0;
        }
        const double tot = warp_sum_d(w[0] + w[1]);
        find_chunk(w, (double)p.u_draft[(size_t)b * k + s] * tot, nc, sm);
        if (lane == 0) sm.m = m;
    }
    __syncthreads();
    if (sm.expired) return false;
    const int ch = sm.chunk;
    if (ch != c && !(ch < 0 && c == 0)) return true;  // uniform: another CTA owns the draw
    int t = -1;
    if (ch >= 0) {
        const float mr = sm.m * kLog2e;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const float z = gr.get(e);
            sm.w[wpos(entry_offset(tid, e))] = z == -INFINITY ? 0.f : fast_exp2(fmaf(z, kLog2e, -mr));
        }
        const int loc = rescan(sm);
        t = loc < 0 ? -1 : ch * kChunk + loc;
    }
    if (tid == 0) {
        p.next_drafts[(size_t)b * k + s] = t;
        if (s == 0) publish_state(p, b, j, v.P + j);  // j* = k: no replacement token
    }
    __syncthreads();
    return true;
}

// Copies (b, q): warp w copies (layer, KV head) pair 8q + w of sequence b.
template <int MODE>
__device__ bool copy_item(const TailParams &p, TailSmem &sm, int b, int q, int how) {
    if (!get_verdict<MODE>(p, sm, b, how)) return false;
    const int pair = q * kWarps + (threadIdx.x >> 5);
    const int j = sm.v.jc;
    if (j > 0 && pair < p.L * p.Hkv) copy_rows(p, pair / p.Hkv, b, pair % p.Hkv, j, sm.v.P);
    return true;
}

// ---------------------------------------------------------------------------------------------------------

template <int MODE, int DT, bool MIX>
__global__ void __launch_bounds__(kStatThreads, 2) tail_kernel(const TailParams p) {
    __shared__ TailSmem sm;
    const int tid = threadIdx.x;
    const int k = p.k, nc = p.nchunk, B = p.B;
    const int G = (int)gridDim.x;
    constexpr bool kVerify = (MODE & kModeVerify) != 0;
    constexpr bool kCommit = (MODE & kModeCommit) != 0;
    if (tid == 0) {
        sm.vb = -1;
        sm.expired = 0;
    }
    __syncthreads();

    // ---- the prefix lengths as they are before any commit ----
    if constexpr (kCommit) {
        for (int b = blockIdx.x; b < B; b += G) {
            if (tid == 0) {
                const int P = p.prefix_len[b];
                st_slot(p.pslot + b, P >= 0 ? P : kPrefixInvalid);
            }
        }
    }

    // ---- A: chunk statistics of the 2k rows of every sequence, and the draft logits ----
    if constexpr (kVerify) {
        constexpr int NP = DT == TIDAR_DT_BF16 ? 2 : 1;  // items in flight per CTA
        const int itemsA = B * 2 * k * nc;
        for (int it0 = blockIdx.x; it0 < itemsA; it0 += NP * G) {
            Raw<DT> tr[NP], qr[MIX ? NP : 1];
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
                imix[x] = MIX && row < k;
                load_raw<DT>(logit_row(row >= k ? p.q_logits : MIX ? p.p_logits : p.t_logits, p.dtype, srow, p.V),
                             p.V, c, tr[x]);
                if (MIX && imix[x]) load_raw<DT>(logit_row(p.q_logits, p.dtype, srow, p.V), p.V, c, qr[MIX ? x : 0]);
            }
            float mx[NP];
#pragma unroll
            for (int x = 0; x < NP; ++x) {
                mx[x] = -INFINITY;
                if (ib[x] < 0) continue;
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    mx[x] = fmaxf(mx[x], item_val<MIX>(tr[x], qr[MIX ? x : 0], imix[x], p.lambda, e));
                // the thread that holds entry d of this row publishes that logit for the ratio test
                const long long off = (long long)id[x] - (long long)ic[x] * kChunk;
                if (off >= 0 && off < kChunk && (((int)off & 2047) >> 3) == tid) {
                    const int ee = ((int)off >> 11) * 8 + ((int)off & 7);
                    float zd = 0.f;
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (e == ee) zd = item_val<MIX>(tr[x], qr[MIX ? x : 0], imix[x], p.lambda, e);
                    st_slot(p.dlogit + (size_t)ib[x] * 2 * k + irow[x], zd);
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
                    for (int e = 0; e < 32; ++e)
                        s += fast_exp2(fmaf(item_val<MIX>(tr[x], qr[MIX ? x : 0], imix[x], p.lambda, e), kLog2e, -ms));
                }
                sz[x] = (double)s;
            }
            block_sum_n<NP>(sz, sm.redd);
            if (tid == 0) {
#pragma unroll
                for (int x = 0; x < NP; ++x)
                    if (ib[x] >= 0) st_stat(p.vstats + ((size_t)ib[x] * 2 * k + irow[x]) * nc + ic[x], mx[x], sz[x]);
            }
        }
    }

    // ---- B: residual chunks, group chunks, copies ----
    const int n_res = kVerify ? B * nc : 0;
    const int n_grp = kCommit ? B * k * nc : 0;
    const int cp_per_seq = kCommit ? (p.L * p.Hkv + kWarps - 1) / kWarps : 0;
    const int nb = n_res + n_grp + B * cp_per_seq;
    for (int it = blockIdx.x; it < nb; it += G) {
        // the verdict: formed once per sequence, by its first residual item, and published; every other item
        // polls that 32-byte slot (a few hundred CTAs polling the statistics themselves would queue on the
        // handful of L2 lines that hold them).  The commit alone forms its own (no statistics to wait for).
        const int how = kVerify ? kVerdictLookup : kVerdictCompute;
        bool ok;
        if (it < n_res) {
            ok = residual_item<MODE, DT, MIX>(p, sm, it / nc, it % nc, how);
        } else if (it < n_res + n_grp) {
            const int t = it - n_res;
            ok = group_item<MODE, DT>(p, sm, t / (nc * k), (t / nc) % k, t % nc, how);
        } else {
            ok = true;
            if constexpr (kCommit) {
                const int t = it - n_res - n_grp;
                ok = copy_item<MODE>(p, sm, t / cp_per_seq, t % cp_per_seq, how);
            }
        }
        if (!ok) return;
    }
}

// ---------------------------------------------------------------------------------------------------------
// Workspace: the slots [vstats | dlogit | parts | gstats | pslot | vslot], 256-byte aligned regions, all filled with
// 0xff bytes (NaN / -1) before every launch.

struct Layout {
    size_t vstats, dlogit, parts, gstats, pslot, vslot, total;
};

Layout layout(int B, int k, int V, int mode) {
    const size_t nc = vocab_chunks(V);
    const bool v = (mode & kModeVerify) != 0, c = (mode & kModeCommit) != 0;
    Layout L;
    size_t o = 0;
    L.vstats = o;
    o += v ? align256(sizeof(double2) * B * 2 * k * nc) : 0;
    L.dlogit = o;
    o += v ? align256(sizeof(float) * B * 2 * k) : 0;
    L.parts = o;
    o += v ? align256(sizeof(double2) * B * nc) : 0;
    L.gstats = o;
    o += c ? align256(sizeof(double2) * B * k * nc) : 0;
    L.pslot = o;
    o += c ? align256(sizeof(int32_t) * B) : 0;
    L.vslot = o;
    o += v ? align256(sizeof(int4) * 2 * B) : 0;
    L.total = o;
    return L;
}

template <int MODE, int DT, bool MIX>
int resident_ctas() {
    static int n = -1;
    if (n >= 0) return n;
    int dev = 0, sms = 0, per = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, tail_kernel<MODE, DT, MIX>, kStatThreads, 0) !=
            cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    n = sms * per;
    return n;
}

template <int MODE, int DT, bool MIX>
cudaError_t launch_mode(TailParams &p, void *ws, cudaStream_t s) {
    const Layout L = layout(p.B, p.k, p.V, MODE);
    uint8_t *w = reinterpret_cast<uint8_t *>(ws);
    p.vstats = reinterpret_cast<double2 *>(w + L.vstats);
    p.dlogit = reinterpret_cast<float *>(w + L.dlogit);
    p.parts = reinterpret_cast<double2 *>(w + L.parts);
    p.gstats = reinterpret_cast<double2 *>(w + L.gstats);
    p.pslot = reinterpret_cast<int32_t *>(w + L.pslot);
    p.vslot = reinterpret_cast<int4 *>(w + L.vslot);
    const int cap = resident_ctas<MODE, DT, MIX>();
    if (cap <= 0) return cudaErrorLaunchFailure;
    // enough CTAs for phase A (two items per CTA) and for every block item at once, at most two per SM, and
    // never fewer than the largest group (nchunk <= 64): the condition of deadlock freedom
    const long nc = p.nchunk;
    long want = 64;
    if (MODE & kModeVerify) want = std::max(want, std::max(((long)p.B * 2 * p.k * nc + 1) / 2, (long)p.B * nc));
    if (MODE & kModeCommit)
        want = std::max(want, (long)p.B * p.k * nc + (long)p.B * ((p.L * p.Hkv + kWarps - 1) / kWarps) +
                                  ((MODE & kModeVerify) ? (long)p.B * nc : 0));
    const int grid = (int)std::min<long>(want, std::min(cap, 2 * kNumSMs));
    if (grid < nc) return cudaErrorLaunchFailure;
    cudaError_t e = cudaMemsetAsync(ws, 0xff, L.total, s);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kStatThreads, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident at once: every poll can complete
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, tail_kernel<MODE, DT, MIX>, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int MODE>
cudaError_t launch(TailParams &p, void *ws, cudaStream_t s) {
    // the target logits are mixed only strictly inside (0, 1); at the endpoints one stored row is the target
    p.t_logits = p.lambda == 0.f ? p.q_logits : p.p_logits;
    if constexpr ((MODE & kModeVerify) != 0) {
        if (p.lambda != 0.f && p.lambda != 1.f)
            return p.dtype == TIDAR_DT_BF16 ? launch_mode<MODE, TIDAR_DT_BF16, true>(p, ws, s)
                                            : launch_mode<MODE, TIDAR_DT_F32, true>(p, ws, s);
    }
    return p.dtype == TIDAR_DT_BF16 ? launch_mode<MODE, TIDAR_DT_BF16, false>(p, ws, s)
                                    : launch_mode<MODE, TIDAR_DT_F32, false>(p, ws, s);
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
