// TiDAR hybrid-mask attention for sm_100a: TMA + tcgen05 (TMEM accumulators).
//
// One CTA owns 128 packed query rows (row m = r*G + g of the G query heads
// sharing KV head kvh: GQA packing, so every K/V byte feeds 128 rows) and a
// contiguous run of 128-key tiles of one sequence.  A sequence's tiles are
// the cached prefix in 128-row tiles (the last one partial) followed by the
// R new keys of this step in 128-row tiles.
//
// Warp roles (12 warps):
//   warps 0, 2  TMA producers of K and of V (128-byte swizzle), each into its
//               own 3-stage ring: prefix tiles from the cache (one 128-row
//               box per 64 columns; with a paged cache one 64-row box per
//               page, two per tile), new-key tiles from K_new/V_new through a
//               3-D tensor map (no head gather).  A K stage is freed when its QK^T completes, a V
//               stage when its PV does, so K runs ahead of V.
//   warp 1      TMEM owner; one thread issues S = Q K^T (tcgen05.mma, both
//               operands in shared memory) into S buffer j % 3.
//   warp 3      one thread issues O += P V with P read from TMEM (A operand
//               in TMEM, V an MN-major operand in shared memory).
//   warps 4-11  softmax: both warpgroups work on every tile, warpgroup w on
//               its columns [64w, 64w+64); thread = query row = TMEM lane.
//               The two halves of a row always hold the same running max,
//               so their exponentials share a scale and PV sums them into
//               the one O.  A tile is exponentiated against that (possibly
//               stale) max -- exact as long as p <= 2^8 fits -- while its row
//               max is taken in the same pass; the halves then exchange
//               maxima through shared memory, and only rows whose max grew
//               by more than 2^8 redo their exponentials and rescale O.  The
//               mask is evaluated from indices.
//   warps 2-11  also load Q when its rows cannot come through TMA.
// TMEM (512 columns): S buffers at [0, 128), [128, 256), [256, 384); O at
// [384, 384+D).  P (bf16) overwrites columns [32, 96) of its S buffer: the P of
// warpgroup w's keys lands in [32 + 32w, 64 + 32w), inside the columns that
// warpgroup w itself read, so neither warpgroup can overwrite scores the other
// has yet to load.
// QK(j) reuses the buffer that PV(j-3) reads and is issued once PV(j-3) has
// completed, so the softmax always has the next two tiles' S ready.
// The S CTAs of a row tile take its key tiles round robin (split s: tiles s,
// s + S, ...), so that a split's first tile does not depend on the prefix.
// At the end each warpgroup reads its half of the columns of O and forms one
// partial row per query row: the half row over its largest magnitude, stored
// as fp16 (|error| <= 2^-12 of that magnitude), with an fp32 scale (that
// magnitude over the row sum) and the row's log2 LSE in fp32.  With one split
// the normalised row is the output.  Otherwise the CTAs that split one row
// tile's keys form a thread-block cluster: each CTA stages its records in its
// own (idle) K/V ring, in the layout of the block every owner receives, and
// sends each owner its block with one shared-to-shared bulk copy that counts
// the bytes on the owner's receive barrier (armed at set-up); every CTA merges
// its slice of rows over the S blocks (LSE weights, fixed order) as soon as
// they have all landed, and writes the final bf16 output and LSE.  One cluster
// barrier (every CTA's ring is idle) comes before the copies; a CTA exits once
// every other CTA has told it (a remote arrival on its "sent" barrier) that
// all its blocks have landed, so no copy still reads its shared memory.
//
// Before the previous kernel in the stream has finished (programmatic
// dependent launch), a CTA sets up its barriers, tensor maps and TMEM; every
// global read (prefix lengths, Q, K/V) waits for that kernel.  Then only the
// first QK's operands (Q and K of the first tile) are requested -- with a
// contiguous cache both at once, before the prefix length is known (the K
// copy is dropped if the prefix ends before that tile); the producers stream
// V and the later tiles once that K has landed, so it is not queued behind
// the start-up burst of every CTA (~20 MB at once).
//
// Every wait is bounded (p.wait_cycles).  On expiry the CTA raises
// TIDAR_DEV_TIMEOUT in dev_status and every role stops; then the producers
// wait for their copies in flight and the MMA issuers for their MMAs (bounded
// waits that ignore the abort), so nothing lands in shared memory or TMEM
// after the CTA frees it.  The softmax warps pass the per-tile named barrier
// on every tile even after an abort, so no warp waits there for one that left.
#include "attn.cuh"
#include "tc.cuh"

namespace tidar {

namespace {

constexpr int TM = 128;
constexpr int TN = 128;
constexpr int BOXR = 64;  // rows of one TMA box of a paged cache (one page): a tile is two boxes
constexpr int STAGES = 3;
constexpr int THREADS = 384;
// Cluster sizes (key splits per row tile): 2..8, and the non-portable 9, 10, 12 and 15 where the device grants
// them -- the larger sizes whose exchange blocks fit the region the portable ones need.
constexpr int kMaxSplits = 15;
__host__ __device__ constexpr bool split_count_ok(int S) {
    return (S >= 1 && S <= 8) || S == 9 || S == 10 || S == 12 || S == 15;
}
constexpr long long kDrainCycles = kAttnWaitCycles;  // bound of the waits that drain issued work
static_assert(BOXR == kPageRows, "a TMA box of the cache is one page");

// Split-KV exchange of an S-CTA cluster.  CTA s merges rows [s*per, (s+1)*per) of the row tile, per =
// ceil(128 / S).  Every CTA sends each owner one block with its partial records of the owner's rows:
//   vals [D/8][pv]  16-byte chunks (8 fp16 of one row, over its half row's largest magnitude), pv = per rounded
//                   up to an odd number, so that reading one chunk of consecutive rows and reading the consecutive
//                   chunks of one row both spread over all shared-memory banks
//   hdr  [per]      float4 (log2 LSE, scale of columns [0, D/2), scale of [D/2, D), unused); a half's scale is
//                   its largest magnitude over the row sum, so value x scale is the normalised partial output
// The owner receives the S blocks in source order.  Both the received blocks and the staged outgoing ones live
// in the CTA's K/V ring, which is idle by then: [row statistics | received | staged].
__host__ __device__ constexpr int xchg_per(int S) { return (TM + S - 1) / S; }
__host__ __device__ constexpr int xchg_vals_bytes(int S, int D) { return (D / 8) * (xchg_per(S) | 1) * 16; }
__host__ __device__ constexpr int xchg_block_bytes(int S, int D) { return xchg_vals_bytes(S, D) + xchg_per(S) * 16; }
constexpr int xchg_region_max(int D) {
    int m = 0;
    for (int S = 2; S <= kMaxSplits; ++S)
        if (split_count_ok(S)) m = S * xchg_block_bytes(S, D) > m ? S * xchg_block_bytes(S, D) : m;
    return (m + 127) / 128 * 128;
}
constexpr int kStatsBytes = 4 * TM * 4;  // row statistics exchanged between the warpgroups (start of the ring)

template <int D>
struct Smem {
    static constexpr int Q_BYTES = TM * D * 2;
    static constexpr int KV_TILE = TN * D * 2;  // one of K or V
    static constexpr int STAGE = 2 * KV_TILE;
    static constexpr int KV_OFF = Q_BYTES;
    static constexpr int RECV_OFF = KV_OFF + kStatsBytes;          // received blocks (inside the idle ring)
    static constexpr int STAGE_OFF = RECV_OFF + xchg_region_max(D);  // staged outgoing blocks (idem)
    static constexpr int BAR_OFF = KV_OFF + STAGES * STAGE;
    // k_full, k_empty, v_full, v_empty, s_full[3], p_full[3], pv_done[2], o_final, q_full, fin_qk, fin_pv, stall,
    // recv, sent, k_spec
    static constexpr int NBARS = 4 * STAGES + 16;
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
    static constexpr int XM_OFF = MISC_OFF + 16;  // row-max exchange between the warpgroups: [2][2][TM] bf16
    static constexpr int TOTAL = XM_OFF + 2 * 2 * TM * 2;
    static constexpr int ALLOC = TOTAL + 1024;  // alignment slack
};

static_assert(Smem<64>::ALLOC <= 227 * 1024 && Smem<128>::ALLOC <= 227 * 1024, "shared memory beyond 227 KB");
static_assert(Smem<64>::STAGE_OFF + xchg_region_max(64) <= Smem<64>::BAR_OFF &&
                  Smem<128>::STAGE_OFF + xchg_region_max(128) <= Smem<128>::BAR_OFF,
              "split-KV exchange larger than the K/V ring");
// the merge's per-row weights fit the row-statistics area: per rows x (S weights x 2 halves + 2)
constexpr bool weights_fit() {
    for (int S = 2; S <= kMaxSplits; ++S)
        if (split_count_ok(S) && xchg_per(S) * (2 * S + 2) * 4 > kStatsBytes) return false;
    return true;
}
static_assert(weights_fit(), "merge weights larger than the row-statistics area");

// Bit i set iff key base+i lies in [a, b) (i = 0..31).
__device__ __forceinline__ uint32_t range_bits(int a, int b, int base) {
    const int lo = max(a - base, 0), hi = min(b - base, 32);
    if (hi <= lo) return 0u;
    const uint32_t below_hi = hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u);
    return below_hi & ~((1u << lo) - 1u);
}

// S(tmem) = Q K^T: D/16 MMAs over the head dimension.  Q and K are K-major with 128-byte swizzle in
// blocks of 64 columns (TM or TN rows x 128 B); within a block a 16-column step is +32 B (+2 in the
// descriptor's address field).
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t d_s, uint64_t dq, uint64_t dk, uint32_t id) {
    constexpr uint64_t kQBlock = (TM * 128) >> 4, kKBlock = (TN * 128) >> 4;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = (kk & 3) * 2;
        tc::mma_ss(d_s, dq + (kk >> 2) * kQBlock + off, dk + (kk >> 2) * kKBlock + off, id, kk > 0 ? 1u : 0u);
    }
}

// First TMEM column of P inside its S buffer (P of 128 keys: 64 columns, two bf16 per column).
constexpr uint32_t kPCol = 32;

// O(tmem) (+)= P(tmem) V: TN/16 MMAs over the keys.  P occupies TN/2 columns of S from kPCol (two bf16 per
// column); V is MN-major, a 16-key step is 16 rows x 128 B (+128 in the descriptor's address field).
template <int D>
__device__ __forceinline__ void issue_pv(uint32_t d_o, uint32_t a_p, uint64_t dv, uint32_t id, bool acc) {
#pragma unroll
    for (int kk = 0; kk < TN / 16; ++kk) tc::mma_ts(d_o, a_p + kk * 8, dv + kk * 128, id, (acc || kk > 0) ? 1u : 0u);
}

// Loads this thread's 64 raw scores (TMEM columns col .. col+63 of its lane) into x.  MASKED: only keys
// kbase + j in [0, lo) and [glo, ghi) are kept; the others (garbage past the sequence included) become -inf.
template <bool MASKED>
__device__ __forceinline__ void half_load(uint32_t col, int kbase, int lo, int glo, int ghi, float (&x)[64]) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        tc::tmem_ld32(col + c * 32, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) x[c * 32 + j] = __uint_as_float(v[j]);
    }
    tc::tmem_wait_ld();
    if constexpr (MASKED) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int base = kbase + c * 32;
            const uint32_t bits = range_bits(0, lo, base) | range_bits(glo, ghi, base);
#pragma unroll
            for (int j = 0; j < 32; ++j) x[c * 32 + j] = (bits >> j) & 1u ? x[c * 32 + j] : -INFINITY;
        }
    }
}

__device__ __forceinline__ float half_max(const float (&x)[64]) {
    float m8[8];  // eight independent chains
#pragma unroll
    for (int j = 0; j < 8; ++j) m8[j] = x[j];
#pragma unroll
    for (int j = 8; j < 64; ++j) m8[j & 7] = fmaxf(m8[j & 7], x[j]);
    return fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
}

// p = 2^(x * sl2 + neg_m) for the 64 scores in x (-inf gives exactly 0), written as 32 bf16 pairs to TMEM
// columns pcol .. pcol+31 (P, the A operand of PV).  Returns the sum of the 64 values of p; *mx receives the
// maximum of x, computed in the same pass (its ALU work hides under the exponentials).
__device__ __forceinline__ float half_exp(uint32_t pcol, const float (&x)[64], float sl2, float neg_m, float *mx) {
    float sum8[8], m8[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        sum8[j] = 0.f;
        m8[j] = -INFINITY;
    }
    uint32_t pk[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float a = fast_exp2(fmaf(x[2 * j], sl2, neg_m));
        const float bb = fast_exp2(fmaf(x[2 * j + 1], sl2, neg_m));
        m8[(2 * j) & 7] = fmaxf(m8[(2 * j) & 7], x[2 * j]);
        m8[(2 * j + 1) & 7] = fmaxf(m8[(2 * j + 1) & 7], x[2 * j + 1]);
        sum8[(2 * j) & 7] += a;
        sum8[(2 * j + 1) & 7] += bb;
        pk[j] = pack_bf16x2(a, bb);
    }
    tc::tmem_st32(pcol, pk);
    *mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
    return ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
}

// Merge of this CTA's rows over the S blocks received (all THREADS threads).  First the weights of every row:
// w_s = exp2(lse_s - max) / sum * scale_s per column half (in the row-statistics area, free by then); then items
// (row, one 16-byte column chunk of each half), consecutive threads on consecutive chunks of one row, so that
// every warp writes whole output rows in one round.  Sources are summed in a fixed order.
template <int D, int S>
__device__ __forceinline__ void merge_rows(const AttnParams &p, const uint8_t *recv, float *wts, int split, int mt,
                                           int b, int kvh, int tid) {
    constexpr int per = xchg_per(S), pv = per | 1, CH = D / 8, VB = xchg_vals_bytes(S, D), BB = xchg_block_bytes(S, D);
    const int row0 = split * per, nrows = max(0, min(TM, row0 + per) - row0);
    for (int rl = tid; rl < nrows; rl += THREADS) {
        float4 hd[S];
        float mx = -INFINITY;
#pragma unroll
        for (int sp = 0; sp < S; ++sp) {
            hd[sp] = reinterpret_cast<const float4 *>(recv + sp * BB + VB)[rl];
            mx = fmaxf(mx, hd[sp].x);
        }
        float wq[S], wsum = 0.f;
#pragma unroll
        for (int sp = 0; sp < S; ++sp) {
            wq[sp] = hd[sp].x == -INFINITY ? 0.f : fast_exp2(hd[sp].x - mx);
            wsum += wq[sp];
        }
        const float winv = wsum > 0.f ? __fdividef(1.f, wsum) : 0.f;
        float *w = wts + rl * (2 * S + 2);
#pragma unroll
        for (int sp = 0; sp < S; ++sp) {
            w[2 * sp] = wq[sp] * winv * hd[sp].y;
            w[2 * sp + 1] = wq[sp] * winv * hd[sp].z;
        }
        w[2 * S] = wsum > 0.f ? (mx + __log2f(wsum)) * kLn2 : -INFINITY;  // natural-log LSE
    }
    __syncthreads();
    // items (row, chunk c of the first column half and chunk c + CH/2 of the second): one round for every row
    constexpr int HC = CH / 2;
    for (int it = tid; it < nrows * HC; it += THREADS) {
        const int rl = it / HC, c = it - rl * HC;
        const float *w = wts + rl * (2 * S + 2);
        float acc[2][8];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[h][e] = 0.f;
#pragma unroll
        for (int sp = 0; sp < S; ++sp) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4 raw = reinterpret_cast<const uint4 *>(recv + sp * BB)[(c + h * HC) * pv + rl];
                const float f = w[2 * sp + h];
                const uint32_t u[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 v = unpack_half2(u[e]);
                    acc[h][2 * e] = fmaf(f, v.x, acc[h][2 * e]);
                    acc[h][2 * e + 1] = fmaf(f, v.y, acc[h][2 * e + 1]);
                }
            }
        }
        const int m = mt * TM + row0 + rl;
        if (m < p.M) {
            const int rq = m / p.G;
            const size_t orow = (size_t)(b * p.R + rq) * p.Hq + kvh * p.G + (m - rq * p.G);
#pragma unroll
            for (int h = 0; h < 2; ++h)
                *reinterpret_cast<uint4 *>(p.out + orow * D + (c + h * HC) * 8) =
                    make_uint4(pack_bf16x2(acc[h][0], acc[h][1]), pack_bf16x2(acc[h][2], acc[h][3]),
                               pack_bf16x2(acc[h][4], acc[h][5]), pack_bf16x2(acc[h][6], acc[h][7]));
            if (c == 0 && p.lse) p.lse[orow] = w[2 * S];
        }
    }
}

// Number of valid keys in tile t (t < TP: prefix tile, else new-key tile).
__device__ __forceinline__ int tile_valid(int t, int TP, int P, int R) {
    return t < TP ? min(TN, P - t * TN) : min(TN, R - (t - TP) * TN);
}

// Key tiles of split `split` out of n_splits for a sequence with prefix length P (TP prefix tiles, then the
// new-key tiles): tiles split, split + n_splits, split + 2 n_splits, ... -- n of them.  Round robin, so that a
// split's first tile does not depend on P.
__device__ __forceinline__ void split_tiles(int P, int R, int split, int n_splits, int &TP, int &n) {
    TP = ceil_div(P, TN);
    const int T = TP + ceil_div(R, TN);
    n = split < T ? (T - split + n_splits - 1) / n_splits : 0;
}

// kLarge: the instantiation for the non-portable cluster sizes (more than 8 splits); the other one has only the
// common sizes' merge, so the large sizes cost it no code.
template <int D, bool kLarge>
__global__ void __launch_bounds__(THREADS, 1)
    attn_sm100_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tm_kc,
                      const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_kn,
                      const __grid_constant__ CUtensorMap tm_vn, const __grid_constant__ CUtensorMap tm_q, int q_tma) {
    using L = Smem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase;
    const uint32_t sKV = sbase + L::KV_OFF;
    const uint32_t bar0 = sbase + L::BAR_OFF;
    auto k_full = [&](int s) { return bar0 + 8u * s; };
    auto k_empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto v_full = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
    auto v_empty = [&](int s) { return bar0 + 8u * (3 * STAGES + s); };
    auto s_full = [&](int sb) { return bar0 + 8u * (4 * STAGES + sb); };      // S buffer sb holds a new S
    auto p_full = [&](int sb) { return bar0 + 8u * (4 * STAGES + 3 + sb); };  // P in S buffer sb is complete
    // pv_done(e): its k-th phase completes with PV(2k + e).  Waiting for PV(i) on pv_done(i & 1) is unambiguous
    // once PV(i-2) has completed, which holds wherever it is waited for (see there).
    auto pv_done = [&](int e) { return bar0 + 8u * (4 * STAGES + 6 + e); };
    const uint32_t o_final = bar0 + 8u * (4 * STAGES + 8);  // one phase: the last PV has completed
    const uint32_t q_full = bar0 + 8u * (4 * STAGES + 9);
    const uint32_t fin_qk = bar0 + 8u * (4 * STAGES + 10);  // the QK issuer's MMAs have all completed
    const uint32_t fin_pv = bar0 + 8u * (4 * STAGES + 11);  // the PV issuer's MMAs have all completed
    const uint32_t stall = bar0 + 8u * (4 * STAGES + 12);   // nothing arrives here (timeout test)
    const uint32_t recv = bar0 + 8u * (4 * STAGES + 13);    // every CTA's block of this CTA's rows has landed
    const uint32_t sent = bar0 + 8u * (4 * STAGES + 14);    // every other CTA has received this CTA's block
    const uint32_t k_spec = bar0 + 8u * (4 * STAGES + 15);  // the early copy of cache tile `split` (below)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::MISC_OFF);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::MISC_OFF + 4);

    const int split = blockIdx.x, mt = blockIdx.y, bh = blockIdx.z;
    const int kvh = bh % p.Hkv;
    int b = bh / p.Hkv;  // (several sequences without splits: reassigned below, longest first)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long wl = p.wait_cycles;
    const int S = p.n_splits;  // cluster size; this CTA's rank is `split`
    // ---- set-up that needs nothing from the previous kernel (programmatic dependent launch) ----
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(k_full(s), 1);
            tc::mbar_init(k_empty(s), 1);
            tc::mbar_init(v_full(s), 1);
            tc::mbar_init(v_empty(s), 1);
        }
        for (int sb = 0; sb < 3; ++sb) {
            tc::mbar_init(s_full(sb), 1);
            tc::mbar_init(p_full(sb), 256);  // both softmax warpgroups
        }
        tc::mbar_init(pv_done(0), 1);
        tc::mbar_init(pv_done(1), 1);
        tc::mbar_init(o_final, 1);
        tc::mbar_init(q_full, q_tma ? 1 : THREADS - 64);
        tc::mbar_init(fin_qk, 1);
        tc::mbar_init(fin_pv, 1);
        tc::mbar_init(stall, 1);
        tc::mbar_init(recv, 1);
        tc::mbar_init(sent, S > 1 ? S - 1 : 1);
        tc::mbar_init(k_spec, 1);
        *abort_flag = 0;
        tc::mbar_fence_init();
        // armed now with the bytes it is to receive (one block from every CTA of the cluster, itself included):
        // its phase completes when the last block lands
        if (S > 1) tc::mbar_arrive_expect_tx(recv, S * xchg_block_bytes(S, D));
        tc::tma_prefetch_desc(&tm_kc);
        tc::tma_prefetch_desc(&tm_vc);
        tc::tma_prefetch_desc(&tm_kn);
        tc::tma_prefetch_desc(&tm_vn);
        // An L2 prefetch of this tile's Q rows, ahead of the wait: L2 is the point of coherence, so the copy
        // after the wait still sees whatever the previous kernel writes there; the prefetch only starts the HBM
        // read early.  (Several sequences without splits choose their sequence after the wait: no prefetch.)
        if (q_tma && !(p.B > 1 && S == 1)) {
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
                tc::tma_prefetch_l2_3d(&tm_q, h * 64, kvh * p.G, b * p.R + mt * (TM / p.G));
        }
    }
    if (warp == 1) tc::tmem_alloc(smem_u32(tmem_slot), 512);
    // every global read below (prefix lengths, Q, K/V) waits for the previous kernel
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    if (p.B > 1 && S == 1) {
        // Several sequences and more row tiles than one wave holds: CTAs are dispatched in grid order, so the
        // r-th group of KV heads takes the sequence with the r-th longest prefix (ties by index).  The first
        // wave runs the longest, and the shortest fill the SMs that free up first.
        int *seq_slot = reinterpret_cast<int *>(smem + L::MISC_OFF + 8);
        const int rank_want = bh / p.Hkv;
        for (int cand = tid; cand < p.B; cand += THREADS) {
            const int pc = p.prefix_len[cand];
            int rank = 0;
            for (int o = 0; o < p.B; ++o) {
                const int po = p.prefix_len[o];
                rank += (po > pc) || (po == pc && o < cand);
            }
            if (rank == rank_want) *seq_slot = cand;
        }
        __syncthreads();
        b = *seq_slot;
    }
    if (tid == 0) {
        // Q does not depend on the prefix length: its copy starts at once
        if (q_tma) {  // rows (r, g) of the tile: box {64 d, G heads, 128/G rows}
            tc::mbar_arrive_expect_tx(q_full, L::Q_BYTES);
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
                tc::tma_load_3d(sQ + h * TM * 128, &tm_q, h * 64, kvh * p.G, b * p.R + mt * (TM / p.G), q_full);
        }
    }
    // With a contiguous cache the first tile of this split, cache tile `split`, does not depend on the prefix
    // length either: its copy starts now too, into the K slot of the ring's last stage, counted on k_spec.  If the
    // prefix reaches that tile it is kept, and tile i of the split goes to stage (i + STAGES - 1) % STAGES;
    // otherwise tile i goes to stage i % STAGES, and the last stage is reused only once the copy has landed.
    // (Rows past the cache read as zeros.)
    const bool spec = !p.block_table;
    if (tid == 0 && spec) {
        tc::mbar_arrive_expect_tx(k_spec, L::KV_TILE);
        const int y = (b * p.Hkv + kvh) * p.P_max + split * TN;
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
            tc::tma_load_2d(sKV + (STAGES - 1) * L::STAGE + h * TN * 128, &tm_kc, h * 64, y, k_spec);
    }
    const int P = p.prefix_len[b];
    int TP = 0, n = 0;
    const bool bad_prefix = P < 0 || P > p.P_max;
    if (!bad_prefix) split_tiles(P, p.R, split, S, TP, n);
    const bool spec_ok = spec && n > 0 && split < TP;  // the early copy is this split's first tile
    const int so = spec_ok ? STAGES - 1 : 0;             // tile i of the split uses ring stage (i + so) % STAGES
    bool bad_page = false;
    if (p.block_table && !bad_prefix) {  // (uniform over the CTA: one sequence)
        // every CTA of the cluster checks every page of the sequence, so that they all take the same exit (the
        // early one below passes no cluster barrier)
        int bad = 0;
        const int np = ceil_div(P, BOXR);  // pages holding rows [0, P)
        const int32_t *row_pages = p.block_table + (size_t)b * p.max_pages;
        for (int pi = tid; pi < np; pi += THREADS) {
            const int pg = row_pages[pi];
            bad |= pg < 0 || pg >= p.num_pages;
        }
        bad_page = __syncthreads_or(bad) != 0;
    }
    if (bad_prefix || bad_page) {
        if (tid == 0 && split == 0 && mt == 0)
            atomicOr(p.dev_status, bad_prefix ? TIDAR_DEV_BAD_PREFIX : TIDAR_DEV_BAD_PAGE);
        if (tid == 0 && q_tma) tc::mbar_wait_drain(q_full, 0, kDrainCycles);  // no copy may land after exit
        if (tid == 0 && spec) tc::mbar_wait_drain(k_spec, 0, kDrainCycles);
        tc::fence_before_sync();
        __syncthreads();
        if (warp == 1) {
            tc::fence_after_sync();
            tc::tmem_dealloc(*tmem_slot, 512);
        }
        return;
    }
    // cache row of box h2 (0, 1: the two 64-row halves) of cache tile t: contiguous, or through the block table
    // (read as the copy is issued; the table is not written during the launch).  The second box of a last tile
    // that ends within its first page has no page of its own: it re-reads the first page (rows past P are
    // excluded from the scores and their V rows zeroed).
    auto cache_row = [&](int t, int h2) {
        if (!p.block_table) return (b * p.Hkv + kvh) * p.P_max + t * TN + h2 * BOXR;
        const int pi = 2 * t + h2;
        const int pg = __ldcg(p.block_table + (size_t)b * p.max_pages + (pi < ceil_div(P, BOXR) ? pi : pi - 1));
        return (pg * p.Hkv + kvh) * BOXR;
    };

    // K (is_v = 0) or V (is_v = 1) of tile i into stage (i + so) % STAGES of its ring
    auto issue_tile = [&](int i, int is_v) {
        const int st = (i + so) % STAGES;
        const uint32_t bar = is_v ? v_full(st) : k_full(st);
        tc::mbar_arrive_expect_tx(bar, L::KV_TILE);
        const int t = split + i * S;
        const uint32_t dst = sKV + st * L::STAGE + is_v * L::KV_TILE;
        if (t < TP && p.block_table) {  // two 64-row boxes, one per page
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int y = cache_row(t, h2);
#pragma unroll
                for (int h = 0; h < D / 64; ++h)
                    tc::tma_load_2d(dst + h * TN * 128 + h2 * BOXR * 128, is_v ? &tm_vc : &tm_kc, h * 64, y, bar);
            }
        } else if (t < TP) {  // one 128-row box per column block
            const int y = (b * p.Hkv + kvh) * p.P_max + t * TN;
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
                tc::tma_load_2d(dst + h * TN * 128, is_v ? &tm_vc : &tm_kc, h * 64, y, bar);
        } else {
            const int z = b * p.R + (t - TP) * TN;
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
                tc::tma_load_3d(dst + h * TN * 128, is_v ? &tm_vn : &tm_kn, h * 64, kvh, z, bar);
        }
    };

    // ---- the first K tile's copy (paged cache: starts now); the producers stream the rest once it has landed ----
    if (tid == 0 && n > 0 && !spec_ok) issue_tile(0, 0);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    if (!q_tma && warp >= 2) {  // Q tile, K-major with 128-byte swizzle: D/64 blocks of [128 rows][128 B]
        constexpr int CH = D / 8;
        for (int idx = tid - 64; idx < TM * CH; idx += THREADS - 64) {
            const int i = idx / CH, c = idx % CH;
            const int m = mt * TM + i;
            const bf16 *src = p.q;
            int bytes = 0;
            if (m < p.M) {
                const int r = m / p.G, g = m - r * p.G;
                src = p.q + ((size_t)(b * p.R + r) * p.Hq + kvh * p.G + g) * D + c * 8;
                bytes = 16;
            }
            const uint32_t dst = sQ + (c >> 3) * TM * 128 + i * 128 + (((c & 7) ^ (i & 7)) << 4);
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
        }
        asm volatile("cp.async.wait_all;\n" ::: "memory");
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(q_full);
    }

    if (warp < 4) {
        if (warp == 0 || warp == 2) {
            // ================= TMA producers: warp 0 streams K, warp 2 streams V =================
            const int is_v = warp == 2;
            if (lane == 0) {
                // the first QK's operands (Q, K of tile 0) are served ahead of the rest of every CTA's burst
                const int first = is_v ? 0 : min(n, 1);
                int issued = first;
                // (kept early copy: it completes the last stage's first K phase; the QK of tile 0 waits on k_spec)
                if (!is_v && spec_ok) tc::mbar_arrive(k_full(so));
                const bool k0_in = n == 0 || tc::mbar_wait(spec_ok ? k_spec : k_full(0), 0, abort_flag, wl);
                for (int i = first; i < n && k0_in; ++i) {
                    const int u = i / STAGES;
                    const int st = (i + so) % STAGES;
                    if (!tc::mbar_wait(is_v ? v_empty(st) : k_empty(st), (u - 1) & 1, abort_flag, wl)) break;
                    // (a dropped early copy: the last stage's K slot is rewritten once it has landed)
                    if (!is_v && spec && !spec_ok && st == STAGES - 1 && u == 0)
                        tc::mbar_wait_drain(k_spec, 0, kDrainCycles);
                    issue_tile(i, is_v);
                    issued = i + 1;
                }
                // drain, whatever happened: only the last copy of each stage can still be in flight (an earlier
                // one completed before its stage was re-armed), and none may land after the CTA exits
                for (int i = max(0, issued - STAGES); i < issued; ++i)
                    tc::mbar_wait_drain(is_v ? v_full((i + so) % STAGES) : k_full((i + so) % STAGES), (i / STAGES) & 1,
                                        kDrainCycles);
                if (!is_v && q_tma) tc::mbar_wait_drain(q_full, 0, kDrainCycles);
                if (!is_v && spec) tc::mbar_wait_drain(k_spec, 0, kDrainCycles);
            }
            __syncwarp();
        } else {
            // ================= MMA issue: QK^T on warp 1, PV on warp 3 (one thread each) =================
            // S of tile j goes to S buffer j % 3.  QK(j), j >= 3, reuses the buffer whose P PV(j-3) reads, so it
            // is issued once PV(j-3) has completed; the softmax still has S(j-2) and S(j-1) to work on.
            constexpr uint64_t kStage = L::STAGE >> 4;  // one ring stage in the descriptor's address field
            const uint32_t tb = tbase;
            if (lane == 0 && warp == 1) {
                constexpr uint32_t id_qk = tc::idesc_bf16_f32(TM, TN, 0, 0);
                // descriptors are built once; a k-step or stage moves the start address, which lives in the
                // low 14 bits (address >> 4; shared memory is < 256 KB, so the add never carries out)
                const uint64_t dq = tc::smem_desc_sw128(sQ, 16, 1024);
                const uint64_t dk = tc::smem_desc_sw128(sKV, 16, 1024);
                bool ok = !p.stall_test || tc::mbar_wait(stall, 0, abort_flag, wl);
                ok = ok && tc::mbar_wait(q_full, 0, abort_flag, wl);
                for (int j = 0; j < n && ok; ++j) {
                    const int sb = j % 3, kst = (j + so) % STAGES;
                    const uint32_t kph = (j / STAGES) & 1;
                    if (j >= 3) {  // PV(j-3) done reading P from buffer sb (PV(j-5) was waited for before)
                        ok = tc::mbar_wait(pv_done((j - 3) & 1), ((j - 3) >> 1) & 1, abort_flag, wl);
                        if (!ok) break;
                    }
                    ok = tc::mbar_wait(j == 0 && spec_ok ? k_spec : k_full(kst), kph, abort_flag, wl);
                    if (!ok) break;
                    tc::fence_after_sync();
                    issue_qk<D>(tb + sb * 128, dq, dk + kst * kStage, id_qk);
                    tc::mma_commit(s_full(sb));
                    tc::mma_commit(k_empty(kst));
                }
                tc::mma_commit(fin_qk);  // every MMA of this thread completes before TMEM is freed
                tc::mbar_wait_drain(fin_qk, 0, kDrainCycles);
            } else if (lane == 0 && warp == 3) {
                constexpr uint32_t id_pv = tc::idesc_bf16_f32(TM, D, 0, 1);
                const uint64_t dv = tc::smem_desc_sw128(sKV + L::KV_TILE, TN * 128, 1024);
                bool ok = true;
                for (int i = 0; i < n && ok; ++i) {
                    const int sb = i % 3, vst = (i + so) % STAGES;
                    const uint32_t vph = (i / STAGES) & 1;
                    ok = tc::mbar_wait(v_full(vst), vph, abort_flag, wl) &&
                         tc::mbar_wait(p_full(sb), (i / 3) & 1, abort_flag, wl);
                    if (!ok) break;
                    tc::fence_after_sync();
                    issue_pv<D>(tb + 384, tb + sb * 128 + kPCol, dv + vst * kStage, id_pv, i > 0);
                    tc::mma_commit(v_empty(vst));
                    tc::mma_commit(pv_done(i & 1));
                    if (i == n - 1) tc::mma_commit(o_final);
                }
                tc::mma_commit(fin_pv);
                tc::mbar_wait_drain(fin_pv, 0, kDrainCycles);
            }
        }
        __syncwarp();
        // these warps are done with the ring (copies drained, MMAs complete): first phase of the cluster barrier
        tc::cluster_arrive_relaxed();
        tc::cluster_wait();
    } else {
        // ================= softmax: both warpgroups on every tile =================
        // Warpgroup w takes columns [64w, 64w+64) of each S tile (thread = query row = TMEM lane).  The two
        // halves of a row agree on one running max through a small exchange in shared memory, so both scale
        // their exponentials alike and PV sums them into the one O accumulator.
        const int w = (warp - 4) >> 2;
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const int m_row = mt * TM + row;
        const int r = m_row / p.G;
        const int wt = tid - 128;  // 0..255
        // visible new keys of row r: [0, vis_lim) and [vis_glo, vis_ghi) (same rule as new_key_visible)
        int vis_lim, vis_glo = 0, vis_ghi = 0;
        if (p.mask_mode == TIDAR_MASK_CAUSAL || r < p.k) {
            vis_lim = r + 1;
        } else {
            const int grp = (r - p.k) / p.k;
            vis_lim = grp;
            vis_glo = p.k + grp * p.k;
            vis_ghi = vis_glo + p.k;
        }
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const uint32_t o_col = tbase + lane_off + 384 + w * (D / 2);  // this warpgroup's half of O
        __nv_bfloat16 *xm = reinterpret_cast<__nv_bfloat16 *>(smem + L::XM_OFF);  // [2 tiles][2 wg][TM]
        const float sl2 = p.scale_log2;  // > 0, so the max of raw scores gives the max of scaled ones
        float m_run = -INFINITY, l_run = 0.f;  // running max (scaled log2 units, shared by both halves), own sum
        bool ok = true;
        for (int i = 0; i < n; ++i) {
            const int sb = i % 3;
            bool have = ok && tc::mbar_wait(s_full(sb), (i / 3) & 1, abort_flag, wl);
            ok = __all_sync(0xffffffffu, have);  // TMEM accesses are warp-collective: decide per warp
            const uint32_t s_col = tbase + lane_off + sb * 128;
            const int t = split + i * S;
            // a partial prefix tile (keys beyond P) or a new-key tile (the TiDAR mask): the visible keys of
            // this row are [0, lo) and [glo, ghi); everything else, garbage included, is excluded by select
            const bool masked = t >= TP - 1 && !(t == TP - 1 && P % TN == 0);
            int lo = TN, glo = 0, ghi = 0;
            if (masked) {
                int end;
                if (t < TP) {
                    lo = end = P - t * TN;
                } else {
                    const int nn0 = (t - TP) * TN;
                    lo = vis_lim - nn0;
                    glo = vis_glo - nn0;
                    ghi = vis_ghi - nn0;
                    end = p.R - nn0;
                }
                lo = min(lo, end);
                ghi = min(ghi, end);
            }
            float x[64];
            // P of keys [64w, 64w+64) over S columns [32 + 32w, 64 + 32w): inside this warpgroup's own scores
            const uint32_t pcol = s_col + kPCol + w * 32;
            const bool fresh = m_run == -INFINITY;  // no visible key so far: no max to reuse
            float hmx = -INFINITY, lt = 0.f;
            if (ok) {
                tc::fence_after_sync();
                if (masked)
                    half_load<true>(s_col + w * 64, w * 64, lo, glo, ghi, x);
                else
                    half_load<false>(s_col + w * 64, w * 64, lo, glo, ghi, x);
                // Exponentials against the running max the two halves already share (stale by design: exact as
                // long as p <= 2^8); the tile's row max comes out of the same pass.  Only a row whose max grew by
                // more than 2^8 -- all rows on the first tile, rarely later -- redoes them with the new max.
                lt = fresh ? 0.f : half_exp(pcol, x, sl2, -m_run, &hmx);
                if (fresh) hmx = half_max(x);
            }
            // both halves' maxima (rounded to bf16 for the exchange: any value the two sides agree on and that
            // is within 2^8 of the true maximum serves); every warp passes this barrier on every tile
            const __nv_bfloat16 hb = __float2bfloat16_rn(hmx);
            xm[((i & 1) * 2 + w) * TM + row] = hb;
            // only the two warps that hold the two halves of these 32 rows (warps 4 + q4 and 8 + q4) meet here
            asm volatile("bar.sync %0, 64;\n" ::"r"(2 + q4) : "memory");
            const __nv_bfloat16 ob = xm[((i & 1) * 2 + (1 - w)) * TM + row];
            if (ok) {
                const float mx = fmaxf(__bfloat162float(hb), __bfloat162float(ob)) * sl2;
                const float m_new = fmaxf(m_run, mx);
                const bool grow = m_new > m_run + 8.f;
                if (__any_sync(0xffffffffu, grow || fresh)) {  // fresh rows have written no P yet
                    if (i >= 1 && __any_sync(0xffffffffu, grow)) {
                        // rescale this half of O once PV(i-1), the last to write it, has completed.  S(i) is
                        // complete, and QK(i) was issued after PV(i-3) completed: the wait below is unambiguous.
                        const bool got =
                            tc::mbar_wait(pv_done((i - 1) & 1), ((i - 1) >> 1) & 1, abort_flag, wl);
                        ok = __all_sync(0xffffffffu, got);
                        if (ok) {
                            tc::fence_after_sync();
                            const float f = grow ? fast_exp2(m_run - m_new) : 1.f;
#pragma unroll 1
                            for (int c = 0; c < D / 64; ++c) {
                                uint32_t v[32];
                                tc::tmem_ld32(o_col + c * 32, v);
                                tc::tmem_wait_ld();
#pragma unroll
                                for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * f);
                                tc::tmem_st32(o_col + c * 32, v);
                            }
                        }
                    }
                    if (ok) {
                        if (grow) {
                            l_run *= fast_exp2(m_run - m_new);
                            m_run = m_new;
                        }
                        tc::tmem_wait_st();  // the redone P overwrites the first pass's
                        float unused;
                        lt = half_exp(pcol, x, sl2, m_run == -INFINITY ? 0.f : -m_run, &unused);
                    }
                }
                l_run += lt;
            }
            const int valid = tile_valid(t, TP, P, p.R);
            if (ok && valid < TN) {
                // keys past the sequence: zero their V rows (0 * garbage could be NaN) before PV reads them
                const int st = (i + so) % STAGES;
                const bool got = tc::mbar_wait(v_full(st), (i / STAGES) & 1, abort_flag, wl);
                ok = __all_sync(0xffffffffu, got);
                if (ok) {
                    uint8_t *vrow = smem + L::KV_OFF + st * L::STAGE + L::KV_TILE;
                    for (int idx = wt; idx < (TN - valid) * (D / 8); idx += 256) {
                        const int j = valid + idx / (D / 8), c = idx % (D / 8);
                        *reinterpret_cast<uint4 *>(vrow + (c >> 3) * TN * 128 + j * 128 + ((c & 7) << 4)) =
                            make_uint4(0, 0, 0, 0);
                    }
                    tc::fence_proxy_async_smem();
                }
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
            if (ok) tc::mbar_arrive(p_full(sb));
        }
        tc::tmem_wait_st();  // (abort path) no TMEM store left in flight
        // the next kernel in the stream may launch now: it waits for this grid before touching memory
        asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
        constexpr int H = D / 2;
        bool fin = ok && n > 0 && tc::mbar_wait(o_final, 0, abort_flag, wl);  // O final
        fin = __all_sync(0xffffffffu, fin);
        tc::fence_after_sync();
        // this CTA's ring is idle (every PV has read its V): first phase of the cluster barrier
        tc::cluster_arrive_relaxed();
        // this half row of O (its copy from TMEM overlaps the row-sum exchange below)
        uint32_t va[H / 32][32];
#pragma unroll
        for (int c = 0; c < H / 32; ++c) {
#pragma unroll
            for (int j = 0; j < 32; ++j) va[c][j] = 0u;
            if (fin) tc::tmem_ld32(o_col + c * 32, va[c]);
        }
        // the row sum is split over the two halves
        float *xl = reinterpret_cast<float *>(smem + L::KV_OFF);  // [2][TM] in the row-statistics area
        xl[w * TM + row] = l_run;
        asm volatile("bar.sync 1, 256;\n" ::: "memory");
        const float ltot = l_run + xl[(1 - w) * TM + row];
        const float inv = ltot > 0.f ? __fdividef(1.f, ltot) : 0.f;
        const float lse2 = ltot > 0.f ? m_run + __log2f(ltot) : -INFINITY;  // log2 of this CTA's row sum
        tc::tmem_wait_ld();
        tc::fence_before_sync();  // (TMEM is freed after a later barrier)
        if (S == 1) {  // the CTA saw every key of its rows: the normalised half row is the output
            if (m_row < p.M) {
                float hv[H];
#pragma unroll
                for (int c = 0; c < H / 32; ++c)
#pragma unroll
                    for (int j = 0; j < 32; ++j) hv[c * 32 + j] = __uint_as_float(va[c][j]) * inv;
                const size_t orow = (size_t)(b * p.R + r) * p.Hq + kvh * p.G + (m_row - r * p.G);
                uint4 *dst = reinterpret_cast<uint4 *>(p.out + orow * D + w * H);
#pragma unroll
                for (int j = 0; j < H / 8; ++j)
                    dst[j] = make_uint4(pack_bf16x2(hv[8 * j], hv[8 * j + 1]),
                                        pack_bf16x2(hv[8 * j + 2], hv[8 * j + 3]),
                                        pack_bf16x2(hv[8 * j + 4], hv[8 * j + 5]),
                                        pack_bf16x2(hv[8 * j + 6], hv[8 * j + 7]));
                if (w == 0 && p.lse) p.lse[orow] = lse2 * kLn2;
            }
            tc::cluster_wait();  // (first phase)
        } else {
            // this row's record, staged in this CTA's (idle) ring in the layout of the block its owner receives:
            // the unnormalised half row over its largest magnitude (so in [-1, 1]), and that magnitude / the row sum
            float am[4] = {0.f, 0.f, 0.f, 0.f};  // four independent chains
#pragma unroll
            for (int j = 0; j < H; ++j) am[j & 3] = fmaxf(am[j & 3], fabsf(__uint_as_float(va[j >> 5][j & 31])));
            const float amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
            const float rs = amax > 0.f ? __fdividef(1.f, amax) : 0.f;
            const float scale = amax * inv;  // the stored value times this is the normalised one
            const int per = xchg_per(S), pv = per | 1;
            const int VB = xchg_vals_bytes(S, D), BB = xchg_block_bytes(S, D);
            const int owner = row / per, rl = row - owner * per;
            uint8_t *stage = smem + L::STAGE_OFF;  // [owner][vals | hdr]
            uint4 *vals = reinterpret_cast<uint4 *>(stage + owner * BB);
#pragma unroll
            for (int j = 0; j < H / 8; ++j) {
                float o8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) o8[e] = __uint_as_float(va[(8 * j + e) >> 5][(8 * j + e) & 31]) * rs;
                vals[(w * (H / 8) + j) * pv + rl] = make_uint4(pack_half2(o8[0], o8[1]), pack_half2(o8[2], o8[3]),
                                                               pack_half2(o8[4], o8[5]), pack_half2(o8[6], o8[7]));
            }
            float *hdr = reinterpret_cast<float *>(stage + owner * BB + VB) + rl * 4;
            hdr[1 + w] = scale;
            if (w == 0) hdr[0] = lse2;
            tc::fence_proxy_async_smem();  // the bulk copies below read the staged records through the async proxy
            asm volatile("bar.sync 1, 256;\n" ::: "memory");
            tc::cluster_wait();  // every CTA's ring is idle: the blocks may land
            if (tid == 128) {  // one block to every owner, this CTA included: it lands as source `split`
                for (int o = 0; o < S; ++o)
                    tc::bulk_copy_s2c(tc::cluster_map(sbase + L::RECV_OFF + split * BB, o), smem_u32(stage + o * BB),
                                      BB, tc::cluster_map(recv, o));
            }
        }
    }

    // ---- merge this CTA's rows over the S blocks received (all threads), once they have all landed ----
    if (S > 1) {
        const bool got = tc::mbar_wait_drain(recv, 0, kDrainCycles);
        if (!got && tid == 0) atomicOr(p.dev_status, TIDAR_DEV_TIMEOUT);
        if (__syncthreads_and(got)) {
            // every other CTA's copy into this CTA has completed, so its source block has been read: each source
            // hears of it at once (lane o of warp 0 tells CTA o; it may exit once all its blocks are in)
            if (warp == 0 && lane < S && lane != split) tc::mbar_arrive_remote(tc::cluster_map(sent, lane));
            const uint8_t *rv = smem + L::RECV_OFF;
            float *wts = reinterpret_cast<float *>(smem + L::KV_OFF);  // row-statistics area, free by now
            if constexpr (kLarge) {
                switch (S) {
                    case 9: merge_rows<D, 9>(p, rv, wts, split, mt, b, kvh, tid); break;
                    case 10: merge_rows<D, 10>(p, rv, wts, split, mt, b, kvh, tid); break;
                    case 12: merge_rows<D, 12>(p, rv, wts, split, mt, b, kvh, tid); break;
                    default: merge_rows<D, 15>(p, rv, wts, split, mt, b, kvh, tid); break;
                }
            } else {
                switch (S) {
                    case 2: merge_rows<D, 2>(p, rv, wts, split, mt, b, kvh, tid); break;
                    case 3: merge_rows<D, 3>(p, rv, wts, split, mt, b, kvh, tid); break;
                    case 4: merge_rows<D, 4>(p, rv, wts, split, mt, b, kvh, tid); break;
                    case 5: merge_rows<D, 5>(p, rv, wts, split, mt, b, kvh, tid); break;
                    case 6: merge_rows<D, 6>(p, rv, wts, split, mt, b, kvh, tid); break;
                    case 7: merge_rows<D, 7>(p, rv, wts, split, mt, b, kvh, tid); break;
                    default: merge_rows<D, 8>(p, rv, wts, split, mt, b, kvh, tid); break;
                }
            }
        }
    }
    if (S > 1) {
        // no copy may still read this CTA's shared memory when it exits: wait until every block it sent has landed
        if (tid == 0 && !tc::mbar_wait_drain(sent, 0, kDrainCycles)) atomicOr(p.dev_status, TIDAR_DEV_TIMEOUT);
    } else {
        // (a cluster of one: every thread is past its TMEM reads before the allocation is freed)
        tc::cluster_arrive_relaxed();
        tc::cluster_wait();
    }
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tbase, 512);
    }
    if (tid == 0 && *abort_flag) atomicOr(p.dev_status, TIDAR_DEV_TIMEOUT);
}

// ---- host side ---------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeTiledFn) nullptr;
        return reinterpret_cast<EncodeTiledFn>(ptr);
    }();
    return fn;
}

// bf16 tensor map, 128-byte swizzle, box {64, ..., TN} (dims innermost first).
bool make_map(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims, const cuuint64_t *strides_bytes,
              const cuuint32_t *box) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides_bytes, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch(const AttnParams &p, cudaStream_t s) {
    CUtensorMap kc, vc, kn, vn, qm;
    const cuuint64_t cache_rows =
        p.block_table ? (cuuint64_t)p.num_pages * p.Hkv * kPageRows : (cuuint64_t)p.B * p.Hkv * p.P_max;
    const cuuint64_t dc[2] = {(cuuint64_t)D, cache_rows};
    const cuuint64_t sc[1] = {(cuuint64_t)D * 2};
    const cuuint32_t bc[2] = {64, (cuuint32_t)(p.block_table ? BOXR : TN)};
    const cuuint64_t dn[3] = {(cuuint64_t)D, (cuuint64_t)p.Hkv, (cuuint64_t)p.B * p.R};
    const cuuint64_t sn[2] = {(cuuint64_t)D * 2, (cuuint64_t)p.Hkv * D * 2};
    const cuuint32_t bn[3] = {64, 1, TN};
    // Q as {D, Hq, B*R}: a box of G heads x 128/G rows is one packed row tile when G divides 128
    const int q_tma = (TM % p.G == 0) ? 1 : 0;
    const cuuint64_t dq[3] = {(cuuint64_t)D, (cuuint64_t)p.Hq, (cuuint64_t)p.B * p.R};
    const cuuint64_t sq[2] = {(cuuint64_t)D * 2, (cuuint64_t)p.Hq * D * 2};
    const cuuint32_t bq[3] = {64, (cuuint32_t)(q_tma ? p.G : 1), (cuuint32_t)(q_tma ? TM / p.G : 1)};
    if (!make_map(&kc, p.k_cache, 2, dc, sc, bc) || !make_map(&vc, p.v_cache, 2, dc, sc, bc) ||
        !make_map(&kn, p.k_new, 3, dn, sn, bn) || !make_map(&vn, p.v_new, 3, dn, sn, bn) ||
        !make_map(&qm, p.q, 3, dq, sq, bq))
        return cudaErrorInvalidValue;
    const int smem = Smem<D>::ALLOC;
    const bool large = p.n_splits > 8;  // (chosen only where the occupancy query granted such clusters)
    const auto kern = large ? attn_sm100_kernel<D, true> : attn_sm100_kernel<D, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (large) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.n_splits, p.Mpad / TM, p.B * p.Hkv);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;  // the splits of one row tile form a cluster
    attr[0].val.clusterDim.x = p.n_splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlap set-up with the previous kernel
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kern, p, kc, vc, kn, vn, qm, q_tma);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Clusters of `S` CTAs of this kernel that can be resident at once (0 if the query fails).
template <int D>
int max_active_clusters(int S) {
    static int cache[kMaxSplits + 1] = {-1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1, -1};
    if (cache[S] >= 0) return cache[S];
    const int smem = Smem<D>::ALLOC;
    const auto kern = S > 8 ? attn_sm100_kernel<D, true> : attn_sm100_kernel<D, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return 0;
    if (S > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        cudaGetLastError();
        cache[S] = 0;
        return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(S, 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cache[S] = n;
    return n;
}

}  // namespace

int attn_sm100_rows_per_tile() { return TM; }
int attn_sm100_keys_per_tile() { return TN; }
int attn_sm100_max_splits() { return kMaxSplits; }

// Key splits per row tile (the cluster size): the largest allowed S (split_count_ok) <= the tile count for which
// all `groups` clusters are resident in one wave; 1 if even single CTAs need several waves.  Sizes above 8
// (non-portable) only where the occupancy query grants them.
int attn_sm100_pick_splits(int D, long groups, int max_tiles) {
    const int hi = max(1, min(kMaxSplits, max_tiles));
    for (int S = hi; S > 1; --S) {
        if (!split_count_ok(S)) continue;
        const int fit = D == 64 ? max_active_clusters<64>(S) : max_active_clusters<128>(S);
        if (fit == 0 && S <= 8 && S * groups <= kNumSMs) return S;  // query unavailable: one CTA per SM
        if (fit >= groups) return S;
    }
    return 1;
}

cudaError_t attn_sm100_launch(const AttnParams &p, cudaStream_t s) {
    return p.D == 64 ? launch<64>(p, s) : launch<128>(p, s);
}

}  // namespace tidar
