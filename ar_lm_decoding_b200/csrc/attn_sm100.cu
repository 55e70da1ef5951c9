// TiDAR hybrid-mask attention for sm_100a: TMA + tcgen05 (TMEM accumulators).
//
// One CTA owns 128 packed query rows (row m = r*G + g of the G query heads
// sharing KV head kvh: GQA packing, so every K/V byte feeds 128 rows) and a
// contiguous run of 128-key tiles of one sequence.  A sequence's tiles are
// the cached prefix in 128-row tiles (the last one partial) followed by the
// R new keys of this step in 128-row tiles.
//
// Warp roles (12 warps):
//   warp 0      TMA producer: K and V tiles (128-byte swizzle) into a
//               3-stage ring; prefix tiles from the cache, new-key tiles from
//               K_new/V_new through a 3-D tensor map (no head gather).
//   warp 1      TMEM owner and MMA issuer (one thread): S = Q K^T into the
//               S columns of the warpgroup that owns the tile, then
//               O += P V with P read from TMEM (tcgen05.mma A-from-TMEM).
//   warps 4-7   softmax warpgroup 0: even tiles;  warps 8-11: odd tiles.
//               Thread = query row = TMEM lane.  Each warpgroup keeps its
//               own online-softmax state and its own O accumulator, so the
//               tensor pipe computes one warpgroup's GEMMs while the other
//               runs its exponentials.  The mask is evaluated from indices;
//               O is rescaled only when the running max grows by more than
//               2^8 (a stale max is exact as long as p <= 2^8 fits).
//   warps 2-3   help load Q, then idle.
// TMEM (512 columns): warpgroup w owns S/P at [256w, 256w+128) and O at
// [256w+128, 256w+128+D).  P (bf16) overwrites the first 64 columns of S; the
// next S into those columns is issued after the PV that reads P, and
// tcgen05.mma executes in issue order.
// At the end the two warpgroups merge their (m, l, O) through shared memory
// and write the normalised partial output and its LSE for the split combine.
//
// Every wait is bounded (clock64 budget); on expiry the CTA raises
// TIDAR_DEV_TIMEOUT in dev_status, drains, frees TMEM and returns.
#include "attn.cuh"
#include "tc.cuh"

namespace tidar {

namespace {

constexpr int TM = 128;
constexpr int TN = 128;
constexpr int STAGES = 3;
constexpr int THREADS = 384;
constexpr long long kWaitCycles = 4000000000LL;

template <int D>
struct Smem {
    static constexpr int Q_BYTES = TM * D * 2;
    static constexpr int KV_TILE = TN * D * 2;  // one of K or V
    static constexpr int STAGE = 2 * KV_TILE;
    static constexpr int KV_OFF = Q_BYTES;
    static constexpr int BAR_OFF = KV_OFF + STAGES * STAGE;
    static constexpr int NBARS = 2 * STAGES + 6;  // kv_full, kv_empty, s_full[2], p_full[2], o_done[2]
    static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
    static constexpr int TOTAL = MISC_OFF + 16;
    static constexpr int ALLOC = TOTAL + 1024;  // alignment slack
};

// Number of valid keys in tile t (t < TP: prefix tile, else new-key tile).
__device__ __forceinline__ int tile_valid(int t, int TP, int P, int R) {
    return t < TP ? min(TN, P - t * TN) : min(TN, R - (t - TP) * TN);
}

template <int D>
__global__ void __launch_bounds__(THREADS, 1)
    attn_sm100_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tm_kc,
                      const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_kn,
                      const __grid_constant__ CUtensorMap tm_vn) {
    using L = Smem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase;
    const uint32_t sKV = sbase + L::KV_OFF;
    const uint32_t bar0 = sbase + L::BAR_OFF;
    auto kv_full = [&](int s) { return bar0 + 8u * s; };
    auto kv_empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto s_full = [&](int w) { return bar0 + 8u * (2 * STAGES + w); };
    auto p_full = [&](int w) { return bar0 + 8u * (2 * STAGES + 2 + w); };
    auto o_done = [&](int w) { return bar0 + 8u * (2 * STAGES + 4 + w); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::MISC_OFF);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::MISC_OFF + 4);

    const int split = blockIdx.x, mt = blockIdx.y, bh = blockIdx.z;
    const int b = bh / p.Hkv, kvh = bh % p.Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int P = p.prefix_len[b];
    if (P < 0 || P > p.P_max) {
        if (tid == 0 && split == 0 && mt == 0) atomicOr(p.dev_status, TIDAR_DEV_BAD_PREFIX);
        return;
    }
    const int TP = ceil_div(P, TN);
    const int T = TP + ceil_div(p.R, TN);
    const int t0 = (int)((long)split * T / p.n_splits);
    const int t1 = (int)((long)(split + 1) * T / p.n_splits);
    const int n = t1 - t0;

    // ---- set-up ----
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(kv_full(s), 1);
            tc::mbar_init(kv_empty(s), 1);
        }
        for (int w = 0; w < 2; ++w) {
            tc::mbar_init(s_full(w), 1);
            tc::mbar_init(p_full(w), 128);
            tc::mbar_init(o_done(w), 1);
        }
        *abort_flag = 0;
        tc::mbar_fence_init();
    }
    if (warp == 0 && lane == 0) {
        tc::tma_prefetch_desc(&tm_kc);
        tc::tma_prefetch_desc(&tm_vc);
        tc::tma_prefetch_desc(&tm_kn);
        tc::tma_prefetch_desc(&tm_vn);
    }
    if (warp == 1) tc::tmem_alloc(smem_u32(tmem_slot), 512);
    if (warp >= 2) {  // Q tile, K-major with 128-byte swizzle: D/64 blocks of [128 rows][128 B]
        constexpr int CH = D / 8;
        for (int idx = tid - 64; idx < TM * CH; idx += THREADS - 64) {
            const int i = idx / CH, c = idx % CH;
            const int m = mt * TM + i;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (m < p.M) {
                const int r = m / p.G, g = m % p.G;
                v = *reinterpret_cast<const uint4 *>(p.q + ((size_t)(b * p.R + r) * p.Hq + kvh * p.G + g) * D + c * 8);
            }
            const int blk = c >> 3, cc = c & 7;
            *reinterpret_cast<uint4 *>(smem + blk * TM * 128 + i * 128 + ((cc ^ (i & 7)) << 4)) = v;
        }
        tc::fence_proxy_async_smem();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;

    if (warp == 0) {
        // ================= TMA producer =================
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < n; ++i) {
                const int st = i % STAGES, u = i / STAGES;
                if (u > 0 && !tc::mbar_wait(kv_empty(st), (u - 1) & 1, abort_flag, kWaitCycles)) break;
                tc::mbar_arrive_expect_tx(kv_full(st), L::STAGE);
                const int t = t0 + i;
                const uint32_t kd = sKV + st * L::STAGE, vd = kd + L::KV_TILE;
                if (t < TP) {
                    const int y = (b * p.Hkv + kvh) * p.P_max + t * TN;
#pragma unroll
                    for (int h = 0; h < D / 64; ++h) {
                        tc::tma_load_2d(kd + h * TN * 128, &tm_kc, h * 64, y, kv_full(st));
                        tc::tma_load_2d(vd + h * TN * 128, &tm_vc, h * 64, y, kv_full(st));
                    }
                } else {
                    const int z = b * p.R + (t - TP) * TN;
#pragma unroll
                    for (int h = 0; h < D / 64; ++h) {
                        tc::tma_load_3d(kd + h * TN * 128, &tm_kn, h * 64, kvh, z, kv_full(st));
                        tc::tma_load_3d(vd + h * TN * 128, &tm_vn, h * 64, kvh, z, kv_full(st));
                    }
                }
                issued = i + 1;
            }
            // drain: no copy may land after the CTA exits
            for (int i = max(0, issued - STAGES); i < issued; ++i)
                tc::mbar_wait(kv_full(i % STAGES), (i / STAGES) & 1, abort_flag, kWaitCycles);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ================= MMA issuer =================
        constexpr uint32_t id_qk = tc::idesc_bf16_f32(TM, TN, 0, 0);
        constexpr uint32_t id_pv = tc::idesc_bf16_f32(TM, D, 0, 1);
        bool ok = true;
        auto issue_qk = [&](int i) {
            const int st = i % STAGES, w = i & 1;
            ok = ok && tc::mbar_wait(kv_full(st), (i / STAGES) & 1, abort_flag, kWaitCycles);
            if (!ok) return;
            const int valid = tile_valid(t0 + i, TP, P, p.R);
            if (valid < TN) {  // keys past the sequence: zero their V rows so that 0 * V stays 0
                uint8_t *vrow = smem + L::KV_OFF + st * L::STAGE + L::KV_TILE;
                for (int idx = lane; idx < (TN - valid) * (D / 8); idx += 32) {
                    const int j = valid + idx / (D / 8), c = idx % (D / 8);
                    *reinterpret_cast<uint4 *>(vrow + (c >> 3) * TN * 128 + j * 128 + ((c & 7) << 4)) =
                        make_uint4(0, 0, 0, 0);
                }
                tc::fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) {
                tc::fence_after_sync();
                const uint32_t kb = sKV + st * L::STAGE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 0 + (kk & 3) * 32;
                    const uint64_t ad = tc::smem_desc_sw128(sQ + (kk >> 2) * TM * 128 + off, 16, 1024);
                    const uint64_t bd = tc::smem_desc_sw128(kb + (kk >> 2) * TN * 128 + off, 16, 1024);
                    tc::mma_ss(tbase + w * 256, ad, bd, id_qk, kk > 0);
                }
                tc::mma_commit(s_full(w));
            }
            __syncwarp();
        };
        auto issue_pv = [&](int i) {
            const int st = i % STAGES, w = i & 1;
            ok = ok && tc::mbar_wait(p_full(w), (i >> 1) & 1, abort_flag, kWaitCycles);
            if (!ok) return;
            if (lane == 0) {
                tc::fence_after_sync();
                const uint32_t vb = sKV + st * L::STAGE + L::KV_TILE;
#pragma unroll
                for (int kk = 0; kk < TN / 16; ++kk) {
                    const uint64_t bd = tc::smem_desc_sw128(vb + kk * 16 * 128, TN * 128, 1024);
                    tc::mma_ts(tbase + w * 256 + 128, tbase + w * 256 + kk * 8, bd, id_pv, (i >= 2 || kk > 0) ? 1u : 0u);
                }
                tc::mma_commit(kv_empty(st));
                if (i + 2 >= n) tc::mma_commit(o_done(w));
            }
            __syncwarp();
        };
        if (n > 0) issue_qk(0);
        if (n > 1) issue_qk(1);
        for (int i = 0; i < n && ok; ++i) {
            issue_pv(i);
            if (i + 2 < n) issue_qk(i + 2);
        }
    } else if (warp >= 4) {
        // ================= softmax warpgroups =================
        const int w = (warp - 4) >> 2;
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const int m_row = mt * TM + row;
        const int r = m_row / p.G;
        const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
        const uint32_t s_col = tbase + lane_off + w * 256;
        const uint32_t o_col = s_col + 128;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int i = w; i < n; i += 2) {
            if (!tc::mbar_wait(s_full(w), (i >> 1) & 1, abort_flag, kWaitCycles)) { ok = false; break; }
            tc::fence_after_sync();
            float x[TN];
#pragma unroll
            for (int c = 0; c < TN / 32; ++c) {
                uint32_t v[32];
                tc::tmem_ld32(s_col + c * 32, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) x[c * 32 + j] = __uint_as_float(v[j]);
            }
            tc::tmem_wait_ld();
            const int t = t0 + i;
            float mx = -INFINITY;
            if (t < TP - 1 || (t == TP - 1 && P % TN == 0)) {  // full prefix tile: no mask
#pragma unroll
                for (int j = 0; j < TN; ++j) {
                    x[j] *= p.scale_log2;
                    mx = fmaxf(mx, x[j]);
                }
            } else if (t < TP) {  // partial prefix tile
                const int valid = P - t * TN;
#pragma unroll
                for (int j = 0; j < TN; ++j) {
                    x[j] = j < valid ? x[j] * p.scale_log2 : -INFINITY;
                    mx = fmaxf(mx, x[j]);
                }
            } else {  // new-key tile: the TiDAR mask
                const int nn0 = (t - TP) * TN;
#pragma unroll
                for (int j = 0; j < TN; ++j) {
                    const int nn = nn0 + j;
                    const bool vis = nn < p.R && new_key_visible(p.mask_mode, p.k, r, nn);
                    x[j] = vis ? x[j] * p.scale_log2 : -INFINITY;
                    mx = fmaxf(mx, x[j]);
                }
            }
            const float m_new = fmaxf(m_run, mx);
            const bool grow = m_new > m_run + 8.f;
            if (i >= 2 && __any_sync(0xffffffffu, grow)) {  // rescale O (last written by the PV of tile i-2)
                const float f = grow ? fast_exp2(m_run - m_new) : 1.f;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t v[32];
                    tc::tmem_ld32(o_col + c * 32, v);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * f);
                    tc::tmem_st32(o_col + c * 32, v);
                }
            }
            if (grow) {
                l_run *= fast_exp2(m_run - m_new);
                m_run = m_new;
            }
            const float m_use = m_run == -INFINITY ? 0.f : m_run;
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < TN / 64; ++c) {
                uint32_t pk[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float a = fast_exp2(x[c * 64 + 2 * j] - m_use);
                    const float bb = fast_exp2(x[c * 64 + 2 * j + 1] - m_use);
                    sum += a + bb;
                    pk[j] = pack_bf16x2(a, bb);
                }
                tc::tmem_st32(s_col + c * 32, pk);
            }
            l_run += sum;
            tc::tmem_wait_st();
            tc::fence_before_sync();
            tc::mbar_arrive(p_full(w));
        }
        // ---- final O of this warpgroup ----
        const bool has = n > w;
        if (ok && has) ok = tc::mbar_wait(o_done(w), 0, abort_flag, kWaitCycles);
        tc::fence_after_sync();
        asm volatile("bar.sync 1, 256;\n" ::: "memory");  // both warpgroups done: the K/V ring is free
        float *xo = reinterpret_cast<float *>(smem + L::KV_OFF);  // [TM][D + 4] exchange rows
        float *xm = xo + TM * (D + 4);                              // [TM] m, then [TM] l
        if (w == 1) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                if (has && ok) {
                    tc::tmem_ld32(o_col + c * 32, v);
                    tc::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = 0u;
                }
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4 *>(xo + row * (D + 4) + c * 32 + j) =
                        make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]),
                                    __uint_as_float(v[j + 3]));
            }
            xm[row] = has ? m_run : -INFINITY;
            xm[TM + row] = has ? l_run : 0.f;
        }
        asm volatile("bar.sync 1, 256;\n" ::: "memory");
        if (w == 0) {
            const float m0 = has ? m_run : -INFINITY, l0 = has ? l_run : 0.f;
            const float m1 = xm[row], l1 = xm[TM + row];
            const float mm = fmaxf(m0, m1);
            const float a0 = m0 == -INFINITY ? 0.f : fast_exp2(m0 - mm);
            const float a1 = m1 == -INFINITY ? 0.f : fast_exp2(m1 - mm);
            const float l = l0 * a0 + l1 * a1;
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const size_t prow = (size_t)(bh * p.n_splits + split) * p.Mpad + mt * TM + row;
            float *dst = p.part_o + prow * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t v[32];
                if (has && ok) {
                    tc::tmem_ld32(o_col + c * 32, v);
                    tc::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = 0u;
                }
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const float4 o1 = *reinterpret_cast<const float4 *>(xo + row * (D + 4) + c * 32 + j);
                    float4 o;
                    o.x = (__uint_as_float(v[j]) * a0 + o1.x * a1) * inv;
                    o.y = (__uint_as_float(v[j + 1]) * a0 + o1.y * a1) * inv;
                    o.z = (__uint_as_float(v[j + 2]) * a0 + o1.z * a1) * inv;
                    o.w = (__uint_as_float(v[j + 3]) * a0 + o1.w * a1) * inv;
                    *reinterpret_cast<float4 *>(dst + c * 32 + j) = o;
                }
            }
            p.part_lse[prow] = l > 0.f ? (mm + __log2f(l)) * kLn2 : -INFINITY;
        }
    }

    // ---- teardown ----
    tc::fence_before_sync();
    __syncthreads();
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
    CUtensorMap kc, vc, kn, vn;
    const cuuint64_t dc[2] = {(cuuint64_t)D, (cuuint64_t)p.B * p.Hkv * p.P_max};
    const cuuint64_t sc[1] = {(cuuint64_t)D * 2};
    const cuuint32_t bc[2] = {64, TN};
    const cuuint64_t dn[3] = {(cuuint64_t)D, (cuuint64_t)p.Hkv, (cuuint64_t)p.B * p.R};
    const cuuint64_t sn[2] = {(cuuint64_t)D * 2, (cuuint64_t)p.Hkv * D * 2};
    const cuuint32_t bn[3] = {64, 1, TN};
    if (!make_map(&kc, p.k_cache, 2, dc, sc, bc) || !make_map(&vc, p.v_cache, 2, dc, sc, bc) ||
        !make_map(&kn, p.k_new, 3, dn, sn, bn) || !make_map(&vn, p.v_new, 3, dn, sn, bn))
        return cudaErrorInvalidValue;
    const int smem = Smem<D>::ALLOC;
    cudaError_t e = cudaFuncSetAttribute(attn_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.n_splits, p.Mpad / TM, p.B * p.Hkv);
    attn_sm100_kernel<D><<<grid, THREADS, smem, s>>>(p, kc, vc, kn, vn);
    return cudaGetLastError();
}

}  // namespace

int attn_sm100_rows_per_tile() { return TM; }
int attn_sm100_keys_per_tile() { return TN; }

cudaError_t attn_sm100_launch(const AttnParams &p, cudaStream_t s) {
    return p.D == 64 ? launch<64>(p, s) : launch<128>(p, s);
}

}  // namespace tidar
