// TiDAR hybrid-mask attention, split-KV (flash-decoding) with GQA row packing,
// on the legacy warp-level tensor-core path (mma.sync m16n8k16, bf16 -> f32).
//
// The R query rows of the G query heads that share one KV head form one
// M = R*G row operand, so every K/V byte a CTA loads is used by up to 64 rows.
// The keys of one sequence are [cached prefix | R new keys]; each CTA takes a
// contiguous, 64-aligned key range, keeps an online softmax per row, and
// writes a normalised partial output plus its log-sum-exp; attn_combine
// merges the ranges.  The mask is evaluated from indices (new_key_visible).
// This kernel is the correctness baseline for the tcgen05 kernel and also
// serves the shapes that kernel does not take.
#include "attn.cuh"

namespace tidar {

namespace {

constexpr int BM = 64;   // query rows per CTA (4 warps x 16)
constexpr int BN = 64;   // keys per tile
constexpr int THREADS = 128;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte chunk c of row `row` in a [rows][D] bf16 tile whose
// chunks are XOR-swizzled by (row & 7) to keep ldmatrix conflict-free.
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int c) {
    return static_cast<uint32_t>(row * (D * 2) + ((c ^ (row & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(THREADS) attn_mma_kernel(const AttnParams p) {
    constexpr int CH = D / 8;  // 16-byte chunks per row
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *sQ = smem;
    uint8_t *sK = sQ + BM * D * 2;
    uint8_t *sV = sK + 2 * BN * D * 2;

    const int split = blockIdx.x, mt = blockIdx.y, bh = blockIdx.z;
    const int b = bh / p.Hkv, kvh = bh % p.Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int P = p.prefix_len[b];
    if (P < 0 || P > p.P_max) {
        if (tid == 0 && split == 0 && mt == 0) atomicOr(p.dev_status, TIDAR_DEV_BAD_PREFIX);
        return;
    }
    const int N = P + p.R;
    const int chunk = round_up(ceil_div(N, p.n_splits), BN);
    const int n0 = split * chunk;
    const int n1 = min(N, n0 + chunk);
    const size_t part_row0 = (size_t)(bh * p.n_splits + split) * p.Mpad;

    // ---- Q tile: rows m = mt*BM + i of the packed (r, g) operand ----
    for (int idx = tid; idx < BM * CH; idx += THREADS) {
        const int i = idx / CH, c = idx % CH;
        const int m = mt * BM + i;
        const bf16 *src = p.q;
        int bytes = 0;
        if (m < p.M) {
            const int r = m / p.G, g = m % p.G;
            src = p.q + ((size_t)(b * p.R + r) * p.Hq + kvh * p.G + g) * D + c * 8;
            bytes = 16;
        }
        cp_async16(smem_u32(sQ + swz<D>(i, c)), src, bytes);
    }
    cp_async_commit();

    auto load_kv = [&](int tile, int stage) {
        const int base = n0 + tile * BN;
        for (int idx = tid; idx < BN * CH; idx += THREADS) {
            const int i = idx / CH, c = idx % CH;
            const int n = base + i;
            const bf16 *ks = p.k_cache, *vs = p.v_cache;
            int bytes = 0;
            if (n < P) {
                const size_t off = ((size_t)(b * p.Hkv + kvh) * p.P_max + n) * D + c * 8;
                ks = p.k_cache + off;
                vs = p.v_cache + off;
                bytes = 16;
            } else if (n < n1) {
                const size_t off = ((size_t)(b * p.R + (n - P)) * p.Hkv + kvh) * D + c * 8;
                ks = p.k_new + off;
                vs = p.v_new + off;
                bytes = 16;
            }
            const uint32_t o = swz<D>(i, c) + stage * BN * D * 2;
            cp_async16(smem_u32(sK + o), ks, bytes);
            cp_async16(smem_u32(sV + o), vs, bytes);
        }
    };

    const int ntiles = n1 > n0 ? ceil_div(n1 - n0, BN) : 0;
    if (ntiles > 0) load_kv(0, 0);
    cp_async_commit();

    float o_acc[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    const int gq = lane >> 2, tq = lane & 3;
    const int row_lo = mt * BM + warp * 16 + gq;  // packed row of c[0], c[1]; +8 for c[2], c[3]
    const int r_lo = row_lo / p.G, r_hi = (row_lo + 8) / p.G;

    uint32_t qf[D / 16][4];
    cp_async_wait<1>();
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int row = warp * 16 + (lane & 15);
        const int c = kk * 2 + (lane >> 4);
        ldsm_x4(smem_u32(sQ + swz<D>(row, c)), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
    }

    for (int t = 0; t < ntiles; ++t) {
        if (t + 1 < ntiles) load_kv(t + 1, (t + 1) & 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const uint8_t *k_st = sK + (t & 1) * BN * D * 2;
        const uint8_t *v_st = sV + (t & 1) * BN * D * 2;

        float s[BN / 8][4];
#pragma unroll
        for (int nt = 0; nt < BN / 8; ++nt) {
            s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < D / 16; kk += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(smem_u32(k_st + swz<D>(nt * 8 + (lane & 7), kk * 2 + (lane >> 3))), b0, b1, b2, b3);
                mma_bf16(s[nt], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
                mma_bf16(s[nt], qf[kk + 1][0], qf[kk + 1][1], qf[kk + 1][2], qf[kk + 1][3], b2, b3);
            }
        }
        // scale (log2 domain) and mask
        const int base = n0 + t * BN;
        const bool edge = base + BN > P;
#pragma unroll
        for (int nt = 0; nt < BN / 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float v = s[nt][e] * p.scale_log2;
                if (edge) {
                    const int n = base + nt * 8 + 2 * tq + (e & 1);
                    const int r = e < 2 ? r_lo : r_hi;
                    if (n >= n1 || (n >= P && !new_key_visible(p.mask_mode, p.k, r, n - P))) v = -INFINITY;
                }
                s[nt][e] = v;
            }
        // online softmax per row (two rows per thread; a row is spread over a quad)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < BN / 8; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * h], s[nt][2 * h + 1]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_run[h], mx);
            const float m_use = m_new == -INFINITY ? 0.f : m_new;
            const float corr = fast_exp2(m_run[h] - m_use);
            float sum = 0.f;
#pragma unroll
            for (int nt = 0; nt < BN / 8; ++nt) {
                s[nt][2 * h] = fast_exp2(s[nt][2 * h] - m_use);
                s[nt][2 * h + 1] = fast_exp2(s[nt][2 * h + 1] - m_use);
                sum += s[nt][2 * h] + s[nt][2 * h + 1];
            }
            l_run[h] = l_run[h] * corr + sum;
            m_run[h] = m_new;
#pragma unroll
            for (int dt = 0; dt < D / 8; ++dt) {
                o_acc[dt][2 * h] *= corr;
                o_acc[dt][2 * h + 1] *= corr;
            }
        }
        // O += P V
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
            const uint32_t a0 = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
            const uint32_t a1 = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
            const uint32_t a2 = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
            const uint32_t a3 = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                uint32_t b0, b1, b2, b3;
                const int row = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                ldsm_x4_t(smem_u32(v_st + swz<D>(row, dp * 2 + (lane >> 4))), b0, b1, b2, b3);
                mma_bf16(o_acc[2 * dp], a0, a1, a2, a3, b0, b1);
                mma_bf16(o_acc[2 * dp + 1], a0, a1, a2, a3, b2, b3);
            }
        }
        __syncthreads();
    }

    // ---- normalised partial output + log-sum-exp (natural log) ----
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float l = l_run[h];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        const int m = row_lo + 8 * h;
        const int i = m - mt * BM;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        float *dst = p.part_o + (part_row0 + (size_t)(mt * BM + i)) * D;
#pragma unroll
        for (int dt = 0; dt < D / 8; ++dt) {
            float2 v = make_float2(o_acc[dt][2 * h] * inv, o_acc[dt][2 * h + 1] * inv);
            *reinterpret_cast<float2 *>(dst + dt * 8 + 2 * tq) = v;
        }
        if (tq == 0) p.part_lse[part_row0 + mt * BM + i] = l > 0.f ? (m_run[h] + __log2f(l)) * kLn2 : -INFINITY;
    }
}

}  // namespace

template <int D>
static cudaError_t launch_mma(const AttnParams &p, cudaStream_t s) {
    const size_t smem = (size_t)(BM + 4 * BN) * D * 2;
    cudaError_t e = cudaFuncSetAttribute(attn_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.n_splits, p.Mpad / BM, p.B * p.Hkv);
    attn_mma_kernel<D><<<grid, THREADS, smem, s>>>(p);
    return cudaGetLastError();
}

int attn_mma_rows_per_tile() { return BM; }

cudaError_t attn_mma_launch(const AttnParams &p, cudaStream_t s) {
    return p.D == 64 ? launch_mma<64>(p, s) : launch_mma<128>(p, s);
}

}  // namespace tidar
