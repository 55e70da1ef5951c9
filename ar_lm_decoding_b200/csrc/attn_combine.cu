// Merge of the per-key-range partial attention outputs (flash-decoding
// combine): LSE = log sum_s exp(LSE_s), O = sum_s exp(LSE_s - LSE) O_s, taken
// over the ranges in a fixed order so the result is deterministic.
#include "attn.cuh"

namespace tidar {

namespace {

template <int D>
__global__ void __launch_bounds__(128) attn_combine_kernel(const AttnParams p) {
    constexpr int PER = D / 32;  // elements per lane
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long gw = (long)blockIdx.x * 4 + warp;
    if (gw >= (long)p.B * p.Hkv * p.M) return;
    const int bh = (int)(gw / p.M), m = (int)(gw % p.M);
    const int b = bh / p.Hkv, kvh = bh % p.Hkv;
    const int P = p.prefix_len[b];
    if (P < 0 || P > p.P_max) return;
    const size_t row0 = (size_t)bh * p.n_splits * p.Mpad + m;

    float mx = -INFINITY;
    for (int s = 0; s < p.n_splits; ++s) mx = fmaxf(mx, p.part_lse[row0 + (size_t)s * p.Mpad]);
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
    float wsum = 0.f;
    for (int s = 0; s < p.n_splits; ++s) {
        const float ls = p.part_lse[row0 + (size_t)s * p.Mpad];
        if (ls == -INFINITY) continue;
        const float w = fast_exp2((ls - mx) * kLog2e);
        wsum += w;
        const float *src = p.part_o + (row0 + (size_t)s * p.Mpad) * D + lane * PER;
        if constexpr (PER == 4) {
            const float4 v = *reinterpret_cast<const float4 *>(src);
            acc[0] += w * v.x;
            acc[1] += w * v.y;
            acc[2] += w * v.z;
            acc[3] += w * v.w;
        } else {
            const float2 v = *reinterpret_cast<const float2 *>(src);
            acc[0] += w * v.x;
            acc[1] += w * v.y;
        }
    }
    const float inv = 1.f / wsum;
    const int r = m / p.G, h = kvh * p.G + m % p.G;
    const size_t orow = ((size_t)(b * p.R + r) * p.Hq + h);
    bf16 *dst = p.out + orow * D + lane * PER;
    if constexpr (PER == 4) {
        uint2 v;
        v.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        v.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
        *reinterpret_cast<uint2 *>(dst) = v;
    } else {
        *reinterpret_cast<uint32_t *>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    }
    if (p.lse && lane == 0) p.lse[orow] = mx + __logf(wsum);
}

}  // namespace

cudaError_t attn_combine_launch(const AttnParams &p, cudaStream_t s) {
    const long rows = (long)p.B * p.Hkv * p.M;
    const unsigned grid = (unsigned)((rows + 3) / 4);
    if (p.D == 64)
        attn_combine_kernel<64><<<grid, 128, 0, s>>>(p);
    else
        attn_combine_kernel<128><<<grid, 128, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace tidar
