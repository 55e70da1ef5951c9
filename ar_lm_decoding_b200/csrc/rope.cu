// Rotary position embedding of a step's rows, fused with the re-layout of the
// QKV projection output into the attention's inputs.
//
// The fused projection output holds, per row, the Hq query heads, then the Hkv
// key heads, then the Hkv value heads.  One thread takes two rotation pairs
// (x_i, x_{i+D/2}), i = 2c, 2c+1, of one head of one row (a warp reads 128
// contiguous bytes of each half): the rotation by pos * theta^(-2i/D) in double
// precision (position times frequency reaches ~1e4 radians, which fp32 would
// resolve to ~1e-3), with the frequencies theta^(-2i/D) computed once on the
// host in double precision.  Value heads are copied.  Row positions follow the TiDAR
// step layout: draft d_i at P + i - 1, slot s of pre-draft group j at P + j + s.
#include <cmath>

#include "common.cuh"

namespace tidar {

namespace {

struct RopeParams {
    const bf16 *qkv;
    const int32_t *prefix_len;
    int B, Hq, Hkv, D, k, R;
    double inv_freq[64];  // theta^(-2i/D), i < D/2
    bf16 *q, *k_new, *v_new;
    int32_t *dev_status;
};

__device__ __forceinline__ int row_position(int k, int P, int r) {
    if (r < k) return P + r;
    const int j = (r - k) / k;
    return P + j + (r - k - j * k);
}

__global__ void __launch_bounds__(256) rope_qkv_kernel(const RopeParams p) {
    const int H = p.Hq + 2 * p.Hkv;
    const int half = p.D / 2;
    const int pairs2 = half / 2;  // threads per head: two pairs each
    const long total = (long)p.B * p.R * H * pairs2;
    const long it = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (it >= total) return;
    const int c = (int)(it % pairs2);
    const int h = (int)((it / pairs2) % H);
    const long row = it / ((long)pairs2 * H);  // b * R + r
    const int b = (int)(row / p.R), r = (int)(row % p.R);
    const bf16 *x = p.qkv + ((size_t)row * H + h) * p.D;
    bf16 *y;
    if (h < p.Hq) y = p.q + ((size_t)row * p.Hq + h) * p.D;
    else if (h < p.Hq + p.Hkv) y = p.k_new + ((size_t)row * p.Hkv + (h - p.Hq)) * p.D;
    else y = p.v_new + ((size_t)row * p.Hkv + (h - p.Hq - p.Hkv)) * p.D;
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(x + 2 * c);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(x + half + 2 * c);
    if (h >= p.Hq + p.Hkv) {  // value head: copied
        *reinterpret_cast<__nv_bfloat162 *>(y + 2 * c) = lo;
        *reinterpret_cast<__nv_bfloat162 *>(y + half + 2 * c) = hi;
        return;
    }
    const int P = p.prefix_len[b];
    if (P < 0) {
        if (c == 0 && h == 0 && r == 0) atomicOr(p.dev_status, TIDAR_DEV_BAD_PREFIX);
        return;
    }
    const double pos = (double)row_position(p.k, P, r);
    const double a0 = __bfloat162float(lo.x), a1 = __bfloat162float(lo.y);
    const double b0 = __bfloat162float(hi.x), b1 = __bfloat162float(hi.y);
    double s0, c0, s1, c1;
    sincos(pos * p.inv_freq[2 * c], &s0, &c0);
    sincos(pos * p.inv_freq[2 * c + 1], &s1, &c1);
    __nv_bfloat162 olo, ohi;
    olo.x = __double2bfloat16(a0 * c0 - b0 * s0);
    olo.y = __double2bfloat16(a1 * c1 - b1 * s1);
    ohi.x = __double2bfloat16(b0 * c0 + a0 * s0);
    ohi.y = __double2bfloat16(b1 * c1 + a1 * s1);
    *reinterpret_cast<__nv_bfloat162 *>(y + 2 * c) = olo;
    *reinterpret_cast<__nv_bfloat162 *>(y + half + 2 * c) = ohi;
}

}  // namespace
}  // namespace tidar

using namespace tidar;

extern "C" tidar_status tidar_rope_qkv(const void *qkv, const int32_t *prefix_len, int B, int Hq, int Hkv, int D, int k,
                                       double theta, void *q, void *k_new, void *v_new, int32_t *dev_status,
                                       void *stream) {
    if (B < 1 || Hq < 1 || Hkv < 1 || k < 1 || !(theta > 1.0) || !std::isfinite(theta)) return TIDAR_ERR_INVALID_ARG;
    if (k > kMaxDraft || (D != 64 && D != 128) || Hq % Hkv) return TIDAR_ERR_UNSUPPORTED;
    if (!qkv || !prefix_len || !q || !k_new || !v_new || !dev_status) return TIDAR_ERR_INVALID_ARG;
    for (const void *ptr : {qkv, (const void *)q, (const void *)k_new, (const void *)v_new})
        if (reinterpret_cast<uintptr_t>(ptr) & 3) return TIDAR_ERR_INVALID_ARG;
    RopeParams p;
    p.qkv = static_cast<const bf16 *>(qkv);
    p.prefix_len = prefix_len;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.D = D;
    p.k = k;
    p.R = k * (k + 2);
    for (int i = 0; i < D / 2; ++i) p.inv_freq[i] = std::pow(theta, -2.0 * i / D);
    p.q = static_cast<bf16 *>(q);
    p.k_new = static_cast<bf16 *>(k_new);
    p.v_new = static_cast<bf16 *>(v_new);
    p.dev_status = dev_status;
    const long total = (long)B * p.R * (Hq + 2 * Hkv) * (D / 4);
    rope_qkv_kernel<<<(unsigned)((total + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? TIDAR_OK : TIDAR_ERR_CUDA;
}
