// Rotary position embedding of a step's rows, fused with the re-layout of the
// QKV projection output into the attention's inputs.
//
// The fused projection output holds, per row, the Hq query heads, then the Hkv
// key heads, then the Hkv value heads.  One thread takes eight rotation pairs
// (x_i, x_{i+D/2}), i = 8c .. 8c+7, of one head of one row: two 16-byte loads,
// the rotation by pos * theta^(-2i/D) in double precision (position times
// frequency reaches ~1e4 radians, which fp32 would resolve to ~1e-3), two
// 16-byte stores.  Value heads are copied.  Row positions follow the TiDAR
// step layout: draft d_i at P + i - 1, slot s of pre-draft group j at P + j + s.
#include <cmath>

#include "common.cuh"

namespace tidar {

namespace {

struct RopeParams {
    const bf16 *qkv;
    const int32_t *prefix_len;
    int B, Hq, Hkv, D, k, R;
    double log2_theta;
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
    const int chunks = p.D / 16;  // 8-pair chunks per head
    const long total = (long)p.B * p.R * H * chunks;
    const long it = (long)blockIdx.x * blockDim.x + threadIdx.x;
    if (it >= total) return;
    const int c = (int)(it % chunks);
    const int h = (int)((it / chunks) % H);
    const long row = it / ((long)chunks * H);  // b * R + r
    const int b = (int)(row / p.R), r = (int)(row % p.R);
    const int half = p.D / 2;
    const bf16 *x = p.qkv + ((size_t)row * H + h) * p.D;
    bf16 *y;
    if (h < p.Hq) y = p.q + ((size_t)row * p.Hq + h) * p.D;
    else if (h < p.Hq + p.Hkv) y = p.k_new + ((size_t)row * p.Hkv + (h - p.Hq)) * p.D;
    else y = p.v_new + ((size_t)row * p.Hkv + (h - p.Hq - p.Hkv)) * p.D;
    const uint4 lo = *reinterpret_cast<const uint4 *>(x + c * 8);
    const uint4 hi = *reinterpret_cast<const uint4 *>(x + half + c * 8);
    if (h >= p.Hq + p.Hkv) {  // value head: copied
        *reinterpret_cast<uint4 *>(y + c * 8) = lo;
        *reinterpret_cast<uint4 *>(y + half + c * 8) = hi;
        return;
    }
    const int P = p.prefix_len[b];
    if (P < 0) {
        if (c == 0 && h == 0 && r == 0) atomicOr(p.dev_status, TIDAR_DEV_BAD_PREFIX);
        return;
    }
    const double pos = (double)row_position(p.k, P, r);
    const bf16 *a = reinterpret_cast<const bf16 *>(&lo);
    const bf16 *bb = reinterpret_cast<const bf16 *>(&hi);
    __align__(16) bf16 oa[8], ob[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const int i = c * 8 + e;
        const double ang = pos * exp2(-2.0 * i / p.D * p.log2_theta);
        double sn, cs;
        sincos(ang, &sn, &cs);
        const double va = (double)__bfloat162float(a[e]), vb = (double)__bfloat162float(bb[e]);
        oa[e] = __double2bfloat16(va * cs - vb * sn);
        ob[e] = __double2bfloat16(vb * cs + va * sn);
    }
    *reinterpret_cast<uint4 *>(y + c * 8) = *reinterpret_cast<const uint4 *>(oa);
    *reinterpret_cast<uint4 *>(y + half + c * 8) = *reinterpret_cast<const uint4 *>(ob);
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
        if (reinterpret_cast<uintptr_t>(ptr) & 15) return TIDAR_ERR_INVALID_ARG;
    RopeParams p;
    p.qkv = static_cast<const bf16 *>(qkv);
    p.prefix_len = prefix_len;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.D = D;
    p.k = k;
    p.R = k * (k + 2);
    p.log2_theta = std::log2(theta);
    p.q = static_cast<bf16 *>(q);
    p.k_new = static_cast<bf16 *>(k_new);
    p.v_new = static_cast<bf16 *>(v_new);
    p.dev_status = dev_status;
    const long total = (long)B * p.R * (Hq + 2 * Hkv) * (D / 16);
    rope_qkv_kernel<<<(unsigned)((total + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? TIDAR_OK : TIDAR_ERR_CUDA;
}
