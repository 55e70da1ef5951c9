// Shared device helpers for the TiDAR decode-step kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tidar.h"

namespace tidar {

typedef __nv_bfloat16 bf16;

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kNumSMs = 148;
constexpr int kMaxDraft = 16;  // longest draft block k every entry point accepts
constexpr int kPageRows = 64;  // rows of a KV-cache page: one key tile of the attention kernel
constexpr int kMaxPagesPerSeq = 1024;  // longest block-table row a paged call accepts (65536 cached tokens)
constexpr int kMaxVocab = 1 << 19;      // largest vocabulary the verify and commit accept (64 chunks of 8192)

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Visibility of new key nn (0..R-1, same order as the query rows) to query
// row r under the TiDAR decode mask: drafts are causal among themselves;
// a slot of pre-draft group j sees drafts d_1..d_j and its own group.
// Cached-prefix keys are visible to every row and never reach this test.
__device__ __forceinline__ bool new_key_visible(int mask_mode, int k, int r, int nn) {
    if (mask_mode == TIDAR_MASK_CAUSAL) return nn <= r;
    if (r < k) return nn <= r;
    const int grp = (r - k) / k;
    if (nn < k) return nn < grp;
    return (nn - k) / k == grp;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float2 unpack_half2(uint32_t u) {
    __half2 v = *reinterpret_cast<__half2 *>(&u);
    return __half22float2(v);
}

// Logit element as float (bf16 or f32 storage).
__device__ __forceinline__ float load_logit(const void *base, int dtype, size_t idx) {
    if (dtype == TIDAR_DT_BF16) return __bfloat162float(reinterpret_cast<const bf16 *>(base)[idx]);
    return reinterpret_cast<const float *>(base)[idx];
}

}  // namespace tidar
