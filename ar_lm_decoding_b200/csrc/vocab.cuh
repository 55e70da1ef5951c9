// Vocabulary-sweep building blocks shared by the verify and the draft
// selection: per-chunk max / sum-exp statistics with 16-byte loads, and the
// chunked inverse CDF (sum of non-negative weights, find the chunk, rescan it).
#pragma once

#include "common.cuh"

namespace tidar {

constexpr int kChunk = 8192;        // vocabulary entries per CTA
constexpr int kStatThreads = 256;   // kChunk / kStatThreads = 32 entries per thread
static_assert(kMaxVocab == 64 * kChunk, "a row's chunk statistics are held two per lane of one warp");

struct ChunkStat {
    float m;   // max logit of the chunk
    float pad;
    double z;  // sum exp(logit - m) over the chunk
};

__host__ __device__ inline int vocab_chunks(int V) { return (V + kChunk - 1) / kChunk; }

// Load this thread's 32 entries of chunk c of a logit row (missing entries =
// -inf).  Entry e of thread t is at c*kChunk + (e/8)*2048 + t*8 + e%8 so that a
// warp reads 512 contiguous bytes (bf16) per step.
__device__ __forceinline__ void load_chunk32(const void *row, int dtype, int V, int c, float (&v)[32]) {
    const int tid = threadIdx.x;
    const int base = c * kChunk;
    const bool full = base + kChunk <= V;
    if (dtype == TIDAR_DT_BF16) {
        const bf16 *r = reinterpret_cast<const bf16 *>(row);
        const bool aligned = ((reinterpret_cast<uintptr_t>(r) & 15) == 0);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i0 = base + j * 2048 + tid * 8;
            if (full && aligned) {
                const uint4 u = __ldg(reinterpret_cast<const uint4 *>(r + i0));
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    v[j * 8 + 2 * e] = __uint_as_float(w[e] << 16);
                    v[j * 8 + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) v[j * 8 + e] = i0 + e < V ? __bfloat162float(r[i0 + e]) : -INFINITY;
            }
        }
    } else {
        const float *r = reinterpret_cast<const float *>(row);
        const bool aligned = ((reinterpret_cast<uintptr_t>(r) & 15) == 0);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i0 = base + j * 2048 + tid * 8;
            if (full && aligned) {
                const float4 a = __ldg(reinterpret_cast<const float4 *>(r + i0));
                const float4 b = __ldg(reinterpret_cast<const float4 *>(r + i0 + 4));
                v[j * 8 + 0] = a.x; v[j * 8 + 1] = a.y; v[j * 8 + 2] = a.z; v[j * 8 + 3] = a.w;
                v[j * 8 + 4] = b.x; v[j * 8 + 5] = b.y; v[j * 8 + 6] = b.z; v[j * 8 + 7] = b.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) v[j * 8 + e] = i0 + e < V ? r[i0 + e] : -INFINITY;
            }
        }
    }
}

// Block-wide max (blockDim.x == kStatThreads).  `red` holds >= 8 floats.
__device__ __forceinline__ float block_max256(float v, float *red) {
    v = warp_max(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int i = 1; i < kStatThreads / 32; ++i) r = fmaxf(r, red[i]);
    return r;
}

// Block-wide sum in double with a fixed order (blockDim.x == nthreads).
template <int NT>
__device__ __forceinline__ double block_sum_d(double v, double *red) {
    v = warp_sum_d(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    double r = 0.0;
#pragma unroll 1
    for (int i = 0; i < NT / 32; ++i) r += red[i];
    return r;
}

// Statistics (max, sum exp) of the 32 values of every thread of the block (missing entries -inf); every
// thread returns them.
__device__ __forceinline__ ChunkStat stat_of(const float (&v)[32], float *redf, double *redd) {
    float mx = -INFINITY;
#pragma unroll
    for (int e = 0; e < 32; ++e) mx = fmaxf(mx, v[e]);
    mx = block_max256(mx, redf);
    const float ms = mx * kLog2e;
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) s += fast_exp2(fmaf(v[e], kLog2e, -ms));
    ChunkStat st;
    st.m = mx;
    st.pad = 0.f;
    st.z = block_sum_d<kStatThreads>((double)s, redd);
    return st;
}

// Statistics (max, sum exp) of chunk c of one logit row; every thread returns them.
__device__ __forceinline__ ChunkStat chunk_stat(const void *row, int dtype, int V, int c, float *redf, double *redd) {
    float v[32];
    load_chunk32(row, dtype, V, c, v);
    return stat_of(v, redf, redd);
}

// The verify's target logits from an AR value zp and a diffusion value zq: lambda * zp + (1 - lambda) * zq,
// with the endpoints taken as stored (an infinite logit never meets a zero weight).
__device__ __forceinline__ float mix_logit(float zp, float zq, float lambda) {
    if (lambda == 1.f) return zp;
    if (lambda == 0.f) return zq;
    return fmaf(lambda, zp, (1.f - lambda) * zq);
}

// Grid-wide barrier of a cooperative launch: every CTA arrives on `counter` (zeroed before the launch, one
// increment per CTA per barrier) and waits until it reaches `target`.  The wait is bounded: after `limit`
// clock cycles the CTA raises TIDAR_DEV_TIMEOUT and returns false.  Writes before the barrier are visible to
// reads after it in every CTA (release on arrival, acquire on the wait; read such data with __ldcg).
__device__ __forceinline__ bool grid_barrier(unsigned *counter, unsigned target, int32_t *dev_status,
                                             long long limit) {
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;\n" ::"l"(counter) : "memory");
        int ok = 1;
        const long long t0 = clock64();
        while (true) {
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(counter) : "memory");
            if (v >= target) break;
            if (clock64() - t0 > limit) {
                atomicOr(dev_status, TIDAR_DEV_TIMEOUT);
                ok = 0;
                break;
            }
            __nanosleep(32);
        }
        __threadfence();
        s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
}

// This thread's 32 consecutive entries (tid*32 .. tid*32+31) of chunk c (256 threads), -inf beyond V.
__device__ __forceinline__ void load_chunk32_contig(const void *row, int dtype, int V, int c, float (&v)[32]) {
    const int i0 = c * kChunk + threadIdx.x * 32;
    if (dtype == TIDAR_DT_BF16) {
        const bf16 *r = reinterpret_cast<const bf16 *>(row);
        if (i0 + 32 <= V && ((reinterpret_cast<uintptr_t>(r + i0) & 15) == 0)) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 u = __ldg(reinterpret_cast<const uint4 *>(r + i0) + q);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    v[q * 8 + 2 * e] = __uint_as_float(w[e] << 16);
                    v[q * 8 + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
                }
            }
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = i0 + e < V ? __bfloat162float(r[i0 + e]) : -INFINITY;
        }
    } else {
        const float *r = reinterpret_cast<const float *>(row);
        if (i0 + 32 <= V && ((reinterpret_cast<uintptr_t>(r + i0) & 15) == 0)) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 a = __ldg(reinterpret_cast<const float4 *>(r + i0) + q);
                v[q * 4 + 0] = a.x; v[q * 4 + 1] = a.y; v[q * 4 + 2] = a.z; v[q * 4 + 3] = a.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = i0 + e < V ? r[i0 + e] : -INFINITY;
        }
    }
}

// Ordered search inside one chunk with 256 threads holding 32 consecutive weights each (entries
// tid*32 .. tid*32+31): the first local index whose inclusive sum exceeds `target`, or the last
// index with positive weight when rounding leaves none (target beyond the chunk's total).
__device__ __forceinline__ int chunk_search256(const double (&w)[32], double target, double *scan_buf, int *pick) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    double loc = 0.0;
#pragma unroll
    for (int e = 0; e < 32; ++e) loc += w[e];
    double incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (tid == 0) { pick[0] = 0x7fffffff; pick[1] = -1; }
    if (lane == 31) scan_buf[warp] = incl;
    __syncthreads();
    double before = 0.0;
    for (int i = 0; i < warp; ++i) before += scan_buf[i];
    double c = before + incl - loc;  // exclusive prefix of this thread
    int first = 0x7fffffff, last = -1;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        c += w[e];
        if (w[e] > 0.0) {
            last = tid * 32 + e;
            if (c > target && first == 0x7fffffff) first = tid * 32 + e;
        }
    }
    if (first != 0x7fffffff) atomicMin(&pick[0], first);
    if (last >= 0) atomicMax(&pick[1], last);
    __syncthreads();
    return pick[0] != 0x7fffffff ? pick[0] : pick[1];
}

// Merge of chunk statistics by up to 32 lanes of one warp (lane c takes chunk c, c + 32, ...):
// every lane returns the row max m and the row sum Z of exp(x - m).
__device__ __forceinline__ void merge_stats_warp(const ChunkStat *st, int n, float &m, double &z) {
    const int lane = threadIdx.x & 31;
    float mx = -INFINITY;
    for (int c = lane; c < n; c += 32) mx = fmaxf(mx, __ldcg(&st[c].m));
    m = warp_max(mx);
    double s = 0.0;
    for (int c = lane; c < n; c += 32) {
        const float mc = __ldcg(&st[c].m);
        if (mc != -INFINITY) s += __ldcg(&st[c].z) * (double)exp2f((mc - m) * kLog2e);
    }
    z = warp_sum_d(s);
}

}  // namespace tidar
