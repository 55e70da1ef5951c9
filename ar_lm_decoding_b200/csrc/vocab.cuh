// Vocabulary chunking shared by the verify and the draft selection.
#pragma once

#include "common.cuh"

namespace tidar {

constexpr int kChunk = 8192;        // vocabulary entries per CTA
constexpr int kStatThreads = 256;   // kChunk / kStatThreads = 32 entries per thread
static_assert(kMaxVocab == 64 * kChunk, "a row's chunk statistics are held two per lane of one warp");

__host__ __device__ inline int vocab_chunks(int V) { return (V + kChunk - 1) / kChunk; }

// The verify's target logits from an AR value zp and a diffusion value zq: lambda * zp + (1 - lambda) * zq,
// with the endpoints taken as stored (an infinite logit never meets a zero weight).
__device__ __forceinline__ float mix_logit(float zp, float zq, float lambda) {
    if (lambda == 1.f) return zp;
    if (lambda == 0.f) return zq;
    return fmaf(lambda, zp, (1.f - lambda) * zq);
}

}  // namespace tidar
