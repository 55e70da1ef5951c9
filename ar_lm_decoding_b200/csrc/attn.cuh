// Parameters shared by the attention kernels and the split combine.
#pragma once

#include "common.cuh"

namespace tidar {

struct AttnParams {
    const bf16 *q, *k_new, *v_new, *k_cache, *v_cache;
    const int32_t *prefix_len;
    int B, Hq, Hkv, D, k, R, G, M, P_max;
    float scale_log2;  // softmax_scale * log2(e)
    int mask_mode;
    int n_splits;      // key ranges per (sequence, KV head, row tile): the cluster size
    int Mpad;          // M rounded up to the row tile
    bf16 *out;         // [B, R, Hq, D]
    float *lse;        // [B, R, Hq] or null
    int32_t *dev_status;
    // paged KV cache (null: contiguous [B, Hkv, P_max, D] caches): cache row n of sequence b is row n % 64 of
    // page block_table[b * max_pages + n / 64] of the pool [num_pages, Hkv, 64, D]; P_max = 64 * max_pages
    const int32_t *block_table;
    int max_pages, num_pages;
    long long wait_cycles;  // bound of every on-chip wait, in SM clock cycles
    int stall_test;         // 1: the QK issuer first waits on a barrier nothing arrives on (timeout test)
};

// Bound of the on-chip waits of a normal launch (about 2 s at the B200's clocks).
constexpr long long kAttnWaitCycles = 4000000000LL;

int attn_sm100_rows_per_tile();
int attn_sm100_keys_per_tile();
int attn_sm100_pick_splits(int D, long groups, int max_tiles);
int attn_sm100_max_splits();
cudaError_t attn_sm100_launch(const AttnParams &p, cudaStream_t s);

}  // namespace tidar
