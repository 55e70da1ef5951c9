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
};

int attn_sm100_rows_per_tile();
int attn_sm100_keys_per_tile();
int attn_sm100_pick_splits(int D, long groups, int max_tiles);
int attn_sm100_max_splits();
cudaError_t attn_sm100_launch(const AttnParams &p, cudaStream_t s);

}  // namespace tidar
