// Decode attention (one query token per (batch row, head) against a cache).
#pragma once

#include "common.cuh"

namespace lwm {

// Number of key chunks (CTAs) per (batch row, head) for a cache of L keys.
int decode_splits(int L);

// Partials: part_m, part_l [B][H][splits], part_acc [B][H][splits][128].
// `half`: q and the cached keys in the rotate-half RoPE layout. `status`:
// device word that records LWM_ERR_TIMEOUT if a load never lands.
cudaError_t launch_decode(const void* q, const void* k_rot, const void* v,
                          const int32_t* kv_start, const int32_t* kv_len,
                          const int32_t* q_pos, const float* table,
                          int max_pos, int B, int L, int H, bool half,
                          void* out, float* lse, float* part_m, float* part_l,
                          float* part_acc, int* status, cudaStream_t st);

}  // namespace lwm
