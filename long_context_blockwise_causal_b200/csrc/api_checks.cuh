// Host-side argument checks shared by the forward entry points.
#pragma once

#include <stdint.h>

namespace lwm {

// Returned by check_fwd_args for a valid call with no work (B, N or H is 0).
constexpr int kFwdNothingToDo = -1;

// Every check lwm_blockattn_fwd makes before it looks at its workspace:
// sizes, RoPE layout, theta, dtype, qk precision, supported shape, max_pos
// and the non-null, 16-byte-aligned input and output pointers. Returns
// LWM_OK, kFwdNothingToDo or the LWM_ERR_* status the call must return.
int check_fwd_args(const void* q, const void* k, const void* v,
                   const int32_t* segment_ids, const int32_t* positions,
                   double theta, int block_q, int block_k, int max_pos, int B,
                   int N, int H, int D, int dtype, int qk_precision,
                   int rope_layout, const void* out, const float* lse);

}  // namespace lwm
