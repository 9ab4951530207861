// Host-side argument checks shared by the attention entry points (internal).  Each returns
// DSA_OK or the status to return, with the reason recorded for dsa_last_error().
#pragma once

#include <stdint.h>

#include "../../include/dsa.h"

namespace dsa {

// dtype, pointers, sizes, gate, sm_scale, head shapes and 16-byte alignment of q/k/v/out/gate
// ([B,S,H,DQK] queries against [B,T,HKV,DQK] keys and [B,T,HKV,DV] values).
dsa_status check_attn_common(dsa_dtype dtype, const void* q, const void* k, const void* v,
                             const void* gate, dsa_gate_mode gm, float sm_scale, int B, int S,
                             int T, int H, int HKV, int DQK, int DV, const void* out);
// The index lists: present, K > 0, 16-byte aligned.
dsa_status check_idx_args(const int32_t* idx, int K);

}  // namespace dsa
