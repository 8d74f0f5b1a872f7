// Launchers of the causal flash-attention kernels (internal to the library).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace gpt {

using bf16 = __nv_bfloat16;

// q, k, v [B, H, T, 128] -> o [B, T, H, 128], lse [B, H, T] (natural log).
// err: device error word for expired waits (may be null).
void launch_attn_fwd(const bf16* q, const bf16* k, const bf16* v, bf16* o, float* lse, int B, int H, int T,
                     cudaStream_t s, int* err);

// Gradients of o w.r.t. q, k, v given dout [B, T, H, 128]: dq (fp32, zeroed
// here, then accumulated), dk, dv [B, H, T, 128]; Dv [B, H, T] is scratch.
void launch_attn_bwd(const bf16* q, const bf16* k, const bf16* v, const bf16* o, const bf16* dout,
                     const float* lse, float* Dv, float* dq, bf16* dk, bf16* dv, int B, int H, int T,
                     cudaStream_t s, int* err);

}  // namespace gpt
