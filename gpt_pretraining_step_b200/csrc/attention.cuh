// Launchers of the causal flash-attention kernels (internal to the library).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace gpt {

using bf16 = __nv_bfloat16;

// q [B, H, T, 128], k, v [B, Hkv, T, 128] -> o [B, T, H, 128], lse [B, H, T]
// (natural log).  Hkv <= 0 means Hkv = H (it must divide H); window < 0 (or
// >= T) is full causal attention, else query t sees keys t - window .. t.
// err: device error word for expired waits (may be null).  sched: a device
// int the persistent kernel hands out its work with (zeroed here, on s); null
// takes one of the library's own.  kv_stride: heads per batch row in the
// k/v (and dk/dv) buffers, kv head j of batch b at row b*kv_stride + j (0:
// Hkv, dense).  wait_cycles: bound of every device-side wait in SM cycles
// (<= 0: the library default).
void launch_attn_fwd(const bf16* q, const bf16* k, const bf16* v, bf16* o, float* lse, int B, int H, int T,
                     cudaStream_t s, int* err, int Hkv = 0, int window = -1, int* sched = nullptr,
                     int kv_stride = 0, long long wait_cycles = 0);

// Gradients of o w.r.t. q, k, v given dout [B, T, H, 128]: dq (fp32
// [B, H, T, 128], zeroed here, then accumulated), dk, dv [B, kv_stride, T,
// 128] with the kv heads at rows h < Hkv (summed over the query heads of each
// kv head); Dv [B, H, T] is scratch; sched as for the forward.
// With dqkv, dk and dv are not written: dV goes to the v columns of the
// token-major gradient rows dqkv [B*T, (H + 2 Hkv) * 128] and dK, taken
// through the backward of the QK RMS norm (k holds the normalised rotated
// keys, rk [B*T, H] their inverse RMS, kv head h at column h) and of the
// rotation (rope [T, 64] (cos, sin) of the pairs (i, 64 + i)), to its k
// columns; the q columns are left to the caller.  d_ready: Dv already holds
// D = rowsum(dout * o) (the dout GEMM's epilogue computed it).
void launch_attn_bwd(const bf16* q, const bf16* k, const bf16* v, const bf16* o, const bf16* dout,
                     const float* lse, float* Dv, float* dq, bf16* dk, bf16* dv, int B, int H, int T,
                     cudaStream_t s, int* err, int Hkv = 0, int window = -1, int* sched = nullptr,
                     int kv_stride = 0, long long wait_cycles = 0, const float* rk = nullptr,
                     const float2* rope = nullptr, bf16* dqkv = nullptr, bool d_ready = false);

}  // namespace gpt
