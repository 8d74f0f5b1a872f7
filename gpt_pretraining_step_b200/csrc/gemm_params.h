// Epilogue kinds and kernel parameters of the tcgen05 GEMM (host and device).
#pragma once

#include <cuda_runtime.h>

namespace gpt {

enum EpiKind : int {
  EPI_STORE = 0,    // out = acc                       (OutT)
  EPI_ACC = 1,      // out += acc                      (fp32)
  EPI_RELU2 = 2,    // out = relu(acc)^2               (bf16)
  EPI_DRELU2 = 3,   // out = acc * 2 sqrt(aux)         (bf16, aux = relu(u)^2 in bf16)
  EPI_AXPBY = 4,    // out = alpha * aux + beta * acc  (OutT, aux AuxT)
  EPI_QKV = 5,      // RoPE + per-head RMSNorm, scatter to q/k/v [B, H, T, 128]
  EPI_LOGITS = 6,   // out = acc (bf16) + per-(row, tile) softmax partials
};

struct GemmParams {
  int M, N, K, batch;
  int tiles_m, tiles_n, kblocks, splits, kb_per_split, sym, units;
  void* out;
  long long ldo, out_bs, split_stride;
  const void* aux;
  long long ld_aux, aux_bs;
  float alpha, beta;
  float gamma;          // AXPBY: added to the diagonal elements (row == column) of every output matrix
  int split_lo;         // 1: the second (fp16) output holds out - fp16(out), the rounding residual of
                        //   the fp16 main output, so that the pair carries ~22 significant bits
  int row_dot;          // STORE, bf16 output, BN 256: also f32a[(b H + h) T + t] = the sum over head h's
                        //   128 columns of row b T + t of the stored values times aux (bf16, ld_aux)
  float* f32a;          // QKV: rstd of q [M, H];   LOGITS: (max, sumexp) pairs [M, tiles_n]
  float* f32b;          // QKV: rstd of k [M, H];   LOGITS: target logit [M]
  const int* tgt;       // LOGITS: targets of the rows
  const float2* rope;   // QKV: (cos, sin) pair-major [64, T]
  void* qkv_out[3];     // QKV: q, k, v [B, H, T, 128] bf16
  void* out_t;          // STORE/AXPBY: optional transposed copy of out, [N][M] with row stride ldo_t
  long long ldo_t;
  const float* dq_a;    // fp8 operands: device inverse scales of A and B; the accumulator is
  const float* dq_b;    //   multiplied by dq_a[z * dq_zs] * dq_b[z * dq_zs] before the epilogue
  int dq_zs;            //   (null: 1; dq_zs 1 = one scale per batch entry z, 0 = one for all)
  unsigned int* amax_out;   // RELU2 / DRELU2: optional 32 fp8 scale words, atomically raised to the
                            //   bits of max |bf16(out)| (each warp in one of them)
  int T, H;
  int Hkv;              // QKV: kv heads (0: H); columns are q (H heads) | k | v (Hkv heads each),
                        //   k and v stored at head rows b*H + j of their [B, H, T, 128] buffers
  int tma_out;          // 1: the main output is written by TMA stores through the output tensor map
  int tma_out2;         // 1: also an fp16 copy of the output, same layout, through the second map
  int tma_mirror;       // symmetric products, 16-bit output: the mirrored (transposed) tiles are
                        //   written by TMA through the second map (box 32 x 64, no swizzle)
  void* out2;           //   (its base; row stride ldo, batch stride out_bs)
  int* err;
  long long wait_cycles;   // bound of every mbarrier wait (SM cycles; <= 0: the library default)
};

}  // namespace gpt
