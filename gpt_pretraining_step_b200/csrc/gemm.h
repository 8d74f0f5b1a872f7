// Host interface of the tcgen05 GEMM (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "gemm_params.h"

namespace gpt {

// D[z](m, n) = sum_k A[z](m, k) B[z](n, k), z < batch.
//   A storage: a_mn ? [K][lda] (m contiguous) : [M][lda] (k contiguous); z stride a_bs
//   B storage: b_mn ? [K][ldb] (n contiguous) : [N][ldb] (k contiguous); z stride b_bs
//   es: operand element size, 2 = bf16 or (f16) fp16 (kind::f16), 4 = fp32 read as tf32 (kind::tf32),
//       1 = fp8 e4m3 (kind::f8f6f4; p.dq_a / p.dq_b dequantise the accumulator)
//   out_es / aux_es: element sizes of the epilogue output and auxiliary input
//   bn: 128 or 256 output columns per tile; splits: K split count (> 1 writes
//   partials at out + s * split_stride); sym: only tiles on or above the
//   diagonal are computed and mirrored (M == N, bn == 128).
struct GemmCall {
  int M = 0, N = 0, K = 0, batch = 1;
  int es = 2;
  bool a_mn = false, b_mn = false;
  const void* A = nullptr;
  long long lda = 0, a_bs = 0;
  const void* B = nullptr;
  long long ldb = 0, b_bs = 0;
  int bn = 256, splits = 1;
  bool sym = false;
  // CTA pairs (2-CTA clusters, M = 256 per tile) where the call allows them:
  // BN 256, 16- or 8-bit operands, a bound on waits of at least
  // kShortWaitCycles, and a compiled paired variant; else one CTA per tile
  bool allow_pair = true;
  bool pair = false;   // set by gemm_run: the call runs on CTA pairs
  int epi = 0, out_es = 4, aux_es = 4;
  bool f16 = false, out_f16 = false, aux_f16 = false;   // 16-bit operands / output / aux are fp16, not bf16
  GemmParams p{};   // epilogue fields (out, ldo, aux, ...) filled by the caller
};

// Returns cudaSuccess or the launch error; cudaErrorInvalidValue for a
// shape/alignment/variant the kernels do not cover.
cudaError_t gemm_run(GemmCall& c, cudaStream_t stream);

// Number of work units a call would launch without a K split.
int gemm_tiles(const GemmCall& c);

int device_sm_count();

// TMA descriptor of a bf16 (es = 2; fp16 with f16) or fp32 (es = 4) tensor [batch][outer][inner]
// with row stride ld and batch stride bs (elements), 128-byte swizzle (or
// none), box box_inner x box_outer.  False if the driver entry point is
// missing or the base/strides are not 16-byte aligned.
bool make_map(CUtensorMap* m, const void* ptr, int es, long long inner, long long outer, long long batch,
              long long ld, long long bs, int box_inner, int box_outer, bool f16 = false, bool swizzle = true);

// 4-D bf16 map, dims {d0 (innermost), d1, d2, d3}, byte strides of dims 1..3,
// box {b0, b1, b2, b3}, 128-byte swizzle.
bool make_map_4d(CUtensorMap* m, const void* ptr, const long long (&dims)[4], const long long (&strides)[3],
                 const int (&box)[4]);

}  // namespace gpt
