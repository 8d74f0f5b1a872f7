// Host side of the tcgen05 GEMM: TMA tensor maps, tile/split bookkeeping and
// the table of compiled variants.
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "gemm.cuh"
#include "gemm.h"

namespace gpt {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

}  // namespace

// 3-D map over [batch][outer][inner] with 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* ptr, int es, long long inner, long long outer, long long batch,
              long long ld, long long bs, int box_inner, int box_outer, bool f16, bool swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  if (bs == 0 || batch == 1) bs = ld * outer;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer),
                        static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld * es), static_cast<cuuint64_t>(bs * es)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (strides[0] & 15) || (strides[1] & 15)) return false;
  const CUtensorMapDataType dt =
      es == 2 ? (f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16)
              : (es == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_UINT8);
  CUresult r = fn(m, dt, 3,
                  const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 4-D bf16 map over dims {d0, d1, d2, d3} (d0 innermost) with byte strides
// s1, s2, s3 of dims 1..3, box {b0, b1, b2, b3}, 128-byte swizzle.
bool make_map_4d(CUtensorMap* m, const void* ptr, const long long (&dims)[4], const long long (&strides)[3],
                 const int (&box)[4]) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[4], gs[3];
  cuuint32_t bx[4], es[4] = {1, 1, 1, 1};
  for (int i = 0; i < 4; ++i) {
    gd[i] = static_cast<cuuint64_t>(dims[i]);
    bx[i] = static_cast<cuuint32_t>(box[i]);
  }
  for (int i = 0; i < 3; ++i) {
    gs[i] = static_cast<cuuint64_t>(strides[i]);
    if (gs[i] & 15) return false;
  }
  if (reinterpret_cast<uintptr_t>(ptr) & 15) return false;
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), gd, gs, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

using bf16 = __nv_bfloat16;
using f16 = __half;

// The paired variants compiled (16- and 8-bit operands, BN 256), one line each:
// operand type, A and B MN-major, epilogue, output and aux types.
#define GPT_GEMM_PAIR_LIST(X)                            \
  X(bf16, false, true, EPI_QKV, bf16, bf16)              \
  X(bf16, false, true, EPI_ACC, float, float)            \
  X(bf16, false, true, EPI_RELU2, bf16, bf16)            \
  X(bf16, false, true, EPI_LOGITS, bf16, bf16)           \
  X(bf16, false, true, EPI_STORE, bf16, bf16)            \
  X(bf16, false, true, EPI_STORE, float, float)          \
  X(bf16, false, false, EPI_DRELU2, bf16, bf16)          \
  X(bf16, false, false, EPI_STORE, float, float)         \
  X(bf16, false, false, EPI_STORE, bf16, bf16)           \
  X(bf16, true, true, EPI_STORE, float, float)           \
  X(bf16, true, true, EPI_ACC, float, float)             \
  X(bf16, true, false, EPI_STORE, float, float)          \
  X(f16, false, true, EPI_AXPBY, f16, float)             \
  X(f16, false, true, EPI_AXPBY, f16, f16)               \
  X(f16, false, true, EPI_AXPBY, float, f16)             \
  X(f16, false, false, EPI_STORE, f16, f16)              \
  X(f16, false, false, EPI_AXPBY, f16, f16)              \
  X(uint8_t, false, true, EPI_ACC, float, float)         \
  X(uint8_t, false, true, EPI_RELU2, bf16, bf16)         \
  X(uint8_t, false, true, EPI_STORE, float, float)       \
  X(uint8_t, false, false, EPI_STORE, float, float)      \
  X(uint8_t, false, false, EPI_DRELU2, bf16, bf16)       \
  X(uint8_t, false, false, EPI_STORE, bf16, bf16)        \
  X(uint8_t, true, true, EPI_STORE, float, float)        \
  X(uint8_t, true, true, EPI_ACC, float, float)

bool pair_variant_exists(const GemmCall& c) {
#define GPT_GEMM_PAIR_HAS(T_, AMN_, BMN_, EPI_, OUT_, AUX_)                                                     \
  if (c.es == (int)sizeof(T_) && c.a_mn == AMN_ && c.b_mn == BMN_ && c.epi == EPI_ &&                          \
      c.out_es == (int)sizeof(OUT_) && c.aux_es == (int)sizeof(AUX_) && c.f16 == std::is_same<T_, f16>::value && \
      c.out_f16 == std::is_same<OUT_, f16>::value && c.aux_f16 == std::is_same<AUX_, f16>::value)                \
    return true;
  GPT_GEMM_PAIR_LIST(GPT_GEMM_PAIR_HAS)
#undef GPT_GEMM_PAIR_HAS
  return false;
}

template <typename T, int BN, bool A_MN, bool B_MN, int EPI, typename OutT, typename AuxT, bool PAIR = false>
cudaError_t launch(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mc, const CUtensorMap& md,
                   const GemmParams& p, cudaStream_t s) {
  using C = GemmCfg<sizeof(T), BN, PAIR>;
  auto kern = gemm_tc_kernel<T, BN, A_MN, B_MN, EPI, OutT, AuxT, PAIR>;
  static std::atomic<unsigned long long> configured{0};
  cudaError_t e = set_smem_limit_once(kern, C::SMEM, configured);
  if (e != cudaSuccess) return e;
  if constexpr (!PAIR) {
    const int grid = p.units < device_sm_count() ? p.units : device_sm_count();
    kern<<<grid, 320, C::SMEM, s>>>(ma, mb, mc, md, p);
  } else {
    // persistent pairs: as many clusters of two as fit at once, at most one per unit
    static std::atomic<int> max_clusters{0};
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(320, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int mc2 = max_clusters.load(std::memory_order_relaxed);
    if (mc2 <= 0) {
      cfg.gridDim = dim3(2 * (device_sm_count() / 2), 1, 1);
      if (cudaOccupancyMaxActiveClusters(&mc2, kern, &cfg) != cudaSuccess || mc2 <= 0) return cudaErrorInvalidValue;
      max_clusters.store(mc2, std::memory_order_relaxed);
    }
    const int nclusters = p.units < mc2 ? p.units : mc2;
    cfg.gridDim = dim3(2 * nclusters, 1, 1);
    e = cudaLaunchKernelEx(&cfg, kern, ma, mb, mc, md, p);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace

int device_sm_count() {
  // per device (a process may drive GPUs of different sizes)
  static std::atomic<int> n[64];
  int dev = 0;
  cudaGetDevice(&dev);
  std::atomic<int>& slot = n[dev & 63];
  int v = slot.load(std::memory_order_relaxed);
  if (v <= 0) {
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (v <= 0) v = 148;
    slot.store(v, std::memory_order_relaxed);
  }
  return v;
}

int gemm_tiles(const GemmCall& c) {
  const int tm = (c.M + 127) / 128;
  const int tn = (c.N + c.bn - 1) / c.bn;
  return (c.sym ? tm * (tm + 1) / 2 : tm * tn) * c.batch;
}

cudaError_t gemm_run(GemmCall& c, cudaStream_t stream) {
  if (c.M <= 0 || c.N <= 0 || c.batch <= 0) return cudaSuccess;
  if (c.K <= 0 || (c.bn != 128 && c.bn != 256) || (c.es != 1 && c.es != 2 && c.es != 4)) return cudaErrorInvalidValue;
  if (c.sym && c.M != c.N) return cudaErrorInvalidValue;
  if (c.N % 8) return cudaErrorInvalidValue;
  // 32-bit operands are staged K-major only (the 128-byte swizzle atom used here
  // describes MN-major layouts of 16-bit types)
  if (c.es == 4 && (c.a_mn || c.b_mn)) return cudaErrorInvalidValue;
  const int bk = 128 / c.es;
  GemmParams& p = c.p;
  p.M = c.M; p.N = c.N; p.K = c.K; p.batch = c.batch;
  p.tiles_m = (c.M + 127) / 128;
  p.tiles_n = (c.N + c.bn - 1) / c.bn;
  p.kblocks = (c.K + bk - 1) / bk;
  int splits = c.splits < 1 ? 1 : c.splits;
  if (splits > p.kblocks) splits = p.kblocks;
  p.kb_per_split = (p.kblocks + splits - 1) / splits;
  p.splits = (p.kblocks + p.kb_per_split - 1) / p.kb_per_split;
  p.sym = c.sym ? 1 : 0;
  c.pair = c.allow_pair && c.bn == 256 && (c.es == 2 || c.es == 1) && c.M > 128 &&
           wait_limit_or_default(p.wait_cycles) >= kShortWaitCycles && pair_variant_exists(c);
  if (c.pair) p.tiles_m = (p.tiles_m + 1) / 2;   // one unit per 256-row block: the kernel's index counts pairs
  const long long ntiles =
      c.sym ? sym_tile_count(p.tiles_m, p.tiles_n, c.pair ? 1 : c.bn / 128) : 1ll * p.tiles_m * p.tiles_n;
  const long long units = ntiles * p.splits * c.batch;
  if (units > 0x7fffffffll) return cudaErrorInvalidValue;
  p.units = static_cast<int>(units);

  CUtensorMap ma, mb;
  const int mn_box = bk;   // 128 bytes of the MN dimension
  bool ok;
  if (!c.a_mn)
    ok = make_map(&ma, c.A, c.es, c.K, c.M, c.batch, c.lda, c.a_bs, bk, 128, c.f16);
  else
    ok = make_map(&ma, c.A, c.es, c.M, c.K, c.batch, c.lda, c.a_bs, mn_box, bk, c.f16);
  if (!ok) return cudaErrorInvalidValue;
  if (!c.b_mn)
    ok = make_map(&mb, c.B, c.es, c.K, c.N, c.batch, c.ldb, c.b_bs, bk, c.pair ? c.bn / 2 : c.bn, c.f16);
  else
    ok = make_map(&mb, c.B, c.es, c.N, c.K, c.batch, c.ldb, c.b_bs, mn_box, bk, c.f16);
  if (!ok) return cudaErrorInvalidValue;

  // Output written by TMA stores of 32-row x 128-byte boxes when the output's
  // base and strides are 16-byte aligned; otherwise by per-thread stores.
  // The map's third dimension is the batch index, or the K split of a
  // split-K partial (never both).
  CUtensorMap mc;
  p.tma_out = 0;
  if (c.epi == EPI_QKV) {
    // q, k, v [B, H, T, 128] bf16 as one 4-D map {dim, t, b*H + head, which};
    // a 32-token box stays inside one sequence when T is a multiple of 32
    const long long gap = static_cast<const char*>(p.qkv_out[1]) - static_cast<const char*>(p.qkv_out[0]);
    const long long gap2 = static_cast<const char*>(p.qkv_out[2]) - static_cast<const char*>(p.qkv_out[1]);
    if (p.T > 0 && p.T % 32 == 0 && c.M % p.T == 0 && gap > 0 && gap == gap2) {
      const long long dims[4] = {128, p.T, 1ll * (c.M / p.T) * p.H, 3};
      const long long strides[3] = {256, 256ll * p.T, gap};
      const int box[4] = {64, 32, 1, 1};
      if (make_map_4d(&mc, p.qkv_out[0], dims, strides, box)) p.tma_out = 1;
    }
  } else if (!(c.batch > 1 && p.splits > 1) && (c.out_es == 2 || c.out_es == 4)) {
    const long long n3 = p.splits > 1 ? p.splits : c.batch;
    const long long s3 = p.splits > 1 ? p.split_stride : p.out_bs;
    if (make_map(&mc, p.out, c.out_es, c.N, c.M, n3, p.ldo, s3, 128 / c.out_es, 32, c.out_f16)) p.tma_out = 1;
  }
  // optional fp16 copy of the output (plain batched layouts only)
  CUtensorMap md;
  p.tma_out2 = 0;
  if (p.split_lo && (!p.out2 || p.out_t || c.out_es != 2 || !c.out_f16 || c.sym)) return cudaErrorInvalidValue;
  if (p.row_dot && (c.epi != EPI_STORE || c.out_es != 2 || c.out_f16 || c.bn != 256 || c.batch != 1 || c.sym ||
                    p.splits > 1 || c.N % 128 || !p.aux || !p.f32a || p.T <= 0 || c.M % p.T || p.H * 128 != c.N ||
                    (p.ld_aux & 7) || (reinterpret_cast<uintptr_t>(p.aux) & 15)))
    return cudaErrorInvalidValue;
  p.tma_mirror = 0;
  if (p.out2) {
    if (c.epi == EPI_QKV || c.epi == EPI_LOGITS || p.splits > 1 || !p.tma_out) return cudaErrorInvalidValue;
    if (!make_map(&md, p.out2, 2, c.N, c.M, c.batch, p.ldo, p.out_bs, 64, 32, true)) return cudaErrorInvalidValue;
    p.tma_out2 = 1;
  } else if (c.sym && p.tma_out && c.out_es == 2 && !p.out_t && p.splits == 1 &&
             make_map(&md, p.out, 2, c.N, c.M, c.batch, p.ldo, p.out_bs, 32, 64, c.out_f16, false)) {
    // the transposed copies of a symmetric product's off-diagonal tiles: a
    // warp's 32 rows x 64 columns land as 64 rows x 32 columns
    p.tma_mirror = 1;
  } else {
    md = ma;   // unused by the kernel
  }
  // fp32 accumulation (out += acc) is done by TMA add-reduction only
  if (c.epi == EPI_ACC && !p.tma_out) return cudaErrorInvalidValue;
  if (!p.tma_out) mc = ma;   // unused by the kernel

#define GPT_GEMM_MATCH(T_, BN_, AMN_, BMN_, EPI_, OUT_, AUX_)                                        \
  (c.es == (int)sizeof(T_) && c.bn == BN_ && c.a_mn == AMN_ && c.b_mn == BMN_ && c.epi == EPI_ &&       \
   c.out_es == (int)sizeof(OUT_) && c.aux_es == (int)sizeof(AUX_) && c.f16 == std::is_same<T_, f16>::value && \
   c.out_f16 == std::is_same<OUT_, f16>::value && c.aux_f16 == std::is_same<AUX_, f16>::value)
#define GPT_GEMM_CASE(T_, BN_, AMN_, BMN_, EPI_, OUT_, AUX_)                                        \
  if (!c.pair && GPT_GEMM_MATCH(T_, BN_, AMN_, BMN_, EPI_, OUT_, AUX_))                            \
    return launch<T_, BN_, AMN_, BMN_, EPI_, OUT_, AUX_>(ma, mb, mc, md, p, stream);
#define GPT_GEMM_PAIR_CASE(T_, AMN_, BMN_, EPI_, OUT_, AUX_)                                       \
  if (c.pair && GPT_GEMM_MATCH(T_, 256, AMN_, BMN_, EPI_, OUT_, AUX_))                             \
    return launch<T_, 256, AMN_, BMN_, EPI_, OUT_, AUX_, true>(ma, mb, mc, md, p, stream);

  // CTA pairs
  GPT_GEMM_PAIR_LIST(GPT_GEMM_PAIR_CASE)

  // forward
  GPT_GEMM_CASE(bf16, 256, false, true, EPI_QKV, bf16, bf16)
  GPT_GEMM_CASE(bf16, 256, false, true, EPI_ACC, float, float)
  GPT_GEMM_CASE(bf16, 256, false, true, EPI_RELU2, bf16, bf16)
  GPT_GEMM_CASE(bf16, 256, false, true, EPI_LOGITS, bf16, bf16)
  GPT_GEMM_CASE(bf16, 256, false, true, EPI_STORE, bf16, bf16)
  GPT_GEMM_CASE(bf16, 256, false, true, EPI_STORE, float, float)
  GPT_GEMM_CASE(bf16, 128, false, true, EPI_STORE, float, float)
  // backward: activation gradients (B is a weight read K-major)
  GPT_GEMM_CASE(bf16, 256, false, false, EPI_DRELU2, bf16, bf16)
  GPT_GEMM_CASE(bf16, 256, false, false, EPI_STORE, float, float)
  GPT_GEMM_CASE(bf16, 256, false, false, EPI_STORE, bf16, bf16)
  // backward: weight gradients (both operands token-major)
  GPT_GEMM_CASE(bf16, 256, true, true, EPI_STORE, float, float)
  GPT_GEMM_CASE(bf16, 256, true, true, EPI_ACC, float, float)
  GPT_GEMM_CASE(bf16, 256, true, false, EPI_STORE, float, float)
  // Newton-Schulz, bf16 steps
  GPT_GEMM_CASE(bf16, 128, false, false, EPI_STORE, bf16, bf16)
  GPT_GEMM_CASE(bf16, 128, false, false, EPI_AXPBY, bf16, bf16)
  GPT_GEMM_CASE(bf16, 256, false, true, EPI_AXPBY, bf16, bf16)
  // Newton-Schulz, tf32 steps
  GPT_GEMM_CASE(float, 128, false, false, EPI_STORE, float, float)
  GPT_GEMM_CASE(float, 128, false, false, EPI_AXPBY, float, float)
  GPT_GEMM_CASE(float, 256, false, false, EPI_AXPBY, float, float)
  GPT_GEMM_CASE(float, 256, false, false, EPI_AXPBY, bf16, float)
  // Newton-Schulz, fp16 steps (iterates as fp16 hi / lo pairs)
  GPT_GEMM_CASE(f16, 128, false, false, EPI_STORE, f16, f16)
  GPT_GEMM_CASE(f16, 128, false, false, EPI_AXPBY, f16, f16)
  GPT_GEMM_CASE(f16, 256, false, false, EPI_STORE, f16, f16)
  GPT_GEMM_CASE(f16, 256, false, false, EPI_AXPBY, f16, f16)
  GPT_GEMM_CASE(bf16, 256, false, false, EPI_AXPBY, bf16, bf16)
  GPT_GEMM_CASE(f16, 256, false, true, EPI_AXPBY, f16, float)   // first step: fp32 X in, hi / lo out
  GPT_GEMM_CASE(f16, 256, false, true, EPI_AXPBY, f16, f16)     // middle steps: lo in, hi / lo out
  GPT_GEMM_CASE(f16, 256, false, true, EPI_AXPBY, float, f16)   // last step: lo in, fp32 X out
  // fp8 e4m3 forward projections (operands as raw bytes)
  GPT_GEMM_CASE(uint8_t, 256, false, true, EPI_QKV, bf16, bf16)
  GPT_GEMM_CASE(uint8_t, 256, false, true, EPI_ACC, float, float)
  GPT_GEMM_CASE(uint8_t, 256, false, true, EPI_RELU2, bf16, bf16)
  GPT_GEMM_CASE(uint8_t, 256, false, true, EPI_STORE, float, float)
  GPT_GEMM_CASE(uint8_t, 256, false, false, EPI_STORE, float, float)
  // fp8 e4m3 backward: activation gradients against K-major weights, and the
  // weight gradients with both operands token-major
  GPT_GEMM_CASE(uint8_t, 256, false, false, EPI_DRELU2, bf16, bf16)
  GPT_GEMM_CASE(uint8_t, 256, false, false, EPI_STORE, bf16, bf16)
  GPT_GEMM_CASE(uint8_t, 256, true, true, EPI_STORE, float, float)
  GPT_GEMM_CASE(uint8_t, 256, true, true, EPI_ACC, float, float)
#undef GPT_GEMM_CASE
#undef GPT_GEMM_PAIR_CASE
#undef GPT_GEMM_MATCH
  return cudaErrorInvalidValue;
}

}  // namespace gpt
