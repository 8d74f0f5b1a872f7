// tcgen05 GEMM for sm_100a: D[z][m][n] = sum_k A[z](m, k) * B[z](n, k), fp32
// accumulators in TMEM, operands staged by TMA into a 128-byte-swizzled
// shared-memory ring, and a fused epilogue.
//
// Roles (320 threads, one CTA per SM, persistent over work units):
//   warp 0      TMA producer (one elected lane)
//   warp 1      TMEM allocator and MMA issuer (one elected lane)
//   warps 2..9  epilogue: two warps per TMEM lane quarter, each thread owning
//               one accumulator row (TMEM lane) and half of the tile's columns
// Two accumulator buffers in TMEM let the epilogue of tile i overlap the
// MMAs of tile i+1.  Every mbarrier wait is bounded; on expiry the CTA
// raises an abort flag, drains its in-flight copies and MMAs, frees TMEM
// and returns with ERRF_TIMEOUT set in the error word.
#pragma once

#include <cuda_fp16.h>

#include <type_traits>

#include "common.cuh"
#include "gemm_params.h"

namespace gpt {

// 16-bit epilogue storage: bf16 or fp16 (pairs packed low element first)
template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (std::is_same<T, __half>::value) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    return pack_bf16x2(lo, hi);
  }
}
template <typename T>
__device__ __forceinline__ float lo16(uint32_t u) {
  if constexpr (std::is_same<T, __half>::value) return __half2float(__ushort_as_half(static_cast<unsigned short>(u & 0xFFFFu)));
  else return bf16_lo(u);
}
template <typename T>
__device__ __forceinline__ float hi16(uint32_t u) {
  if constexpr (std::is_same<T, __half>::value) return __half2float(__ushort_as_half(static_cast<unsigned short>(u >> 16)));
  else return bf16_hi(u);
}

template <int ES, int BN, bool PAIR = false>
struct GemmCfg {
  static constexpr int BK = 128 / ES;                 // elements of K per stage (one 128 B row)
  static constexpr int MMA_K = 32 / ES;               // K per tcgen05.mma (16 bf16, 8 tf32, 32 fp8)
  static constexpr int A_BYTES = 128 * 128;
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;   // rows (N) of B this CTA stages
  static constexpr int B_BYTES = B_ROWS * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = B_ROWS == 256 ? 4 : 6;
  static constexpr int CHUNK_BYTES = BK * 128;        // one MN-major box: BK rows of 128 B
  static constexpr int TMEM_COLS = 2 * BN;
  // output staging: one 32-row x 128-byte box per epilogue warp
  static constexpr int STG_BYTES = 8 * 4096;
  static constexpr int SMEM = STAGES * STAGE_BYTES + STG_BYTES + 1024 + 256;
};

// Tiles of a symmetric product (M == N) on or above the diagonal: row block m
// (128 rows) needs the column blocks (BN wide) from m / (BN / 128) on.
__host__ __device__ __forceinline__ int sym_tile_count(int tiles_m, int tiles_n, int rows_per_col_block) {
  int n = 0;
  for (int m = 0; m < tiles_m; ++m) n += tiles_n - m / rows_per_col_block;
  return n;
}

// (PAIR: mb counts 256-row blocks, so a row block of a symmetric product needs
// the column blocks from mb on)
template <int BN, bool PAIR = false>
__device__ __forceinline__ void decode_unit(const GemmParams& p, int u, int& z, int& mb, int& nb,
                                            int& kb0, int& kb1, int& split) {
  constexpr int R = PAIR ? 1 : BN / 128;
  const int ntiles = p.sym ? sym_tile_count(p.tiles_m, p.tiles_n, R) : p.tiles_m * p.tiles_n;
  const int per_z = ntiles * p.splits;
  z = u / per_z;
  int r = u - z * per_z;
  split = r / ntiles;
  int t = r - split * ntiles;
  if (p.sym) {
    int m = 0;
    while (t >= p.tiles_n - m / R) {
      t -= p.tiles_n - m / R;
      ++m;
    }
    mb = m;
    nb = m / R + t;
  } else {
    // Groups of 16 row blocks.  Inside a group, tiles that follow one another
    // go to CTAs (clusters) with adjacent indices, which in practice sit on
    // the same die and its half of L2, so they share the larger operand: the
    // column blocks of a row one after another when A (M x K) is the larger,
    // else the row blocks of a column (sharing the other way read the larger
    // operand from DRAM about twice, and for M << N many times over)
    constexpr int G = 16;
    const int gsz = G * p.tiles_n;
    const int g = t / gsz;
    const int first = g * G;
    const int gm = min(G, p.tiles_m - first);
    const int tt = t - g * gsz;
    if (p.tiles_m >= p.tiles_n) {
      mb = first + tt / p.tiles_n;
      nb = tt % p.tiles_n;
    } else {
      mb = first + tt % gm;
      nb = tt / gm;
    }
  }
  kb0 = split * p.kb_per_split;
  kb1 = min(p.kblocks, kb0 + p.kb_per_split);
}

// ------------------------------------------------------------ epilogue stores

template <typename OutT>
__device__ __forceinline__ void store_row32(OutT* dst, const float (&v)[32], int nvalid) {
  if constexpr (sizeof(OutT) == 2) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (8 * g < nvalid) {
        uint4 w;
        w.x = pack2<OutT>(v[8 * g + 0], v[8 * g + 1]);
        w.y = pack2<OutT>(v[8 * g + 2], v[8 * g + 3]);
        w.z = pack2<OutT>(v[8 * g + 4], v[8 * g + 5]);
        w.w = pack2<OutT>(v[8 * g + 6], v[8 * g + 7]);
        *reinterpret_cast<uint4*>(dst + 8 * g) = w;
      }
    }
  } else {
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      if (4 * g < nvalid)
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(dst) + 4 * g) =
            make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
    }
  }
}

template <typename AuxT>
__device__ __forceinline__ void load_row32(const AuxT* src, float (&v)[32], int nvalid) {
  if constexpr (sizeof(AuxT) == 2) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint4 w = make_uint4(0, 0, 0, 0);
      if (8 * g < nvalid)
        w = *reinterpret_cast<const uint4*>(src + 8 * g);
      v[8 * g + 0] = lo16<AuxT>(w.x); v[8 * g + 1] = hi16<AuxT>(w.x);
      v[8 * g + 2] = lo16<AuxT>(w.y); v[8 * g + 3] = hi16<AuxT>(w.y);
      v[8 * g + 4] = lo16<AuxT>(w.z); v[8 * g + 5] = hi16<AuxT>(w.z);
      v[8 * g + 6] = lo16<AuxT>(w.w); v[8 * g + 7] = hi16<AuxT>(w.w);
    }
  } else {
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
      if (4 * g < nvalid) w = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(src) + 4 * g);
      v[4 * g] = w.x; v[4 * g + 1] = w.y; v[4 * g + 2] = w.z; v[4 * g + 3] = w.w;
    }
  }
}

template <typename OutT>
__device__ __forceinline__ void store_scalar(OutT* dst, float x) {
  if constexpr (std::is_same<OutT, __half>::value)
    *reinterpret_cast<__half*>(dst) = __float2half_rn(x);
  else if constexpr (sizeof(OutT) == 2)
    *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(x);
  else
    *reinterpret_cast<float*>(dst) = x;
}

// Online (max, sum of exp) of one row's 32-column logits chunk starting at
// column col0 (columns >= n are ignored), and the target's logit if it falls
// in the chunk.
__device__ __forceinline__ void logits_chunk(const float (&v)[32], int col0, int n, int tg, float& mx, float& sm,
                                             float& zt, bool& have_t) {
  const int nvalid = min(32, n - col0);
  if (nvalid <= 0) return;
  float cm = -INFINITY;
#pragma unroll
  for (int j = 0; j < 32; ++j) if (j < nvalid) cm = fmaxf(cm, v[j]);
  if (cm > mx) { sm *= __expf(mx - cm); mx = cm; }
#pragma unroll
  for (int j = 0; j < 32; ++j) if (j < nvalid) sm += __expf(v[j] - mx);
  if (tg >= col0 && tg < col0 + 32) {
    // select without an indexed access, which would move v to local memory
    const int idx = tg - col0;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      asm("{\n\t.reg .pred q;\n\tsetp.eq.s32 q, %2, %3;\n\tselp.f32 %0, %1, %0, q;\n\t}"
          : "+f"(zt)
          : "f"(v[j]), "r"(j), "r"(idx));
    have_t = true;
  }
}

// ------------------------------------------------------------------ kernel

// PAIR: a cluster of two CTAs per M = 256 tile (see common.cuh); units then
// count tile pairs and p.tiles_m counts 256-row blocks.
template <typename T, int BN, bool A_MN, bool B_MN, int EPI, typename OutT, typename AuxT, bool PAIR = false>
__global__ void __launch_bounds__(320, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmD,
                   const __grid_constant__ GemmParams p) {
  constexpr int ES = sizeof(T);
  using C = GemmCfg<ES, BN, PAIR>;
  static_assert(!PAIR || ((ES == 2 || ES == 1) && BN == 256), "CTA pairs: 16- or 8-bit operands, 256-wide tiles");
  constexpr uint32_t IDESC = make_idesc(ES == 2 ? (std::is_same<T, __half>::value ? 0 : 1) : (ES == 4 ? 2 : 0), BN,
                                        A_MN, B_MN, PAIR ? 256 : 128);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stg_base = smem + C::STAGES * C::STAGE_BYTES;   // 1024-aligned output staging
  uint64_t* full = reinterpret_cast<uint64_t*>(stg_base + C::STG_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = warp_id();
  const int lane = lane_id();
  const long long wlim = wait_limit_or_default(p.wait_cycles);
  // work units: CTA pairs take every (gridDim.x / 2)-th unit, rank 1 the upper 128 rows
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int u_first = PAIR ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
  const int u_step = PAIR ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], PAIR ? 512 : 256);   // every epilogue thread (of both CTAs of a pair)
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (p.tma_out) tma_prefetch_desc(&tmC);
    if (p.tma_out2) tma_prefetch_desc(&tmD);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_holder, C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_holder, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();   // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  float amax = 0.f;   // DRELU2 epilogue: this thread's max |out| (of the bf16-rounded values) over its tiles

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int u = u_first; u < p.units && ok; u += u_step) {
        int z, mb, nb, kb0, kb1, split;
        decode_unit<BN, PAIR>(p, u, z, mb, nb, kb0, kb1, split);
        if constexpr (PAIR) mb = 2 * mb + static_cast<int>(rank);
        const int n0 = nb * BN + (PAIR ? 128 * static_cast<int>(rank) : 0);   // first B row staged here
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, wlim)) { ok = false; break; }
          uint8_t* sA = smem + stage * C::STAGE_BYTES;
          uint8_t* sB = sA + C::A_BYTES;
          const int k0 = kb * C::BK;
          if constexpr (PAIR) {
            // both CTAs' bytes complete on the leader's barrier, which the leader expects
            const uint32_t cb = cluster_addr(&full[stage], 0);
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
            if constexpr (!A_MN) {
              tma_load_3d_pair(sA, &tmA, cb, k0, mb * 128, z);
            } else {
#pragma unroll
              for (int j = 0; j < 128 / C::BK; ++j)
                tma_load_3d_pair(sA + j * C::CHUNK_BYTES, &tmA, cb, mb * 128 + j * C::BK, k0, z);
            }
            if constexpr (!B_MN) {
              tma_load_3d_pair(sB, &tmB, cb, k0, n0, z);
            } else {
#pragma unroll
              for (int j = 0; j < C::B_ROWS / C::BK; ++j)
                tma_load_3d_pair(sB + j * C::CHUNK_BYTES, &tmB, cb, n0 + j * C::BK, k0, z);
            }
          } else {
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          if constexpr (!A_MN) {
            tma_load_3d(sA, &tmA, &full[stage], k0, mb * 128, z);
          } else {
#pragma unroll
            for (int j = 0; j < 128 / C::BK; ++j)
              tma_load_3d(sA + j * C::CHUNK_BYTES, &tmA, &full[stage], mb * 128 + j * C::BK, k0, z);
          }
          if constexpr (!B_MN) {
            tma_load_3d(sB, &tmB, &full[stage], k0, n0, z);
          } else {
#pragma unroll
            for (int j = 0; j < BN / C::BK; ++j)
              tma_load_3d(sB + j * C::CHUNK_BYTES, &tmB, &full[stage], n0 + j * C::BK, k0, z);
          }
          }
          ++issued;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok && (!PAIR || leader)) {
        // let every copy this thread started land before the CTA exits (a pair's
        // copies complete on the leader's barriers, so only the leader can tell;
        // the closing cluster barrier keeps the other CTA until then)
        for (int s = 0; s < C::STAGES; ++s) {
          const bool used = s < stage || issued >= C::STAGES;
          const uint32_t par = s < stage ? phase : (phase ^ 1u);
          if (used) {
            for (uint32_t i = 0; i < (1u << 20) && !mbar_try_wait(&full[s], par); ++i) {}
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ----------------------------------------------------------------- MMA
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int u = u_first; u < p.units && ok; u += u_step, ++local) {
        int z, mb, nb, kb0, kb1, split;
        decode_unit<BN, PAIR>(p, u, z, mb, nb, kb0, kb1, split);
        const int acc = local & 1;
        const uint32_t acc_par = (local >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_par ^ 1u, abort_flag, p.err, wlim)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err, wlim)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t b0 = a0 + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = A_MN ? smem_desc_sw128(a0 + kk * C::MMA_K * 128, C::CHUNK_BYTES, 1024)
                                     : smem_desc_sw128(a0 + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? smem_desc_sw128(b0 + kk * C::MMA_K * 128, C::CHUNK_BYTES, 1024)
                                     : smem_desc_sw128(b0 + kk * 32, 16, 1024);
            const uint32_t accum = (kb > kb0 || kk > 0) ? 1u : 0u;
            if constexpr (PAIR && ES == 2)
              umma_f16_pair(d_tmem, ad, bd, IDESC, accum);
            else if constexpr (PAIR)
              umma_f8_pair(d_tmem, ad, bd, IDESC, accum);
            else if constexpr (ES == 2)
              umma_f16(d_tmem, ad, bd, IDESC, accum);
            else if constexpr (ES == 4)
              umma_tf32(d_tmem, ad, bd, IDESC, accum);
            else
              umma_f8(d_tmem, ad, bd, IDESC, accum);
          }
          if constexpr (PAIR)
            umma_commit_pair_both(&empty[stage]);
          else
            umma_commit(&empty[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if constexpr (PAIR)
          umma_commit_pair_both(&tfull[acc]);
        else
          umma_commit(&tfull[acc]);
      }
      // all MMAs of this thread complete before TMEM is released
      if constexpr (PAIR)
        umma_commit_pair_own(drain);
      else
        umma_commit(drain);
      for (uint32_t i = 0; i < (1u << 22) && !mbar_try_wait(drain, 0); ++i) {}
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int quarter = warp & 3;                 // TMEM lanes 32*quarter .. +31
    const int half = (warp - 2) >> 2;             // which half of the tile's columns
    const int r = quarter * 32 + lane;            // accumulator row within the tile
    constexpr int NCH = BN / 64;                  // 32-column chunks per half
    const int c_begin = half * NCH, c_end = c_begin + NCH;
    // This warp's output box: 32 rows x 128 bytes (32 fp32 or 64 bf16 columns),
    // laid out with the 128-byte swizzle of the output tensor map: 16-byte unit
    // u of box row i sits at unit u ^ (i & 7).  Lane i owns box row i.
    uint8_t* stg = stg_base + (warp - 2) * 4096;
    uint8_t* stg_row = stg + lane * 128;
    const int stg_sw = lane & 7;
    auto box_open = [&]() {
      if (lane == 0) bulk_wait_read_all();   // the previous box has been read by TMA
      __syncwarp();
    };
    auto box_put = [&](int u, uint4 w) { *reinterpret_cast<uint4*>(stg_row + ((u ^ stg_sw) << 4)) = w; };
    auto box_close = [&](const CUtensorMap* map, bool reduce, int col0, int row0, int z3) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && row0 < p.M && col0 < p.N) {
        if (reduce)
          tma_reduce_add_3d(map, stg, col0, row0, z3);
        else
          tma_store_3d(map, stg, col0, row0, z3);
        bulk_commit();
      }
    };
    // 64 accumulator columns (two 32-column halves) to boxes of type OT
    // through `map`: one 16-bit box or two fp32 boxes
    auto emit64_to = [&](auto tag, const CUtensorMap* map, bool reduce, const float (&v0)[32],
                         const float (&v1)[32], int col0, int row0, int z3) {
      using OT = decltype(tag);
      if constexpr (sizeof(OT) == 2) {
        box_open();
#pragma unroll
        for (int u = 0; u < 4; ++u)
          box_put(u, make_uint4(pack2<OT>(v0[8 * u], v0[8 * u + 1]), pack2<OT>(v0[8 * u + 2], v0[8 * u + 3]),
                                pack2<OT>(v0[8 * u + 4], v0[8 * u + 5]), pack2<OT>(v0[8 * u + 6], v0[8 * u + 7])));
#pragma unroll
        for (int u = 0; u < 4; ++u)
          box_put(4 + u, make_uint4(pack2<OT>(v1[8 * u], v1[8 * u + 1]), pack2<OT>(v1[8 * u + 2], v1[8 * u + 3]),
                                    pack2<OT>(v1[8 * u + 4], v1[8 * u + 5]), pack2<OT>(v1[8 * u + 6], v1[8 * u + 7])));
        box_close(map, reduce, col0, row0, z3);
      } else {
        box_open();
#pragma unroll
        for (int u = 0; u < 8; ++u)
          box_put(u, make_uint4(__float_as_uint(v0[4 * u]), __float_as_uint(v0[4 * u + 1]),
                                __float_as_uint(v0[4 * u + 2]), __float_as_uint(v0[4 * u + 3])));
        box_close(map, reduce, col0, row0, z3);
        box_open();
#pragma unroll
        for (int u = 0; u < 8; ++u)
          box_put(u, make_uint4(__float_as_uint(v1[4 * u]), __float_as_uint(v1[4 * u + 1]),
                                __float_as_uint(v1[4 * u + 2]), __float_as_uint(v1[4 * u + 3])));
        box_close(map, reduce, col0 + 32, row0, z3);
      }
    };
    // the main output (EPI_ACC adds into it)
    auto emit64 = [&](const float (&v0)[32], const float (&v1)[32], int col0, int row0, int z3) {
      emit64_to(OutT{}, &tmC, EPI == EPI_ACC, v0, v1, col0, row0, z3);
    };
    int local = 0;
    for (int u = u_first; u < p.units; u += u_step, ++local) {
      int z, mb, nb, kb0, kb1, split;
      decode_unit<BN, PAIR>(p, u, z, mb, nb, kb0, kb1, split);
      if constexpr (PAIR) mb = 2 * mb + static_cast<int>(rank);
      const int acc = local & 1;
      const uint32_t acc_par = (local >> 1) & 1;
      if constexpr (EPI == EPI_DRELU2 || EPI == EPI_AXPBY) {
        // pull this row's slice of the epilogue input into L2 while the MMAs run
        const int prow = mb * 128 + r;
        const int pcol = nb * BN + half * (BN / 2);
        if (prow < p.M && pcol < p.N) {
          const AuxT* src = reinterpret_cast<const AuxT*>(p.aux) + static_cast<long long>(z) * p.aux_bs +
                            static_cast<long long>(prow) * p.ld_aux + pcol;
          const uint32_t bytes = static_cast<uint32_t>(min(BN / 2, p.N - pcol) * sizeof(AuxT));
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
        }
      }
      bool got = mbar_wait(&tfull[acc], acc_par, abort_flag, p.err, wlim);
      __syncwarp();   // tcgen05.ld is warp-collective: reconverge after the spin
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN;
      const int row = mb * 128 + r;
      const bool row_ok = row < p.M;
      const int box_row0 = mb * 128 + quarter * 32;
      const int z3 = p.splits > 1 ? split : z;   // third coordinate of the output map
      float dqs = 1.f;   // dequantisation of fp8 operands
      if constexpr (ES == 1)
        dqs = (p.dq_a ? p.dq_a[z * p.dq_zs] : 1.f) * (p.dq_b ? p.dq_b[z * p.dq_zs] : 1.f);
      if constexpr (EPI == EPI_QKV) {
        // BN = 256: the tile holds heads 2*nb and 2*nb+1 of the H + 2 Hkv heads
        // of q|k|v for 128 tokens; the four warps of column half `half` own one
        // head whole, so the per-head norm needs no exchange between warps
        const int gh = 2 * nb + half;
        const int hkv = p.Hkv > 0 ? p.Hkv : p.H;
        if (gh < p.H + 2 * hkv) {
          const int which = gh < p.H ? 0 : (gh < p.H + hkv ? 1 : 2);
          const int head = gh - (which == 0 ? 0 : (which == 1 ? p.H : p.H + hkv));
          const int b = row / p.T;
          const int t = row - b * p.T;
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.qkv_out[which]) +
                               ((static_cast<long long>(b) * p.H + head) * p.T + t) * 128;
          const uint32_t hb = tbase + half * 128;   // TMEM columns of this head
          // the output box of 32 tokens x 64 dims at dims col0 (TMA path)
          const int bb = box_row0 / p.T, bt = box_row0 - bb * p.T;
          auto put_box = [&](int col0) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && box_row0 < p.M) {
              tma_store_4d(&tmC, stg, col0, bt, bb * p.H + head, which);
              bulk_commit();
            }
          };
          if (which == 2) {
#pragma unroll 1
            for (int c = 0; c < 4; c += 2) {
              float v0[32], v1[32];
              tmem_load32(hb + c * 32, v0);
              tmem_load32(hb + (c + 1) * 32, v1);
              if constexpr (ES == 1) {
#pragma unroll
                for (int j = 0; j < 32; ++j) { v0[j] *= dqs; v1[j] *= dqs; }
              }
              if (p.tma_out) {
                box_open();
#pragma unroll
                for (int u = 0; u < 4; ++u)
                  box_put(u, make_uint4(pack2<OutT>(v0[8 * u], v0[8 * u + 1]), pack2<OutT>(v0[8 * u + 2], v0[8 * u + 3]),
                                        pack2<OutT>(v0[8 * u + 4], v0[8 * u + 5]),
                                        pack2<OutT>(v0[8 * u + 6], v0[8 * u + 7])));
#pragma unroll
                for (int u = 0; u < 4; ++u)
                  box_put(4 + u, make_uint4(pack2<OutT>(v1[8 * u], v1[8 * u + 1]),
                                            pack2<OutT>(v1[8 * u + 2], v1[8 * u + 3]),
                                            pack2<OutT>(v1[8 * u + 4], v1[8 * u + 5]),
                                            pack2<OutT>(v1[8 * u + 6], v1[8 * u + 7])));
                put_box(c * 32);
              } else if (row_ok) {
                store_row32(dst + c * 32, v0, 32);
                store_row32(dst + (c + 1) * 32, v1, 32);
              }
            }
          } else {
            // a rotation keeps the sum of squares, so the norm is taken before RoPE
            float ss = 0.f;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              float v[32];
              tmem_load32(hb + c * 32, v);
#pragma unroll
              for (int j = 0; j < 32; ++j) ss = fmaf(v[j], v[j], ss);
            }
            ss *= dqs * dqs;
            const float rstd = rsqrtf(ss * (1.f / 128.f) + 1e-6f);
            if (row_ok) (which == 0 ? p.f32a : p.f32b)[static_cast<long long>(row) * p.H + head] = rstd;
            const float sc = rstd * dqs;
            // RoPE pairs (i, i + 64): each (cos, sin) is read once and gives output
            // dims i (into the staging box) and 64 + i (kept packed until the
            // first box has gone out)
            uint32_t keep[32];
            if (p.tma_out) box_open();
#pragma unroll 1
            for (int pc = 0; pc < 2; ++pc) {
              float lo[32], hi[32];
              tmem_load32(hb + pc * 32, lo);
              tmem_load32(hb + 64 + pc * 32, hi);
              // pair-major table: the warp's 32 consecutive tokens read one pair coalesced
              const float2* cs = p.rope + static_cast<long long>(pc * 32) * p.T + t;
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                float o0[8], o1[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                  const int j = 8 * u + jj;
                  const float2 e = row_ok ? cs[static_cast<long long>(j) * p.T] : make_float2(1.f, 0.f);
                  o0[jj] = (lo[j] * e.x - hi[j] * e.y) * sc;
                  o1[jj] = (lo[j] * e.y + hi[j] * e.x) * sc;
                }
                const uint4 w0 = make_uint4(pack2<OutT>(o0[0], o0[1]), pack2<OutT>(o0[2], o0[3]),
                                            pack2<OutT>(o0[4], o0[5]), pack2<OutT>(o0[6], o0[7]));
                const uint4 w1 = make_uint4(pack2<OutT>(o1[0], o1[1]), pack2<OutT>(o1[2], o1[3]),
                                            pack2<OutT>(o1[4], o1[5]), pack2<OutT>(o1[6], o1[7]));
                if (p.tma_out) {
                  box_put(4 * pc + u, w0);
                  keep[16 * pc + 4 * u] = w1.x; keep[16 * pc + 4 * u + 1] = w1.y;
                  keep[16 * pc + 4 * u + 2] = w1.z; keep[16 * pc + 4 * u + 3] = w1.w;
                } else if (row_ok) {
                  *reinterpret_cast<uint4*>(dst + pc * 32 + 8 * u) = w0;
                  *reinterpret_cast<uint4*>(dst + 64 + pc * 32 + 8 * u) = w1;
                }
              }
            }
            if (p.tma_out) {
              put_box(0);
              box_open();
#pragma unroll
              for (int u = 0; u < 8; ++u)
                box_put(u, make_uint4(keep[4 * u], keep[4 * u + 1], keep[4 * u + 2], keep[4 * u + 3]));
              put_box(64);
            }
          }
        }
      } else if constexpr (EPI == EPI_LOGITS) {
        float mx = -INFINITY, sm = 0.f, zt = 0.f;
        bool have_t = false;
        const int tg = row_ok ? p.tgt[row] : -1;
        OutT* orow = reinterpret_cast<OutT*>(p.out) + static_cast<long long>(row) * p.ldo;
#pragma unroll 1
        for (int c = c_begin; c < c_end; c += 2) {
          uint32_t ra[32], rb[32];
          tmem_load32_async(tbase + c * 32, ra);
          tmem_load32_async(tbase + (c + 1) * 32, rb);
          tmem_wait_ld();
          float v0[32], v1[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            v0[j] = __uint_as_float(ra[j]);
            v1[j] = __uint_as_float(rb[j]);
          }
          auto stats = [&](const float (&v)[32], int col0) {
            logits_chunk(v, col0, p.N, tg, mx, sm, zt, have_t);
            if (!p.tma_out && row_ok && col0 < p.N) store_row32(orow + col0, v, min(32, p.N - col0));
          };
          stats(v0, nb * BN + c * 32);
          stats(v1, nb * BN + c * 32 + 32);
          if (p.tma_out) emit64(v0, v1, nb * BN + c * 32, box_row0, 0);
        }
        if (row_ok) {
          // one (max, sumexp) partial per half tile
          reinterpret_cast<float2*>(p.f32a)[static_cast<long long>(row) * (2 * p.tiles_n) + 2 * nb + half] =
              make_float2(mx, sm);
          if (have_t) p.f32b[row] = zt;
        }
      } else {
        OutT* obase = reinterpret_cast<OutT*>(p.out) + static_cast<long long>(z) * p.out_bs +
                      static_cast<long long>(split) * p.split_stride;
        // Symmetric products: the tiles that hold diagonal elements are written
        // whole, and the tiles wholly above the diagonal are written and
        // mirrored whole, so each element is written exactly once (with 128 x
        // 256 tiles the two row blocks of a diagonal 256-column block are both
        // computed and together cover it).  The mirror goes by TMA when the
        // host built its map, else by per-thread stores.
        constexpr bool kRect = BN == 256;
        const bool sym_cross = kRect ? nb * BN < mb * 128 + 128 : nb == mb;
        const bool mirror = p.sym && !sym_cross;
        const bool tma_here = p.tma_out;
        // Auxiliary input of the epilogue, prefetched one 32-column chunk ahead to
        // hide its load latency.  (EPI_ACC adds into the output by TMA
        // add-reduction and reads nothing.)
        constexpr bool HAS_AUX = EPI == EPI_DRELU2 || EPI == EPI_AXPBY;
        using AT = AuxT;
        const AT* abase = nullptr;
        if constexpr (HAS_AUX)
          abase = reinterpret_cast<const AT*>(p.aux) + static_cast<long long>(z) * p.aux_bs +
                  static_cast<long long>(row) * p.ld_aux;
        constexpr int AUX_VEC = HAS_AUX ? (32 * static_cast<int>(sizeof(AT))) / 16 : 1;   // uint4 per chunk
        uint4 pf[AUX_VEC];
        auto prefetch = [&](int c) {
          if constexpr (HAS_AUX) {
            const int col0 = nb * BN + c * 32;
            const int nvalid = min(32, p.N - col0);
            constexpr int EPV = 16 / static_cast<int>(sizeof(AT));   // elements per uint4
#pragma unroll
            for (int g = 0; g < AUX_VEC; ++g) {
              pf[g] = make_uint4(0, 0, 0, 0);
              if (row_ok && g * EPV < nvalid) pf[g] = reinterpret_cast<const uint4*>(abase + col0)[g];
            }
          }
        };
        prefetch(c_begin);
        float rdot = 0.f;   // row_dot: this row's <out, aux> over the thread's 128 columns
        // (N is a multiple of 128, so the thread's columns are all inside or all past N)
        const bool dot_here = p.row_dot && row_ok && nb * BN + c_begin * 32 < p.N;
#pragma unroll 1
        for (int c = c_begin; c < c_end; c += 2) {
          uint32_t ra[32], rb[32];
          tmem_load32_async(tbase + c * 32, ra);
          tmem_load32_async(tbase + (c + 1) * 32, rb);
          tmem_wait_ld();
          float v[2][32];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int cc = c + hh;
            float a[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[hh][j] = __uint_as_float(hh ? rb[j] : ra[j]) * dqs;
            if constexpr (HAS_AUX) {
#pragma unroll
              for (int g = 0; g < AUX_VEC; ++g) {
                const uint32_t w[4] = {pf[g].x, pf[g].y, pf[g].z, pf[g].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  if constexpr (sizeof(AT) == 2) {
                    a[8 * g + 2 * e] = lo16<AT>(w[e]);
                    a[8 * g + 2 * e + 1] = hi16<AT>(w[e]);
                  } else {
                    a[4 * g + e] = __uint_as_float(w[e]);
                  }
                }
              }
              if (cc + 1 < c_end) prefetch(cc + 1);
            }
            if constexpr (EPI == EPI_RELU2) {
#pragma unroll
              for (int j = 0; j < 32; ++j) { const float t = fmaxf(v[hh][j], 0.f); v[hh][j] = t * t; }
              if (p.amax_out && row_ok) {
                const int nv = min(32, p.N - (nb * BN + cc * 32));
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (j < nv) amax = fmaxf(amax, fabsf(__bfloat162float(__float2bfloat16_rn(v[hh][j]))));
              }
            } else if constexpr (EPI == EPI_DRELU2) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                // relu(u) = sqrt(h); h = relu(u)^2 is exact zero on half the entries, where
                // the IEEE sqrt takes its slow path, so use the single-instruction form
                float rt;
                asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(rt) : "f"(a[j]));
                v[hh][j] *= 2.f * rt;
              }
              if (p.amax_out && row_ok) {
                const int nv = min(32, p.N - (nb * BN + cc * 32));
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (j < nv) amax = fmaxf(amax, fabsf(__bfloat162float(__float2bfloat16_rn(v[hh][j]))));
              }
            } else if constexpr (EPI == EPI_AXPBY) {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[hh][j] = p.alpha * a[j] + p.beta * v[hh][j];
              if (p.gamma != 0.f) {
                const int dj = row - (nb * BN + cc * 32);   // this row's diagonal column in the chunk
                if (dj >= 0 && dj < 32) {
#pragma unroll
                  for (int j = 0; j < 32; ++j)
                    if (j == dj) v[hh][j] += p.gamma;
                }
              }
            }
          }
          if (tma_here) emit64(v[0], v[1], nb * BN + c * 32, box_row0, z3);
          if (mirror && p.tma_mirror) {
            // this warp's 32 rows x 64 columns transposed: staging row j (column
            // nb BN + 32 c + j) holds the 32 rows, 64 bytes, for a 32 x 64 box
            box_open();
            OutT* st = reinterpret_cast<OutT*>(stg);
#pragma unroll
            for (int j = 0; j < 32; ++j) store_scalar(st + j * 32 + lane, v[0][j]);
#pragma unroll
            for (int j = 0; j < 32; ++j) store_scalar(st + (32 + j) * 32 + lane, v[1][j]);
            box_close(&tmD, false, box_row0, nb * BN + c * 32, z3);
          }
          if constexpr (EPI == EPI_STORE && std::is_same<OutT, __nv_bfloat16>::value) {
            if (dot_here) {
              // the stored (bf16-rounded) values against the same columns of aux
              const uint4* arow = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.aux) +
                                                                 static_cast<long long>(row) * p.ld_aux +
                                                                 nb * BN + c * 32);
#pragma unroll
              for (int g = 0; g < 8; ++g) {
                const uint4 w = __ldg(arow + g);
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
                const float (&vv)[32] = v[g >> 2];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int j = (g & 3) * 8 + 2 * e;
                  rdot += __bfloat162float(__float2bfloat16_rn(vv[j])) * __uint_as_float(ws[e] << 16) +
                          __bfloat162float(__float2bfloat16_rn(vv[j + 1])) * __uint_as_float(ws[e] & 0xFFFF0000u);
                }
              }
            }
          }
          // optional fp16 copy of the output in the same layout, or the rounding
          // residual of an fp16 main output (then the TMA path alone stores v)
          if (p.tma_out2) {
            if (p.split_lo) {
#pragma unroll
              for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int j = 0; j < 32; ++j) v[hh][j] -= __half2float(__float2half_rn(v[hh][j]));
            }
            emit64_to(__half{}, &tmD, false, v[0], v[1], nb * BN + c * 32, box_row0, z3);
          }
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int col0 = nb * BN + (c + hh) * 32;
            const int nvalid = min(32, p.N - col0);
            if (!row_ok || nvalid <= 0) continue;
            if (!tma_here) store_row32(obase + static_cast<long long>(row) * p.ldo + col0, v[hh], nvalid);
            if (p.out_t) {
              OutT* tb = reinterpret_cast<OutT*>(p.out_t) + static_cast<long long>(z) * p.out_bs;
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j < nvalid) store_scalar(tb + static_cast<long long>(col0 + j) * p.ldo_t + row, v[hh][j]);
            }
            if (mirror && !p.tma_mirror) {
              // the transposed tile of a symmetric product: lanes write consecutive columns
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j < nvalid) store_scalar(obase + static_cast<long long>(col0 + j) * p.ldo + row, v[hh][j]);
            }
          }
        }
        if constexpr (EPI == EPI_STORE && std::is_same<OutT, __nv_bfloat16>::value) {
          // one 128-column head per thread: D[(b H + h) T + t] for row b T + t
          if (dot_here) {
            const int b = row / p.T, t = row - b * p.T, h = (nb * BN + c_begin * 32) >> 7;
            p.f32a[(static_cast<long long>(b) * p.H + h) * p.T + t] = rdot;
          }
        }
      }
      tc_fence_before();
      if constexpr (PAIR)
        mbar_arrive_cluster(cluster_addr(&tempty[acc], 0));   // the leader's MMAs refill this TMEM
      else
        mbar_arrive(&tempty[acc]);
    }
  }

  if constexpr (EPI == EPI_DRELU2 || EPI == EPI_RELU2) {
    if (warp >= 2 && p.amax_out) {
      const float m = warp_max(amax);
      if (lane == 0) atomicMax(p.amax_out + ((blockIdx.x * 8 + warp) & 31), __float_as_uint(m));
    }
  }
  if (warp >= 2 && lane == 0) bulk_wait_all();   // output boxes written before the CTA exits
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();   // neither CTA leaves while the other may still signal it
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else
      tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace gpt
