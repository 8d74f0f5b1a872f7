// Causal flash attention, forward and backward, head_dim 128, bf16 operands
// with fp32 softmax and accumulation (online softmax; the forward saves the
// row log-sum-exp, the backward recomputes P from it).
//
// Layouts: q, k, v, dk, dv are [B, H, T, 128]; the forward output O and the
// incoming gradient dO are token-major [B, T, H, 128] (the rows of the
// projection GEMMs); dq is accumulated in fp32 [B, H, T, 128]; lse and
// D = rowsum(dO * O) are [B, H, T].
//
// The forward runs on tcgen05 with TMEM accumulators; the backward issues
// warp-level mma.sync m16n8k16 tiles from a swizzled shared-memory ring
// filled by cp.async.
#include "attention.cuh"
#include "common.cuh"
#include "gemm.h"

namespace gpt {

namespace {

constexpr int HD = 128;

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool pred) {
  const uint32_t d = smem_u32(dst);
  const int n = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Row r, 16-byte chunk c of a [rows][128] bf16 tile, chunks XOR-swizzled by r % 8.
__device__ __forceinline__ uint32_t swz(int r, int c) { return r * 256 + ((c ^ (r & 7)) << 4); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Copy rows [r0, r0 + nrows) of a 128-wide bf16 tile; rows >= limit are zero-filled.
__device__ __forceinline__ void load_tile(uint8_t* sm, const bf16* g, long long row_stride, int r0, int nrows,
                                          int limit, int tid, int nthreads) {
  for (int i = tid; i < nrows * 16; i += nthreads) {
    const int r = i >> 4, c = i & 15;
    const bool ok = r0 + r < limit;
    const bf16* src = g + static_cast<long long>(ok ? r0 + r : 0) * row_stride + c * 8;
    cp_async16(sm + swz(r, c), src, ok);
  }
}

// ------------------------------------------------- forward on tcgen05 / TMEM
//
// One CTA per (128-query tile, batch*head), 192 threads:
//   warp 0      TMA: Q once, K_j and V_j through two-slot rings
//   warp 1      TMEM owner and MMA issuer: S_j = Q K_j^T into one of two TMEM
//               S buffers and O += P_j V_j into the TMEM output accumulator;
//               S_{j+1} is issued before P_j is ready so the tensor cores
//               keep working while the softmax runs
//   warps 2..5  softmax, one query row (TMEM lane) per thread: the block max
//               from a first pass over the S row, exp2 into bf16 P written to
//               shared memory (128-byte swizzle, the A operand of P V).
// The reference max of a row only moves when the block max exceeds it by
// more than 8 (log2 units), so P stays below 2^8; when it moves, the warp
// rescales its rows of O in TMEM after the previous P V has completed.
// TMEM: S0 @ col 0, S1 @ 128, O @ 256 (fp32, lane = query row).

constexpr int TF_TILE = 16384;                // one [128 rows][128 B] swizzled tile
constexpr int TF_BUF = 2 * TF_TILE;           // 128 x 128 bf16 as two 64-column tiles
constexpr int TF_SMEM = 7 * TF_BUF + 1024 + 512;
constexpr float TF_RESCALE = 8.f;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_store32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__global__ void __launch_bounds__(192, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, bf16* __restrict__ o, float* __restrict__ lse,
                       int H, int T, float scale_log2, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = sm;
  uint8_t* sK = sm + TF_BUF;         // two slots
  uint8_t* sV = sm + 3 * TF_BUF;     // two slots
  uint8_t* sP = sm + 5 * TF_BUF;     // two slots
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + 7 * TF_BUF);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* k_empty = bars + 3;   // [2]
  uint64_t* v_full = bars + 5;    // [2]
  uint64_t* v_empty = bars + 7;   // [2]
  uint64_t* s_full = bars + 9;    // [2]
  uint64_t* s_free = bars + 11;   // [2]
  uint64_t* p_full = bars + 13;   // [2]
  uint64_t* pv_done = bars + 15;  // [2]: P slot may be rewritten; O may be rescaled or read
  uint64_t* drain = bars + 17;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 18);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = warp_id(), lane = lane_id();
  const int qt = (gridDim.x - 1) - blockIdx.x;    // longest rows first
  const int bh = blockIdx.y;
  const int q0 = qt * 128;
  const int nkv = qt + 1;                          // causal: key blocks 0..qt

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1); mbar_init(&s_free[i], 128);
      mbar_init(&p_full[i], 128); mbar_init(&pv_done[i], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // -------------------------------------------------------------- TMA
      bool ok = true;
      int issued_k = 0, issued_v = 0;
      mbar_arrive_expect_tx(q_full, TF_BUF);
      tma_load_3d(sQ, &tq, q_full, 0, q0, bh);
      tma_load_3d(sQ + TF_TILE, &tq, q_full, 64, q0, bh);
      for (int j = 0; j < nkv && ok; ++j) {
        const int s = j & 1;
        const uint32_t par = (j >> 1) & 1;
        if (!mbar_wait(&k_empty[s], par ^ 1u, abort_flag, err)) { ok = false; break; }
        mbar_arrive_expect_tx(&k_full[s], TF_BUF);
        tma_load_3d(sK + s * TF_BUF, &tk, &k_full[s], 0, j * 128, bh);
        tma_load_3d(sK + s * TF_BUF + TF_TILE, &tk, &k_full[s], 64, j * 128, bh);
        ++issued_k;
        if (!mbar_wait(&v_empty[s], par ^ 1u, abort_flag, err)) { ok = false; break; }
        mbar_arrive_expect_tx(&v_full[s], TF_BUF);
        tma_load_3d(sV + s * TF_BUF, &tv, &v_full[s], 0, j * 128, bh);
        tma_load_3d(sV + s * TF_BUF + TF_TILE, &tv, &v_full[s], 64, j * 128, bh);
        ++issued_v;
      }
      if (!ok) {
        // let the copies already started land before the CTA exits
        for (uint32_t i = 0; i < (1u << 20) && !mbar_try_wait(q_full, 0); ++i) {}
        for (int j = (issued_k > 2 ? issued_k - 2 : 0); j < issued_k; ++j)
          for (uint32_t i = 0; i < (1u << 20) && !mbar_try_wait(&k_full[j & 1], (j >> 1) & 1); ++i) {}
        for (int j = (issued_v > 2 ? issued_v - 2 : 0); j < issued_v; ++j)
          for (uint32_t i = 0; i < (1u << 20) && !mbar_try_wait(&v_full[j & 1], (j >> 1) & 1); ++i) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // -------------------------------------------------------------- MMA
      constexpr uint32_t IDESC_S = make_idesc(1, 128, false, false);
      constexpr uint32_t IDESC_O = make_idesc(1, 128, false, true);
      const uint32_t q_addr = smem_u32(sQ);
      bool ok = mbar_wait(q_full, 0, abort_flag, err);
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1;
        const uint32_t par = (j >> 1) & 1;
        if (!mbar_wait(&k_full[s], par, abort_flag, err)) return false;
        if (!mbar_wait(&s_free[s], par ^ 1u, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + s * TF_BUF);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * TF_TILE + (kk & 3) * 32;
          umma_f16(tmem + s * 128, smem_desc_sw128(q_addr + off, 16, 1024),
                   smem_desc_sw128(k_addr + off, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[s]);
        umma_commit(&k_empty[s]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int s = j & 1;
        const uint32_t par = (j >> 1) & 1;
        if (!mbar_wait(&p_full[s], par, abort_flag, err)) return false;
        if (!mbar_wait(&v_full[s], par, abort_flag, err)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sV + s * TF_BUF);
        const uint32_t p_addr = smem_u32(sP + s * TF_BUF);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = (kk >> 2) * TF_TILE + (kk & 3) * 32;
          umma_f16(tmem + 256, smem_desc_sw128(p_addr + aoff, 16, 1024),
                   smem_desc_sw128(v_addr + kk * 2048, TF_TILE, 1024), IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&v_empty[s]);
        umma_commit(&pv_done[s]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < nkv && ok; ++j) {
        if (j + 1 < nkv) ok = issue_s(j + 1);
        if (ok) ok = issue_pv(j);
      }
      umma_commit(drain);
      for (uint32_t i = 0; i < (1u << 22) && !mbar_try_wait(drain, 0); ++i) {}
    }
  } else {
    // ---------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int q = q0 + r;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_o = tmem + lane_base + 256;
    float m_ref = -INFINITY, l = 0.f;   // reference max (log2 units) and row sum relative to it
    bool ok = true;
    auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
      const bool got = mbar_wait(bar, par, abort_flag, err);
      __syncwarp();
      return __all_sync(0xffffffffu, got);
    };
    for (int j = 0; j < nkv && ok; ++j) {
      const int s = j & 1;
      if (!wait_all(&s_full[s], (j >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      // the whole S row at once; the S buffer is free again as soon as it is read
      uint32_t sr[128];
      {
        const uint32_t ts = tmem + lane_base + s * 128;
        uint32_t (&r0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
        uint32_t (&r1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
        uint32_t (&r2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[64]);
        uint32_t (&r3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[96]);
        tmem_load32_async(ts, r0);
        tmem_load32_async(ts + 32, r1);
        tmem_load32_async(ts + 64, r2);
        tmem_load32_async(ts + 96, r3);
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(&s_free[s]);
      const int kbase = j * 128;
      if ((j == qt) || (kbase + 128 > T)) {
        // causal diagonal / ragged tail: masked scores become -inf
#pragma unroll
        for (int k = 0; k < 128; ++k) {
          const int key = kbase + k;
          if (key > q || key >= T) sr[k] = __float_as_uint(-INFINITY);
        }
      }
      // block max of the raw scores (the scale is positive), eight independent chains
      float mx8[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) mx8[t] = __uint_as_float(sr[t]);
#pragma unroll
      for (int k = 8; k < 128; ++k) mx8[k & 7] = fmaxf(mx8[k & 7], __uint_as_float(sr[k]));
      const float mraw = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float mblk = mraw * scale_log2;
      const bool move = mblk > m_ref + TF_RESCALE;   // always true on the first block
      const float m_new = move ? mblk : m_ref;
      const float factor = ex2_approx(m_ref - m_new);  // 1 when the reference stays, 0 on the first block
      // O may only be rescaled once the previous P V has accumulated into it
      if (j >= 1 && __any_sync(0xffffffffu, move)) {
        if (!wait_all(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t ra[32];
          tmem_load32_async(t_o + c * 32, ra);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) ra[k] = __float_as_uint(__uint_as_float(ra[k]) * factor);
          tmem_store32(t_o + c * 32, ra);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
      }
      // the P slot is free once the P V two blocks back has read it
      if (j >= 2 && !wait_all(&pv_done[s], ((j >> 1) & 1) ^ 1u)) { ok = false; break; }
      // probabilities relative to the reference, row sum, bf16 P tile (masked scores give 0)
      const float bias = -m_new;
      float rs8[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) rs8[t] = 0.f;
      uint8_t* pslot = sP + s * TF_BUF;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c * 32 + k]), scale_log2, bias));
          const float p1 = ex2_approx(fmaf(__uint_as_float(sr[c * 32 + k + 1]), scale_log2, bias));
          rs8[(k >> 1) & 7] += p0 + p1;
          pk[k >> 1] = pack_bf16x2(p0, p1);
        }
        uint8_t* prow = pslot + (c >> 1) * TF_TILE + r * 128;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int unit = ((c & 1) * 4 + t) ^ (r & 7);
          *reinterpret_cast<uint4*>(prow + unit * 16) =
              make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&p_full[s]);
      const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
      l = l * factor + rs;
      m_ref = m_new;
    }
    // epilogue: O / l once the last P V has landed
    if (ok) ok = wait_all(&pv_done[(nkv - 1) & 1], ((nkv - 1) >> 1) & 1);
    if (ok) {
      tc_fence_after();
      const int b = bh / H, h = bh - (bh / H) * H;
      const float inv = 1.f / l;
      bf16* orow = o + (static_cast<long long>(b) * T + q) * (static_cast<long long>(H) * 128) + h * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t ra[32];
        tmem_load32_async(t_o + c * 32, ra);
        tmem_wait_ld();
        if (q < T) {
#pragma unroll
          for (int k = 0; k < 32; k += 8) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(ra[k]) * inv, __uint_as_float(ra[k + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(ra[k + 2]) * inv, __uint_as_float(ra[k + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(ra[k + 4]) * inv, __uint_as_float(ra[k + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(ra[k + 6]) * inv, __uint_as_float(ra[k + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c * 32 + k) = w;
          }
        }
      }
      if (q < T) lse[static_cast<long long>(bh) * T + q] = (m_ref + log2f(l)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------- backward prepass

// D[b, h, t] = sum_i dO[b, t, h, i] * O[b, t, h, i]
__global__ void attn_bwd_dot_kernel(const bf16* __restrict__ o, const bf16* __restrict__ dout,
                                    float* __restrict__ Dv, int B, int H, int T) {
  const long long w = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + warp_id();
  if (w >= static_cast<long long>(B) * H * T) return;
  const int t = static_cast<int>(w % T);
  const int h = static_cast<int>((w / T) % H);
  const int b = static_cast<int>(w / (static_cast<long long>(T) * H));
  const long long off = ((static_cast<long long>(b) * T + t) * H + h) * HD + lane_id() * 4;
  const uint2 x = *reinterpret_cast<const uint2*>(o + off);
  const uint2 y = *reinterpret_cast<const uint2*>(dout + off);
  float s = bf16_lo(x.x) * bf16_lo(y.x) + bf16_hi(x.x) * bf16_hi(y.x) + bf16_lo(x.y) * bf16_lo(y.y) +
            bf16_hi(x.y) * bf16_hi(y.y);
  s = warp_sum(s);
  if (lane_id() == 0) Dv[w] = s;
}

// --------------------------------------------------------------- backward

// One CTA per (128-key block, b, h); loops over 64-query blocks at or below
// the diagonal.  Warp w owns keys 16w..16w+15 for S^T, dP^T, dV and dK; for
// dQ it owns query rows 16(w%4).. and head columns 64(w/4)...
constexpr int BWD_BN = 128, BWD_BM = 64, BWD_THREADS = 256;

__global__ void __launch_bounds__(BWD_THREADS, 1)
    attn_bwd_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                    const bf16* __restrict__ dout, const float* __restrict__ lse, const float* __restrict__ Dv,
                    float* __restrict__ dq, bf16* __restrict__ dk, bf16* __restrict__ dv, int B, int H, int T,
                    float scale) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sK = smem;                          // 128 x 128
  uint8_t* sV = sK + BWD_BN * 256;             // 128 x 128
  uint8_t* sQ = sV + BWD_BN * 256;             // 2 x 64 x 128
  uint8_t* sO = sQ + 2 * BWD_BM * 256;         // 2 x 64 x 128 (dO)
  uint8_t* sS = sO + 2 * BWD_BM * 256;         // dS^T: 128 keys x 64 queries bf16, 128 B rows
  float* sL = reinterpret_cast<float*>(sS + BWD_BN * 128);   // 2 x 64 lse
  float* sD = sL + 2 * BWD_BM;                               // 2 x 64 D

  const int kblk = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / H, h = bh % H;
  const int k0 = kblk * BWD_BN;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const long long head_off = static_cast<long long>(bh) * T * HD;
  const long long dstride = static_cast<long long>(H) * HD;
  const bf16* qg = q + head_off;
  const bf16* dog = dout + static_cast<long long>(b) * T * dstride + h * HD;
  const float* lg = lse + static_cast<long long>(bh) * T;
  const float* Dg = Dv + static_cast<long long>(bh) * T;

  load_tile(sK, k + head_off, HD, k0, BWD_BN, T, tid, BWD_THREADS);
  load_tile(sV, v + head_off, HD, k0, BWD_BN, T, tid, BWD_THREADS);
  const int qb_first = k0 / BWD_BM;
  const int nqb = (T + BWD_BM - 1) / BWD_BM;
  auto load_q = [&](int qb, int buf) {
    load_tile(sQ + buf * BWD_BM * 256, qg, HD, qb * BWD_BM, BWD_BM, T, tid, BWD_THREADS);
    load_tile(sO + buf * BWD_BM * 256, dog, dstride, qb * BWD_BM, BWD_BM, T, tid, BWD_THREADS);
    if (tid < BWD_BM) {
      const int r = qb * BWD_BM + tid;
      sL[buf * BWD_BM + tid] = r < T ? lg[r] : 0.f;
      sD[buf * BWD_BM + tid] = r < T ? Dg[r] : 0.f;
    }
  };
  if (qb_first < nqb) load_q(qb_first, 0);
  cp_async_commit();

  float dK[16][4], dV[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) dK[j][e] = dV[j][e] = 0.f;

  const uint32_t kbase = smem_u32(sK), vbase = smem_u32(sV), sbase = smem_u32(sS);
  const int key_a = k0 + warp * 16 + g, key_b = key_a + 8;   // this thread's two key rows
  const float scale_log2 = scale * 1.4426950408889634f;

  for (int qb = qb_first; qb < nqb; ++qb) {
    const int buf = (qb - qb_first) & 1;
    if (qb + 1 < nqb) {
      load_q(qb + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t qbase = smem_u32(sQ + buf * BWD_BM * 256);
    const uint32_t obase = smem_u32(sO + buf * BWD_BM * 256);
    const float* L = sL + buf * BWD_BM;
    const float* Dd = sD + buf * BWD_BM;
    const int q0 = qb * BWD_BM;

    // S^T = K Q^T and dP^T = V dO^T for 16 keys x 64 queries
    float st[8][4], dpt[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) st[j][e] = dpt[j][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t a0, a1, a2, a3, c0, c1, c2, c3;
      const int ar = warp * 16 + (lane & 15);
      const int ac = kk * 2 + (lane >> 4);
      ldsm_x4(kbase + swz(ar, ac), a0, a1, a2, a3);
      ldsm_x4(vbase + swz(ar, ac), c0, c1, c2, c3);
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        uint32_t b0, b1, b2, b3;
        const int r = j * 8 + (lane & 7) + ((lane >> 4) << 3);
        const int c = kk * 2 + ((lane >> 3) & 1);
        ldsm_x4(qbase + swz(r, c), b0, b1, b2, b3);
        mma16816(st[j], a0, a1, a2, a3, b0, b1);
        mma16816(st[j + 1], a0, a1, a2, a3, b2, b3);
        ldsm_x4(obase + swz(r, c), b0, b1, b2, b3);
        mma16816(dpt[j], c0, c1, c2, c3, b0, b1);
        mma16816(dpt[j + 1], c0, c1, c2, c3, b2, b3);
      }
    }
    // P^T = exp(S^T * scale - lse[q]) masked; dS^T = P^T (dP^T - D[q]) * scale
    uint32_t pf[8][2], sf[8][2];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float pv[4], dsv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qi = j * 8 + 2 * t4 + (e & 1);
        const int key = (e < 2) ? key_a : key_b;
        const int qrow = q0 + qi;
        float p = exp2f(st[j][e] * scale_log2 - L[qi] * 1.4426950408889634f);
        if (key > qrow || qrow >= T || key >= T) p = 0.f;
        pv[e] = p;
        dsv[e] = p * (dpt[j][e] - Dd[qi]) * scale;
      }
      pf[j][0] = pack_bf16x2(pv[0], pv[1]);
      pf[j][1] = pack_bf16x2(pv[2], pv[3]);
      sf[j][0] = pack_bf16x2(dsv[0], dsv[1]);
      sf[j][1] = pack_bf16x2(dsv[2], dsv[3]);
      // dS^T rows (keys) to shared memory for the dQ product: 64 queries x 2 B = 128 B per key row
      const int kr_a = warp * 16 + g, kr_b = kr_a + 8;
      const int chunk = j;   // 8 queries = 16 B
      *reinterpret_cast<uint32_t*>(sS + kr_a * 128 + (((chunk ^ (kr_a & 7)) << 4)) + t4 * 4) = sf[j][0];
      *reinterpret_cast<uint32_t*>(sS + kr_b * 128 + (((chunk ^ (kr_b & 7)) << 4)) + t4 * 4) = sf[j][1];
    }
    // dV += P^T dO, dK += dS^T Q (k = 64 queries in 4 steps)
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const uint32_t pa0 = pf[2 * ks][0], pa1 = pf[2 * ks][1], pa2 = pf[2 * ks + 1][0], pa3 = pf[2 * ks + 1][1];
      const uint32_t sa0 = sf[2 * ks][0], sa1 = sf[2 * ks][1], sa2 = sf[2 * ks + 1][0], sa3 = sf[2 * ks + 1][1];
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        uint32_t b0, b1, b2, b3;
        const int r = ks * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int c = j + (lane >> 4);
        ldsm_x4_t(obase + swz(r, c), b0, b1, b2, b3);
        mma16816(dV[j], pa0, pa1, pa2, pa3, b0, b1);
        mma16816(dV[j + 1], pa0, pa1, pa2, pa3, b2, b3);
        ldsm_x4_t(qbase + swz(r, c), b0, b1, b2, b3);
        mma16816(dK[j], sa0, sa1, sa2, sa3, b0, b1);
        mma16816(dK[j + 1], sa0, sa1, sa2, sa3, b2, b3);
      }
    }
    __syncthreads();   // dS^T complete
    // dQ[q0 + 16(w%4) .., 64(w/4) ..] += dS K: A = dS (rows = queries) read transposed from dS^T
    {
      float dqa[8][4];
#pragma unroll
      for (int j = 0; j < 8; ++j) dqa[j][0] = dqa[j][1] = dqa[j][2] = dqa[j][3] = 0.f;
      const int qr0 = (warp & 3) * 16;
      const int hc0 = (warp >> 2) * 64;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {   // 128 keys in steps of 16
        // A fragment rows = queries qr0.., cols = keys 16ks..; stored as dS^T[key][query]
        uint32_t a0, a1, a2, a3;
        {
          const int key = ks * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int qc = qr0 + (((lane >> 3) & 1) << 3);   // query chunk start (8 queries)
          const int chunk = qc >> 3;
          ldsm_x4_t(sbase + key * 128 + ((chunk ^ (key & 7)) << 4), a0, a1, a2, a3);
        }
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
          uint32_t b0, b1, b2, b3;
          const int r = ks * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
          const int c = (hc0 >> 3) + j + (lane >> 4);
          ldsm_x4_t(kbase + swz(r, c), b0, b1, b2, b3);
          mma16816(dqa[j], a0, a1, a2, a3, b0, b1);
          mma16816(dqa[j + 1], a0, a1, a2, a3, b2, b3);
        }
      }
      const int qa = q0 + qr0 + g, qb2 = qa + 8;
      float* dqh = dq + head_off;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int col = hc0 + j * 8 + 2 * t4;
        if (qa < T) {
          atomicAdd(dqh + static_cast<long long>(qa) * HD + col, dqa[j][0]);
          atomicAdd(dqh + static_cast<long long>(qa) * HD + col + 1, dqa[j][1]);
        }
        if (qb2 < T) {
          atomicAdd(dqh + static_cast<long long>(qb2) * HD + col, dqa[j][2]);
          atomicAdd(dqh + static_cast<long long>(qb2) * HD + col + 1, dqa[j][3]);
        }
      }
    }
    __syncthreads();   // buffers of this query block may be refilled
  }
  // write dK, dV for this warp's 16 keys
  if (key_a < T) {
    bf16* kr = dk + head_off + static_cast<long long>(key_a) * HD;
    bf16* vr = dv + head_off + static_cast<long long>(key_a) * HD;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      *reinterpret_cast<uint32_t*>(kr + j * 8 + 2 * t4) = pack_bf16x2(dK[j][0], dK[j][1]);
      *reinterpret_cast<uint32_t*>(vr + j * 8 + 2 * t4) = pack_bf16x2(dV[j][0], dV[j][1]);
    }
  }
  if (key_b < T) {
    bf16* kr = dk + head_off + static_cast<long long>(key_b) * HD;
    bf16* vr = dv + head_off + static_cast<long long>(key_b) * HD;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      *reinterpret_cast<uint32_t*>(kr + j * 8 + 2 * t4) = pack_bf16x2(dK[j][2], dK[j][3]);
      *reinterpret_cast<uint32_t*>(vr + j * 8 + 2 * t4) = pack_bf16x2(dV[j][2], dV[j][3]);
    }
  }
}

}  // namespace

void launch_attn_fwd(const bf16* q, const bf16* k, const bf16* v, bf16* o, float* lse, int B, int H, int T,
                     cudaStream_t s, int* err) {
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TF_SMEM);
    configured = true;
  }
  CUtensorMap mq, mk, mv;
  const long long bh = 1ll * B * H;
  if (!make_map(&mq, q, 2, HD, T, bh, HD, 1ll * T * HD, 64, 128) ||
      !make_map(&mk, k, 2, HD, T, bh, HD, 1ll * T * HD, 64, 128) ||
      !make_map(&mv, v, 2, HD, T, bh, HD, 1ll * T * HD, 64, 128)) {
    if (err) cudaMemsetAsync(err, 0xff, sizeof(int), s);   // latched as a device error
    return;
  }
  dim3 grid((T + 127) / 128, B * H);
  const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(HD));
  attn_fwd_tc_kernel<<<grid, 192, TF_SMEM, s>>>(mq, mk, mv, o, lse, H, T, scale_log2, err);
}

void launch_attn_bwd(const bf16* q, const bf16* k, const bf16* v, const bf16* o, const bf16* dout,
                     const float* lse, float* Dv, float* dq, bf16* dk, bf16* dv, int B, int H, int T,
                     cudaStream_t s) {
  static bool configured = false;
  constexpr int smem = 2 * BWD_BN * 256 + 4 * BWD_BM * 256 + BWD_BN * 128 + 4 * BWD_BM * 4;
  if (!configured) {
    cudaFuncSetAttribute(attn_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    configured = true;
  }
  const long long rows = 1ll * B * H * T;
  attn_bwd_dot_kernel<<<static_cast<int>((rows + 7) / 8), 256, 0, s>>>(o, dout, Dv, B, H, T);
  cudaMemsetAsync(dq, 0, static_cast<size_t>(rows) * HD * sizeof(float), s);
  dim3 grid((T + BWD_BN - 1) / BWD_BN, B * H);
  attn_bwd_kernel<<<grid, BWD_THREADS, smem, s>>>(q, k, v, dout, lse, Dv, dq, dk, dv, B, H, T,
                                                  1.f / sqrtf(static_cast<float>(HD)));
}

}  // namespace gpt
