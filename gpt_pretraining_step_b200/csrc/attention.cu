// Causal flash attention, forward and backward, head_dim 128, bf16 operands
// with fp32 softmax and accumulation (online softmax; the forward saves the
// row log-sum-exp, the backward recomputes P from it).
//
// Layouts: q, k, v, dk, dv are [B, H, T, 128]; the forward output O and the
// incoming gradient dO are token-major [B, T, H, 128] (the rows of the
// projection GEMMs); dq is accumulated in fp32 [B, H, T, 128]; lse and
// D = rowsum(dO * O) are [B, H, T].
//
// This version issues warp-level mma.sync m16n8k16 tiles from a swizzled
// shared-memory ring filled by cp.async.
#include "attention.cuh"
#include "common.cuh"

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

// ------------------------------------------------------------------ forward

constexpr int FWD_BM = 128, FWD_BN = 64, FWD_THREADS = 256;

__global__ void __launch_bounds__(FWD_THREADS, 1)
    attn_fwd_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                    bf16* __restrict__ o, float* __restrict__ lse, int B, int H, int T, float scale_log2) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sQ = smem;                              // 128 x 128
  uint8_t* sK = sQ + FWD_BM * 256;                 // 2 x 64 x 128
  uint8_t* sV = sK + 2 * FWD_BN * 256;             // 2 x 64 x 128
  const int qb = (gridDim.x - 1) - blockIdx.x;     // longest rows first
  const int bh = blockIdx.y;
  const int b = bh / H, h = bh % H;
  const int q0 = qb * FWD_BM;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long head_off = static_cast<long long>(bh) * T * HD;
  const bf16* qg = q + head_off;
  const bf16* kg = k + head_off;
  const bf16* vg = v + head_off;

  load_tile(sQ, qg, HD, q0, FWD_BM, T, tid, FWD_THREADS);
  const int q_end = min(T, q0 + FWD_BM);
  const int nkb = (q_end + FWD_BN - 1) / FWD_BN;
  load_tile(sK, kg, HD, 0, FWD_BN, T, tid, FWD_THREADS);
  load_tile(sV, vg, HD, 0, FWD_BN, T, tid, FWD_THREADS);
  cp_async_commit();

  const int g = lane >> 2, t4 = lane & 3;
  const int row_a = q0 + warp * 16 + g;   // this thread's two query rows
  const int row_b = row_a + 8;
  float acc[16][4];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
  uint32_t qf[8][4];

  for (int kb = 0; kb < nkb; ++kb) {
    if (kb + 1 < nkb) {
      const int nb = (kb + 1) & 1;
      load_tile(sK + nb * FWD_BN * 256, kg, HD, (kb + 1) * FWD_BN, FWD_BN, T, tid, FWD_THREADS);
      load_tile(sV + nb * FWD_BN * 256, vg, HD, (kb + 1) * FWD_BN, FWD_BN, T, tid, FWD_THREADS);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (kb == 0) {
      const uint32_t qbase = smem_u32(sQ);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int r = warp * 16 + (lane & 15);
        const int c = kk * 2 + (lane >> 4);
        ldsm_x4(qbase + swz(r, c), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
    }
    const uint32_t kbase = smem_u32(sK + (kb & 1) * FWD_BN * 256);
    const uint32_t vbase = smem_u32(sV + (kb & 1) * FWD_BN * 256);
    const int k0 = kb * FWD_BN;
    // S = Q K^T for this warp's 16 rows x 64 keys
    float s[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        uint32_t b0, b1, b2, b3;
        const int r = j * 8 + (lane & 7) + ((lane >> 4) << 3);
        const int c = kk * 2 + ((lane >> 3) & 1);
        ldsm_x4(kbase + swz(r, c), b0, b1, b2, b3);
        mma16816(s[j], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
        mma16816(s[j + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
      }
    }
    // mask (causal and ragged tail), online softmax in the log2 domain
    float mx_a = m_a, mx_b = m_b;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c0 = k0 + j * 8 + 2 * t4;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int col = c0 + e;
        float va = s[j][e] * scale_log2, vb = s[j][2 + e] * scale_log2;
        if (col > row_a || col >= T) va = -INFINITY;
        if (col > row_b || col >= T) vb = -INFINITY;
        s[j][e] = va;
        s[j][2 + e] = vb;
        mx_a = fmaxf(mx_a, va);
        mx_b = fmaxf(mx_b, vb);
      }
    }
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
    const float base_a = mx_a == -INFINITY ? 0.f : mx_a;
    const float base_b = mx_b == -INFINITY ? 0.f : mx_b;
    const float alpha_a = exp2f(m_a - base_a), alpha_b = exp2f(m_b - base_b);
    m_a = mx_a;
    m_b = mx_b;
    l_a *= alpha_a;
    l_b *= alpha_b;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      acc[j][0] *= alpha_a; acc[j][1] *= alpha_a;
      acc[j][2] *= alpha_b; acc[j][3] *= alpha_b;
    }
    uint32_t pf[8][2];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float p0 = exp2f(s[j][0] - base_a), p1 = exp2f(s[j][1] - base_a);
      const float p2 = exp2f(s[j][2] - base_b), p3 = exp2f(s[j][3] - base_b);
      l_a += p0 + p1;
      l_b += p2 + p3;
      pf[j][0] = pack_bf16x2(p0, p1);
      pf[j][1] = pack_bf16x2(p2, p3);
    }
    // O += P V
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const uint32_t a0 = pf[2 * ks][0], a1 = pf[2 * ks][1], a2 = pf[2 * ks + 1][0], a3 = pf[2 * ks + 1][1];
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        uint32_t b0, b1, b2, b3;
        const int r = ks * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int c = j + (lane >> 4);
        ldsm_x4_t(vbase + swz(r, c), b0, b1, b2, b3);
        mma16816(acc[j], a0, a1, a2, a3, b0, b1);
        mma16816(acc[j + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();
  }
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  const float inv_a = l_a > 0.f ? 1.f / l_a : 0.f, inv_b = l_b > 0.f ? 1.f / l_b : 0.f;
  const long long d = static_cast<long long>(H) * HD;
  if (row_a < T) {
    bf16* orow = o + (static_cast<long long>(b) * T + row_a) * d + h * HD;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      *reinterpret_cast<uint32_t*>(orow + j * 8 + 2 * t4) = pack_bf16x2(acc[j][0] * inv_a, acc[j][1] * inv_a);
    if (t4 == 0) lse[static_cast<long long>(bh) * T + row_a] = (m_a + log2f(l_a)) * 0.69314718055994531f;
  }
  if (row_b < T) {
    bf16* orow = o + (static_cast<long long>(b) * T + row_b) * d + h * HD;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      *reinterpret_cast<uint32_t*>(orow + j * 8 + 2 * t4) = pack_bf16x2(acc[j][2] * inv_b, acc[j][3] * inv_b);
    if (t4 == 0) lse[static_cast<long long>(bh) * T + row_b] = (m_b + log2f(l_b)) * 0.69314718055994531f;
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
                     cudaStream_t s) {
  static bool configured = false;
  constexpr int smem = FWD_BM * 256 + 4 * FWD_BN * 256;
  if (!configured) {
    cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    configured = true;
  }
  dim3 grid((T + FWD_BM - 1) / FWD_BM, B * H);
  const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(HD));
  attn_fwd_kernel<<<grid, FWD_THREADS, smem, s>>>(q, k, v, o, lse, B, H, T, scale_log2);
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
