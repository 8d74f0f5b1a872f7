// Bandwidth-bound kernels of the step: embedding, RMSNorm, QK-norm/RoPE
// backward, cross-entropy finish, deterministic reductions, AdamW and the
// elementwise parts of Muon.  Rows are processed one warp per row with
// 16-byte vector accesses; grids are sized from the row count.
#include <cuda_fp8.h>
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

#include <cuda_fp16.h>
#include <type_traits>

namespace gpt {

namespace {

inline int cdiv(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

__device__ __forceinline__ void store_bf16x4(bf16* dst, float4 v) {
  uint2 w;
  w.x = pack_bf16x2(v.x, v.y);
  w.y = pack_bf16x2(v.z, v.w);
  *reinterpret_cast<uint2*>(dst) = w;
}

__device__ __forceinline__ float4 load_bf16x4(const bf16* src) {
  const uint2 w = *reinterpret_cast<const uint2*>(src);
  return make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
}

// ------------------------------------------------------------------ RoPE

// (cos, sin) of t * 10000^(-2i/128) for positions t < T and pairs i < 64, in
// two layouts: token-major tab[t][i] and pair-major tab[T * 64 + i * T + t]
// (the latter lets a warp of consecutive tokens read one pair coalesced)
__global__ void rope_table_kernel(float2* tab, int T) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= T * 64) return;
  const int t = idx / 64, i = idx % 64;
  const double inv_freq = pow(10000.0, -2.0 * i / 128.0);
  double sn, cs;
  sincos(static_cast<double>(t) * inv_freq, &sn, &cs);
  const float2 e = make_float2(static_cast<float>(cs), static_cast<float>(sn));
  tab[idx] = e;
  tab[static_cast<long long>(T) * 64 + static_cast<long long>(i) * T + t] = e;
}

// ------------------------------------------------------------- embedding

__global__ void embed_fwd_kernel(const int* __restrict__ tok, const bf16* __restrict__ wte,
                                 float* __restrict__ x, int M, int d, int V, int* err) {
  const int row = blockIdx.x * (blockDim.x / 32) + warp_id();
  if (row >= M) return;
  int t = tok[row];
  const bool bad = t < 0 || t >= V;
  if (bad) {
    if (lane_id() == 0) atomicOr(err, ERRF_TOKEN_RANGE);
  }
  const bf16* src = wte + static_cast<long long>(bad ? 0 : t) * d;
  float* dst = x + static_cast<long long>(row) * d;
  for (int c = lane_id() * 4; c < d; c += 128) {
    float4 v = bad ? make_float4(0.f, 0.f, 0.f, 0.f) : load_bf16x4(src + c);
    *reinterpret_cast<float4*>(dst + c) = v;
  }
}

// Single-CTA bitonic sort of (token, position) keys of one chunk of <= 32768 positions.
constexpr int kEmbChunk = 32768;

__global__ void __launch_bounds__(1024) embed_sort_kernel(const int* __restrict__ tok, int n, int npow2,
                                                          uint32_t* __restrict__ keys_out, int V) {
  extern __shared__ uint32_t keys[];
  for (int i = threadIdx.x; i < npow2; i += blockDim.x) {
    uint32_t k = 0xFFFFFFFFu;
    if (i < n) {
      int t = tok[i];
      t = (t < 0 || t >= V) ? 0 : t;
      k = static_cast<uint32_t>(t) * kEmbChunk + static_cast<uint32_t>(i);
    }
    keys[i] = k;
  }
  __syncthreads();
  for (int size = 2; size <= npow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < npow2 / 2; i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint32_t a = keys[lo], b = keys[hi];
        if ((a > b) == up) {
          keys[lo] = b;
          keys[hi] = a;
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < n; i += blockDim.x) keys_out[i] = keys[i];
}

// Segmented sum of dx rows by token over the sorted keys, robust to skewed
// token histograms (natural text puts thousands of rows on a few tokens).
// The sorted positions are cut into aligned chunks of kEmbPiece rows; a run
// of equal tokens is split at the chunk boundaries into pieces, each summed
// by one warp per 128 columns in position order.  A run inside one chunk is
// added to its row of dwte directly; the pieces of a run that crosses
// chunks leave partial sums in the workspace (slot 2c for the piece at the
// start of chunk c, 2c + 1 for a piece that starts inside chunk c and runs
// on into the next one), which embed_join_kernel adds in position order.
// Every sum has a fixed order, so the result is deterministic.
constexpr int kEmbPiece = 64;

__device__ __forceinline__ uint32_t emb_tok(const uint32_t* keys, int i) { return keys[i] / kEmbChunk; }

__global__ void embed_piece_kernel(const uint32_t* __restrict__ keys, int n, const float* __restrict__ dx, int base,
                                   float* __restrict__ dwte, float* __restrict__ part, int d) {
  const int nchunk = d / 128;
  const long long gw = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + warp_id();
  const int w = static_cast<int>(gw / nchunk);
  const int c0 = static_cast<int>(gw - static_cast<long long>(w) * nchunk) * 128;
  if (w >= n) return;
  const uint32_t tw = emb_tok(keys, w);
  const bool at_chunk = w % kEmbPiece == 0;
  const bool run_start = w == 0 || emb_tok(keys, w - 1) != tw;
  if (!at_chunk && !run_start) return;
  // the piece ends at the run's end or the chunk's end, whichever is first
  const int cend = min(n, (w / kEmbPiece + 1) * kEmbPiece);
  int e = cend;
  for (int j0 = w + 1; j0 < cend; j0 += 32) {
    const int j = j0 + lane_id();
    const bool other = j < cend && emb_tok(keys, j) != tw;
    const unsigned m = __ballot_sync(0xffffffffu, other);
    if (m) { e = j0 + __ffs(m) - 1; break; }
  }
  const bool continues_before = at_chunk && !run_start;
  const bool continues_after = e == cend && cend < n && emb_tok(keys, cend) == tw;
  const int c = lane_id() * 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = w; j < e; j += 8) {
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j + u < e) {
        const int m = base + static_cast<int>(keys[j + u] % kEmbChunk);
        v[u] = *reinterpret_cast<const float4*>(dx + static_cast<long long>(m) * d + c0 + c);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      acc.x += v[u].x; acc.y += v[u].y; acc.z += v[u].z; acc.w += v[u].w;
    }
  }
  if (!continues_before && !continues_after) {
    float* dst = dwte + static_cast<long long>(tw) * d + c0 + c;
    const float4 o = *reinterpret_cast<const float4*>(dst);
    *reinterpret_cast<float4*>(dst) = make_float4(o.x + acc.x, o.y + acc.y, o.z + acc.z, o.w + acc.w);
    return;
  }
  const int slot = 2 * (w / kEmbPiece) + (at_chunk ? 0 : 1);
  *reinterpret_cast<float4*>(part + static_cast<long long>(slot) * d + c0 + c) = acc;
}

// One warp per (run that crosses a chunk boundary, 128 columns): the sum of
// its pieces' partials in position order, added to the token's row.
__global__ void embed_join_kernel(const uint32_t* __restrict__ keys, int n, const float* __restrict__ part,
                                  float* __restrict__ dwte, int d) {
  const int nchunk = d / 128;
  const long long gw = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + warp_id();
  const int w = static_cast<int>(gw / nchunk);
  const int c0 = static_cast<int>(gw - static_cast<long long>(w) * nchunk) * 128;
  if (w >= n) return;
  const uint32_t tw = emb_tok(keys, w);
  if (w > 0 && emb_tok(keys, w - 1) == tw) return;           // not a run start
  const int b = (w / kEmbPiece + 1) * kEmbPiece;               // the next chunk boundary
  if (b >= n || emb_tok(keys, b) != tw) return;              // the run stays inside its chunk
  // the run's last position: the last key of token tw
  int lo = b, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (emb_tok(keys, mid) == tw) lo = mid; else hi = mid - 1;
  }
  const int c = lane_id() * 4;
  const float* p0 = part + static_cast<long long>(2 * (w / kEmbPiece) + (w % kEmbPiece == 0 ? 0 : 1)) * d + c0 + c;
  float4 acc = *reinterpret_cast<const float4*>(p0);
  for (int ch = b / kEmbPiece; ch <= lo / kEmbPiece; ++ch) {
    const float4 v = *reinterpret_cast<const float4*>(part + static_cast<long long>(2 * ch) * d + c0 + c);
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  float* dst = dwte + static_cast<long long>(tw) * d + c0 + c;
  const float4 o = *reinterpret_cast<const float4*>(dst);
  *reinterpret_cast<float4*>(dst) = make_float4(o.x + acc.x, o.y + acc.y, o.z + acc.z, o.w + acc.w);
}

// --------------------------------------------------------------- RMSNorm
//
// One warp per row of d = 128 * NV fp32 values; every load of the row is
// issued before the warp reduction so one memory latency covers the row.

// Largest |value| of a warp's bf16-rounded outputs into one of 32 slots of an
// fp8 scale word set (32 slots spread the atomics; the quantiser takes the
// max over them).  m: this lane's max.
__device__ __forceinline__ void amax_slot_update(unsigned int* slots, float m, long long key) {
  m = warp_max(m);
  if (lane_id() == 0) atomicMax(slots + (key & 31), __float_as_uint(m));
}

__device__ __forceinline__ float abs_bf16(float v) { return fabsf(__bfloat162float(__float2bfloat16_rn(v))); }

template <int NV>
__global__ void __launch_bounds__(128) rmsnorm_fwd_kernel(const float* __restrict__ x, bf16* __restrict__ y,
                                                          float* __restrict__ rstd, int M,
                                                          unsigned int* __restrict__ amax) {
  constexpr int d = 128 * NV;
  const int row = blockIdx.x * 4 + warp_id();
  if (row >= M) return;
  const float* xr = x + static_cast<long long>(row) * d;
  float4 buf[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) buf[i] = *reinterpret_cast<const float4*>(xr + (i * 32 + lane_id()) * 4);
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) ss += buf[i].x * buf[i].x + buf[i].y * buf[i].y + buf[i].z * buf[i].z + buf[i].w * buf[i].w;
  ss = warp_sum(ss);
  const float r = rsqrtf(ss * (1.f / d) + 1e-6f);
  bf16* yr = y + static_cast<long long>(row) * d;
#pragma unroll
  for (int i = 0; i < NV; ++i)
    store_bf16x4(yr + (i * 32 + lane_id()) * 4, make_float4(buf[i].x * r, buf[i].y * r, buf[i].z * r, buf[i].w * r));
  if (lane_id() == 0) rstd[row] = r;
  if (amax) {
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i)
      m = fmaxf(m, fmaxf(fmaxf(abs_bf16(buf[i].x * r), abs_bf16(buf[i].y * r)),
                         fmaxf(abs_bf16(buf[i].z * r), abs_bf16(buf[i].w * r))));
    amax_slot_update(amax, m, row);
  }
}

template <int NV>
__global__ void __launch_bounds__(128) rmsnorm_bwd_kernel(const float* __restrict__ dy, const bf16* __restrict__ y,
                                                          const float* __restrict__ rstd, float* __restrict__ dx,
                                                          bf16* __restrict__ dxb, int M, int accumulate,
                                                          unsigned int* __restrict__ amax) {
  constexpr int d = 128 * NV;
  const int row = blockIdx.x * 4 + warp_id();
  if (row >= M) return;
  const long long off = static_cast<long long>(row) * d;
  float4 g[NV], p[NV];
  uint2 yy[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (i * 32 + lane_id()) * 4;
    g[i] = *reinterpret_cast<const float4*>(dy + off + c);
    yy[i] = *reinterpret_cast<const uint2*>(y + off + c);
    p[i] = accumulate ? *reinterpret_cast<const float4*>(dx + off + c) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const float r = rstd[row];
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i)
    dot += g[i].x * bf16_lo(yy[i].x) + g[i].y * bf16_hi(yy[i].x) + g[i].z * bf16_lo(yy[i].y) + g[i].w * bf16_hi(yy[i].y);
  dot = warp_sum(dot) * (1.f / d);
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (i * 32 + lane_id()) * 4;
    float4 o;
    o.x = p[i].x + r * (g[i].x - bf16_lo(yy[i].x) * dot);
    o.y = p[i].y + r * (g[i].y - bf16_hi(yy[i].x) * dot);
    o.z = p[i].z + r * (g[i].z - bf16_lo(yy[i].y) * dot);
    o.w = p[i].w + r * (g[i].w - bf16_hi(yy[i].y) * dot);
    *reinterpret_cast<float4*>(dx + off + c) = o;
    store_bf16x4(dxb + off + c, o);
    if (amax) m = fmaxf(m, fmaxf(fmaxf(abs_bf16(o.x), abs_bf16(o.y)), fmaxf(abs_bf16(o.z), abs_bf16(o.w))));
  }
  if (amax) amax_slot_update(amax, m, row);
}

// ------------------------------------------- residual scales and backout
//
// Per-layer residual scaling and backout ("¿Cómo Entrenar Tu Propio ChatGPT
// por $50?", section "1. Modelo GPT", efficiency tricks 1 and 3).  lam holds
// (resid[0..L), x0[0..L), backout).

// Before block l: x_in[l] = x; x = resid[l] x + x0[l] x0 (block 0 also
// stores x0 = x, the embedding output).
__global__ void resid_fwd_kernel(float* __restrict__ x, float* __restrict__ x_in, float* __restrict__ x0,
                                 const float* __restrict__ lam, int l, int L, long long n4, int first) {
  const float a = lam[l], b = lam[L + l];
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(x)[i];
    reinterpret_cast<float4*>(x_in)[i] = v;
    float4 z;
    if (first) {
      z = v;
      reinterpret_cast<float4*>(x0)[i] = v;
    } else {
      z = reinterpret_cast<const float4*>(x0)[i];
    }
    reinterpret_cast<float4*>(x)[i] =
        make_float4(a * v.x + b * z.x, a * v.y + b * z.y, a * v.z + b * z.z, a * v.w + b * z.w);
  }
}

// After the last block: x -= backout * x_mid.
__global__ void backout_fwd_kernel(float* __restrict__ x, const float* __restrict__ x_mid,
                                   const float* __restrict__ lam, int L, long long n4) {
  const float c = lam[2 * L];
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float4 v = reinterpret_cast<float4*>(x)[i];
    const float4 m = reinterpret_cast<const float4*>(x_mid)[i];
    v.x -= c * m.x; v.y -= c * m.y; v.z -= c * m.z; v.w -= c * m.w;
    reinterpret_cast<float4*>(x)[i] = v;
  }
}

// Block sum of two per-thread values into part_a[blockIdx.x], part_b[blockIdx.x]
// (a fixed grid and a fixed reduction tree, so the result does not depend on
// scheduling).
__device__ __forceinline__ void block_sum2(float sa, float sb, float* part_a, float* part_b) {
  __shared__ float ra[32], rb[32];
  sa = warp_sum(sa);
  sb = warp_sum(sb);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    ra[w] = sa;
    rb[w] = sb;
  }
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    float a = lane < nw ? ra[lane] : 0.f, b = lane < nw ? rb[lane] : 0.f;
    a = warp_sum(a);
    b = warp_sum(b);
    if (lane == 0) {
      if (part_a) part_a[blockIdx.x] = a;
      if (part_b) part_b[blockIdx.x] = b;
    }
  }
}

// Backward through x' = resid[l] x_in + x0[l] x0 given g = dL/dx' in dx:
// partial sums of x_in . g and x0 . g, dx0 (+)= x0[l] g, dx = resid[l] g
// (minus backout * dx_final for the block whose input the backout read), and
// the bf16 copy of dx for the block below; for block 0 dx also takes dx0 (the
// embedding output fed every block through x0).
__global__ void __launch_bounds__(256) resid_bwd_kernel(float* __restrict__ dx, const float* __restrict__ x_in,
                                                        const float* __restrict__ x0, float* __restrict__ dx0,
                                                        const float* __restrict__ dx_final,
                                                        const float* __restrict__ lam, int l, int L, long long n4,
                                                        bf16* __restrict__ gout, float* __restrict__ part_r,
                                                        float* __restrict__ part_0, int first, int last) {
  const float a = lam[l], b = lam[L + l], c = dx_final ? lam[2 * L] : 0.f;
  float sr = 0.f, s0 = 0.f;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 g = reinterpret_cast<const float4*>(dx)[i];
    const float4 xi = reinterpret_cast<const float4*>(x_in)[i];
    const float4 z = reinterpret_cast<const float4*>(x0)[i];
    sr += xi.x * g.x + xi.y * g.y + xi.z * g.z + xi.w * g.w;
    s0 += z.x * g.x + z.y * g.y + z.z * g.z + z.w * g.w;
    float4 d0 = first ? make_float4(0.f, 0.f, 0.f, 0.f) : reinterpret_cast<const float4*>(dx0)[i];
    d0.x += b * g.x; d0.y += b * g.y; d0.z += b * g.z; d0.w += b * g.w;
    float4 o = make_float4(a * g.x, a * g.y, a * g.z, a * g.w);
    if (dx_final) {
      const float4 f = reinterpret_cast<const float4*>(dx_final)[i];
      o.x -= c * f.x; o.y -= c * f.y; o.z -= c * f.z; o.w -= c * f.w;
    }
    if (last) {
      o.x += d0.x; o.y += d0.y; o.z += d0.z; o.w += d0.w;
    } else {
      reinterpret_cast<float4*>(dx0)[i] = d0;
    }
    reinterpret_cast<float4*>(dx)[i] = o;
    store_bf16x4(gout + 4 * i, o);
  }
  block_sum2(sr, s0, part_r, part_0);
}

// Partial sums of a . b (the backout scale's gradient is -sum x_mid . dx_final).
__global__ void __launch_bounds__(256) dot_partial_kernel(const float* __restrict__ a, const float* __restrict__ b,
                                                          long long n4, float* __restrict__ part) {
  float s = 0.f;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 x = reinterpret_cast<const float4*>(a)[i];
    const float4 y = reinterpret_cast<const float4*>(b)[i];
    s += x.x * y.x + x.y * y.y + x.z * y.z + x.w * y.w;
  }
  block_sum2(s, 0.f, part, nullptr);
}

// Smear (efficiency trick 2): x[t] = e[t] + gate[t] e[t-1] for t > 0 within
// a sequence, gate[t] = lam_s * sigmoid(w . e[t, :24]) with lam_s = lam[2L+1]
// and w = lam[2L+2 .. 2L+26).  One warp per token; sig[t] is kept for the
// backward.
constexpr int kSmearChannels = 24;

__global__ void __launch_bounds__(256) smear_fwd_kernel(const float* __restrict__ e, float* __restrict__ x,
                                                        float* __restrict__ sig, const float* __restrict__ lam,
                                                        int L, int T, int M, int d) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= M) return;
  const float* er = e + static_cast<long long>(t) * d;
  float z = lane < kSmearChannels ? lam[2 * L + 2 + lane] * er[lane] : 0.f;
  z = warp_sum(z);
  const float sg = 1.f / (1.f + expf(-z));
  const float gate = (t % T) > 0 ? lam[2 * L + 1] * sg : 0.f;
  if (lane == 0) sig[t] = sg;
  float* xr = x + static_cast<long long>(t) * d;
  for (int c = 4 * lane; c < d; c += 128) {
    const float4 v = *reinterpret_cast<const float4*>(er + c);
    float4 o = v;
    if (gate != 0.f) {
      const float4 p = *reinterpret_cast<const float4*>(er - d + c);
      o.x += gate * p.x; o.y += gate * p.y; o.z += gate * p.z; o.w += gate * p.w;
    }
    *reinterpret_cast<float4*>(xr + c) = o;
  }
}

// Backward of the smear: g = dL/dx, output de = dL/de; partial sums of the
// smear scale's and gate weights' gradients per block (part[j * nb + block]
// for scalar j = 2L+1 .. 2L+25).  A fixed grid of warps strides over the
// tokens, so the sums do not depend on scheduling.
__global__ void __launch_bounds__(256) smear_bwd_kernel(const float* __restrict__ g, const float* __restrict__ e,
                                                        const float* __restrict__ sig, const float* __restrict__ lam,
                                                        float* __restrict__ de, float* __restrict__ part, int L,
                                                        int T, int M, int d) {
  __shared__ float acc[8][kSmearChannels + 1];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float lam_s = lam[2 * L + 1];
  const float wc = lane < kSmearChannels ? lam[2 * L + 2 + lane] : 0.f;
  float a_lam = 0.f, a_w = 0.f;   // this lane's share: the scale (lane 0) and gate weight `lane`
  for (int t = blockIdx.x * 8 + w; t < M; t += gridDim.x * 8) {
    const long long off = static_cast<long long>(t) * d;
    const int pos = t % T;
    // s = dL/dgate[t] = g[t] . e[t-1]
    float sdot = 0.f;
    if (pos > 0) {
      for (int c = 4 * lane; c < d; c += 128) {
        const float4 a = *reinterpret_cast<const float4*>(g + off + c);
        const float4 b = *reinterpret_cast<const float4*>(e + off - d + c);
        sdot += a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
      }
    }
    sdot = warp_sum(sdot);
    const float sg = sig[t];
    const float dz = sdot * lam_s * sg * (1.f - sg);
    const float gnext = (pos + 1 < T && t + 1 < M) ? lam_s * sig[t + 1] : 0.f;   // e[t] feeds position t + 1
    for (int c = 4 * lane; c < d; c += 128) {
      float4 o = *reinterpret_cast<const float4*>(g + off + c);
      if (gnext != 0.f) {
        const float4 n = *reinterpret_cast<const float4*>(g + off + d + c);
        o.x += gnext * n.x; o.y += gnext * n.y; o.z += gnext * n.z; o.w += gnext * n.w;
      }
      *reinterpret_cast<float4*>(de + off + c) = o;
    }
    __syncwarp();
    if (lane < kSmearChannels) {
      // the gate reads channels 0..23: d(de[t, c]) = dz w[c]; dw[c] += dz e[t, c]
      de[off + lane] += dz * wc;
      a_w += dz * e[off + lane];
    }
    a_lam += sdot * sg;
  }
  if (lane < kSmearChannels) acc[w][1 + lane] = a_w;
  if (lane == 0) acc[w][0] = a_lam;
  __syncthreads();
  if (threadIdx.x < kSmearChannels + 1) {
    float sum = 0.f;
    for (int k = 0; k < 8; ++k) sum += acc[k][threadIdx.x];
    part[static_cast<long long>(2 * L + 1 + threadIdx.x) * gridDim.x + blockIdx.x] = sum;
  }
}

// Value embeddings (section "1. Modelo GPT", value residual): on a value-
// embedding layer, v[t, h] += 3 sigmoid(xn1[t, :C] . Wg[:, h]) ve[tok[t], h].
// v is [B, H, T, 128] bf16 (the attention input), ve the bf16 copy of the
// layer's [V, d] table, Wg [C, H] fp32.  One warp per token; sig [M, H] is
// kept for the backward.  Ids outside [0, V) read row 0 (they are latched as
// errors by the range check).
__global__ void __launch_bounds__(256) ve_fwd_kernel(const bf16* __restrict__ xn1, const int* __restrict__ tok,
                                                     const bf16* __restrict__ ve, const float* __restrict__ wg,
                                                     float* __restrict__ sig, bf16* __restrict__ v, int M, int T,
                                                     int H, int Hkv, int C, int V) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= M) return;
  const int d = H * 128, kvd = Hkv * 128;
  const int b = t / T, pos = t - b * T;
  int id = tok[t];
  id = static_cast<unsigned>(id) < static_cast<unsigned>(V) ? id : 0;
  const bf16* xr = xn1 + static_cast<long long>(t) * d;
  const bf16* er = ve + static_cast<long long>(id) * kvd;
  for (int h = 0; h < Hkv; ++h) {   // kv head h sits at head row b*H + h of v
    float z = 0.f;
    for (int c = lane; c < C; c += 32) z += __bfloat162float(xr[c]) * wg[c * Hkv + h];
    z = warp_sum(z);
    const float sg = 1.f / (1.f + expf(-z));
    if (lane == 0) sig[static_cast<long long>(t) * Hkv + h] = sg;
    const float gate = 3.f * sg;
    bf16* vr = v + ((static_cast<long long>(b) * H + h) * T + pos) * 128 + 4 * lane;
    const uint2 a = *reinterpret_cast<const uint2*>(vr);
    const uint2 e = *reinterpret_cast<const uint2*>(er + h * 128 + 4 * lane);
    uint2 o;
    o.x = pack_bf16x2(bf16_lo(a.x) + gate * bf16_lo(e.x), bf16_hi(a.x) + gate * bf16_hi(e.x));
    o.y = pack_bf16x2(bf16_lo(a.y) + gate * bf16_lo(e.y), bf16_hi(a.y) + gate * bf16_hi(e.y));
    *reinterpret_cast<uint2*>(vr) = o;
  }
}

// Backward, given dv [B, H, T, 128] (the gradient at the attention input):
// dve[t, h] = 3 sig dv[t, h] (fp32 [M, d], scattered into the table's
// gradient afterwards) and dz[t, h] = (ve[t, h] . dv[t, h]) 3 sig (1 - sig).
__global__ void __launch_bounds__(256) ve_bwd_kernel(const bf16* __restrict__ dv, long long ldv,
                                                     const int* __restrict__ tok, const bf16* __restrict__ ve,
                                                     const float* __restrict__ sig, float* __restrict__ dve,
                                                     float* __restrict__ dz, int M, int Hkv, int V) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= M) return;
  const int kvd = Hkv * 128;
  int id = tok[t];
  id = static_cast<unsigned>(id) < static_cast<unsigned>(V) ? id : 0;
  const bf16* er = ve + static_cast<long long>(id) * kvd;
  for (int h = 0; h < Hkv; ++h) {
    const uint2 g = *reinterpret_cast<const uint2*>(dv + static_cast<long long>(t) * ldv + h * 128 + 4 * lane);
    const uint2 e = *reinterpret_cast<const uint2*>(er + h * 128 + 4 * lane);
    const float g0 = bf16_lo(g.x), g1 = bf16_hi(g.x), g2 = bf16_lo(g.y), g3 = bf16_hi(g.y);
    float dot = g0 * bf16_lo(e.x) + g1 * bf16_hi(e.x) + g2 * bf16_lo(e.y) + g3 * bf16_hi(e.y);
    dot = warp_sum(dot);
    const float sg = sig[static_cast<long long>(t) * Hkv + h];
    const float gate = 3.f * sg;
    *reinterpret_cast<float4*>(dve + static_cast<long long>(t) * kvd + h * 128 + 4 * lane) =
        make_float4(gate * g0, gate * g1, gate * g2, gate * g3);
    if (lane == 0) dz[static_cast<long long>(t) * Hkv + h] = dot * 3.f * sg * (1.f - sg);
  }
}

// Partial sums of dWg[c, h] = sum_t xn1[t, c] dz[t, h]: block k takes a fixed
// range of tokens, thread (c, h) its own pair (C * H <= blockDim.x);
// part[(c * H + h) * gridDim.x + k].
__global__ void __launch_bounds__(1024) ve_gate_grad_kernel(const bf16* __restrict__ xn1,
                                                            const float* __restrict__ dz, float* __restrict__ part,
                                                            int M, int d, int H, int C) {
  const int pair = threadIdx.x;
  const int per = (M + gridDim.x - 1) / gridDim.x;
  const int t0 = blockIdx.x * per, t1 = min(M, t0 + per);
  if (pair >= C * H) return;
  const int c = pair / H, h = pair - (pair / H) * H;
  float s = 0.f;
  for (int t = t0; t < t1; ++t)
    s += __bfloat162float(xn1[static_cast<long long>(t) * d + c]) * dz[static_cast<long long>(t) * H + h];
  part[static_cast<long long>(pair) * gridDim.x + blockIdx.x] = s;
}

// dxn1[t, c] += sum_h dz[t, h] Wg[c, h] for c < C (the gate reads xn1[:, :C]).
__global__ void __launch_bounds__(256) ve_dxn_kernel(float* __restrict__ dxn, const float* __restrict__ dz,
                                                     const float* __restrict__ wg, int M, int d, int H, int C) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= M) return;
  for (int c = lane; c < C; c += 32) {
    float s = 0.f;
    for (int h = 0; h < H; ++h) s += dz[static_cast<long long>(t) * H + h] * wg[c * H + h];
    dxn[static_cast<long long>(t) * d + c] += s;
  }
}

// Scalar gradients from their partial sums (nb per scalar, summed in a fixed
// order by one warp each): grad[j] (+)= sum_k part[j][k], negated for j =
// neg_index (the backout scale, whose partials are sums of x_mid . dx).
__global__ void scalar_grad_finish_kernel(const float* __restrict__ part, int nb, int count, int neg_index,
                                          float* __restrict__ grad, int accumulate) {
  const int j = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (j >= count) return;
  float s = 0.f;
  for (int k = lane; k < nb; k += 32) s += part[static_cast<long long>(j) * nb + k];
  s = warp_sum(s);
  if (lane == 0) {
    if (j == neg_index) s = -s;
    grad[j] = accumulate ? grad[j] + s : s;
  }
}

// -------------------------------------------------- QK-norm / RoPE backward

// kGrouped: fewer kv heads than query heads (the plain case keeps the
// unconditional k/v path).
template <bool kGrouped>
__global__ void qk_bwd_kernel(const float* __restrict__ dq, const bf16* __restrict__ dk,
                              const bf16* __restrict__ dv, const bf16* __restrict__ qn,
                              const bf16* __restrict__ kn, const float* __restrict__ rq,
                              const float* __restrict__ rk, const float2* __restrict__ rope,
                              bf16* __restrict__ dqkv, int B, int T, int H, int Hkv,
                              unsigned int* __restrict__ amax) {
  const long long w = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + warp_id();
  const long long total = static_cast<long long>(B) * H * T;
  if (w >= total) return;
  // w enumerates (b, h, t) in the head-major layout of q/k/v
  const int t = static_cast<int>(w % T);
  const int h = static_cast<int>((w / T) % H);
  const int b = static_cast<int>(w / (static_cast<long long>(T) * H));
  const long long m = static_cast<long long>(b) * T + t;
  const int d = H * 128, kvd = Hkv * 128;
  const long long src = w * 128;   // k/v heads j < Hkv sit at the same head rows as q's
  const int i0 = 2 * lane_id();
  const float2 e0 = rope[t * 64 + i0], e1 = rope[t * 64 + i0 + 1];
  // row of dqkv: q (d) | k (kvd) | v (kvd); head h of k and v only for h < Hkv
  bf16* out = dqkv + m * (d + 2 * kvd) + h * 128;
  const bool has_kv = dk && (!kGrouped || h < Hkv);   // no dk: the k and v columns are written elsewhere
  float am = 0.f;   // max |written value| (for fp8 scales)
#pragma unroll
  for (int which = 0; which < 2; ++which) {
    if (which == 1 && !has_kv) break;
    const bf16* yv = which == 0 ? qn : kn;
    const float r = (which == 0 ? rq : rk)[m * H + h];
    float gl0, gl1, gh0, gh1;
    if (which == 0) {
      const float2 a = *reinterpret_cast<const float2*>(dq + src + i0);
      const float2 c = *reinterpret_cast<const float2*>(dq + src + 64 + i0);
      gl0 = a.x; gl1 = a.y; gh0 = c.x; gh1 = c.y;
    } else {
      const uint32_t glo = *reinterpret_cast<const uint32_t*>(dk + src + i0);
      const uint32_t ghi = *reinterpret_cast<const uint32_t*>(dk + src + 64 + i0);
      gl0 = bf16_lo(glo); gl1 = bf16_hi(glo); gh0 = bf16_lo(ghi); gh1 = bf16_hi(ghi);
    }
    const uint32_t ylo = *reinterpret_cast<const uint32_t*>(yv + src + i0);
    const uint32_t yhi = *reinterpret_cast<const uint32_t*>(yv + src + 64 + i0);
    float yl0 = bf16_lo(ylo), yl1 = bf16_hi(ylo), yh0 = bf16_lo(yhi), yh1 = bf16_hi(yhi);
    float dot = gl0 * yl0 + gl1 * yl1 + gh0 * yh0 + gh1 * yh1;
    dot = warp_sum(dot) * (1.f / 128.f);
    // gradient w.r.t. the rotated vector, then the transposed rotation
    const float rl0 = r * (gl0 - yl0 * dot), rl1 = r * (gl1 - yl1 * dot);
    const float rh0 = r * (gh0 - yh0 * dot), rh1 = r * (gh1 - yh1 * dot);
    const float ol0 = rl0 * e0.x + rh0 * e0.y, oh0 = -rl0 * e0.y + rh0 * e0.x;
    const float ol1 = rl1 * e1.x + rh1 * e1.y, oh1 = -rl1 * e1.y + rh1 * e1.x;
    *reinterpret_cast<uint32_t*>(out + which * d + i0) = pack_bf16x2(ol0, ol1);
    *reinterpret_cast<uint32_t*>(out + which * d + 64 + i0) = pack_bf16x2(oh0, oh1);
    if (amax) am = fmaxf(am, fmaxf(fmaxf(abs_bf16(ol0), abs_bf16(ol1)), fmaxf(abs_bf16(oh0), abs_bf16(oh1))));
  }
  if (has_kv) {
    const uint2 vv = *reinterpret_cast<const uint2*>(dv + src + 4 * lane_id());
    *reinterpret_cast<uint2*>(out + d + kvd + 4 * lane_id()) = vv;
    if (amax)
      am = fmaxf(am, fmaxf(fmaxf(fabsf(bf16_lo(vv.x)), fabsf(bf16_hi(vv.x))),
                           fmaxf(fabsf(bf16_lo(vv.y)), fabsf(bf16_hi(vv.y)))));
  }
  if (amax) amax_slot_update(amax, am, w);
}

// q alone (the attention backward writes the k and v columns): half a warp
// per (b, h, t) row, lane l of the half holding dims 4l..4l+3 and
// 64+4l..64+4l+3, so that each rotation pair (i, i + 64) sits in one thread
// and every access is a 16- or 8-byte vector; 32-bit indices (the launcher
// checks the row count).
__global__ void __launch_bounds__(256) qk_bwd_q_kernel(const float* __restrict__ dq, const bf16* __restrict__ qn,
                                                       const float* __restrict__ rq, const float2* __restrict__ rope,
                                                       bf16* __restrict__ dqkv, int total, int T, int H, int row_len,
                                                       unsigned int* __restrict__ amax) {
  const int w = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 4);
  if ((w & ~1) >= total) return;   // both rows of the warp past the end
  const bool valid = w < total;
  const int l = threadIdx.x & 15;
  const int t = w % T, bh = w / T;
  const int h = bh % H, b = bh / H;
  const int m = b * T + t;
  float am = 0.f;
  float g[8], y[8];
  float4 e[4];   // (cos, sin) of dims 4l .. 4l+3 as float2 pairs
  float r = 0.f;
  if (valid) {
    const long long src = static_cast<long long>(w) * 128 + 4 * l;
    const float4 a = *reinterpret_cast<const float4*>(dq + src);
    const float4 c = *reinterpret_cast<const float4*>(dq + src + 64);
    const uint2 ylo = *reinterpret_cast<const uint2*>(qn + src);
    const uint2 yhi = *reinterpret_cast<const uint2*>(qn + src + 64);
    const float4* ep = reinterpret_cast<const float4*>(rope + static_cast<long long>(t) * 64 + 4 * l);
    e[0] = ep[0]; e[1] = ep[1];
    r = rq[static_cast<long long>(m) * H + h];
    g[0] = a.x; g[1] = a.y; g[2] = a.z; g[3] = a.w;
    g[4] = c.x; g[5] = c.y; g[6] = c.z; g[7] = c.w;
    y[0] = bf16_lo(ylo.x); y[1] = bf16_hi(ylo.x); y[2] = bf16_lo(ylo.y); y[3] = bf16_hi(ylo.y);
    y[4] = bf16_lo(yhi.x); y[5] = bf16_hi(yhi.x); y[6] = bf16_lo(yhi.y); y[7] = bf16_hi(yhi.y);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) g[i] = y[i] = 0.f;
    e[0] = e[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) dot += g[i] * y[i];
  // sum over the half warp's 16 lanes
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  dot *= 1.f / 128.f;
  if (valid) {
    // gradient w.r.t. the rotated vector, then the transposed rotation
    const float cs[4] = {e[0].x, e[0].z, e[1].x, e[1].z};
    const float sn[4] = {e[0].y, e[0].w, e[1].y, e[1].w};
    float ol[4], oh[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float rl = r * (g[i] - y[i] * dot), rh = r * (g[4 + i] - y[4 + i] * dot);
      ol[i] = rl * cs[i] + rh * sn[i];
      oh[i] = -rl * sn[i] + rh * cs[i];
    }
    bf16* out = dqkv + static_cast<long long>(m) * row_len + h * 128 + 4 * l;
    *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf16x2(ol[0], ol[1]), pack_bf16x2(ol[2], ol[3]));
    *reinterpret_cast<uint2*>(out + 64) = make_uint2(pack_bf16x2(oh[0], oh[1]), pack_bf16x2(oh[2], oh[3]));
    if (amax)
#pragma unroll
      for (int i = 0; i < 4; ++i) am = fmaxf(am, fmaxf(abs_bf16(ol[i]), abs_bf16(oh[i])));
  }
  if (amax) amax_slot_update(amax, am, w);
}

// ------------------------------------------------------- cross-entropy finish

__global__ void __launch_bounds__(256) ce_finish_kernel(bf16* __restrict__ z, const float2* __restrict__ stats,
                                                        const float* __restrict__ zt, const int* __restrict__ tgt,
                                                        float* __restrict__ row_loss, int V, int tiles_n,
                                                        float inv_count) {
  __shared__ float red[8];
  __shared__ float bc;
  const int row = blockIdx.x;
  const float2* st = stats + static_cast<long long>(row) * tiles_n;
  float mx = -INFINITY;
  for (int i = threadIdx.x; i < tiles_n; i += blockDim.x) mx = fmaxf(mx, st[i].x);
  mx = warp_max(mx);
  if (lane_id() == 0) red[warp_id()] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = red[0];
    for (int i = 1; i < 8; ++i) m = fmaxf(m, red[i]);
    bc = m;
  }
  __syncthreads();
  mx = bc;
  float s = 0.f;
  for (int i = threadIdx.x; i < tiles_n; i += blockDim.x) s += st[i].y * __expf(st[i].x - mx);
  s = warp_sum(s);
  __syncthreads();
  if (lane_id() == 0) red[warp_id()] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < 8; ++i) t += red[i];
    const float lse = mx + logf(t);
    bc = lse;
    row_loss[row] = lse - zt[row];
  }
  __syncthreads();
  const float lse = bc;
  const int tg = tgt[row];
  bf16* zr = z + static_cast<long long>(row) * V;
  for (int c = threadIdx.x * 8; c < V; c += blockDim.x * 8) {
    uint4 w = *reinterpret_cast<const uint4*>(zr + c);
    uint32_t* u = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float a = __expf(bf16_lo(u[j]) - lse), b = __expf(bf16_hi(u[j]) - lse);
      if (c + 2 * j == tg) a -= 1.f;
      if (c + 2 * j + 1 == tg) b -= 1.f;
      u[j] = pack_bf16x2(a * inv_count, b * inv_count);
    }
    *reinterpret_cast<uint4*>(zr + c) = w;
  }
}

__global__ void __launch_bounds__(1024) sum_scale_kernel(const float* __restrict__ v, int n, float scale,
                                                         float* __restrict__ out) {
  __shared__ float red[32];
  float s = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s += v[i];
  s = warp_sum(s);
  if (lane_id() == 0) red[warp_id()] = s;
  __syncthreads();
  if (warp_id() == 0) {
    float t = lane_id() < static_cast<int>(blockDim.x / 32) ? red[lane_id()] : 0.f;
    t = warp_sum(t);
    if (lane_id() == 0) *out = t * scale;
  }
}

// ---------------------------------------------------------------- split-K

__global__ void splitk_reduce_kernel(const float* __restrict__ part, int splits, long long stride, long long n4,
                                     float* __restrict__ out, int accumulate) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float4 a = accumulate ? reinterpret_cast<const float4*>(out)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < splits; ++s) {
      const float4 b = reinterpret_cast<const float4*>(part + s * stride)[i];
      a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
    }
    reinterpret_cast<float4*>(out)[i] = a;
  }
}

// ------------------------------------------------------------------ AdamW

__global__ void adamw_kernel(float* __restrict__ p, const float* __restrict__ g, float* __restrict__ m,
                             float* __restrict__ v, bf16* __restrict__ pb, long long n4, float lr, float b1,
                             float b2, float eps, float wd, float bc1, float bc2) {
  const float decay = 1.f - lr * wd;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float4 pp = reinterpret_cast<float4*>(p)[i];
    const float4 gg = reinterpret_cast<const float4*>(g)[i];
    float4 mm = reinterpret_cast<float4*>(m)[i];
    float4 vv = reinterpret_cast<float4*>(v)[i];
    float* pa = &pp.x; const float* ga = &gg.x; float* ma = &mm.x; float* va = &vv.x;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      ma[j] = b1 * ma[j] + (1.f - b1) * ga[j];
      va[j] = b2 * va[j] + (1.f - b2) * ga[j] * ga[j];
      const float mh = ma[j] / bc1;
      const float vh = va[j] / bc2;
      pa[j] = pa[j] * decay - lr * mh / (sqrtf(vh) + eps);
    }
    reinterpret_cast<float4*>(p)[i] = pp;
    reinterpret_cast<float4*>(m)[i] = mm;
    reinterpret_cast<float4*>(v)[i] = vv;
    store_bf16x4(pb + 4 * i, pp);
  }
}

// ------------------------------------------------------------------- Muon

constexpr int kNormBlocks = 64;

__global__ void __launch_bounds__(256) muon_momentum_kernel(float* __restrict__ mom, const float* __restrict__ g,
                                                            long long n4, float beta, float* __restrict__ part) {
  const int z = blockIdx.y;
  float4* mz = reinterpret_cast<float4*>(mom) + z * n4;
  const float4* gz = reinterpret_cast<const float4*>(g) + z * n4;
  float ss = 0.f;
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n4; i += kNormBlocks * 256ll) {
    float4 a = mz[i];
    const float4 b = gz[i];
    a.x = beta * a.x + b.x; a.y = beta * a.y + b.y; a.z = beta * a.z + b.z; a.w = beta * a.w + b.w;
    mz[i] = a;
    ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
  }
  __shared__ float red[8];
  ss = warp_sum(ss);
  if (lane_id() == 0) red[warp_id()] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int i = 0; i < 8; ++i) t += red[i];
    part[z * kNormBlocks + blockIdx.x] = t;
  }
}

__global__ void muon_norm_kernel(const float* __restrict__ part, int nmat, float eps, float* __restrict__ inv_norm) {
  const int z = blockIdx.x;
  if (z >= nmat) return;
  float s = 0.f;
  for (int i = lane_id(); i < kNormBlocks; i += 32) s += part[z * kNormBlocks + i];
  s = warp_sum(s);
  if (lane_id() == 0) inv_norm[z] = 1.f / (sqrtf(s) + eps);
}

// Both Muon elementwise passes work on 64 x 64 tiles with 256 threads: thread
// (tx, ty) = (threadIdx.x % 16, threadIdx.x / 16) covers columns 4 tx .. 4 tx + 3
// of rows ty, ty + 16, ty + 32, ty + 48, and a transposed write goes through a
// padded shared-memory tile.  Matrix extents are multiples of 4.

template <typename T>
__device__ __forceinline__ void store4(T* p, float a, float b, float c, float d) {
  if constexpr (std::is_same<T, __half>::value) {
    __half2 h0 = __floats2half2_rn(a, b), h1 = __floats2half2_rn(c, d);
    uint2 w;
    w.x = *reinterpret_cast<uint32_t*>(&h0);
    w.y = *reinterpret_cast<uint32_t*>(&h1);
    *reinterpret_cast<uint2*>(p) = w;
  } else if constexpr (sizeof(T) == 2) {
    uint2 w;
    w.x = pack_bf16x2(a, b);
    w.y = pack_bf16x2(c, d);
    *reinterpret_cast<uint2*>(p) = w;
  } else {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
  }
}

template <typename T>
__device__ __forceinline__ float4 load4(const T* p) {
  if constexpr (sizeof(T) == 2) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    return make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
  } else {
    return *reinterpret_cast<const float4*>(p);
  }
}

// From the momentum mom[z] (rows x cols): `same` = s_z mom[z] in the same
// layout and `trans` = (s_z mom[z])^T (cols x rows), s_z = inv_norm[z], in
// storage type T1, and the same pair in T2; any output may be null.  One read
// of the momentum serves all of them.
template <typename T1, typename T2>
__global__ void __launch_bounds__(256) muon_make_x_kernel(const float* __restrict__ mom,
                                                          const float* __restrict__ inv_norm, T1* __restrict__ same1,
                                                          T1* __restrict__ trans1, T2* __restrict__ same2,
                                                          T2* __restrict__ trans2, int rows, int cols) {
  __shared__ float tile[64][65];
  const int z = blockIdx.z;
  const float s = inv_norm[z];
  const long long n = static_cast<long long>(rows) * cols;
  const float* mz = mom + z * n;
  const int r0 = blockIdx.y * 64, c0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int cc = c0 + 4 * tx;
  const bool want_t = trans1 || trans2;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int rr = r0 + ty + 16 * k;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (rr < rows && cc < cols) {
      v = *reinterpret_cast<const float4*>(mz + static_cast<long long>(rr) * cols + cc);
      v.x *= s; v.y *= s; v.z *= s; v.w *= s;
      const long long o = z * n + static_cast<long long>(rr) * cols + cc;
      if (same1) store4(same1 + o, v.x, v.y, v.z, v.w);
      if (same2) store4(same2 + o, v.x, v.y, v.z, v.w);
    }
    if (want_t) {
      tile[ty + 16 * k][4 * tx] = v.x;
      tile[ty + 16 * k][4 * tx + 1] = v.y;
      tile[ty + 16 * k][4 * tx + 2] = v.z;
      tile[ty + 16 * k][4 * tx + 3] = v.w;
    }
  }
  if (!want_t) return;
  __syncthreads();
  // rows of the transpose are columns of the tile
  const int oc = r0 + 4 * tx;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int orow = c0 + ty + 16 * k, tc = ty + 16 * k;
    if (orow < cols && oc < rows) {
      const long long o = z * n + static_cast<long long>(orow) * rows + oc;
      const float a = tile[4 * tx][tc], b = tile[4 * tx + 1][tc], c = tile[4 * tx + 2][tc], d = tile[4 * tx + 3][tc];
      if (trans1) store4(trans1 + o, a, b, c, d);
      if (trans2) store4(trans2 + o, a, b, c, d);
    }
  }
}

// NorMuon ("¿Cómo Entrenar Tu Propio ChatGPT por $50?", section "2. Optimizador
// Muon", NorMuon variance reduction).  The orthogonalised update X[z] is held
// with its shorter axis as rows (r <= c), so the per-neuron second moment is a
// mean over each row.  First pass: the sum of squares of every row, one warp
// per row (c is a multiple of 4).
template <typename XT>
__global__ void __launch_bounds__(256) row_sumsq_kernel(const XT* __restrict__ X, int r, int c,
                                                        float* __restrict__ out) {
  const int z = blockIdx.y;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= r) return;
  const XT* xr = X + (static_cast<long long>(z) * r + row) * c;
  float acc = 0.f;
  for (int j = 4 * lane; j < c; j += 128) {
    const float4 u = load4(xr + j);
    acc = fmaf(u.x, u.x, acc);
    acc = fmaf(u.y, u.y, acc);
    acc = fmaf(u.z, u.z, acc);
    acc = fmaf(u.w, u.w, acc);
  }
  acc = warp_sum(acc);
  if (lane == 0) out[static_cast<long long>(z) * r + row] = acc;
}

// Second pass, one block per matrix: v_mean = sumsq / c;
// V <- beta2 V + (1 - beta2) v_mean; s = max(V, 1e-10)^(-1/2); the factor
// f = s * ||v_mean||^(1/2) / max(||v_mean s^2||^(1/2), 1e-10) (sums over the
// rows) keeps the Frobenius norm of the update.  f overwrites the sums.
__global__ void __launch_bounds__(1024) normuon_factor_kernel(float* __restrict__ ss_f, float* __restrict__ V, int r,
                                                              int c, float beta2) {
  __shared__ float red[2][32];
  const int z = blockIdx.x;
  float* sf = ss_f + static_cast<long long>(z) * r;
  float* v = V + static_cast<long long>(z) * r;
  const float inv_c = 1.f / static_cast<float>(c);
  float sum_m = 0.f, sum_ms = 0.f;
  for (int i = threadIdx.x; i < r; i += blockDim.x) {
    const float m = sf[i] * inv_c;
    const float vn = fmaf(beta2, v[i], (1.f - beta2) * m);
    v[i] = vn;
    const float vc = fmaxf(vn, 1e-10f);
    sum_m += m;
    sum_ms += m / vc;
  }
  sum_m = warp_sum(sum_m);
  sum_ms = warp_sum(sum_ms);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    red[0][w] = sum_m;
    red[1][w] = sum_ms;
  }
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    float a = lane < nw ? red[0][lane] : 0.f, b = lane < nw ? red[1][lane] : 0.f;
    a = warp_sum(a);
    b = warp_sum(b);
    if (lane == 0) {
      red[0][0] = a;
      red[1][0] = b;
    }
  }
  __syncthreads();
  const float ratio = sqrtf(red[0][0]) / fmaxf(sqrtf(red[1][0]), 1e-10f);
  for (int i = threadIdx.x; i < r; i += blockDim.x) sf[i] = ratio / sqrtf(fmaxf(v[i], 1e-10f));
}

// W[z] <- decay W[z] - step U with U = X[z] (r x c, W in the same layout) or
// U = X[z]^T (W is c x r); also refreshes the bf16 working copy.  With rowf,
// row i of X[z] is first scaled by rowf[z r + i] (the NorMuon factor).
template <typename XT>
__global__ void __launch_bounds__(256) muon_apply_kernel(float* __restrict__ W, bf16* __restrict__ Wb,
                                                         const XT* __restrict__ X, const float* __restrict__ rowf,
                                                         int r, int c, int transpose, float decay, float step) {
  __shared__ float tile[64][65];
  const int z = blockIdx.z;
  const long long n = static_cast<long long>(r) * c;
  float* wz = W + z * n;
  bf16* wbz = Wb + z * n;
  const XT* xz = X + z * n;
  const int r0 = blockIdx.y * 64, c0 = blockIdx.x * 64;   // a tile of X
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  auto update = [&](long long o, float4 u) {
    float4 w = *reinterpret_cast<const float4*>(wz + o);
    w.x = w.x * decay - step * u.x; w.y = w.y * decay - step * u.y;
    w.z = w.z * decay - step * u.z; w.w = w.w * decay - step * u.w;
    *reinterpret_cast<float4*>(wz + o) = w;
    store4(wbz + o, w.x, w.y, w.z, w.w);
  };
  const int cc = c0 + 4 * tx;
  if (!transpose) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int rr = r0 + ty + 16 * k;
      if (rr < r && cc < c) {
        const long long o = static_cast<long long>(rr) * c + cc;
        float4 u = load4(xz + o);
        if (rowf) {
          const float f = rowf[static_cast<long long>(z) * r + rr];
          u.x *= f; u.y *= f; u.z *= f; u.w *= f;
        }
        update(o, u);
      }
    }
    return;
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int rr = r0 + ty + 16 * k;
    float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
    if (rr < r && cc < c) {
      u = load4(xz + static_cast<long long>(rr) * c + cc);
      if (rowf) {
        const float f = rowf[static_cast<long long>(z) * r + rr];
        u.x *= f; u.y *= f; u.z *= f; u.w *= f;
      }
    }
    tile[ty + 16 * k][4 * tx] = u.x;
    tile[ty + 16 * k][4 * tx + 1] = u.y;
    tile[ty + 16 * k][4 * tx + 2] = u.z;
    tile[ty + 16 * k][4 * tx + 3] = u.w;
  }
  __syncthreads();
  // W row = X column (c0 + ...), W columns = X rows (r0 + 4 tx ..)
  const int wc = r0 + 4 * tx;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int wr = c0 + ty + 16 * k, tc = ty + 16 * k;
    if (wr < c && wc < r)
      update(static_cast<long long>(wr) * r + wc,
             make_float4(tile[4 * tx][tc], tile[4 * tx + 1][tc], tile[4 * tx + 2][tc], tile[4 * tx + 3][tc]));
  }
}

// ------------------------------------------------------- fp8 e4m3 quantisation
//
// Per-tensor dynamic scaling: scale = 448 / amax(|x|) of the tensor being
// quantised, q = e4m3(x * scale) rounded to nearest even and saturated at
// +-448, and the inverse scale amax / 448 kept for the GEMM epilogue.

// amax of nmat matrices of n bf16 values each (z = blockIdx.y); the maxima of
// non-negative floats order like their bit patterns, so an integer atomicMax
// gives the same result in any order.  amax_bits must start at zero.
__global__ void __launch_bounds__(256) amax_bf16_kernel(const bf16* __restrict__ x, long long n,
                                                        unsigned int* __restrict__ amax_bits) {
  const bf16* xz = x + blockIdx.y * n;
  float m = 0.f;
  const long long n8 = n / 8;
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n8; i += gridDim.x * 256ll) {
    const uint4 w = reinterpret_cast<const uint4*>(xz)[i];
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) m = fmaxf(m, fmaxf(fabsf(bf16_lo(u[e])), fabsf(bf16_hi(u[e]))));
  }
  for (long long i = n8 * 8 + blockIdx.x * 256ll + threadIdx.x; i < n; i += gridDim.x * 256ll)
    m = fmaxf(m, fabsf(__bfloat162float(xz[i])));
  m = warp_max(m);
  __shared__ float red[8];
  if (lane_id() == 0) red[warp_id()] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = red[0];
    for (int i = 1; i < 8; ++i) t = fmaxf(t, red[i]);
    atomicMax(amax_bits + blockIdx.y, __float_as_uint(t));
  }
}

// amax of matrix z: the max over its nslots words (1: one word per matrix)
__global__ void __launch_bounds__(256) quantize_e4m3_kernel(const bf16* __restrict__ x, long long n,
                                                            const unsigned int* __restrict__ amax_bits,
                                                            uint8_t* __restrict__ q, float* __restrict__ inv,
                                                            int nslots) {
  const int z = blockIdx.y;
  unsigned int ab = 0;
  for (int i = 0; i < nslots; ++i) ab = max(ab, amax_bits[z * nslots + i]);
  const float amax = __uint_as_float(ab);
  const float sc = amax > 0.f ? 448.f / amax : 1.f;
  if (blockIdx.x == 0 && threadIdx.x == 0) inv[z] = amax > 0.f ? amax / 448.f : 1.f;
  const bf16* xz = x + z * n;
  uint8_t* qz = q + z * n;
  const long long n8 = n / 8;
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n8; i += gridDim.x * 256ll) {
    const uint4 w = reinterpret_cast<const uint4*>(xz)[i];
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
    uint32_t o[2] = {0, 0};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_fp8x2_storage_t pr =
          __nv_cvt_float2_to_fp8x2(make_float2(bf16_lo(u[e]) * sc, bf16_hi(u[e]) * sc), __NV_SATFINITE, __NV_E4M3);
      o[e >> 1] |= static_cast<uint32_t>(pr) << (16 * (e & 1));
    }
    reinterpret_cast<uint2*>(qz)[i] = make_uint2(o[0], o[1]);
  }
  for (long long i = n8 * 8 + blockIdx.x * 256ll + threadIdx.x; i < n; i += gridDim.x * 256ll)
    qz[i] = __nv_cvt_float_to_fp8(__bfloat162float(xz[i]) * sc, __NV_SATFINITE, __NV_E4M3);
}

__global__ void cast_bf16_kernel(const float* __restrict__ src, bf16* __restrict__ dst, long long n) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

int stream_grid(long long work, int threads) {
  // a few resident blocks per SM, never more than the work needs
  long long g = (work + threads - 1) / threads;
  const long long cap = 148ll * 8;
  return static_cast<int>(g < cap ? (g > 0 ? g : 1) : cap);
}

}  // namespace

void launch_rope_table(float2* tab, int T, cudaStream_t s) {
  rope_table_kernel<<<cdiv(T * 64, 256), 256, 0, s>>>(tab, T);
}

void launch_embed_fwd(const int* tok, const bf16* wte, float* x, int M, int d, int V, int* err, cudaStream_t s) {
  embed_fwd_kernel<<<cdiv(M, 8), 256, 0, s>>>(tok, wte, x, M, d, V, err);
}

#define GPT_NV_CASES(X) X(1) X(2) X(3) X(4) X(5) X(6) X(7) X(8) X(9) X(10) X(11) X(12) X(13) X(14) X(15) X(16)

void launch_rmsnorm_fwd(const float* x, bf16* y, float* rstd, int M, int d, cudaStream_t s, unsigned int* amax) {
  if (M <= 0) return;
  switch (d / 128) {
#define GPT_FWD_CASE(n) case n: rmsnorm_fwd_kernel<n><<<cdiv(M, 4), 128, 0, s>>>(x, y, rstd, M, amax); break;
    GPT_NV_CASES(GPT_FWD_CASE)
#undef GPT_FWD_CASE
    default: break;
  }
}

void launch_rmsnorm_bwd(const float* dy, const bf16* y, const float* rstd, float* dx, bf16* dxb, int M, int d,
                        bool accumulate, cudaStream_t s, unsigned int* amax) {
  if (M <= 0) return;
  switch (d / 128) {
#define GPT_BWD_CASE(n) \
  case n: rmsnorm_bwd_kernel<n><<<cdiv(M, 4), 128, 0, s>>>(dy, y, rstd, dx, dxb, M, accumulate ? 1 : 0, amax); break;
    GPT_NV_CASES(GPT_BWD_CASE)
#undef GPT_BWD_CASE
    default: break;
  }
}

void launch_qk_bwd(const float* dq, const bf16* dk, const bf16* dv, const bf16* qn, const bf16* kn, const float* rq,
                   const float* rk, const float2* rope, bf16* dqkv, int B, int T, int H, cudaStream_t s, int Hkv,
                   unsigned int* amax) {
  const long long rows = 1ll * B * H * T;
  if (!dk && rows <= 0x3fffffffll) {
    // q alone: two rows per warp
    const int d = H * 128, kvd = (Hkv <= 0 ? H : Hkv) * 128;
    qk_bwd_q_kernel<<<static_cast<int>(cdiv(rows, 16)), 256, 0, s>>>(dq, qn, rq, rope, dqkv, static_cast<int>(rows), T,
                                                                      H, d + 2 * kvd, amax);
    return;
  }
  if (Hkv <= 0 || Hkv == H)
    qk_bwd_kernel<false><<<cdiv(rows, 8), 256, 0, s>>>(dq, dk, dv, qn, kn, rq, rk, rope, dqkv, B, T, H, H, amax);
  else
    qk_bwd_kernel<true><<<cdiv(rows, 8), 256, 0, s>>>(dq, dk, dv, qn, kn, rq, rk, rope, dqkv, B, T, H, Hkv, amax);
}

void launch_ce_finish(bf16* z, const float2* stats, const float* zt, const int* tgt, float* row_loss, int rows,
                      int V, int tiles_n, float inv_count, cudaStream_t s) {
  if (rows <= 0) return;
  ce_finish_kernel<<<rows, 256, 0, s>>>(z, stats, zt, tgt, row_loss, V, tiles_n, inv_count);
}

void launch_sum_scale(const float* v, int n, float scale, float* out, cudaStream_t s) {
  sum_scale_kernel<<<1, 1024, 0, s>>>(v, n, scale, out);
}

// the sort runs in chunks of kEmbChunk tokens, so the workspace does not grow
// with M: the sorted keys, then two partial rows of d floats per piece chunk
size_t embed_bwd_workspace(int /*M*/, int d) {
  return static_cast<size_t>(kEmbChunk) * sizeof(uint32_t) +
         static_cast<size_t>(2 * (kEmbChunk / kEmbPiece)) * d * sizeof(float) + 256;
}

void launch_embed_bwd(const int* tok, const float* dx, float* dwte, int M, int d, int V, void* ws, bool accumulate,
                      cudaStream_t s) {
  static std::atomic<unsigned long long> configured{0};
  set_smem_limit_once(embed_sort_kernel, kEmbChunk * 4, configured);   // a failure shows at the launch
  if (!accumulate) cudaMemsetAsync(dwte, 0, static_cast<size_t>(V) * d * sizeof(float), s);
  uint32_t* keys = static_cast<uint32_t*>(ws);
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + static_cast<size_t>(kEmbChunk) * sizeof(uint32_t));
  const int nchunk = d / 128;
  for (int base = 0; base < M; base += kEmbChunk) {
    const int n = M - base < kEmbChunk ? M - base : kEmbChunk;
    int npow2 = 1;
    while (npow2 < n) npow2 <<= 1;
    embed_sort_kernel<<<1, 1024, npow2 * 4, s>>>(tok + base, n, npow2, keys, V);
    const long long warps = static_cast<long long>(n) * nchunk;
    embed_piece_kernel<<<static_cast<int>((warps + 7) / 8), 256, 0, s>>>(keys, n, dx, base, dwte, part, d);
    embed_join_kernel<<<static_cast<int>((warps + 7) / 8), 256, 0, s>>>(keys, n, part, dwte, d);
  }
}

void launch_splitk_reduce(const float* part, int splits, long long stride, long long n, float* out, bool accumulate,
                          cudaStream_t s) {
  const long long n4 = n / 4;
  splitk_reduce_kernel<<<stream_grid(n4, 256), 256, 0, s>>>(part, splits, stride, n4, out, accumulate ? 1 : 0);
}

constexpr int kResidBlocks = 4 * 148;

int resid_partial_blocks() { return kResidBlocks; }

void launch_resid_fwd(float* x, float* x_in, float* x0, const float* lam, int l, int L, long long n, bool first,
                      cudaStream_t s) {
  resid_fwd_kernel<<<stream_grid(n / 4, 256), 256, 0, s>>>(x, x_in, x0, lam, l, L, n / 4, first ? 1 : 0);
}

void launch_backout_fwd(float* x, const float* x_mid, const float* lam, int L, long long n, cudaStream_t s) {
  backout_fwd_kernel<<<stream_grid(n / 4, 256), 256, 0, s>>>(x, x_mid, lam, L, n / 4);
}

void launch_resid_bwd(float* dx, const float* x_in, const float* x0, float* dx0, const float* dx_final,
                      const float* lam, int l, int L, long long n, bf16* gout, float* part, bool first, bool last,
                      cudaStream_t s) {
  // partial sums of scalar j go to part[j * kResidBlocks ...]
  resid_bwd_kernel<<<kResidBlocks, 256, 0, s>>>(dx, x_in, x0, dx0, dx_final, lam, l, L, n / 4, gout,
                                                part + static_cast<long long>(l) * kResidBlocks,
                                                part + static_cast<long long>(L + l) * kResidBlocks, first ? 1 : 0,
                                                last ? 1 : 0);
}

void launch_backout_grad_partial(const float* x_mid, const float* dx_final, int L, long long n, float* part,
                                 cudaStream_t s) {
  dot_partial_kernel<<<kResidBlocks, 256, 0, s>>>(x_mid, dx_final, n / 4,
                                                  part + static_cast<long long>(2 * L) * kResidBlocks);
}

void launch_scalar_grad_finish(const float* part, int L, float* grad, bool accumulate, cudaStream_t s) {
  const int count = 2 * L + 26;
  scalar_grad_finish_kernel<<<cdiv(count, 8), 256, 0, s>>>(part, kResidBlocks, count, 2 * L, grad,
                                                           accumulate ? 1 : 0);
}

void launch_ve_fwd(const bf16* xn1, const int* tok, const bf16* ve, const float* wg, float* sig, bf16* v, int M,
                   int T, int H, int Hkv, int C, int V, cudaStream_t s) {
  ve_fwd_kernel<<<cdiv(M, 8), 256, 0, s>>>(xn1, tok, ve, wg, sig, v, M, T, H, Hkv, C, V);
}

void launch_ve_bwd(const bf16* dv, long long ldv, const int* tok, const bf16* ve, const float* sig, float* dve,
                   float* dz, int M, int Hkv, int V, cudaStream_t s) {
  ve_bwd_kernel<<<cdiv(M, 8), 256, 0, s>>>(dv, ldv, tok, ve, sig, dve, dz, M, Hkv, V);
}

void launch_ve_gate_grad(const bf16* xn1, const float* dz, float* part, float* grad, int M, int d, int H, int C,
                         bool accumulate, cudaStream_t s) {
  ve_gate_grad_kernel<<<kResidBlocks, 1024, 0, s>>>(xn1, dz, part, M, d, H, C);
  scalar_grad_finish_kernel<<<cdiv(C * H, 8), 256, 0, s>>>(part, kResidBlocks, C * H, -1, grad, accumulate ? 1 : 0);
}

void launch_ve_dxn(float* dxn, const float* dz, const float* wg, int M, int d, int H, int C, cudaStream_t s) {
  ve_dxn_kernel<<<cdiv(M, 8), 256, 0, s>>>(dxn, dz, wg, M, d, H, C);
}

void launch_smear_fwd(const float* e, float* x, float* sig, const float* lam, int L, int T, int M, int d,
                      cudaStream_t s) {
  smear_fwd_kernel<<<cdiv(M, 8), 256, 0, s>>>(e, x, sig, lam, L, T, M, d);
}

void launch_smear_bwd(const float* g, const float* e, const float* sig, const float* lam, float* de, float* part,
                      int L, int T, int M, int d, cudaStream_t s) {
  smear_bwd_kernel<<<kResidBlocks, 256, 0, s>>>(g, e, sig, lam, de, part, L, T, M, d);
}

void launch_adamw(float* p, const float* g, float* m, float* v, bf16* pb, long long n, float lr, float b1, float b2,
                  float eps, float wd, float bc1, float bc2, cudaStream_t s) {
  const long long n4 = n / 4;
  adamw_kernel<<<stream_grid(n4, 256), 256, 0, s>>>(p, g, m, v, pb, n4, lr, b1, b2, eps, wd, bc1, bc2);
}

size_t muon_norm_workspace(int nmat) { return static_cast<size_t>(nmat) * kNormBlocks * sizeof(float); }

void launch_muon_momentum(float* mom, const float* g, long long n, int nmat, float beta, float eps, float* inv_norm,
                          void* ws, cudaStream_t s) {
  float* part = static_cast<float*>(ws);
  muon_momentum_kernel<<<dim3(kNormBlocks, nmat), 256, 0, s>>>(mom, g, n / 4, beta, part);
  muon_norm_kernel<<<nmat, 32, 0, s>>>(part, nmat, eps, inv_norm);
}

void launch_muon_make_x(const float* mom, const float* inv_norm, void* same, void* trans, int out_es, int nmat,
                        int rows, int cols, cudaStream_t s, __half* same16, __half* trans16) {
  const dim3 grid(cdiv(cols, 64), cdiv(rows, 64), nmat);
  if (out_es == 2)
    muon_make_x_kernel<bf16, __half><<<grid, 256, 0, s>>>(mom, inv_norm, static_cast<bf16*>(same),
                                                          static_cast<bf16*>(trans), same16, trans16, rows, cols);
  else
    muon_make_x_kernel<float, __half><<<grid, 256, 0, s>>>(mom, inv_norm, static_cast<float*>(same),
                                                           static_cast<float*>(trans), same16, trans16, rows, cols);
}

void launch_muon_apply(float* W, bf16* Wb, const void* X, int x_es, int nmat, int r, int c, bool transpose,
                       float lr, float wd, float scale, cudaStream_t s, const float* rowf) {
  const dim3 grid(cdiv(c, 64), cdiv(r, 64), nmat);
  const float decay = 1.f - lr * wd, step = lr * scale;
  if (x_es == 2)
    muon_apply_kernel<bf16><<<grid, 256, 0, s>>>(W, Wb, static_cast<const bf16*>(X), rowf, r, c, transpose, decay,
                                                 step);
  else
    muon_apply_kernel<float><<<grid, 256, 0, s>>>(W, Wb, static_cast<const float*>(X), rowf, r, c, transpose, decay,
                                                  step);
}

void launch_normuon_factor(const void* X, int x_es, int nmat, int r, int c, float* V, float beta2, float* ws,
                           cudaStream_t s) {
  if (nmat <= 0 || r <= 0) return;
  const dim3 grid(cdiv(r, 8), nmat);
  if (x_es == 2)
    row_sumsq_kernel<bf16><<<grid, 256, 0, s>>>(static_cast<const bf16*>(X), r, c, ws);
  else
    row_sumsq_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(X), r, c, ws);
  normuon_factor_kernel<<<nmat, 1024, 0, s>>>(ws, V, r, c, beta2);
}

void launch_quantize_e4m3(const bf16* x, long long n, int nmat, unsigned int* amax_bits, uint8_t* q, float* inv,
                          cudaStream_t s) {
  if (n <= 0 || nmat <= 0) return;
  cudaMemsetAsync(amax_bits, 0, static_cast<size_t>(nmat) * sizeof(unsigned int), s);
  const int blocks = static_cast<int>(std::min<long long>((n / 8 + 255) / 256 + 1, 4 * 148));
  amax_bf16_kernel<<<dim3(blocks, nmat), 256, 0, s>>>(x, n, amax_bits);
  quantize_e4m3_kernel<<<dim3(blocks, nmat), 256, 0, s>>>(x, n, amax_bits, q, inv, 1);
}

void launch_amax_slots(const bf16* x, long long n, unsigned int* slots, cudaStream_t s) {
  if (n <= 0) return;
  const int blocks = static_cast<int>(std::min<long long>((n / 8 + 255) / 256 + 1, 4 * 148));
  amax_bf16_kernel<<<dim3(blocks, 1), 256, 0, s>>>(x, n, slots);
}

void launch_quantize_e4m3_slots(const bf16* x, long long n, const unsigned int* slots, uint8_t* q, float* inv,
                                cudaStream_t s) {
  if (n <= 0) return;
  const int blocks = static_cast<int>(std::min<long long>((n / 8 + 255) / 256 + 1, 4 * 148));
  quantize_e4m3_kernel<<<dim3(blocks, 1), 256, 0, s>>>(x, n, slots, q, inv, kAmaxSlots);
}

void launch_cast_bf16(const float* src, bf16* dst, long long n, cudaStream_t s) {
  cast_bf16_kernel<<<stream_grid(n, 256), 256, 0, s>>>(src, dst, n);
}

}  // namespace gpt
