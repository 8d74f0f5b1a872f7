// C ABI of the step library: configuration, the caller-owned memory plan,
// the forward/backward schedule, Muon and AdamW, tensor access and the
// op-level entry points.  See include/gpt.h for the contract.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/gpt.h"
#include "attention.cuh"
#include "common.cuh"
#include "gemm.h"
#include "kernels.cuh"
#include "polar_express_table.h"

using namespace gpt;

namespace {

thread_local std::string g_last_error;

int fail(int code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

#define GPT_CK(expr)                                                                            \
  do {                                                                                          \
    cudaError_t e_ = (expr);                                                                    \
    if (e_ != cudaSuccess)                                                                      \
      return fail(GPT_ECUDA, std::string(#expr) + ": " + cudaGetErrorString(e_));               \
  } while (0)

constexpr size_t kAlign = 256;

struct Dims {
  int L, d, H, F, V, B, T, M, Mc, tiles_lm, n_tf32, fp8;
  int Hkv, qc;   // kv heads; columns of the fused projection: d + 2 * 128 * Hkv
  int short_window, n_pat;
  char pat[12];
  int extras;   // residual / x0 scales, backout and smear (2L+26 scalars)
  int nsc;      // scalar count rounded up to a multiple of 4
  int veC, nve, ngp;   // value embeddings: gate width, layers with a table, gate values (padded to 4)
  // value-embedding slot of layer l, or -1
  int ve_slot(int l) const { return veC > 0 && l % 2 == 0 ? l / 2 : -1; }
  // attention window of layer l: short_window for an 'S' layer, -1 = full causal
  int window(int l) const { return n_pat > 0 && pat[l % n_pat] == 'S' ? short_window : -1; }
};

// Offsets (bytes) into the three caller buffers.
struct Plan {
  // params: fp32 masters then bf16 copies
  size_t w[6], wb[6];   // 0 wte, 1 lm_head, 2 qkv, 3 proj, 4 fc, 5 mproj (per-group contiguous over layers)
  size_t param_bytes;
  // state
  size_t g[6], mom[6], am[2], av[2];
  size_t nv;            // NorMuon second moments: 4 groups x L matrices x d floats
  size_t ws, wsb, gs, ams, avs;   // residual-extras scalars: master, bf16 scratch, grad, AdamW m, v
  size_t wve, wveb, gve, amve, avve;   // value-embedding tables [nve][V][d]
  size_t wg, wgb, gg, amg, avg;        // their gates [nve * C][H]
  size_t state_bytes;
  // activations
  size_t x, xn1, r1, q, k, v, rq, rk, o, lse, xn2, r2, h;   // per-layer arrays (stride below)
  size_t xf, rf, z, stats, zt, row_loss, loss;
  size_t dx, dxb, dxn, du, dy, dqf, Dv, dqkv, gx;
  size_t splitk, embws, X0, X1, XT0, XT1, Abuf, Bbuf, inv_norm, normws, nfac, sched, rope, err, tok, tgt;
  size_t x0, xin, dx0, dxfin, scws, xe, sig;   // residual extras (allocated only when on)
  size_t vesig, vedz, vepart;                  // value embeddings (allocated only when on)
  size_t wq8[4], winv, wamax;   // fp8 copies of the block weights with their scales (precision 1)
  // fp8 per-layer copies of the four GEMM activations (xn1, o, xn2, h) and the
  // four gradients they meet (dqkv, the gradient at the attention output and
  // at the block output, du), kept for the batched weight-gradient GEMMs
  size_t act8[4], grad8[4];
  size_t f8slots, f8inv;   // [8][L][kAmaxSlots] scale words, [8][L] inverse scales: acts 0..3, grads 4..7
  size_t act_bytes;
  size_t splitk_elems;
  int splits_lm;      // lm_head dx split-K factor
};

size_t al(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Bump {
  size_t off = 0;
  size_t take(size_t bytes) {
    size_t o = off;
    off = al(off + bytes);
    return o;
  }
};

int choose_splits(long long tiles, long long kblocks) {
  const int sms = 148;
  int best = 1;
  double best_cost = 1e30;
  for (int s = 1; s <= 16; ++s) {
    if (kblocks / s < 8 && s > 1) break;
    const double waves = std::ceil(static_cast<double>(tiles * s) / sms);
    const double cost = waves * std::ceil(static_cast<double>(kblocks) / s) * (s > 1 ? 1.03 : 1.0);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

int dims_from(const gpt_config* c, Dims& D) {
  if (!c) return fail(GPT_EINVAL, "null config");
  if (c->depth < 1 || c->depth > 256) return fail(GPT_EINVAL, "depth out of range");
  if (c->head_dim != 128) return fail(GPT_EINVAL, "head_dim must be 128");
  if (c->mlp_mult != 4) return fail(GPT_EINVAL, "mlp_mult must be 4");
  if (c->precision != 0 && c->precision != 1) return fail(GPT_EINVAL, "precision must be 0 (bf16) or 1 (fp8)");
  if (c->ns_tf32_steps < -1 || c->ns_tf32_steps > 5) return fail(GPT_EINVAL, "ns_tf32_steps must be in -1..5");
  D.L = c->depth;
  D.d = c->d_model ? c->d_model : 64 * c->depth;
  if (D.d % 128 || D.d > 2048) return fail(GPT_EINVAL, "d_model must be a multiple of 128, at most 2048");
  D.H = D.d / 128;
  D.F = 4 * D.d;
  D.V = c->vocab;
  if (D.V < 8 || D.V % 8 || D.V > 131072) return fail(GPT_EINVAL, "vocab must be a multiple of 8 in [8, 131072]");
  D.B = c->batch;
  D.T = c->seq_len;
  if (D.B < 1 || D.T < 1) return fail(GPT_EINVAL, "batch and seq_len must be positive");
  const long long M = 1ll * D.B * D.T;
  if (M > (1ll << 30)) return fail(GPT_EINVAL, "batch * seq_len too large");
  D.M = static_cast<int>(M);
  D.Mc = c->lm_chunk_rows > 0 ? c->lm_chunk_rows : 8192;
  D.Mc = std::min(D.Mc, D.M);
  D.tiles_lm = (D.V + 255) / 256;
  D.n_tf32 = c->ns_tf32_steps;
  D.fp8 = c->precision == 1;
  D.n_pat = 0;
  bool any_s = false;
  for (int i = 0; i < 12 && c->window_pattern[i]; ++i) {
    const char ch = c->window_pattern[i];
    if (ch != 'S' && ch != 'L') return fail(GPT_EINVAL, "window_pattern may hold only 'S' and 'L'");
    any_s = any_s || ch == 'S';
    D.pat[D.n_pat++] = ch;
  }
  if (D.n_pat == 12) return fail(GPT_EINVAL, "window_pattern must be NUL-terminated within 12 bytes");
  if (any_s && (c->short_window < 0 || c->short_window >= (1 << 30)))
    return fail(GPT_EINVAL, "short_window must be in [0, 2^30) when the pattern has an 'S' layer");
  D.short_window = c->short_window;
  if (c->residual_extras != 0 && c->residual_extras != 1) return fail(GPT_EINVAL, "residual_extras must be 0 or 1");
  D.extras = c->residual_extras;
  D.nsc = (2 * D.L + 26 + 3) / 4 * 4;
  if (c->ve_gate_channels < 0 || c->ve_gate_channels > std::min(D.d, 128) || c->ve_gate_channels * D.H > 1024)
    return fail(GPT_EINVAL, "ve_gate_channels must be in [0, min(d_model, 128)] with channels * heads <= 1024");
  if (c->n_kv_head < 0 || (c->n_kv_head > 0 && D.H % c->n_kv_head))
    return fail(GPT_EINVAL, "n_kv_head must divide the number of heads (0: as many as the heads)");
  D.Hkv = c->n_kv_head ? c->n_kv_head : D.H;
  D.qc = D.d + 2 * 128 * D.Hkv;
  if (c->ve_gate_channels * D.Hkv > 1024) return fail(GPT_EINVAL, "ve_gate_channels * kv heads must be <= 1024");
  D.veC = c->ve_gate_channels;
  D.nve = D.veC ? (D.L + 1) / 2 : 0;
  D.ngp = (D.nve * D.veC * D.Hkv + 3) / 4 * 4;
  return GPT_OK;
}

void make_plan(const Dims& D, Plan& P) {
  const size_t L = D.L, d = D.d, F = D.F, V = D.V, M = D.M, H = D.H;
  const size_t qc = D.qc, kvd = 128 * static_cast<size_t>(D.Hkv);
  const size_t numel[6] = {V * d, d * V, L * d * qc, L * d * d, L * d * F, L * F * d};
  Bump pb;
  for (int i = 0; i < 6; ++i) P.w[i] = pb.take(numel[i] * 4);
  for (int i = 0; i < 6; ++i) P.wb[i] = pb.take(numel[i] * 2);
  const size_t nsc = D.extras ? static_cast<size_t>(D.nsc) : 0;
  P.ws = pb.take(std::max<size_t>(nsc, 4) * 4);
  P.wsb = pb.take(std::max<size_t>(nsc, 4) * 2);
  const size_t nvel = static_cast<size_t>(D.nve) * V * kvd;
  const size_t ngp = std::max<size_t>(D.ngp, 4);
  P.wve = pb.take(std::max<size_t>(nvel, 4) * 4);
  P.wveb = pb.take(std::max<size_t>(nvel, 4) * 2);
  P.wg = pb.take(ngp * 4);
  P.wgb = pb.take(ngp * 2);
  P.param_bytes = pb.off;
  Bump sb;
  // gradients: lm_head, embedding, the scalars and value-embedding tables and
  // gates, then the block matrices (one span; everything before the first
  // block gradient goes to AdamW).  The order is that of the buckets in which
  // the backward completes them: lm_head first, the block kinds after the
  // backward sweep, the embedding and the extras last (gpt_grad_bucket).
  P.g[1] = sb.take(numel[1] * 4);
  P.g[0] = sb.take(numel[0] * 4);
  P.gs = sb.take(std::max<size_t>(nsc, 4) * 4);
  P.gve = sb.take(std::max<size_t>(nvel, 4) * 4);
  P.gg = sb.take(ngp * 4);
  for (int i = 2; i < 6; ++i) P.g[i] = sb.take(numel[i] * 4);
  P.mom[0] = P.mom[1] = 0;
  for (int i = 2; i < 6; ++i) P.mom[i] = sb.take(numel[i] * 4);
  for (int i = 0; i < 2; ++i) {
    P.am[i] = sb.take(numel[i] * 4);
    P.av[i] = sb.take(numel[i] * 4);
  }
  P.nv = sb.take(4 * L * d * 4);
  P.ams = sb.take(std::max<size_t>(nsc, 4) * 4);
  P.avs = sb.take(std::max<size_t>(nsc, 4) * 4);
  P.amve = sb.take(std::max<size_t>(nvel, 4) * 4);
  P.avve = sb.take(std::max<size_t>(nvel, 4) * 4);
  P.amg = sb.take(ngp * 4);
  P.avg = sb.take(ngp * 4);
  P.state_bytes = sb.off;

  // split-K plan of the lm_head input gradient (contraction over the vocabulary)
  size_t sk = 0;
  {
    const long long tiles = ((D.Mc + 127) / 128) * ((d + 255) / 256);
    P.splits_lm = choose_splits(tiles, (V + 63) / 64);
    if (P.splits_lm > 1) sk = std::max<size_t>(sk, static_cast<size_t>(P.splits_lm) * D.Mc * d);
  }
  P.splitk_elems = sk;

  Bump ab;
  P.x = ab.take(M * d * 4);
  P.xn1 = ab.take(L * M * d * 2);
  P.r1 = ab.take(L * M * 4);
  P.q = ab.take(L * M * d * 2);
  P.k = ab.take(L * M * d * 2);
  P.v = ab.take(L * M * d * 2);
  P.rq = ab.take(L * M * H * 4);
  P.rk = ab.take(L * M * H * 4);
  P.o = ab.take(L * M * d * 2);
  P.lse = ab.take(L * M * H * 4);
  P.xn2 = ab.take(L * M * d * 2);
  P.r2 = ab.take(L * M * 4);
  P.h = ab.take(L * M * F * 2);
  P.xf = ab.take(M * d * 2);
  P.rf = ab.take(M * 4);
  P.z = ab.take(static_cast<size_t>(D.Mc) * V * 2);
  P.stats = ab.take(static_cast<size_t>(D.Mc) * D.tiles_lm * 2 * 8);   // one partial per half tile
  P.zt = ab.take(static_cast<size_t>(D.Mc) * 4);
  P.row_loss = ab.take(M * 4);
  P.loss = ab.take(16);
  P.dx = ab.take(M * d * 4);
  P.dxb = ab.take(M * d * 2);
  // per-layer gradient inputs of the weight-gradient GEMMs, which run batched
  // over the layers after the backward sweep: the bf16 residual gradient at the
  // attention output (slot 2l) and at the block output (slot 2l+1), du, dqkv
  P.gx = ab.take(2 * L * M * d * 2);
  P.dxn = ab.take(M * d * 4);
  P.du = ab.take(L * M * F * 2);
  P.dy = ab.take(M * d * 2);
  P.dqf = ab.take(M * d * 4);
  P.Dv = ab.take(M * H * 4);
  P.dqkv = ab.take(L * M * qc * 2);
  P.splitk = ab.take(std::max<size_t>(sk, 4) * 4);
  P.embws = ab.take(embed_bwd_workspace(D.M, std::max(d, kvd)));
  const size_t xelems = std::max({L * d * qc, L * d * d, 2 * L * d * F});
  P.X0 = ab.take(xelems * 4);
  P.X1 = ab.take(xelems * 4);
  // fp16 operand copies of the Newton-Schulz iterates (fp16 mode), or the
  // transposed fp32 copies read K-major by its tf32 steps
  const size_t xt_bytes0 = D.n_tf32 < 0 ? xelems * 2 : (D.n_tf32 > 0 ? xelems * 4 : 16);
  const size_t xt_bytes1 = D.n_tf32 < 0 ? xelems * 2 : (D.n_tf32 > 1 ? xelems * 4 : 16);
  P.XT0 = ab.take(xt_bytes0);
  P.XT1 = ab.take(xt_bytes1);
  P.Abuf = ab.take(2 * L * d * d * 4);
  P.Bbuf = ab.take(2 * L * d * d * 4);
  P.inv_norm = ab.take(4 * L * 4);
  P.normws = ab.take(muon_norm_workspace(4 * D.L));
  P.nfac = ab.take(2 * L * d * 4);
  P.sched = ab.take(64);   // work counters of the persistent attention kernels
  if (D.extras) {
    P.x0 = ab.take(M * d * 4);
    P.xin = ab.take(L * M * d * 4);
    P.dx0 = ab.take(M * d * 4);
    P.dxfin = ab.take(M * d * 4);
    P.scws = ab.take(static_cast<size_t>(2 * L + 26) * resid_partial_blocks() * 4);
    P.xe = ab.take(M * d * 4);
    P.sig = ab.take(M * 4);
  } else {
    P.x0 = P.xin = P.dx0 = P.dxfin = P.scws = P.xe = P.sig = 0;
  }
  if (D.nve) {
    P.vesig = ab.take(static_cast<size_t>(D.nve) * M * D.Hkv * 4);
    P.vedz = ab.take(M * D.Hkv * 4);
    P.vepart = ab.take(static_cast<size_t>(D.veC) * D.Hkv * resid_partial_blocks() * 4);
  } else {
    P.vesig = P.vedz = P.vepart = 0;
  }
  P.rope = ab.take(static_cast<size_t>(D.T) * 64 * 8 * 2);   // token-major and pair-major
  P.err = ab.take(16);
  P.tok = ab.take(M * 4);
  P.tgt = ab.take(M * 4);
  {
    // fp8 e4m3 copies of the block weights, of every layer's GEMM activations
    // and of the gradients they meet, with their scales
    const bool f8 = D.fp8 != 0;
    const size_t wn[4] = {L * d * qc, L * d * d, L * d * F, L * F * d};
    for (int i = 0; i < 4; ++i) P.wq8[i] = ab.take(f8 && i > 0 ? wn[i] : 16);   // q|k|v stays bf16
    P.winv = ab.take(4 * L * 4);
    P.wamax = ab.take(4 * L * 4);
    const size_t acols[4] = {d, d, d, F}, gcols[4] = {qc, d, F, d};
    for (int i = 0; i < 4; ++i) {
      P.act8[i] = ab.take(f8 && i > 0 ? L * M * acols[i] : 16);
      P.grad8[i] = ab.take(f8 && i > 0 ? L * M * gcols[i] : 16);
    }
    P.f8slots = ab.take(8 * L * kAmaxSlots * 4);
    P.f8inv = ab.take(8 * L * 4);
  }
  P.act_bytes = ab.off;
}

// ------------------------------------------------------- device-side init

__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

__global__ void init_normal_kernel(float* w, bf16* wb, long long n, uint64_t seed, uint64_t stream_id, float std) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint64_t h1 = splitmix64(seed ^ splitmix64(stream_id * 0x100000001B3ull + 2 * i));
    const uint64_t h2 = splitmix64(seed ^ splitmix64(stream_id * 0x100000001B3ull + 2 * i + 1));
    const double u1 = (static_cast<double>(h1 >> 11) + 1.0) * (1.0 / 9007199254740992.0);
    const double u2 = static_cast<double>(h2 >> 11) * (1.0 / 9007199254740992.0);
    const float g = static_cast<float>(sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2)) * std;
    const bf16 b = __float2bfloat16_rn(g);
    wb[i] = b;
    w[i] = __bfloat162float(b);
  }
}

__global__ void check_range_kernel(const int* v, int n, int V, int* err) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    if (v[i] < 0 || v[i] >= V) atomicOr(err, ERRF_TOKEN_RANGE);
}

// targets out of range are clamped to 0 (the error word already records them)
__global__ void clamp_targets_kernel(const int* src, int* dst, int n, int V) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int t = src[i];
    dst[i] = (t < 0 || t >= V) ? 0 : t;
  }
}

}  // namespace

struct gpt_ctx {
  gpt_config cfg;
  Dims D;
  Plan P;
  uint8_t* pbuf;
  uint8_t* sbuf;
  uint8_t* abuf;
  cudaStream_t stream;
  long long wait_cycles = 0;   // bound of the kernels' device-side waits (<= 0: the default)
  cudaEvent_t grad_ev[GPT_GRAD_BUCKETS] = {};   // caller's events, recorded as gradient buckets complete
  int n_grad_ev = 0;
  void grad_ready(int bucket) {
    if (bucket < n_grad_ev && grad_ev[bucket]) cudaEventRecord(grad_ev[bucket], stream);
  }
  long long adam_step = 0;
  int64_t launches = 0;
  // event profiler
  uint32_t prof_mask = 0;
  struct Rec { cudaEvent_t a, b; int cat; };
  std::vector<Rec> recs;
  size_t recs_used = 0;
  double prof_ms[GPT_PROF_COUNT] = {};
  int64_t prof_n[GPT_PROF_COUNT] = {};
  ~gpt_ctx() {
    for (Rec& r : recs) {
      cudaEventDestroy(r.a);
      cudaEventDestroy(r.b);
    }
  }
  Rec* next_rec() {
    if (recs_used == recs.size()) {
      Rec r{};
      if (cudaEventCreate(&r.a) != cudaSuccess || cudaEventCreate(&r.b) != cudaSuccess) return nullptr;
      recs.push_back(r);
    }
    return &recs[recs_used++];
  }

  template <typename T = float>
  T* W(int i) const { return reinterpret_cast<T*>(pbuf + P.w[i]); }
  bf16* Wb(int i) const { return reinterpret_cast<bf16*>(pbuf + P.wb[i]); }
  float* G(int i) const { return reinterpret_cast<float*>(sbuf + P.g[i]); }
  float* Mom(int i) const { return reinterpret_cast<float*>(sbuf + P.mom[i]); }
  // residual-extras scalars (fp32, in the parameter buffer)
  float* Scal() const { return reinterpret_cast<float*>(pbuf + P.ws); }
  // value-embedding table i (fp32 master, bf16 copy, gradient) and gate block i
  size_t ve_elems() const { return static_cast<size_t>(D.V) * 128 * D.Hkv; }   // one table [V, 128 Hkv]
  float* VeW(int i) const { return reinterpret_cast<float*>(pbuf + P.wve) + i * ve_elems(); }
  bf16* VeWb(int i) const { return reinterpret_cast<bf16*>(pbuf + P.wveb) + i * ve_elems(); }
  float* VeG(int i) const { return reinterpret_cast<float*>(sbuf + P.gve) + i * ve_elems(); }
  float* GateW(int i) const { return reinterpret_cast<float*>(pbuf + P.wg) + static_cast<size_t>(i) * D.veC * D.Hkv; }
  float* GateG(int i) const { return reinterpret_cast<float*>(sbuf + P.gg) + static_cast<size_t>(i) * D.veC * D.Hkv; }
  // NorMuon second moments of block group i (2..5): L vectors of d floats
  float* NV(int i) const { return reinterpret_cast<float*>(sbuf + P.nv) + static_cast<size_t>(i - 2) * D.L * D.d; }
  template <typename T>
  T* A(size_t off) const { return reinterpret_cast<T*>(abuf + off); }
  int* err() const { return A<int>(P.err); }
};

namespace {

// Records a pair of events around the launches in its scope when the
// category is enabled.
struct ProfScope {
  gpt_ctx* c;
  gpt_ctx::Rec* r = nullptr;
  ProfScope(gpt_ctx* ctx, int cat) : c(ctx) {
    if (c && ((c->prof_mask >> cat) & 1u)) {
      r = c->next_rec();
      if (r) {
        r->cat = cat;
        cudaEventRecord(r->a, c->stream);
      }
    }
  }
  ~ProfScope() {
    if (r) cudaEventRecord(r->b, c->stream);
  }
};

// group index (0..5) and element offset of tensor id
bool locate(const gpt_ctx* c, int id, int& grp, size_t& off, int& rows, int& cols) {
  const Dims& D = c->D;
  if (id == 0) { grp = 0; off = 0; rows = D.V; cols = D.d; return true; }
  if (id == 1) { grp = 1; off = 0; rows = D.d; cols = D.V; return true; }
  const int k = id - 2;
  if (k >= 4 * D.L) {
    int x = k - 4 * D.L;
    if (D.extras) {
      if (x == 0) {   // the residual-extras scalars
        grp = 6; off = 0; rows = 1; cols = 2 * D.L + 26;
        return true;
      }
      --x;
    }
    if (x < D.nve) {   // value-embedding table x
      grp = 7; off = static_cast<size_t>(x) * D.V * 128 * D.Hkv; rows = D.V; cols = 128 * D.Hkv;
      return true;
    }
    if (D.nve && x == D.nve) {   // all gates, stacked
      grp = 8; off = 0; rows = D.nve * D.veC; cols = D.Hkv;
      return true;
    }
    return false;
  }
  if (k < 0) return false;
  const int l = k / 4, j = k % 4;
  const int shp[4][2] = {{D.d, D.qc}, {D.d, D.d}, {D.d, D.F}, {D.F, D.d}};
  grp = 2 + j;
  rows = shp[j][0];
  cols = shp[j][1];
  off = static_cast<size_t>(l) * rows * cols;
  return true;
}

GemmCall base_call(int M, int N, int K) {
  GemmCall c;
  c.M = M; c.N = N; c.K = K;
  return c;
}

// gemm_run with the caller's bound on the kernel's waits
cudaError_t run_gemm(GemmCall& g, cudaStream_t s, long long wait_cycles) {
  g.p.wait_cycles = wait_cycles;
  return gemm_run(g, s);
}

// fp32 output [M][N] (contiguous), optionally split over K with a deterministic reduce.
int run_f32(gpt_ctx* c, GemmCall g, float* out, bool accumulate, int splits, int cat) {
  ProfScope ps(c, cat);
  g.out_es = 4;
  g.aux_es = 4;
  g.p.err = c->err();
  if (splits <= 1) {
    g.epi = accumulate ? EPI_ACC : EPI_STORE;
    g.splits = 1;
    g.p.out = out;
    g.p.ldo = g.N;
    GPT_CK(run_gemm(g, c->stream, c->wait_cycles));
    c->launches += 1;
    return GPT_OK;
  }
  float* part = c->A<float>(c->P.splitk);
  const long long n = 1ll * g.M * g.N;
  if (static_cast<size_t>(n) * splits > c->P.splitk_elems) return fail(GPT_EINVAL, "split-K scratch too small");
  g.epi = EPI_STORE;
  g.splits = splits;
  g.p.out = part;
  g.p.ldo = g.N;
  g.p.split_stride = n;
  GPT_CK(run_gemm(g, c->stream, c->wait_cycles));
  launch_splitk_reduce(part, g.p.splits, n, n, out, accumulate, c->stream);
  c->launches += 2;
  return GPT_OK;
}

int forward_backward(gpt_ctx* c, const int* tok, const int* tgt_in, float* loss_out, bool acc) {
  const Dims& D = c->D;
  const Plan& P = c->P;
  cudaStream_t s = c->stream;
  const int M = D.M, d = D.d, F = D.F, V = D.V, H = D.H, L = D.L;
  const size_t Md = static_cast<size_t>(M) * d;
  float* x = c->A<float>(P.x);
  bf16* xn1 = c->A<bf16>(P.xn1);
  bf16* xn2 = c->A<bf16>(P.xn2);
  float* r1 = c->A<float>(P.r1);
  float* r2 = c->A<float>(P.r2);
  bf16* q = c->A<bf16>(P.q);
  bf16* k = c->A<bf16>(P.k);
  bf16* v = c->A<bf16>(P.v);
  float* rq = c->A<float>(P.rq);
  float* rk = c->A<float>(P.rk);
  bf16* o = c->A<bf16>(P.o);
  float* lse = c->A<float>(P.lse);
  bf16* h = c->A<bf16>(P.h);
  bf16* xf = c->A<bf16>(P.xf);
  float* rf = c->A<float>(P.rf);
  const float2* rope = c->A<float2>(P.rope);
  int* tgt = c->A<int>(P.tgt);
  int* err = c->err();

  // ids: range check (latched), targets clamped into the private copy
  {
    ProfScope ps(c, GPT_PROF_EMBED);
    check_range_kernel<<<64, 256, 0, s>>>(tgt_in, M, V, err);
    if (tgt_in != tgt) clamp_targets_kernel<<<64, 256, 0, s>>>(tgt_in, tgt, M, V);
    else clamp_targets_kernel<<<64, 256, 0, s>>>(tgt, tgt, M, V);
    launch_embed_fwd(tok, c->Wb(0), x, M, d, V, err, s);
  }
  if (D.extras) {
    // smear: the embedding is kept for the backward, x takes the smeared one
    ProfScope ps(c, GPT_PROF_EMBED);
    GPT_CK(cudaMemcpyAsync(c->A<float>(P.xe), x, static_cast<size_t>(M) * d * 4, cudaMemcpyDeviceToDevice, s));
    launch_smear_fwd(c->A<float>(P.xe), x, c->A<float>(P.sig), c->Scal(), L, D.T, M, d, s);
    c->launches += 1;
  }
  // fp8 ("3. Gestión de Precisión": FP8 with per-tensor scaling): e4m3 copies
  // of every block matrix, one scale per matrix; every GEMM operand that is an
  // activation or an activation gradient is quantised per tensor with the
  // amax its producer kept (scale words zeroed here, once per step)
  float* winv = c->A<float>(P.winv);
  unsigned int* f8slots = c->A<unsigned int>(P.f8slots);
  float* f8inv = c->A<float>(P.f8inv);
  const long long wn[4] = {1ll * d * D.qc, 1ll * d * d, 1ll * d * F, 1ll * F * d};
  const long long acols[4] = {d, d, d, F}, gcols[4] = {D.qc, d, F, d};
  // tensor t of layer l: activations t = 0..3 (xn1, o, xn2, h), gradients 4..7
  // (dqkv, the gradients at the attention output and at the block output, du)
  // in the order of the weight kinds they meet
  auto slots8 = [&](int t, int l) { return D.fp8 ? f8slots + (static_cast<size_t>(t) * L + l) * kAmaxSlots : nullptr; };
  auto inv8 = [&](int t, int l) { return f8inv + t * L + l; };
  // the q|k|v projection (weight kind 0) stays bf16: its rounding error enters
  // the QK-normalised attention logits, which the softmax amplifies
  auto f8 = [&](int k) { return D.fp8 && k != 0; };
  auto act8 = [&](int k, int l) { return c->A<uint8_t>(P.act8[k]) + static_cast<size_t>(l) * M * acols[k]; };
  auto grad8 = [&](int k, int l) { return c->A<uint8_t>(P.grad8[k]) + static_cast<size_t>(l) * M * gcols[k]; };
  if (D.fp8) {
    ProfScope ps(c, GPT_PROF_FP8_QUANT);
    GPT_CK(cudaMemsetAsync(f8slots, 0, static_cast<size_t>(8) * L * kAmaxSlots * 4, s));
    for (int gi = 1; gi < 4; ++gi)
      launch_quantize_e4m3(c->Wb(2 + gi), wn[gi], L, c->A<unsigned int>(P.wamax) + gi * L,
                           c->A<uint8_t>(P.wq8[gi]), winv + gi * L, s);
    c->launches += 6;
  }
  // operand A of a forward projection of weight kind k: bf16 as it is, or its
  // e4m3 copy (kept for the weight gradient) with the weight's e4m3 copy as B
  auto fwd_a = [&](GemmCall& g, const bf16* a, long long rows, long long cols, int grp, int l) {
    const int k = grp - 2;
    if (!f8(k)) {
      g.A = a;
      return;
    }
    {
      ProfScope ps(c, GPT_PROF_FP8_QUANT);
      if (k == 1) {   // the attention output keeps no amax of its own
        launch_amax_slots(a, rows * cols, slots8(k, l), s);
        c->launches += 1;
      }
      launch_quantize_e4m3_slots(a, rows * cols, slots8(k, l), act8(k, l), inv8(k, l), s);
      c->launches += 1;
    }
    g.es = 1;
    g.A = act8(k, l);
    g.B = c->A<uint8_t>(P.wq8[k]) + static_cast<size_t>(l) * wn[k];
    g.p.dq_a = inv8(k, l);
    g.p.dq_b = winv + k * L + l;
  };
  // operand A of an activation-gradient GEMM against weight kind k: the bf16
  // gradient, or its e4m3 copy with the weight's e4m3 copy as B (K-major)
  auto bwd_a = [&](GemmCall& g, const bf16* a, long long cols, int k, int l) {
    if (!f8(k)) {
      g.A = a;
      return;
    }
    {
      ProfScope ps(c, GPT_PROF_FP8_QUANT);
      launch_quantize_e4m3_slots(a, 1ll * M * cols, slots8(4 + k, l), grad8(k, l), inv8(4 + k, l), s);
      c->launches += 1;
    }
    g.es = 1;
    g.A = grad8(k, l);
    g.B = c->A<uint8_t>(P.wq8[k]) + static_cast<size_t>(l) * wn[k];
    g.p.dq_a = inv8(4 + k, l);
    g.p.dq_b = winv + k * L + l;
  };
  c->launches += 3;

  // ---------------------------------------------------------------- forward
  for (int l = 0; l < L; ++l) {
    bf16* xn1l = xn1 + l * Md;
    bf16* xn2l = xn2 + l * Md;
    bf16* ql = q + l * Md;
    bf16* kl = k + l * Md;
    bf16* vl = v + l * Md;
    bf16* ol = o + l * Md;
    bf16* hl = h + static_cast<size_t>(l) * M * F;
    float* lsel = lse + static_cast<size_t>(l) * M * H;
    if (D.extras) {
      ProfScope ps(c, GPT_PROF_NORM);
      launch_resid_fwd(x, c->A<float>(P.xin) + l * Md, c->A<float>(P.x0), c->Scal(), l, L,
                       static_cast<long long>(Md), l == 0, s);
      c->launches += 1;
    }
    {
      ProfScope ps(c, GPT_PROF_NORM);
      launch_rmsnorm_fwd(x, xn1l, r1 + static_cast<size_t>(l) * M, M, d, s);
    }
    {
      GemmCall g = base_call(M, D.qc, d);
      g.B = c->Wb(2) + static_cast<size_t>(l) * d * D.qc; g.b_mn = true; g.ldb = D.qc;
      fwd_a(g, xn1l, M, d, 2, l); g.lda = d;
      ProfScope ps(c, GPT_PROF_QKV_GEMM);
      g.bn = 256; g.epi = EPI_QKV; g.out_es = 2; g.aux_es = 2;
      g.p.qkv_out[0] = ql; g.p.qkv_out[1] = kl; g.p.qkv_out[2] = vl;
      g.p.f32a = rq + static_cast<size_t>(l) * M * H;
      g.p.f32b = rk + static_cast<size_t>(l) * M * H;
      g.p.rope = rope + static_cast<size_t>(D.T) * 64; g.p.T = D.T; g.p.H = H; g.p.Hkv = D.Hkv; g.p.err = err;
      GPT_CK(run_gemm(g, s, c->wait_cycles));
    }
    if (D.ve_slot(l) >= 0) {
      // value embedding: v += 3 sigmoid(gate) ve[tok] per head
      const int i = D.ve_slot(l);
      ProfScope ps(c, GPT_PROF_EMBED);
      launch_ve_fwd(xn1l, tok, c->VeWb(i), c->GateW(i), c->A<float>(P.vesig) + static_cast<size_t>(i) * M * D.Hkv, vl,
                    M, D.T, H, D.Hkv, D.veC, V, s);
      c->launches += 1;
    }
    {
      ProfScope ps(c, GPT_PROF_ATTN_FWD);
      launch_attn_fwd(ql, kl, vl, ol, lsel, D.B, H, D.T, s, err, D.Hkv, D.window(l), c->A<int>(P.sched), H,
                      c->wait_cycles);
    }
    {
      GemmCall g = base_call(M, d, d);
      g.B = c->Wb(3) + static_cast<size_t>(l) * d * d; g.b_mn = true; g.ldb = d;
      fwd_a(g, ol, M, d, 3, l); g.lda = d;
      ProfScope ps(c, GPT_PROF_PROJ_GEMM);
      g.epi = EPI_ACC; g.out_es = 4; g.aux_es = 4;
      g.p.out = x; g.p.ldo = d; g.p.err = err;
      GPT_CK(run_gemm(g, s, c->wait_cycles));
    }
    {
      ProfScope ps(c, GPT_PROF_NORM);
      launch_rmsnorm_fwd(x, xn2l, r2 + static_cast<size_t>(l) * M, M, d, s, slots8(2, l));
    }
    {
      GemmCall g = base_call(M, F, d);
      g.B = c->Wb(4) + static_cast<size_t>(l) * d * F; g.b_mn = true; g.ldb = F;
      fwd_a(g, xn2l, M, d, 4, l); g.lda = d;
      ProfScope ps(c, GPT_PROF_FC_GEMM);
      g.epi = EPI_RELU2; g.out_es = 2; g.aux_es = 2;
      g.p.out = hl; g.p.ldo = F; g.p.err = err; g.p.amax_out = slots8(3, l);
      GPT_CK(run_gemm(g, s, c->wait_cycles));
    }
    {
      GemmCall g = base_call(M, d, F);
      g.B = c->Wb(5) + static_cast<size_t>(l) * F * d; g.b_mn = true; g.ldb = d;
      fwd_a(g, hl, M, F, 5, l); g.lda = F;
      ProfScope ps(c, GPT_PROF_DOWN_GEMM);
      g.epi = EPI_ACC; g.out_es = 4; g.aux_es = 4;
      g.p.out = x; g.p.ldo = d; g.p.err = err;
      GPT_CK(run_gemm(g, s, c->wait_cycles));
    }
    c->launches += 7;
  }
  if (D.extras) {
    ProfScope ps(c, GPT_PROF_NORM);
    launch_backout_fwd(x, c->A<float>(P.xin) + static_cast<size_t>(L / 2) * Md, c->Scal(), L,
                       static_cast<long long>(Md), s);
    c->launches += 1;
  }
  {
    ProfScope ps(c, GPT_PROF_NORM);
    launch_rmsnorm_fwd(x, xf, rf, M, d, s);
  }
  c->launches += 1;

  // ------------------------------------- fused lm_head + cross-entropy, chunked
  float* dxn = c->A<float>(P.dxn);
  bf16* z = c->A<bf16>(P.z);
  float* row_loss = c->A<float>(P.row_loss);
  for (int r0 = 0; r0 < M; r0 += D.Mc) {
    const int rows = std::min(D.Mc, M - r0);
    {
      ProfScope ps(c, GPT_PROF_LOGITS_GEMM);
      GemmCall g = base_call(rows, V, d);
      g.A = xf + static_cast<size_t>(r0) * d; g.lda = d;
      g.B = c->Wb(1); g.b_mn = true; g.ldb = V;
      g.epi = EPI_LOGITS; g.out_es = 2; g.aux_es = 2;
      g.p.out = z; g.p.ldo = V;
      g.p.f32a = c->A<float>(P.stats); g.p.f32b = c->A<float>(P.zt); g.p.tgt = tgt + r0; g.p.err = err;
      GPT_CK(run_gemm(g, s, c->wait_cycles));
    }
    {
      ProfScope ps(c, GPT_PROF_CE_FINISH);
      launch_ce_finish(z, c->A<float2>(P.stats), c->A<float>(P.zt), tgt + r0, row_loss + r0, rows, V,
                       2 * D.tiles_lm, 1.f / static_cast<float>(M), s);
    }
    c->launches += 2;
    {
      // dxf rows = dz W_lm^T  (contraction over the vocabulary)
      GemmCall g = base_call(rows, d, V);
      g.A = z; g.lda = V;
      g.B = c->Wb(1); g.ldb = V;   // B(n = model dim, k = vocab) = W_lm[n][k]
      int rc = run_f32(c, g, dxn + static_cast<size_t>(r0) * d, false, P.splits_lm, GPT_PROF_LM_DX_GEMM);
      if (rc) return rc;
    }
    {
      // dW_lm += xf^T dz  (contraction over the rows of the chunk)
      GemmCall g = base_call(d, V, rows);
      g.A = xf + static_cast<size_t>(r0) * d; g.a_mn = true; g.lda = d;
      g.B = z; g.b_mn = true; g.ldb = V;
      int rc = run_f32(c, g, c->G(1), acc || r0 > 0, 1, GPT_PROF_LM_DW_GEMM);
      if (rc) return rc;
    }
  }
  launch_sum_scale(row_loss, M, 1.f / static_cast<float>(M), loss_out, s);
  c->launches += 1;
  c->grad_ready(0);   // the lm_head gradient is complete

  // --------------------------------------------------------------- backward
  float* dx = c->A<float>(P.dx);
  bf16* dy = c->A<bf16>(P.dy);
  float* dqf = c->A<float>(P.dqf);
  bf16* gx = c->A<bf16>(P.gx);
  bf16* du_all = c->A<bf16>(P.du);
  bf16* dqkv_all = c->A<bf16>(P.dqkv);
  auto gatt = [&](int l) { return gx + (2 * static_cast<size_t>(l)) * Md; };       // grad at attention output
  auto gmlp = [&](int l) { return gx + (2 * static_cast<size_t>(l) + 1) * Md; };   // grad at block output
  {
    ProfScope ps(c, GPT_PROF_NORM);
    launch_rmsnorm_bwd(dxn, xf, rf, dx, gmlp(L - 1), M, d, false, s, slots8(7, L - 1));
  }
  c->launches += 1;
  if (D.extras) {
    // the backout output's gradient, kept for the block whose input it read
    ProfScope ps(c, GPT_PROF_NORM);
    GPT_CK(cudaMemcpyAsync(c->A<float>(P.dxfin), dx, Md * 4, cudaMemcpyDeviceToDevice, s));
    launch_backout_grad_partial(c->A<float>(P.xin) + static_cast<size_t>(L / 2) * Md, dx, L,
                                static_cast<long long>(Md), c->A<float>(P.scws), s);
    c->launches += 1;
  }
  for (int l = L - 1; l >= 0; --l) {
    bf16* xn2l = xn2 + l * Md;
    bf16* hl = h + static_cast<size_t>(l) * M * F;
    bf16* ol = o + l * Md;
    bf16* du = du_all + static_cast<size_t>(l) * M * F;
    bf16* dqkv = dqkv_all + static_cast<size_t>(l) * M * D.qc;
    // MLP down: dh = dx W_d^T, du = dh * 2 relu(u) with relu(u) = sqrt(h)
    {
      GemmCall g = base_call(M, F, d);
      g.B = c->Wb(5) + static_cast<size_t>(l) * F * d; g.ldb = d;   // B(n = F index, k = d index)
      bwd_a(g, gmlp(l), d, 3, l); g.lda = d;
      ProfScope ps(c, GPT_PROF_DX_GEMM);
      g.epi = EPI_DRELU2; g.out_es = 2; g.aux_es = 2;
      g.p.out = du; g.p.ldo = F; g.p.aux = hl; g.p.ld_aux = F; g.p.err = err; g.p.amax_out = slots8(6, l);
      GPT_CK(run_gemm(g, s, c->wait_cycles));
      c->launches += 1;
    }
    {
      GemmCall g = base_call(M, d, F);   // dxn2 = du W_fc^T
      g.B = c->Wb(4) + static_cast<size_t>(l) * d * F; g.ldb = F;
      bwd_a(g, du, F, 2, l); g.lda = F;
      int rc = run_f32(c, g, dxn, false, 1, GPT_PROF_DX_GEMM);
      if (rc) return rc;
    }
    {
      ProfScope ps(c, GPT_PROF_NORM);
      launch_rmsnorm_bwd(dxn, xn2l, r2 + static_cast<size_t>(l) * M, dx, gatt(l), M, d, true, s, slots8(5, l));
    }
    c->launches += 1;
    // attention output projection
    {
      GemmCall g = base_call(M, d, d);   // dy = dx W_o^T
      g.B = c->Wb(3) + static_cast<size_t>(l) * d * d; g.ldb = d;
      bwd_a(g, gatt(l), d, 1, l); g.lda = d;
      ProfScope ps(c, GPT_PROF_DX_GEMM);
      g.epi = EPI_STORE; g.out_es = 2; g.aux_es = 2;
      g.p.out = dy; g.p.ldo = d; g.p.err = err;
      // and the attention backward's D = rowsum(dO * O) per head
      g.p.row_dot = 1; g.p.aux = ol; g.p.ld_aux = d; g.p.f32a = c->A<float>(P.Dv); g.p.T = D.T; g.p.H = H;
      GPT_CK(run_gemm(g, s, c->wait_cycles));
      c->launches += 1;
    }
    {
      ProfScope ps(c, GPT_PROF_ATTN_BWD);
      // dK (through the QK-norm and rotation backward) and dV go straight to
      // their columns of the q|k|v gradient rows
      launch_attn_bwd(q + l * Md, k + l * Md, v + l * Md, ol, dy, lse + static_cast<size_t>(l) * M * H,
                      c->A<float>(P.Dv), dqf, nullptr, nullptr, D.B, H, D.T, s, err, D.Hkv, D.window(l), c->A<int>(P.sched), H,
                      c->wait_cycles, rk + static_cast<size_t>(l) * M * H, rope, dqkv, true);
    }
    {
      ProfScope ps(c, GPT_PROF_QK_BWD);
      launch_qk_bwd(dqf, nullptr, nullptr, q + l * Md, k + l * Md, rq + static_cast<size_t>(l) * M * H,
                    rk + static_cast<size_t>(l) * M * H, rope, dqkv, D.B, D.T, H, s, D.Hkv);
    }
    c->launches += 2;
    const int vs = D.ve_slot(l);
    if (vs >= 0) {
      // value embedding: the table's gradient (3 sigmoid dv, from the v columns
      // of the q|k|v gradient rows, scattered by token through the fp32
      // buffer the attention backward no longer needs) and the gate's
      ProfScope ps(c, GPT_PROF_EMBED);
      launch_ve_bwd(dqkv + d + 128 * D.Hkv, D.qc, tok, c->VeWb(vs),
                    c->A<float>(P.vesig) + static_cast<size_t>(vs) * M * D.Hkv, dqf, c->A<float>(P.vedz), M, D.Hkv, V,
                    s);
      launch_embed_bwd(tok, dqf, c->VeG(vs), M, 128 * D.Hkv, V, c->A<void>(P.embws), acc, s);
      launch_ve_gate_grad(xn1 + l * Md, c->A<float>(P.vedz), c->A<float>(P.vepart), c->GateG(vs), M, d, D.Hkv,
                          D.veC, acc, s);
      c->launches += 3 + 3 * ((M + 32767) / 32768);
    }
    {
      GemmCall g = base_call(M, d, D.qc);   // dxn1 = dqkv W_qkv^T
      g.B = c->Wb(2) + static_cast<size_t>(l) * d * D.qc; g.ldb = D.qc;
      bwd_a(g, dqkv, D.qc, 0, l); g.lda = D.qc;
      int rc = run_f32(c, g, dxn, false, 1, GPT_PROF_DX_GEMM);
      if (rc) return rc;
    }
    if (vs >= 0) {
      ProfScope ps(c, GPT_PROF_EMBED);
      launch_ve_dxn(dxn, c->A<float>(P.vedz), c->GateW(vs), M, d, D.Hkv, D.veC, s);   // the gate read xn1[:, :C]
      c->launches += 1;
    }
    {
      ProfScope ps(c, GPT_PROF_NORM);
      // the bf16 copy feeds the next (lower) block; below block 0 only the fp32 gradient is used
      launch_rmsnorm_bwd(dxn, xn1 + l * Md, r1 + static_cast<size_t>(l) * M, dx,
                         l > 0 ? gmlp(l - 1) : c->A<bf16>(P.dxb), M, d, true, s,
                         l > 0 && !D.extras ? slots8(7, l - 1) : nullptr);
    }
    c->launches += 1;
    if (D.extras) {
      // through x' = resid[l] x_in + x0s[l] x0: dx becomes the gradient at
      // block l's unscaled input, and its bf16 copy replaces the one above
      ProfScope ps(c, GPT_PROF_NORM);
      launch_resid_bwd(dx, c->A<float>(P.xin) + l * Md, c->A<float>(P.x0), c->A<float>(P.dx0),
                       l == L / 2 ? c->A<float>(P.dxfin) : nullptr, c->Scal(), l, L,
                       static_cast<long long>(Md), l > 0 ? gmlp(l - 1) : c->A<bf16>(P.dxb), c->A<float>(P.scws),
                       l == L - 1, l == 0, s);
      c->launches += 1;
      if (D.fp8 && l > 0) {   // the bf16 copy was rewritten: its amax anew
        launch_amax_slots(gmlp(l - 1), static_cast<long long>(Md), slots8(7, l - 1), s);
        c->launches += 1;
      }
    }
  }
  // weight gradients of every block matrix, each kind as one GEMM batched over the layers:
  // dW[l] = act[l]^T grad[l], contraction over the M tokens
  {
    ProfScope ps(c, GPT_PROF_DW_GEMM);
    struct DW { const bf16* a; long long lda, a_bs; const bf16* b; long long ldb, b_bs; int rows, cols; float* out; };
    const DW dws[4] = {
        {xn1, d, static_cast<long long>(Md), dqkv_all, D.qc, 1ll * M * D.qc, d, D.qc, c->G(2)},
        {o, d, static_cast<long long>(Md), gx, d, 2 * static_cast<long long>(Md), d, d, c->G(3)},
        {xn2, d, static_cast<long long>(Md), du_all, F, 1ll * M * F, d, F, c->G(4)},
        {h, F, 1ll * M * F, gx + Md, d, 2 * static_cast<long long>(Md), F, d, c->G(5)},
    };
    for (int kind = 0; kind < 4; ++kind) {
      const DW& w = dws[kind];
      GemmCall g = base_call(w.rows, w.cols, M);
      g.batch = L;
      g.A = w.a; g.a_mn = true; g.lda = w.lda; g.a_bs = w.a_bs;
      g.B = w.b; g.b_mn = true; g.ldb = w.ldb; g.b_bs = w.b_bs;
      if (f8(kind)) {
        // e4m3 copies of the activations and gradients, one scale pair per layer
        g.es = 1;
        g.A = act8(kind, 0); g.lda = acols[kind]; g.a_bs = 1ll * M * acols[kind];
        g.B = grad8(kind, 0); g.ldb = gcols[kind]; g.b_bs = 1ll * M * gcols[kind];
        g.p.dq_a = inv8(kind, 0);
        g.p.dq_b = inv8(4 + kind, 0);
        g.p.dq_zs = 1;
      }
      g.epi = acc ? EPI_ACC : EPI_STORE; g.out_es = 4; g.aux_es = 4;
      g.p.out = w.out; g.p.ldo = w.cols; g.p.out_bs = 1ll * w.rows * w.cols; g.p.err = err;
      GPT_CK(run_gemm(g, s, c->wait_cycles));
      c->grad_ready(1 + kind);   // this block matrix kind's gradients, every layer
    }
    c->launches += 4;
  }
  // the embedding's gradient: through the smear when the extras are on
  float* demb = dx;
  if (D.extras) {
    ProfScope ps(c, GPT_PROF_EMBED);
    demb = c->A<float>(P.dx0);   // free once block 0 has added it into dx
    launch_smear_bwd(dx, c->A<float>(P.xe), c->A<float>(P.sig), c->Scal(), demb, c->A<float>(P.scws), L, D.T, M, d,
                     s);
    launch_scalar_grad_finish(c->A<float>(P.scws), L, reinterpret_cast<float*>(c->sbuf + P.gs), acc, s);
    c->launches += 2;
  }
  {
    ProfScope ps(c, GPT_PROF_EMBED);
    launch_embed_bwd(tok, demb, c->G(0), M, d, V, c->A<void>(P.embws), acc, s);
  }
  c->launches += 3 * ((M + 32767) / 32768);
  c->grad_ready(5);   // the embedding and the extras
  GPT_CK(cudaGetLastError());
  return GPT_OK;
}

// Five Polar Express steps on X0 ([z][r][c], es0-typed); returns the buffer
// and element size holding the result.  Steps run on tf32 (fp32 storage) while
// t < n_tf32, then on bf16.  A tf32 step reads X^T (XT0, [z][c][r]) as its
// K-major B operand and, when the next step is tf32 too, writes X'^T beside X'.
int newton_schulz(gpt_ctx* pc, int nz, int r, int cc, void* X0, void* X1, void* XT0, void* XT1, void* Ab,
                  void* Bb, int n_tf32, cudaStream_t s, int* err, void** out, int* out_es, int64_t* launches,
                  long long wait_cycles) {
  ProfScope ps(pc, GPT_PROF_NS_GEMM);
  const double (*kPolarCoef)[3] = polar_coefficients();
  if (n_tf32 < 0) {
    // fp16 operands at the full tensor rate.  The iterate is carried as an
    // unevaluated pair X = hi + lo of fp16 matrices (hi = fp16(X), lo = the
    // rounding residual), ~22 significant bits, so that the update's epilogue
    // reads and writes 6 bytes per element instead of an fp32 X plus its fp16
    // copy (10).  The step X' = a X + B X becomes X' = (a I + B) hi + a lo: the
    // tensor cores multiply by hi only, as they did with the fp16 copy, and the
    // diagonal a I is folded into B by the polynomial's epilogue.  The first
    // step reads the fp32 X0 (with its fp16 copy hi in XT0) and the last writes
    // fp32.  The two lo buffers share X1's bytes.  The normalised X keeps every
    // operand far inside fp16's range.
    const size_t nx = static_cast<size_t>(nz) * r * cc;
    void* hi[2] = {XT0, XT1};
    void* lo[2] = {X1, static_cast<uint8_t*>(X1) + nx * 2};
    for (int t = 0; t < kPolarSteps; ++t) {
      const bool first = t == 0, last = t + 1 == kPolarSteps;
      const double a = kPolarCoef[t][0], b = kPolarCoef[t][1], cf = kPolarCoef[t][2];
      void* curH = hi[t & 1];
      {
        GemmCall g = base_call(r, r, cc);   // A = hi hi^T
        g.batch = nz; g.es = 2; g.f16 = true;
        g.A = curH; g.lda = cc; g.a_bs = 1ll * r * cc;
        g.B = curH; g.ldb = cc; g.b_bs = 1ll * r * cc;
        g.bn = 256; g.sym = true; g.epi = EPI_STORE;
        g.out_es = 2; g.out_f16 = true; g.aux_es = 2; g.aux_f16 = true;
        g.p.out = Ab; g.p.ldo = r; g.p.out_bs = 1ll * r * r; g.p.err = err;
        GPT_CK(run_gemm(g, s, wait_cycles));
      }
      {
        GemmCall g = base_call(r, r, r);    // B = b A + c A A (+ a I after the first step)
        g.batch = nz; g.es = 2; g.f16 = true;
        g.A = Ab; g.lda = r; g.a_bs = 1ll * r * r;
        g.B = Ab; g.ldb = r; g.b_bs = 1ll * r * r;
        g.bn = 256; g.sym = true; g.epi = EPI_AXPBY;
        g.out_es = 2; g.out_f16 = true; g.aux_es = 2; g.aux_f16 = true;
        g.p.out = Bb; g.p.ldo = r; g.p.out_bs = 1ll * r * r;
        g.p.aux = Ab; g.p.ld_aux = r; g.p.aux_bs = 1ll * r * r;
        g.p.alpha = static_cast<float>(b); g.p.beta = static_cast<float>(cf); g.p.err = err;
        g.p.gamma = first ? 0.f : static_cast<float>(a);
        GPT_CK(run_gemm(g, s, wait_cycles));
      }
      {
        GemmCall g = base_call(r, cc, r);   // X' = B hi + a X  (first step),  (a I + B) hi + a lo  (later)
        g.batch = nz; g.es = 2; g.f16 = true;
        g.A = Bb; g.lda = r; g.a_bs = 1ll * r * r;
        g.B = curH; g.b_mn = true; g.ldb = cc; g.b_bs = 1ll * r * cc;
        g.bn = 256; g.epi = EPI_AXPBY;
        if (first) {
          g.aux_es = 4; g.p.aux = X0;
        } else {
          g.aux_es = 2; g.aux_f16 = true; g.p.aux = lo[(t + 1) & 1];
        }
        g.p.ld_aux = cc; g.p.aux_bs = 1ll * r * cc;
        if (last) {
          g.out_es = 4; g.p.out = X0;
        } else {
          g.out_es = 2; g.out_f16 = true; g.p.out = hi[(t + 1) & 1];
          g.p.out2 = lo[t & 1]; g.p.split_lo = 1;
        }
        g.p.ldo = cc; g.p.out_bs = 1ll * r * cc;
        g.p.alpha = static_cast<float>(a); g.p.beta = 1.f; g.p.err = err;
        GPT_CK(run_gemm(g, s, wait_cycles));
      }
      *launches += 3;
    }
    *out = X0;
    *out_es = 4;
    return GPT_OK;
  }
  void* cur = X0;
  void* nxt = X1;
  void* curT = XT0;
  void* nxtT = XT1;
  for (int t = 0; t < kPolarSteps; ++t) {
    const int es = t < n_tf32 ? 4 : 2;
    const bool last = t + 1 == kPolarSteps;
    const int es_next = last ? es : ((t + 1) < n_tf32 ? 4 : 2);
    const bool next_T = !last && (t + 1) < n_tf32;
    const double a = kPolarCoef[t][0], b = kPolarCoef[t][1], cf = kPolarCoef[t][2];
    {
      GemmCall g = base_call(r, r, cc);   // A = X X^T
      g.batch = nz; g.es = es;
      g.A = cur; g.lda = cc; g.a_bs = 1ll * r * cc;
      g.B = cur; g.ldb = cc; g.b_bs = 1ll * r * cc;
      g.bn = es == 4 ? 128 : 256; g.sym = true; g.epi = EPI_STORE; g.out_es = es; g.aux_es = es;
      g.p.out = Ab; g.p.ldo = r; g.p.out_bs = 1ll * r * r; g.p.err = err;
      GPT_CK(run_gemm(g, s, wait_cycles));
    }
    {
      GemmCall g = base_call(r, r, r);    // B = b A + c A A
      g.batch = nz; g.es = es;
      g.A = Ab; g.lda = r; g.a_bs = 1ll * r * r;
      g.B = Ab; g.ldb = r; g.b_bs = 1ll * r * r;
      g.bn = es == 4 ? 128 : 256; g.sym = true; g.epi = EPI_AXPBY; g.out_es = es; g.aux_es = es;
      g.p.out = Bb; g.p.ldo = r; g.p.out_bs = 1ll * r * r;
      g.p.aux = Ab; g.p.ld_aux = r; g.p.aux_bs = 1ll * r * r;
      g.p.alpha = static_cast<float>(b); g.p.beta = static_cast<float>(cf); g.p.err = err;
      GPT_CK(run_gemm(g, s, wait_cycles));
    }
    {
      GemmCall g = base_call(r, cc, r);   // X' = a X + B X
      g.batch = nz; g.es = es;
      g.A = Bb; g.lda = r; g.a_bs = 1ll * r * r;
      if (es == 4) {
        g.B = curT; g.b_mn = false; g.ldb = r; g.b_bs = 1ll * r * cc;   // B(n, k) = X[k][n] = X^T[n][k]
      } else {
        g.B = cur; g.b_mn = true; g.ldb = cc; g.b_bs = 1ll * r * cc;
      }
      g.bn = 256; g.epi = EPI_AXPBY; g.out_es = es_next; g.aux_es = es;
      g.p.out = nxt; g.p.ldo = cc; g.p.out_bs = 1ll * r * cc;
      if (next_T) {
        g.p.out_t = nxtT;
        g.p.ldo_t = r;
      }
      g.p.aux = cur; g.p.ld_aux = cc; g.p.aux_bs = 1ll * r * cc;
      g.p.alpha = static_cast<float>(a); g.p.beta = 1.f; g.p.err = err;
      GPT_CK(run_gemm(g, s, wait_cycles));
    }
    *launches += 3;
    std::swap(cur, nxt);
    std::swap(curT, nxtT);
    *out_es = es_next;
  }
  *out = cur;
  return GPT_OK;
}

int check_ctx(const gpt_ctx* c) { return c ? GPT_OK : fail(GPT_EINVAL, "null context"); }

}  // namespace

// ======================================================================== ABI

extern "C" {

const char* gpt_last_error(void) { return g_last_error.c_str(); }

int gpt_workspace_size(const gpt_config* cfg, size_t* param_bytes, size_t* state_bytes, size_t* act_bytes) {
  Dims D;
  int rc = dims_from(cfg, D);
  if (rc) return rc;
  Plan P;
  make_plan(D, P);
  if (param_bytes) *param_bytes = P.param_bytes;
  if (state_bytes) *state_bytes = P.state_bytes;
  if (act_bytes) *act_bytes = P.act_bytes;
  return GPT_OK;
}

int gpt_init(const gpt_config* cfg, void* param_buf, void* state_buf, void* act_buf, void* stream, gpt_ctx** out) {
  if (!out) return fail(GPT_EINVAL, "null output pointer");
  *out = nullptr;
  Dims D;
  int rc = dims_from(cfg, D);
  if (rc) return rc;
  if (!param_buf || !state_buf || !act_buf) return fail(GPT_EINVAL, "null buffer");
  if ((reinterpret_cast<uintptr_t>(param_buf) | reinterpret_cast<uintptr_t>(state_buf) |
       reinterpret_cast<uintptr_t>(act_buf)) & (kAlign - 1))
    return fail(GPT_EINVAL, "buffers must be 256-byte aligned");
  gpt_ctx* c = new gpt_ctx();
  c->cfg = *cfg;
  c->D = D;
  make_plan(D, c->P);
  c->pbuf = static_cast<uint8_t*>(param_buf);
  c->sbuf = static_cast<uint8_t*>(state_buf);
  c->abuf = static_cast<uint8_t*>(act_buf);
  c->stream = static_cast<cudaStream_t>(stream);
  cudaStream_t s = c->stream;
  auto bad = [&](cudaError_t e, const char* what) {
    delete c;
    return fail(GPT_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
  };
  cudaError_t e;
  if ((e = cudaMemsetAsync(c->sbuf, 0, c->P.state_bytes, s)) != cudaSuccess) return bad(e, "zero state");
  if ((e = cudaMemsetAsync(c->A<int>(c->P.err), 0, 16, s)) != cudaSuccess) return bad(e, "zero error word");
  const size_t numel[6] = {static_cast<size_t>(D.V) * D.d, static_cast<size_t>(D.d) * D.V,
                           static_cast<size_t>(D.L) * D.d * D.qc, static_cast<size_t>(D.L) * D.d * D.d,
                           static_cast<size_t>(D.L) * D.d * D.F, static_cast<size_t>(D.L) * D.F * D.d};
  for (int i = 0; i < 6; ++i) {
    init_normal_kernel<<<1024, 256, 0, s>>>(c->W(i), c->Wb(i), static_cast<long long>(numel[i]), cfg->seed, i, 0.02f);
  }
  launch_rope_table(c->A<float2>(c->P.rope), D.T, s);
  if (D.nve) {
    // value-embedding tables N(0, 0.02) like the token embedding; gates zero
    init_normal_kernel<<<1024, 256, 0, s>>>(c->VeW(0), c->VeWb(0), static_cast<long long>(D.nve * c->ve_elems()),
                                            cfg->seed, 7, 0.02f);
    if ((e = cudaMemsetAsync(c->pbuf + c->P.wg, 0, static_cast<size_t>(D.ngp) * 4, s)) != cudaSuccess)
      return bad(e, "zero gates");
  }
  std::vector<float> sc0;
  if (D.extras) {
    // residual scales 1, x0 and backout scales 0 (and zero padding): the plain network
    sc0.assign(D.nsc, 0.f);
    for (int l = 0; l < D.L; ++l) sc0[l] = 1.f;
    if ((e = cudaMemcpyAsync(c->pbuf + c->P.ws, sc0.data(), sc0.size() * 4, cudaMemcpyHostToDevice, s)) != cudaSuccess)
      return bad(e, "init scalars");
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return bad(e, "init kernels");
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return bad(e, "init sync");
  c->launches = 7;
  *out = c;
  return GPT_OK;
}

int gpt_fwd_bwd(gpt_ctx* c, const int32_t* tokens, const int32_t* targets, float* loss_out, int accumulate) {
  int rc = check_ctx(c);
  if (rc) return rc;
  if (!tokens || !targets || !loss_out) return fail(GPT_EINVAL, "null pointer");
  if ((reinterpret_cast<uintptr_t>(tokens) | reinterpret_cast<uintptr_t>(targets)) & 3)
    return fail(GPT_EINVAL, "token/target pointers must be 4-byte aligned");
  return forward_backward(c, tokens, targets, loss_out, accumulate != 0);
}

// Muon over the block matrices of layers [l0, l1); with normuon the
// orthogonalised updates get the NorMuon per-neuron scaling (second-moment
// EMA with factor beta2) first.  Every matrix is updated on its own, so a
// range gives bit-for-bit the result the whole set gives for those layers.
static int muon_update(gpt_ctx* c, float lr, float momentum, float weight_decay, bool normuon, float beta2, int l0,
                       int l1) {
  int rc = check_ctx(c);
  if (rc) return rc;
  const Dims& D = c->D;
  const Plan& P = c->P;
  if (l0 < 0 || l1 > D.L || l0 > l1) return fail(GPT_EINVAL, "layer range out of bounds");
  if (l0 == l1) return GPT_OK;
  cudaStream_t s = c->stream;
  const int L = D.L, d = D.d, F = D.F;
  const int nl = l1 - l0;
  float* inv = c->A<float>(P.inv_norm);
  // momentum and Frobenius norms of every block matrix in the range
  const long long ne[4] = {1ll * d * D.qc, 1ll * d * d, 1ll * d * F, 1ll * F * d};
  {
    ProfScope ps(c, GPT_PROF_MUON_ELEM);
    for (int j = 0; j < 4; ++j)
      launch_muon_momentum(c->Mom(2 + j) + l0 * ne[j], c->G(2 + j) + l0 * ne[j], ne[j], nl, momentum, 1e-7f,
                           inv + j * L + l0, c->A<void>(P.normws), s);
  }
  c->launches += 8;
  // first Newton-Schulz iterate: fp32 for the fp16 and tf32 modes, bf16 otherwise
  const int es0 = D.n_tf32 != 0 ? 4 : 2;
  void* X0 = c->A<void>(P.X0);
  void* X1 = c->A<void>(P.X1);
  void* XT0 = c->A<void>(P.XT0);
  void* XT1 = c->A<void>(P.XT1);
  void* Ab = c->A<void>(P.Abuf);
  void* Bb = c->A<void>(P.Bbuf);
  // three Newton-Schulz batches, all with r = d rows: q|k|v (c = 3d), attention
  // output (c = d), and MLP up plus transposed MLP down (c = 4d)
  struct Member { int grp; bool transpose; };
  struct Batch { int nz; int cc; Member m[2]; int nm; };
  const Batch batches[3] = {{nl, D.qc, {{2, false}}, 1}, {nl, d, {{3, false}}, 1},
                            {2 * nl, F, {{4, false}, {5, true}}, 2}};
  for (const Batch& bt : batches) {
    const size_t per = static_cast<size_t>(d) * bt.cc;
    for (int i = 0; i < bt.nm; ++i) {
      ProfScope ps(c, GPT_PROF_MUON_ELEM);
      const Member& mm = bt.m[i];
      // X (d x cc) and, for tf32 steps, its transpose, from one read of the
      // momentum, which is stored d x cc, or cc x d for the MLP down matrix
      void* dst = static_cast<uint8_t*>(X0) + static_cast<size_t>(i) * nl * per * es0;
      void* dstT = D.n_tf32 > 0 ? static_cast<uint8_t*>(XT0) + static_cast<size_t>(i) * nl * per * es0 : nullptr;
      // fp16 mode: the fp16 operand copy of X, same layout as X
      __half* dstH = D.n_tf32 < 0 ? reinterpret_cast<__half*>(XT0) + static_cast<size_t>(i) * nl * per : nullptr;
      const float* mom = c->Mom(mm.grp) + l0 * per;
      const float* invg = inv + (mm.grp - 2) * L + l0;
      if (!mm.transpose)
        launch_muon_make_x(mom, invg, dst, dstT, es0, nl, d, bt.cc, s, dstH, nullptr);
      else
        launch_muon_make_x(mom, invg, dstT, dst, es0, nl, bt.cc, d, s, nullptr, dstH);
      c->launches += 1;
    }
    void* res = nullptr;
    int res_es = es0;
    rc = newton_schulz(c, bt.nz, d, bt.cc, X0, X1, XT0, XT1, Ab, Bb, D.n_tf32, s, c->err(), &res, &res_es,
                       &c->launches, c->wait_cycles);
    if (rc) return rc;
    for (int i = 0; i < bt.nm; ++i) {
      ProfScope ps(c, GPT_PROF_MUON_ELEM);
      const Member& mm = bt.m[i];
      const int rows = mm.grp == 5 ? F : d;
      const int cols = mm.grp == 2 ? D.qc : (mm.grp == 3 ? d : (mm.grp == 4 ? F : d));
      const float scale = sqrtf(std::max(1.f, static_cast<float>(rows) / static_cast<float>(cols)));
      const void* src = static_cast<const uint8_t*>(res) + static_cast<size_t>(i) * nl * per * res_es;
      // NorMuon: one factor per row of res (the shorter axis of every matrix)
      float* rowf = nullptr;
      if (normuon) {
        rowf = c->A<float>(P.nfac) + static_cast<size_t>(i) * nl * d;
        launch_normuon_factor(src, res_es, nl, d, bt.cc, c->NV(mm.grp) + static_cast<size_t>(l0) * d, beta2, rowf, s);
        c->launches += 2;
      }
      launch_muon_apply(c->W(mm.grp) + l0 * per, c->Wb(mm.grp) + l0 * per, src, res_es, nl, d, bt.cc, mm.transpose,
                        lr, weight_decay, scale, s, rowf);
      c->launches += 1;
    }
  }
  GPT_CK(cudaGetLastError());
  return GPT_OK;
}

int muon_step(gpt_ctx* c, float lr, float momentum, float weight_decay) {
  int rc = check_ctx(c);
  if (rc) return rc;
  return muon_update(c, lr, momentum, weight_decay, false, 0.f, 0, c->D.L);
}

int muon_step_normuon(gpt_ctx* c, float lr, float momentum, float weight_decay, float beta2) {
  int rc = check_ctx(c);
  if (rc) return rc;
  if (!(beta2 >= 0.f && beta2 < 1.f)) return fail(GPT_EINVAL, "NorMuon beta2 must be in [0, 1)");
  return muon_update(c, lr, momentum, weight_decay, true, beta2, 0, c->D.L);
}

int muon_step_layers(gpt_ctx* c, float lr, float momentum, float weight_decay, float normuon_beta2, int l0,
                     int l1) {
  int rc = check_ctx(c);
  if (rc) return rc;
  if (!(normuon_beta2 < 1.f)) return fail(GPT_EINVAL, "NorMuon beta2 must be below 1 (negative: plain Muon)");
  return muon_update(c, lr, momentum, weight_decay, normuon_beta2 >= 0.f, normuon_beta2, l0, l1);
}

int gpt_block_region(const gpt_ctx* c, int what, int kind, int l0, int l1, size_t* offset_bytes,
                     size_t* size_bytes) {
  int rc = check_ctx(c);
  if (rc) return rc;
  if (kind < 0 || kind > 3) return fail(GPT_EINVAL, "block matrix kind must be 0..3");
  if (what < GPT_REGION_MASTER || what > GPT_REGION_GRAD) return fail(GPT_EINVAL, "unknown region");
  if (l0 < 0 || l1 > c->D.L || l0 > l1) return fail(GPT_EINVAL, "layer range out of bounds");
  const int grp = 2 + kind;
  const size_t d = c->D.d, F = c->D.F;
  const size_t per[4] = {d * static_cast<size_t>(c->D.qc), d * d, d * F, F * d};
  const size_t es = what == GPT_REGION_BF16 ? 2 : 4;
  const size_t base = what == GPT_REGION_MASTER ? c->P.w[grp] : (what == GPT_REGION_BF16 ? c->P.wb[grp] : c->P.g[grp]);
  if (offset_bytes) *offset_bytes = base + static_cast<size_t>(l0) * per[kind] * es;
  if (size_bytes) *size_bytes = static_cast<size_t>(l1 - l0) * per[kind] * es;
  return GPT_OK;
}

// AdamW of the embedding and lm_head rows of share `part` of `nparts` (rows
// [part R / nparts, (part + 1) R / nparts) of each), and of every other
// AdamW tensor whole.
static int adamw_update(gpt_ctx* c, float lr, float beta1, float beta2, float eps, float weight_decay, int part,
                        int nparts) {
  c->adam_step += 1;
  const double t = static_cast<double>(c->adam_step);
  const float bc1 = static_cast<float>(1.0 - pow(static_cast<double>(beta1), t));
  const float bc2 = static_cast<float>(1.0 - pow(static_cast<double>(beta2), t));
  ProfScope ps(c, GPT_PROF_ADAMW);
  for (int i = 0; i < 2; ++i) {
    const long long rows = i == 0 ? c->D.V : c->D.d, cols = i == 0 ? c->D.d : c->D.V;
    const long long r0 = rows * part / nparts, r1 = rows * (part + 1) / nparts;
    if (r1 <= r0) continue;
    const size_t off = static_cast<size_t>(r0 * cols);
    launch_adamw(c->W(i) + off, c->G(i) + off, reinterpret_cast<float*>(c->sbuf + c->P.am[i]) + off,
                 reinterpret_cast<float*>(c->sbuf + c->P.av[i]) + off, c->Wb(i) + off, (r1 - r0) * cols, lr, beta1,
                 beta2, eps, weight_decay, bc1, bc2, c->stream);
    c->launches += 1;
  }
  if (c->D.nve) {
    // value-embedding tables and their gates
    launch_adamw(c->VeW(0), c->VeG(0), reinterpret_cast<float*>(c->sbuf + c->P.amve),
                 reinterpret_cast<float*>(c->sbuf + c->P.avve), c->VeWb(0),
                 static_cast<long long>(c->D.nve * c->ve_elems()), lr, beta1, beta2, eps, weight_decay, bc1, bc2,
                 c->stream);
    launch_adamw(c->GateW(0), c->GateG(0), reinterpret_cast<float*>(c->sbuf + c->P.amg),
                 reinterpret_cast<float*>(c->sbuf + c->P.avg), reinterpret_cast<bf16*>(c->pbuf + c->P.wgb), c->D.ngp,
                 lr, beta1, beta2, eps, weight_decay, bc1, bc2, c->stream);
    c->launches += 2;
  }
  if (c->D.extras) {
    // the scalars (zero padding stays zero: zero gradient, zero value)
    launch_adamw(reinterpret_cast<float*>(c->pbuf + c->P.ws), reinterpret_cast<float*>(c->sbuf + c->P.gs),
                 reinterpret_cast<float*>(c->sbuf + c->P.ams), reinterpret_cast<float*>(c->sbuf + c->P.avs),
                 reinterpret_cast<bf16*>(c->pbuf + c->P.wsb), c->D.nsc, lr, beta1, beta2, eps, weight_decay, bc1, bc2,
                 c->stream);
    c->launches += 1;
  }
  GPT_CK(cudaGetLastError());
  return GPT_OK;
}

int gpt_tensor_region(const gpt_ctx* c, int what, int id, int row0, int row1, size_t* offset_bytes,
                      size_t* size_bytes) {
  int rc = check_ctx(c);
  if (rc) return rc;
  if (what < GPT_REGION_MASTER || what > GPT_REGION_GRAD) return fail(GPT_EINVAL, "unknown region");
  int grp, rows, cols;
  size_t off;
  if (!locate(c, id, grp, off, rows, cols) || grp >= 6)
    return fail(GPT_EINVAL, "tensor id must name the embedding, the lm_head or a block matrix");
  if (row0 < 0 || row1 > rows || row0 > row1) return fail(GPT_EINVAL, "row range out of bounds");
  const size_t es = what == GPT_REGION_BF16 ? 2 : 4;
  const size_t base = what == GPT_REGION_MASTER ? c->P.w[grp] : (what == GPT_REGION_BF16 ? c->P.wb[grp] : c->P.g[grp]);
  if (offset_bytes) *offset_bytes = base + (off + static_cast<size_t>(row0) * cols) * es;
  if (size_bytes) *size_bytes = static_cast<size_t>(row1 - row0) * cols * es;
  return GPT_OK;
}

int adamw_step(gpt_ctx* c, float lr, float beta1, float beta2, float eps, float weight_decay) {
  int rc = check_ctx(c);
  if (rc) return rc;
  return adamw_update(c, lr, beta1, beta2, eps, weight_decay, 0, 1);
}

int adamw_step_shard(gpt_ctx* c, float lr, float beta1, float beta2, float eps, float weight_decay, int part,
                     int nparts) {
  int rc = check_ctx(c);
  if (rc) return rc;
  if (nparts < 1 || part < 0 || part >= nparts) return fail(GPT_EINVAL, "need 0 <= part < nparts");
  return adamw_update(c, lr, beta1, beta2, eps, weight_decay, part, nparts);
}

int gpt_set_grad_events(gpt_ctx* c, void* const* events, int n) {
  int rc = check_ctx(c);
  if (rc) return rc;
  if (n < 0 || n > GPT_GRAD_BUCKETS || (n > 0 && !events)) return fail(GPT_EINVAL, "0..GPT_GRAD_BUCKETS events");
  for (int i = 0; i < GPT_GRAD_BUCKETS; ++i) c->grad_ev[i] = i < n ? static_cast<cudaEvent_t>(events[i]) : nullptr;
  c->n_grad_ev = n;
  return GPT_OK;
}

int gpt_grad_bucket(const gpt_ctx* c, int bucket, size_t* offset_bytes, size_t* size_bytes) {
  int rc = check_ctx(c);
  if (rc) return rc;
  const Plan& P = c->P;
  const Dims& D = c->D;
  size_t b = 0, e = 0;
  if (bucket == 0) {
    b = P.g[1];
    e = P.g[1] + static_cast<size_t>(D.d) * D.V * 4;
  } else if (bucket >= 1 && bucket <= 4) {
    const size_t d = D.d, F = D.F;
    const size_t per[4] = {d * static_cast<size_t>(D.qc), d * d, d * F, F * d};
    b = P.g[1 + bucket];
    e = b + static_cast<size_t>(D.L) * per[bucket - 1] * 4;
  } else if (bucket == 5) {
    b = P.g[0];
    e = P.g[2];   // the embedding, then the extras' gradients, up to the first block gradient
  } else {
    return fail(GPT_EINVAL, "bucket must be 0..GPT_GRAD_BUCKETS-1");
  }
  if (offset_bytes) *offset_bytes = b;
  if (size_bytes) *size_bytes = e - b;
  return GPT_OK;
}

int gpt_train_step_host(gpt_ctx* c, const int32_t* tokens_host, const int32_t* targets_host, const gpt_hparams* hp,
                        float* loss_host) {
  int rc = check_ctx(c);
  if (rc) return rc;
  if (!tokens_host || !targets_host || !hp || !loss_host) return fail(GPT_EINVAL, "null pointer");
  const size_t bytes = static_cast<size_t>(c->D.M) * 4;
  int* tok = c->A<int>(c->P.tok);
  int* tgt = c->A<int>(c->P.tgt);
  GPT_CK(cudaMemcpyAsync(tok, tokens_host, bytes, cudaMemcpyHostToDevice, c->stream));
  GPT_CK(cudaMemcpyAsync(tgt, targets_host, bytes, cudaMemcpyHostToDevice, c->stream));
  float* loss = c->A<float>(c->P.loss);
  rc = forward_backward(c, tok, tgt, loss, false);
  if (rc) return rc;
  rc = muon_step(c, hp->muon_lr, hp->muon_momentum, hp->muon_wd);
  if (rc) return rc;
  rc = adamw_step(c, hp->adam_lr, hp->adam_beta1, hp->adam_beta2, hp->adam_eps, hp->adam_wd);
  if (rc) return rc;
  GPT_CK(cudaMemcpyAsync(loss_host, loss, sizeof(float), cudaMemcpyDeviceToHost, c->stream));
  GPT_CK(cudaStreamSynchronize(c->stream));
  return gpt_check(c);
}

int gpt_get_adam_step(const gpt_ctx* c, int64_t* step) {
  int rc = check_ctx(c);
  if (rc) return rc;
  if (!step) return fail(GPT_EINVAL, "null destination");
  *step = c->adam_step;
  return GPT_OK;
}

int gpt_set_adam_step(gpt_ctx* c, int64_t step) {
  int rc = check_ctx(c);
  if (rc) return rc;
  if (step < 0) return fail(GPT_EINVAL, "the AdamW step count cannot be negative");
  c->adam_step = step;
  return GPT_OK;
}

int gpt_num_tensors(const gpt_ctx* c) {
  return c ? 2 + 4 * c->D.L + c->D.extras + (c->D.nve ? c->D.nve + 1 : 0) : 0;
}

int gpt_tensor_info(const gpt_ctx* c, int id, int32_t* rows, int32_t* cols, int32_t* group) {
  int rc = check_ctx(c);
  if (rc) return rc;
  int grp, r, cc;
  size_t off;
  if (!locate(c, id, grp, off, r, cc)) return fail(GPT_EINVAL, "tensor id out of range");
  if (rows) *rows = r;
  if (cols) *cols = cc;
  if (group) *group = (grp < 2 || grp >= 6) ? GPT_GROUP_ADAMW : GPT_GROUP_MUON;
  return GPT_OK;
}

static int tensor_ptr(gpt_ctx* c, int id, int kind, float** p, size_t* n, int* grp_out, size_t* off_out) {
  int grp, r, cc;
  size_t off;
  if (!locate(c, id, grp, off, r, cc)) return fail(GPT_EINVAL, "tensor id out of range");
  float* base = nullptr;
  if (grp == 7 || grp == 8) {
    const size_t pw = grp == 7 ? c->P.wve : c->P.wg, gw = grp == 7 ? c->P.gve : c->P.gg;
    const size_t am = grp == 7 ? c->P.amve : c->P.amg, av = grp == 7 ? c->P.avve : c->P.avg;
    switch (kind) {
      case GPT_KIND_PARAM: *p = reinterpret_cast<float*>(c->pbuf + pw) + off; break;
      case GPT_KIND_GRAD: *p = reinterpret_cast<float*>(c->sbuf + gw) + off; break;
      case GPT_KIND_ADAM_M: *p = reinterpret_cast<float*>(c->sbuf + am) + off; break;
      case GPT_KIND_ADAM_V: *p = reinterpret_cast<float*>(c->sbuf + av) + off; break;
      default: return fail(GPT_EINVAL, "value embeddings have a value, a gradient and AdamW moments only");
    }
    *n = static_cast<size_t>(r) * cc;
    *grp_out = grp;
    *off_out = off;
    return GPT_OK;
  }
  if (grp == 6) {
    size_t o;
    switch (kind) {
      case GPT_KIND_PARAM: *p = reinterpret_cast<float*>(c->pbuf + c->P.ws); break;
      case GPT_KIND_GRAD: o = c->P.gs; *p = reinterpret_cast<float*>(c->sbuf + o); break;
      case GPT_KIND_ADAM_M: o = c->P.ams; *p = reinterpret_cast<float*>(c->sbuf + o); break;
      case GPT_KIND_ADAM_V: o = c->P.avs; *p = reinterpret_cast<float*>(c->sbuf + o); break;
      default: return fail(GPT_EINVAL, "the scalars have a value, a gradient and AdamW moments only");
    }
    *n = static_cast<size_t>(r) * cc;
    *grp_out = grp;
    *off_out = 0;
    return GPT_OK;
  }
  switch (kind) {
    case GPT_KIND_PARAM: base = c->W(grp); break;
    case GPT_KIND_GRAD: base = c->G(grp); break;
    case GPT_KIND_MOM:
      if (grp < 2) return fail(GPT_EINVAL, "momentum exists only for block matrices");
      base = c->Mom(grp);
      break;
    case GPT_KIND_ADAM_M:
    case GPT_KIND_ADAM_V:
      if (grp >= 2) return fail(GPT_EINVAL, "AdamW moments exist only for the embedding and lm_head");
      base = reinterpret_cast<float*>(c->sbuf + (kind == GPT_KIND_ADAM_M ? c->P.am[grp] : c->P.av[grp]));
      break;
    case GPT_KIND_NORMUON_V: {
      // one d-vector per matrix (its shorter axis): layer l's is the l-th
      if (grp < 2) return fail(GPT_EINVAL, "NorMuon state exists only for block matrices");
      const size_t l = off / (static_cast<size_t>(r) * cc);
      *p = c->NV(grp) + l * c->D.d;
      *n = static_cast<size_t>(c->D.d);
      *grp_out = grp;
      *off_out = off;
      return GPT_OK;
    }
    default:
      return fail(GPT_EINVAL, "unknown tensor kind");
  }
  *p = base + off;
  *n = static_cast<size_t>(r) * cc;
  *grp_out = grp;
  *off_out = off;
  return GPT_OK;
}

int gpt_get_tensor(gpt_ctx* c, int id, int kind, float* dst) {
  int rc = check_ctx(c);
  if (rc) return rc;
  if (!dst) return fail(GPT_EINVAL, "null destination");
  float* p;
  size_t n, off;
  int grp;
  rc = tensor_ptr(c, id, kind, &p, &n, &grp, &off);
  if (rc) return rc;
  GPT_CK(cudaMemcpyAsync(dst, p, n * 4, cudaMemcpyDeviceToDevice, c->stream));
  return GPT_OK;
}

int gpt_set_tensor(gpt_ctx* c, int id, int kind, const float* src) {
  int rc = check_ctx(c);
  if (rc) return rc;
  if (!src) return fail(GPT_EINVAL, "null source");
  float* p;
  size_t n, off;
  int grp;
  rc = tensor_ptr(c, id, kind, &p, &n, &grp, &off);
  if (rc) return rc;
  GPT_CK(cudaMemcpyAsync(p, src, n * 4, cudaMemcpyDeviceToDevice, c->stream));
  if (kind == GPT_KIND_PARAM && (grp < 6 || grp == 7)) {   // scalars and gates are read in fp32
    launch_cast_bf16(p, grp == 7 ? reinterpret_cast<bf16*>(c->pbuf + c->P.wveb) + off : c->Wb(grp) + off,
                     static_cast<long long>(n), c->stream);
    c->launches += 1;
  }
  GPT_CK(cudaGetLastError());
  return GPT_OK;
}

int gpt_grad_region(const gpt_ctx* c, size_t* offset_bytes, size_t* size_bytes) {
  int rc = check_ctx(c);
  if (rc) return rc;
  const size_t last = c->P.g[5] + static_cast<size_t>(c->D.L) * c->D.F * c->D.d * 4;
  if (offset_bytes) *offset_bytes = c->P.g[1];
  if (size_bytes) *size_bytes = al(last) - c->P.g[1];
  return GPT_OK;
}

int gpt_get_row_loss(gpt_ctx* c, float* dst) {
  int rc = check_ctx(c);
  if (rc) return rc;
  if (!dst) return fail(GPT_EINVAL, "null destination");
  GPT_CK(cudaMemcpyAsync(dst, c->A<float>(c->P.row_loss), static_cast<size_t>(c->D.M) * 4,
                         cudaMemcpyDeviceToDevice, c->stream));
  return GPT_OK;
}

int gpt_check(gpt_ctx* c) {
  int rc = check_ctx(c);
  if (rc) return rc;
  GPT_CK(cudaStreamSynchronize(c->stream));
  int flag = 0;
  GPT_CK(cudaMemcpy(&flag, c->err(), sizeof(int), cudaMemcpyDeviceToHost));
  if (flag) GPT_CK(cudaMemset(c->err(), 0, sizeof(int)));
  if (flag & ERRF_TIMEOUT) return fail(GPT_ETIMEOUT, "a bounded device wait expired");
  if (flag & ERRF_TOKEN_RANGE) return fail(GPT_ERANGE, "token or target id outside [0, vocab)");
  if (flag) return fail(GPT_ECUDA, "device error flag set");
  return GPT_OK;
}

int64_t gpt_launch_count(const gpt_ctx* c) { return c ? c->launches : 0; }

int gpt_profile_enable(gpt_ctx* c, uint32_t mask) {
  int rc = check_ctx(c);
  if (rc) return rc;
  c->prof_mask = mask & ((1u << GPT_PROF_COUNT) - 1u);
  return GPT_OK;
}

int gpt_profile_read(gpt_ctx* c, double* ms, int64_t* launches) {
  int rc = check_ctx(c);
  if (rc) return rc;
  GPT_CK(cudaStreamSynchronize(c->stream));
  for (size_t i = 0; i < c->recs_used; ++i) {
    float t = 0.f;
    GPT_CK(cudaEventElapsedTime(&t, c->recs[i].a, c->recs[i].b));
    c->prof_ms[c->recs[i].cat] += t;
    c->prof_n[c->recs[i].cat] += 1;
  }
  c->recs_used = 0;
  for (int k = 0; k < GPT_PROF_COUNT; ++k) {
    if (ms) ms[k] = c->prof_ms[k];
    if (launches) launches[k] = c->prof_n[k];
    c->prof_ms[k] = 0.0;
    c->prof_n[k] = 0;
  }
  return GPT_OK;
}

void gpt_destroy(gpt_ctx* c) { delete c; }

// ------------------------------------------------------------ op-level calls
//
// The op-level entry points have no context, so the library keeps their
// device error word itself: one word per device (a __device__ variable
// exists once on every GPU that loads the library), ORed into by every
// op-level kernel and read and cleared by gpt_op_check.  Their wait bound is
// one process-wide value.

}  // extern "C"

namespace {

__device__ int g_op_err_word[4];
std::atomic<long long> g_op_wait_cycles{0};

// Device address of the op-level error word on the current device, looked
// up on every call (cheap once the library's device code is loaded), so a
// context created after a device reset gets its own address.
int op_err(int** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_op_err_word);
  if (e != cudaSuccess || !p)
    return fail(GPT_ECUDA, std::string("cudaGetSymbolAddress of the op-level error word: ") + cudaGetErrorString(e));
  *out = static_cast<int*>(p);
  return GPT_OK;
}

}  // namespace

extern "C" {

int gpt_op_set_wait_limit(long long cycles) {
  g_op_wait_cycles.store(cycles > 0 ? cycles : 0);
  return GPT_OK;
}

int gpt_op_check(void* stream) {
  GPT_CK(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  int* word = nullptr;
  int rc = op_err(&word);
  if (rc) return rc;
  int flag = 0;
  GPT_CK(cudaMemcpy(&flag, word, sizeof(int), cudaMemcpyDeviceToHost));
  if (flag) GPT_CK(cudaMemset(word, 0, sizeof(int)));
  if (flag & ERRF_TIMEOUT) return fail(GPT_ETIMEOUT, "a bounded device wait of an op-level call expired");
  if (flag & ERRF_TOKEN_RANGE) return fail(GPT_ERANGE, "token or target id outside [0, vocab)");
  if (flag) return fail(GPT_ECUDA, "op-level device error flag set");
  return GPT_OK;
}

int gpt_set_wait_limit(gpt_ctx* c, long long cycles) {
  int rc = check_ctx(c);
  if (rc) return rc;
  c->wait_cycles = cycles > 0 ? cycles : 0;
  return GPT_OK;
}

int gpt_op_matmul_bf16(const void* A, const void* B, float* C, int M, int N, int K, int batch, int a_trans,
                       int b_trans, void* stream) {
  if (!A || !B || !C) return fail(GPT_EINVAL, "null pointer");
  if (M < 0 || N < 0 || K <= 0 || batch < 1 || N % 8 || K % 8) return fail(GPT_EINVAL, "bad matmul shape");
  if (a_trans && M % 8) return fail(GPT_EINVAL, "M must be a multiple of 8 when A is transposed");
  GemmCall g = base_call(M, N, K);
  g.batch = batch;
  g.A = A; g.a_mn = a_trans != 0; g.lda = a_trans ? M : K; g.a_bs = 1ll * M * K;
  g.B = B; g.b_mn = b_trans == 0; g.ldb = b_trans ? K : N; g.b_bs = 1ll * K * N;
  g.epi = EPI_STORE; g.out_es = 4; g.aux_es = 4;
  g.p.out = C; g.p.ldo = N; g.p.out_bs = 1ll * M * N;
  int rc = op_err(&g.p.err);
  if (rc) return rc;
  GPT_CK(run_gemm(g, static_cast<cudaStream_t>(stream), g_op_wait_cycles.load()));
  return GPT_OK;
}

int gpt_op_matmul_tf32(const float* A, const float* B, float* C, int M, int N, int K, int b_trans, void* stream) {
  if (!A || !B || !C) return fail(GPT_EINVAL, "null pointer");
  if (M < 0 || N < 0 || K <= 0 || N % 8 || K % 4) return fail(GPT_EINVAL, "bad matmul shape");
  if (!b_trans) return fail(GPT_EINVAL, "tf32 operands must be K-major: pass B as [N, K] with b_trans = 1");
  GemmCall g = base_call(M, N, K);
  g.es = 4;
  g.A = A; g.lda = K;
  g.B = B; g.ldb = K;
  g.bn = 128; g.epi = EPI_STORE; g.out_es = 4; g.aux_es = 4;
  g.p.out = C; g.p.ldo = N;
  int rc = op_err(&g.p.err);
  if (rc) return rc;
  GPT_CK(run_gemm(g, static_cast<cudaStream_t>(stream), g_op_wait_cycles.load()));
  return GPT_OK;
}

int gpt_op_quantize_e4m3(const void* x, long long n, void* q, float* inv, unsigned int* amax_scratch, void* stream) {
  if (!x || !q || !inv || !amax_scratch) return fail(GPT_EINVAL, "null pointer");
  if (n < 0) return fail(GPT_EINVAL, "negative size");
  if (reinterpret_cast<uintptr_t>(x) & 15 || reinterpret_cast<uintptr_t>(q) & 7)
    return fail(GPT_EINVAL, "x must be 16-byte and q 8-byte aligned");
  launch_quantize_e4m3(static_cast<const bf16*>(x), n, 1, amax_scratch, static_cast<uint8_t*>(q), inv,
                       static_cast<cudaStream_t>(stream));
  GPT_CK(cudaGetLastError());
  return GPT_OK;
}

int gpt_op_matmul_fp8(const void* A, const void* B, float* C, int M, int N, int K, const float* inv_a,
                      const float* inv_b, int b_trans, void* stream) {
  if (!A || !B || !C || !inv_a || !inv_b) return fail(GPT_EINVAL, "null pointer");
  if (M < 0 || N < 0 || K <= 0 || N % 16 || K % 16) return fail(GPT_EINVAL, "bad matmul shape (N, K multiples of 16)");
  GemmCall g = base_call(M, N, K);
  g.es = 1;
  g.A = A; g.lda = K;
  g.B = B; g.b_mn = b_trans == 0; g.ldb = b_trans ? K : N;
  g.epi = EPI_STORE; g.out_es = 4; g.aux_es = 4;
  g.p.out = C; g.p.ldo = N; g.p.dq_a = inv_a; g.p.dq_b = inv_b;
  int rc = op_err(&g.p.err);
  if (rc) return rc;
  GPT_CK(run_gemm(g, static_cast<cudaStream_t>(stream), g_op_wait_cycles.load()));
  return GPT_OK;
}

int gpt_op_attention_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                            int T, int window, void* stream) {
  if (!q || !k || !v || !o || !lse) return fail(GPT_EINVAL, "null pointer");
  if (B < 1 || H < 1 || T < 1) return fail(GPT_EINVAL, "bad attention shape");
  if (Hkv < 1 || H % Hkv) return fail(GPT_EINVAL, "kv heads must divide the query heads");
  if (static_cast<long long>(B) * H * T > (1ll << 31) - 1) return fail(GPT_EINVAL, "attention too large");
  int* err = nullptr;
  int rc = op_err(&err);
  if (rc) return rc;
  launch_attn_fwd(static_cast<const bf16*>(q), static_cast<const bf16*>(k), static_cast<const bf16*>(v),
                  static_cast<bf16*>(o), lse, B, H, T, static_cast<cudaStream_t>(stream), err, Hkv, window, nullptr,
                  0, g_op_wait_cycles.load());
  GPT_CK(cudaGetLastError());
  return GPT_OK;
}

int gpt_op_attention_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int T,
                         void* stream) {
  return gpt_op_attention_fwd_ex(q, k, v, o, lse, B, H, H, T, -1, stream);
}

int gpt_op_attention_bwd_ex(const void* q, const void* k, const void* v, const void* o, const void* dout,
                            const float* lse, float* Dscratch, float* dq, void* dk, void* dv, int B, int H, int Hkv,
                            int T, int window, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !Dscratch || !dq || !dk || !dv) return fail(GPT_EINVAL, "null pointer");
  if (B < 1 || H < 1 || T < 1) return fail(GPT_EINVAL, "bad attention shape");
  if (Hkv < 1 || H % Hkv) return fail(GPT_EINVAL, "kv heads must divide the query heads");
  if (static_cast<long long>(B) * H * T > (1ll << 31) - 1) return fail(GPT_EINVAL, "attention too large");
  int* err = nullptr;
  int rc = op_err(&err);
  if (rc) return rc;
  launch_attn_bwd(static_cast<const bf16*>(q), static_cast<const bf16*>(k), static_cast<const bf16*>(v),
                  static_cast<const bf16*>(o), static_cast<const bf16*>(dout), lse, Dscratch, dq,
                  static_cast<bf16*>(dk), static_cast<bf16*>(dv), B, H, T, static_cast<cudaStream_t>(stream), err,
                  Hkv, window, nullptr, 0, g_op_wait_cycles.load());
  GPT_CK(cudaGetLastError());
  return GPT_OK;
}

int gpt_op_attention_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                         const float* lse, float* Dscratch, float* dq, void* dk, void* dv, int B, int H, int T,
                         void* stream) {
  return gpt_op_attention_bwd_ex(q, k, v, o, dout, lse, Dscratch, dq, dk, dv, B, H, H, T, -1, stream);
}

int gpt_op_rmsnorm_fwd(const float* x, void* y, float* rstd, int M, int d, void* stream) {
  if (!x || !y || !rstd) return fail(GPT_EINVAL, "null pointer");
  if (M < 0 || d < 128 || d % 128 || d > 2048) return fail(GPT_EINVAL, "bad rmsnorm shape (d: a multiple of 128 up to 2048)");
  launch_rmsnorm_fwd(x, static_cast<bf16*>(y), rstd, M, d, static_cast<cudaStream_t>(stream));
  GPT_CK(cudaGetLastError());
  return GPT_OK;
}

size_t gpt_op_embedding_bwd_scratch(int M, int d) {
  return M < 0 || d < 128 || d % 128 ? 0 : embed_bwd_workspace(M, d);
}

int gpt_op_embedding_bwd(const int32_t* tokens, const float* dx, float* dwte, int M, int d, int vocab, int accumulate,
                         void* scratch, void* stream) {
  if (!tokens || !dx || !dwte || !scratch) return fail(GPT_EINVAL, "null pointer");
  if (M < 0 || d < 128 || d % 128 || vocab < 1 || vocab > 131072)
    return fail(GPT_EINVAL, "bad embedding shape (d: a multiple of 128; vocab in [1, 131072])");
  if ((reinterpret_cast<uintptr_t>(dx) | reinterpret_cast<uintptr_t>(dwte)) & 15)
    return fail(GPT_EINVAL, "dx and dwte must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(scratch) & (kAlign - 1)) return fail(GPT_EINVAL, "scratch must be 256-byte aligned");
  launch_embed_bwd(tokens, dx, dwte, M, d, vocab, scratch, accumulate != 0, static_cast<cudaStream_t>(stream));
  GPT_CK(cudaGetLastError());
  return GPT_OK;
}

size_t gpt_op_newton_schulz_scratch(int batch, int rows, int cols) {
  const size_t r = std::min(rows, cols), cc = std::max(rows, cols), n = static_cast<size_t>(batch) * r * cc;
  return 4 * al(n * 4) + 2 * al(static_cast<size_t>(batch) * r * r * 4) + al(batch * 4) +
         al(muon_norm_workspace(batch)) + al(n * 2);
}

int gpt_op_newton_schulz(const float* G, float* X, int batch, int rows, int cols, int tf32_steps, void* scratch,
                         void* stream) {
  if (!G || !X || !scratch) return fail(GPT_EINVAL, "null pointer");
  if (batch < 1 || rows < 8 || cols < 8 || rows % 8 || cols % 8) return fail(GPT_EINVAL, "bad matrix shape");
  if (tf32_steps < -1 || tf32_steps > 5) return fail(GPT_EINVAL, "tf32_steps must be in -1..5");
  if (reinterpret_cast<uintptr_t>(scratch) & (kAlign - 1)) return fail(GPT_EINVAL, "scratch must be 256-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool tr = rows > cols;
  const int r = tr ? cols : rows, cc = tr ? rows : cols;
  const size_t n = static_cast<size_t>(batch) * r * cc;
  Bump b;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  void* X0 = base + b.take(n * 4);
  void* X1 = base + b.take(n * 4);
  void* XT0 = base + b.take(n * 4);
  void* XT1 = base + b.take(n * 4);
  void* Ab = base + b.take(static_cast<size_t>(batch) * r * r * 4);
  void* Bb = base + b.take(static_cast<size_t>(batch) * r * r * 4);
  float* inv = reinterpret_cast<float*>(base + b.take(batch * 4));
  void* normws = base + b.take(muon_norm_workspace(batch));
  bf16* Xb = reinterpret_cast<bf16*>(base + b.take(n * 2));
  int* err = nullptr;
  int rc = op_err(&err);
  if (rc) return rc;
  GPT_CK(cudaMemsetAsync(X, 0, n * 4, s));
  launch_muon_momentum(X, G, static_cast<long long>(rows) * cols, batch, 0.f, 1e-7f, inv, normws, s);
  const int es0 = tf32_steps != 0 ? 4 : 2;
  // X (r x cc) and, for tf32 steps, its transpose or, for fp16 steps, its fp16
  // copy; the input is stored r x cc, or cc x r when it was transposed to put
  // the smaller side first
  void* xT = tf32_steps > 0 ? XT0 : nullptr;
  __half* xH = tf32_steps < 0 ? static_cast<__half*>(XT0) : nullptr;
  if (!tr)
    launch_muon_make_x(X, inv, X0, xT, es0, batch, r, cc, s, xH, nullptr);
  else
    launch_muon_make_x(X, inv, xT, X0, es0, batch, cc, r, s, nullptr, xH);
  GPT_CK(cudaMemsetAsync(X, 0, n * 4, s));
  void* res = nullptr;
  int res_es = es0;
  int64_t launches = 0;
  rc = newton_schulz(nullptr, batch, r, cc, X0, X1, XT0, XT1, Ab, Bb, tf32_steps, s, err, &res, &res_es,
                     &launches, g_op_wait_cycles.load());
  if (rc) return rc;
  // X = 0 * (1 - 0) + 1 * NS(G): the apply kernel with lr = -1 writes the (un-transposed) result
  launch_muon_apply(X, Xb, res, res_es, batch, r, cc, tr, -1.f, 0.f, 1.f, s);
  GPT_CK(cudaGetLastError());
  return GPT_OK;
}

// ----------------------------------------------- Newton-Schulz without allocation
//
// Some callers cannot hand this library device scratch: code whose device
// memory is entirely owned by another allocator (a framework's caching pool
// that has already reserved the GPU), runtimes that forbid cudaMalloc after
// start-up, and C callers whose interface has no place for a scratch buffer.
// This variant keeps its scratch in a fixed array in device global memory
// that is part of the loaded library instead.

namespace {

constexpr long long kNsStaticMaxElems = 1ll << 18;   // batch * rows * cols
constexpr int kNsStaticMaxBatch = 64;
constexpr size_t align256(size_t x) { return (x + 255) / 256 * 256; }
// layout of gpt_op_newton_schulz's scratch at the largest accepted size
// (its r x r products never exceed the r x c inputs)
constexpr size_t kNsStaticBytes = 6 * align256(kNsStaticMaxElems * 4) + align256(kNsStaticMaxBatch * 4) +
                                  align256(kNsStaticMaxBatch * 64 * 4) + align256(kNsStaticMaxElems * 2);

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_ns_static_scratch[kNsStaticBytes];

// Device address of the array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// the device current, on every call: the lookup is cheap once the library's
// device code is loaded on that device (the first lookup loads it), and a
// context created after a device reset gets its own address instead of a
// stale one.
int ns_static_scratch(void** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_ns_static_scratch);
  if (e != cudaSuccess || !p)
    return fail(GPT_ECUDA, std::string("cudaGetSymbolAddress of the static scratch: ") + cudaGetErrorString(e));
  *out = p;
  return GPT_OK;
}

}  // namespace

int gpt_op_newton_schulz_noalloc(const float* G, float* X, int batch, int rows, int cols, int tf32_steps,
                                 void* stream) {
  if (batch < 1 || rows < 8 || cols < 8) return fail(GPT_EINVAL, "bad matrix shape");
  const long long n = 1ll * batch * rows * cols;
  if (n > kNsStaticMaxElems || batch > kNsStaticMaxBatch)
    return fail(GPT_EINVAL, "gpt_op_newton_schulz_noalloc accepts at most 262144 elements (batch * rows * cols) "
                            "and batch <= 64; use gpt_op_newton_schulz with caller scratch for larger inputs");
  if (gpt_op_newton_schulz_scratch(batch, rows, cols) > kNsStaticBytes)
    return fail(GPT_EINVAL, "input needs more scratch than the static array holds");
  void* scratch = nullptr;
  int rc = ns_static_scratch(&scratch);
  if (rc) return rc;
  // The same computation as gpt_op_newton_schulz on the static array.  It
  // clears the output before use; every scratch region is written before it
  // is read, so leftovers of an earlier call cannot leak into this one.
  // Expired device waits are latched in the op-level error word
  // (gpt_op_check).
  return gpt_op_newton_schulz(G, X, batch, rows, cols, tf32_steps, scratch, stream);
}

}  // extern "C"
