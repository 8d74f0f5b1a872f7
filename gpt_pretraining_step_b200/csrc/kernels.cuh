// Launchers of the bandwidth-bound kernels (internal to the library).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gpt {

using bf16 = __nv_bfloat16;

// (cos, sin) of t * 10000^(-2i/128) for t < T, i < 64, evaluated in fp64.
void launch_rope_table(float2* tab, int T, cudaStream_t s);

// x[m, :] = wte[tok[m], :] (bf16 weights into the fp32 residual stream).
void launch_embed_fwd(const int* tok, const bf16* wte, float* x, int M, int d, int V, int* err,
                      cudaStream_t s);

// fp8 scale words: a tensor's amax is kept in kAmaxSlots words (zeroed before
// its producer runs) that the producer raises with atomicMax on the bits of
// max |bf16 output|; the quantiser takes the max over them.
constexpr int kAmaxSlots = 32;

// y = x / sqrt(mean(x^2) + 1e-6) per row (bf16 out), rstd saved; d a multiple
// of 128, <= 2048; amax: optional scale words of y.
void launch_rmsnorm_fwd(const float* x, bf16* y, float* rstd, int M, int d, cudaStream_t s,
                        unsigned int* amax = nullptr);

// dx (+)= rstd * (dy - y * mean(dy * y)); also writes dx in bf16 (amax:
// optional scale words of that copy).
void launch_rmsnorm_bwd(const float* dy, const bf16* y, const float* rstd, float* dx, bf16* dx_bf16,
                        int M, int d, bool accumulate, cudaStream_t s, unsigned int* amax = nullptr);

// Per-head QK-norm and RoPE backward plus the v copy, into dqkv [M, d + 2
// Hkv 128] (dq is the fp32 attention-backward accumulator, dk and dv bf16,
// kv head j of batch b at head row b*H + j; Hkv 0 = H).  With dk null only
// the q columns are written (the attention backward wrote the k and v ones).
void launch_qk_bwd(const float* dq, const bf16* dk, const bf16* dv, const bf16* qn, const bf16* kn,
                   const float* rq, const float* rk, const float2* rope, bf16* dqkv, int B, int T, int H,
                   cudaStream_t s, int Hkv = 0, unsigned int* amax = nullptr);

// Per row: lse from the (max, sumexp) tile partials, row loss = lse - z[target],
// and z <- (softmax(z) - onehot(target)) * inv_count in place.
void launch_ce_finish(bf16* z, const float2* stats, const float* zt, const int* tgt, float* row_loss,
                      int rows, int V, int tiles_n, float inv_count, cudaStream_t s);

// loss = sum(row_loss) * scale, deterministic single-block reduction.
void launch_sum_scale(const float* v, int n, float scale, float* out, cudaStream_t s);

// Deterministic embedding gradient: dwte (+)= scatter of dx rows by token
// (d a multiple of 128; the workspace holds the sorted ids and the partial
// sums of tokens with many rows).  Three launches per 32768 tokens.
size_t embed_bwd_workspace(int M, int d);
void launch_embed_bwd(const int* tok, const float* dx, float* dwte, int M, int d, int V, void* ws,
                      bool accumulate, cudaStream_t s);

// out (+)= sum over splits of part[s*stride + i], i < n.
void launch_splitk_reduce(const float* part, int splits, long long stride, long long n, float* out,
                          bool accumulate, cudaStream_t s);

// AdamW over n elements; writes the bf16 working copy.
void launch_adamw(float* p, const float* g, float* m, float* v, bf16* pb, long long n, float lr, float b1,
                  float b2, float eps, float wd, float bc1, float bc2, cudaStream_t s);

// Muon: mom = beta * mom + g over a batch of nmat matrices of n elements each,
// then inv_norm[z] = 1 / (||mom[z]||_F + eps) (deterministic two-level sum).
size_t muon_norm_workspace(int nmat);
void launch_muon_momentum(float* mom, const float* g, long long n, int nmat, float beta, float eps,
                          float* inv_norm, void* ws, cudaStream_t s);

// X[z] = mom[z] * inv_norm[z], stored [r][c] (transpose: mom is [c][r]); bf16 or fp32 out.
// X = mom / ||mom|| per matrix (rows x cols as stored) into `same` (same
// layout) and/or `trans` (transposed), both of element size out_es (2: bf16,
// 4: fp32), and optionally fp16 copies same16 / trans16; null outputs are skipped.
void launch_muon_make_x(const float* mom, const float* inv_norm, void* same, void* trans, int out_es, int nmat,
                        int rows, int cols, cudaStream_t s, __half* same16 = nullptr, __half* trans16 = nullptr);

// W[z] = W[z] (1 - lr wd) - lr * scale * diag(rowf[z]) X[z] (X is [r][c]; W is
// [c][r] when transpose; rowf null = no row factor).
void launch_muon_apply(float* W, bf16* Wb, const void* X, int x_es, int nmat, int r, int c, bool transpose,
                       float lr, float wd, float scale, cudaStream_t s, const float* rowf = nullptr);

// NorMuon row factors of nmat orthogonalised updates X[z] ([r][c], r <= c,
// element size x_es): updates the second-moment EMA V[z] (r floats each) and
// leaves the factor of row i of X[z] in ws[z r + i] (ws: nmat * r floats).
void launch_normuon_factor(const void* X, int x_es, int nmat, int r, int c, float* V, float beta2, float* ws,
                           cudaStream_t s);

// Residual extras (per-layer residual / x0 scales, backout, smear); lam holds
// (resid[0..L), x0[0..L), backout, smear scale, smear gate weights[24]), n is
// the element count (multiple of 4).
void launch_resid_fwd(float* x, float* x_in, float* x0, const float* lam, int l, int L, long long n, bool first,
                      cudaStream_t s);
void launch_backout_fwd(float* x, const float* x_mid, const float* lam, int L, long long n, cudaStream_t s);
// dx holds dL/dx' on entry and dL/dx_in on return (for block 0 plus dx0);
// part: (2L+26) x resid_partial_blocks() floats of partial sums.
void launch_resid_bwd(float* dx, const float* x_in, const float* x0, float* dx0, const float* dx_final,
                      const float* lam, int l, int L, long long n, bf16* gout, float* part, bool first, bool last,
                      cudaStream_t s);
void launch_backout_grad_partial(const float* x_mid, const float* dx_final, int L, long long n, float* part,
                                 cudaStream_t s);
void launch_scalar_grad_finish(const float* part, int L, float* grad, bool accumulate, cudaStream_t s);
// Smear: x = e + lam_s sigmoid(w . e[:, :24]) e(previous position); sig [M]
// kept for the backward, which writes de = dL/de and the partial sums of the
// smear scalars' gradients.
void launch_smear_fwd(const float* e, float* x, float* sig, const float* lam, int L, int T, int M, int d,
                      cudaStream_t s);
void launch_smear_bwd(const float* g, const float* e, const float* sig, const float* lam, float* de, float* part,
                      int L, int T, int M, int d, cudaStream_t s);
int resid_partial_blocks();

// Value embeddings: v[t, h] += 3 sigmoid(xn1[t, :C] . wg[:, h]) ve[tok[t], h]
// for the Hkv kv heads (v [B, H, T, 128] bf16 with kv head h at head row
// b*H + h, xn1 [M, 128 H], ve the bf16 [V, 128 Hkv] table, wg [C, Hkv]); the
// backward writes dve (fp32 [M, 128 Hkv], to be scattered into the table's
// gradient) and dz [M, Hkv]; the gate gradient (C * Hkv <= 1024, the H
// argument of launch_ve_gate_grad / launch_ve_dxn is Hkv) and the xn1
// gradient correction.
void launch_ve_fwd(const bf16* xn1, const int* tok, const bf16* ve, const float* wg, float* sig, bf16* v, int M,
                   int T, int H, int Hkv, int C, int V, cudaStream_t s);
// (dv: the v gradient of token t, kv head h at dv[t * ldv + h * 128 ..])
void launch_ve_bwd(const bf16* dv, long long ldv, const int* tok, const bf16* ve, const float* sig, float* dve,
                   float* dz, int M, int Hkv, int V, cudaStream_t s);
void launch_ve_gate_grad(const bf16* xn1, const float* dz, float* part, float* grad, int M, int d, int H, int C,
                         bool accumulate, cudaStream_t s);
void launch_ve_dxn(float* dxn, const float* dz, const float* wg, int M, int d, int H, int C, cudaStream_t s);

// Per-tensor e4m3 quantisation of nmat matrices of n bf16 values each (z-th at
// x + z n): q = e4m3(x * 448 / amax) with round-to-nearest-even and saturation,
// inv[z] = amax / 448 (1 for an all-zero matrix).  amax_bits: nmat words of scratch.
void launch_quantize_e4m3(const bf16* x, long long n, int nmat, unsigned int* amax_bits, uint8_t* q, float* inv,
                          cudaStream_t s);

// fp8 with precomputed scale words: the amax of x (n bf16 values) into slot 0
// of `slots` (for a tensor whose producer does not keep it), and the e4m3
// quantisation of x with the max over the kAmaxSlots words.
void launch_amax_slots(const bf16* x, long long n, unsigned int* slots, cudaStream_t s);
void launch_quantize_e4m3_slots(const bf16* x, long long n, const unsigned int* slots, uint8_t* q, float* inv,
                                cudaStream_t s);

// dst = bf16(src), n elements.
void launch_cast_bf16(const float* src, bf16* dst, long long n, cudaStream_t s);

}  // namespace gpt
