// Causal flash attention, forward and backward, head_dim 128, bf16 operands
// with fp32 softmax and accumulation (online softmax; the forward saves the
// row log-sum-exp, the backward recomputes P from it).  Optional sliding
// window (query t sees keys t - window .. t) and grouped kv heads (query head
// h reads kv head h / (H / Hkv)), the two attention variants of "¿Cómo
// Entrenar Tu Propio ChatGPT por $50?", section "1. Modelo GPT".
//
// Layouts: q is [B, H, T, 128], k, v, dk, dv are [B, Hkv, T, 128]; the forward output O and the
// incoming gradient dO are token-major [B, T, H, 128] (the rows of the
// projection GEMMs); dq is accumulated in fp32 [B, H, T, 128]; lse and
// D = rowsum(dO * O) are [B, H, T].
//
// Both directions run on the 5th-generation tensor cores (tcgen05.mma with
// TMEM accumulators), fed by TMA; softmax work runs in dedicated warps that
// exchange tiles with the MMA issuer through mbarriers.
#include <algorithm>
#include <type_traits>

#include "attention.cuh"
#include "common.cuh"
#include "gemm.h"

namespace gpt {

namespace {

constexpr int HD = 128;

// ------------------------------------------------- forward on tcgen05 / TMEM
//
// Persistent: one CTA per SM takes work items, a pair of 128-query tiles
// (A = 2p, B = 2p + 1) of one batch*head, until none are left; the pair
// shares every K and V block it loads.  Items are numbered head-major, the
// longest pair of a head first, so the CTAs running at one time share the
// K/V of a few heads in L2; a scheduler word in device memory hands them out
// in that order (an atomic counter, zeroed before the launch), and with no
// word each CTA takes every gridDim.x-th item.  The next item's Q loads and
// first S = Q K^T run while the softmax warps finish the previous item, so
// the per-item load and pipeline-fill latency is hidden.
// 384 threads in three warp groups; the first (TMA, MMA and two idle warps)
// gives registers to the two softmax groups (setmaxnreg 56 / 224 / 224, which
// adds up to the 168 per thread the block is launched with), so each softmax
// thread keeps its whole S row in registers.
//   warp 0      TMA: takes the items and publishes their numbers in a shared
//               ring, loads Q_A and Q_B of each (once every warp has read the
//               item number and the previous Q is no longer read), K_j and
//               V_j through two-slot rings that run on across items
//   warp 1      TMEM owner and MMA issuer.  TMEM columns: S_A [0,128),
//               S_B [128,256), O_A [256,384), O_B [384,512).  Per key block
//               j: O_A += P_A V_j and O_B += P_B V_j, with P read from TMEM
//               (the softmax warps write it as packed bf16 over the first 64
//               columns of S), then S_A = Q_A K_{j+1}^T once O_A's product
//               has read P_A, and then the same for B; the tensor cores thus
//               work on one tile while the other tile's softmax runs.
//   warps 4..7  softmax of tile A, warps 8..11 of tile B, one query row (TMEM
//               lane) per thread: the block max from a first pass over the S
//               row, exp2 into bf16 P (three of every eight exponentials by a
//               polynomial on the FMA pipe), the row sum; after the last
//               block, O / l and the log-sum-exp.
// The reference max of a row only moves when the block max exceeds it by
// more than 8 (log2 units), so P stays below 2^8; when it moves, the warp
// rescales its rows of O in TMEM (the previous P V has completed by then:
// S of this block was issued after it).

// Exponentials per group of 8 scores evaluated on the MUFU unit (the rest by
// the polynomial on the FMA pipe): forward, alternating between two values
// over consecutive groups; backward, one value.  Even numbers (pairs).
#ifndef GPT_FWD_MUFU_EVEN
#define GPT_FWD_MUFU_EVEN 8
#endif
#ifndef GPT_FWD_MUFU_ODD
#define GPT_FWD_MUFU_ODD 8
#endif
#ifndef GPT_BWD_MUFU
#define GPT_BWD_MUFU 8
#endif

constexpr int TF_TILE = 16384;                // one [128 rows][128 B] swizzled tile
constexpr int TF_BUF = 2 * TF_TILE;           // 128 x 128 bf16 as two 64-column tiles
constexpr int TF_SMEM = 6 * TF_BUF + 256;
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

// Item n: batch*head bh and the pair's first query tile, key blocks j0 ..
// (causal end), per tile counts nkvA, nkvB (0: tile B past the sequence).
struct FwdItem {
  int bh, bkv, qtA, j0, nkvA, nkvB, nkv;
  bool hasB;
};

__device__ __forceinline__ FwdItem fwd_item(int n, int nq, int H, int Hkv, int kvs, int wl) {
  FwdItem it;
  const int npairs = (nq + 1) / 2;
  it.bh = n / npairs;
  const int pair = npairs - 1 - (n - it.bh * npairs);
  // k/v row of this query head's kv head: batch rows of kvs heads each
  it.bkv = (it.bh / H) * kvs + (it.bh - (it.bh / H) * H) / (H / Hkv);
  it.qtA = 2 * pair;
  it.hasB = it.qtA + 1 < nq;
  // both tiles start at the first key block any row of tile A sees; rows for
  // which a block lies wholly outside their window see only masked scores
  it.j0 = max(0, it.qtA * 128 - wl) / 128;
  it.nkvA = it.qtA + 1 - it.j0;
  it.nkvB = it.hasB ? it.qtA + 2 - it.j0 : 0;
  it.nkv = it.hasB ? it.nkvB : it.nkvA;
  return it;
}

// S row of query row 32 Q + lane of a causal diagonal block: keys 32 Q + lane
// + 1 .. 127 become -inf (the keys of chunk Q above the lane, then every
// later chunk); Q is the warp's TMEM lane quarter, so no branch diverges.
template <int Q>
__device__ __forceinline__ void causal_mask_row(uint32_t (&sr)[128], int lane) {
#pragma unroll
  for (int k = 0; k < 32; ++k)
    if (k > lane) sr[32 * Q + k] = __float_as_uint(-INFINITY);
#pragma unroll
  for (int k = 32 * (Q + 1); k < 128; ++k) sr[k] = __float_as_uint(-INFINITY);
}

template <bool kFine>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, bf16* __restrict__ o, float* __restrict__ lse,
                       int H, int Hkv, int kvs, int T, int wl, float scale_log2, int n_items, int* sched,
                       int* err, long long wait_cycles) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the 128-byte-swizzled tiles need a 1024-byte-aligned base, which the
  // dynamic shared memory window provides; refuse to run otherwise
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0 && err) atomicOr(err, ERRF_SHAPE);
    return;
  }
  uint8_t* sm = smem_raw;
  uint8_t* sQ = sm;                  // two tiles: A, B
  uint8_t* sK = sm + 2 * TF_BUF;     // two slots
  uint8_t* sV = sm + 4 * TF_BUF;     // two slots
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + 6 * TF_BUF);
  uint64_t* q_full = bars + 0;    // Q of item n landed (or the end marker)
  uint64_t* q_empty = bars + 1;   // item n's S products done and every warp has its number
  uint64_t* k_full = bars + 2;    // [2]
  uint64_t* k_empty = bars + 4;   // [2]
  uint64_t* v_full = bars + 6;    // [2]
  uint64_t* v_empty = bars + 8;   // [2]
  uint64_t* s_full = bars + 10;   // [2] per tile: S of a block in TMEM
  uint64_t* p_full = bars + 12;   // [2] per tile: P of a block in TMEM
  uint64_t* pv_done = bars + 14;  // [2] per tile: P V of a block complete
  uint64_t* drain = bars + 16;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 17);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* item_ring = reinterpret_cast<volatile int*>(tmem_holder + 2);   // [4]

  const int warp = warp_id(), lane = lane_id();
  const int nq = (T + 127) / 128;
  const long long wlim = wait_limit_or_default(wait_cycles);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1 + 8);   // the MMA commit and one arrival per softmax warp
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1); mbar_init(&p_full[i], 128); mbar_init(&pv_done[i], 1);
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

  if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 56;\n" ::: "memory");
  if (warp == 0) {
    if (lane == 0) {
      // -------------------------------------------------------------- TMA
      bool ok = true;
      int g = 0, last_q = -1;   // ring position of the next K/V block; last item whose Q was loaded
      for (int n = 0;; ++n) {
        // the previous item's Q is no longer read and every warp has its number
        if (n > 0 && !mbar_wait_t<kFine>(q_empty, (n - 1) & 1, abort_flag, err, wlim)) { ok = false; break; }
        int idx = sched ? atomicAdd(sched, 1) : n * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x);
        if (idx >= n_items) idx = -1;
        item_ring[n & 3] = idx;
        if (idx < 0) {
          mbar_arrive(q_full);   // end marker: releases the ring entry
          break;
        }
        const FwdItem it = fwd_item(idx, nq, H, Hkv, kvs, wl);
        mbar_arrive_expect_tx(q_full, it.hasB ? 2 * TF_BUF : TF_BUF);
        tma_load_3d(sQ, &tq, q_full, 0, it.qtA * 128, it.bh);
        tma_load_3d(sQ + TF_TILE, &tq, q_full, 64, it.qtA * 128, it.bh);
        if (it.hasB) {
          tma_load_3d(sQ + TF_BUF, &tq, q_full, 0, it.qtA * 128 + 128, it.bh);
          tma_load_3d(sQ + TF_BUF + TF_TILE, &tq, q_full, 64, it.qtA * 128 + 128, it.bh);
        }
        last_q = n;
        for (int j = 0; j < it.nkv; ++j) {
          const int s = g & 1;
          const uint32_t par = (g >> 1) & 1;
          const int kc = (it.j0 + j) * 128;
          if (!mbar_wait_t<kFine>(&k_empty[s], par ^ 1u, abort_flag, err, wlim)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[s], TF_BUF);
          tma_load_3d(sK + s * TF_BUF, &tk, &k_full[s], 0, kc, it.bkv);
          tma_load_3d(sK + s * TF_BUF + TF_TILE, &tk, &k_full[s], 64, kc, it.bkv);
          if (!mbar_wait_t<kFine>(&v_empty[s], par ^ 1u, abort_flag, err, wlim)) {
            // K of this block is in flight: count it, V is not
            for (uint32_t i = 0; i < (1u << 20) && !mbar_try_wait(&k_full[s], par); ++i) {}
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&v_full[s], TF_BUF);
          tma_load_3d(sV + s * TF_BUF, &tv, &v_full[s], 0, kc, it.bkv);
          tma_load_3d(sV + s * TF_BUF + TF_TILE, &tv, &v_full[s], 64, kc, it.bkv);
          ++g;
        }
        if (!ok) break;
      }
      if (!ok) {
        // let the copies already started land before the CTA exits
        if (last_q >= 0)
          for (uint32_t i = 0; i < (1u << 20) && !mbar_try_wait(q_full, last_q & 1); ++i) {}
        for (int x = (g > 2 ? g - 2 : 0); x < g; ++x) {
          for (uint32_t i = 0; i < (1u << 20) && !mbar_try_wait(&k_full[x & 1], (x >> 1) & 1); ++i) {}
          for (uint32_t i = 0; i < (1u << 20) && !mbar_try_wait(&v_full[x & 1], (x >> 1) & 1); ++i) {}
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // -------------------------------------------------------------- MMA
      constexpr uint32_t IDESC_S = make_idesc(1, 128, false, false);
      constexpr uint32_t IDESC_O = make_idesc(1, 128, false, true);
      // The descriptors of a product are its first one plus the byte offset / 16
      // (the start address field); the empty asm keeps the compiler from
      // hoisting every descriptor of the kernel into registers.
      // S_t = Q_t K^T (K in ring slot ks) into TMEM columns 128 t
      auto issue_s = [&](int t, int ks) {
        uint64_t dq = smem_desc_sw128(smem_u32(sQ + t * TF_BUF), 16, 1024);
        uint64_t dk = smem_desc_sw128(smem_u32(sK + ks * TF_BUF), 16, 1024);
        asm volatile("" : "+l"(dq), "+l"(dk));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off16 = ((kk >> 2) * TF_TILE + (kk & 3) * 32) >> 4;
          umma_f16(tmem + t * 128, dq + off16, dk + off16, IDESC_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[t]);
      };
      // O_t (+)= P_t V (V in ring slot vs), P_t from TMEM (16 keys = 8 packed columns per step)
      auto issue_pv = [&](int t, int vs, bool acc) {
        uint64_t dv = smem_desc_sw128(smem_u32(sV + vs * TF_BUF), TF_TILE, 1024);
        asm volatile("" : "+l"(dv));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_f16_tmem_a(tmem + 256 + t * 128, tmem + t * 128 + kk * 8, dv + ((kk * 2048) >> 4), IDESC_O,
                          (acc || kk > 0) ? 1u : 0u);
        umma_commit(&pv_done[t]);
      };
      bool ok = true;
      int g0 = 0;                  // ring position of the item's first key block
      uint32_t npv[2] = {0u, 0u};  // P V products issued per tile so far
      for (int n = 0; ok; ++n) {
        if (!mbar_wait_t<kFine>(q_full, n & 1, abort_flag, err, wlim)) { ok = false; break; }
        const int idx = item_ring[n & 3];
        if (idx < 0) break;
        const FwdItem it = fwd_item(idx, nq, H, Hkv, kvs, wl);
        // S of the first block on both tiles, each once its previous P V (which
        // reads P from the same columns) has completed
        if (!mbar_wait_t<kFine>(&k_full[g0 & 1], (g0 >> 1) & 1, abort_flag, err, wlim)) { ok = false; break; }
        for (int t = 0; t < 2 && ok; ++t) {
          if (t == 1 && !it.hasB) break;
          if (npv[t] > 0 && !mbar_wait_t<kFine>(&pv_done[t], (npv[t] - 1) & 1, abort_flag, err, wlim)) { ok = false; break; }
          tc_fence_after();
          issue_s(t, g0 & 1);
        }
        if (!ok) break;
        if (it.nkv == 1) umma_commit(q_empty);   // the item's last S
        umma_commit(&k_empty[g0 & 1]);
        for (int j = 0; j < it.nkv && ok; ++j) {
          const int gj = g0 + j;
          const int s = gj & 1;
          const int s1 = (gj + 1) & 1;
          if (!mbar_wait_t<kFine>(&v_full[s], (gj >> 1) & 1, abort_flag, err, wlim)) { ok = false; break; }
          if (j + 1 < it.nkv && !mbar_wait_t<kFine>(&k_full[s1], ((gj + 1) >> 1) & 1, abort_flag, err, wlim)) { ok = false; break; }
          // per tile: O += P V_j, then S of the next block over P once that product
          // has read it (tile B's softmax trails tile A's, so A goes first)
          for (int t = 0; t < 2; ++t) {
            const int nkv_t = t ? it.nkvB : it.nkvA;
            if (j >= nkv_t) continue;
            if (!mbar_wait_t<kFine>(&p_full[t], npv[t] & 1, abort_flag, err, wlim)) { ok = false; break; }
            tc_fence_after();
            issue_pv(t, s, j > 0);
            ++npv[t];
            if (j + 1 < nkv_t) {
              if (!mbar_wait_t<kFine>(&pv_done[t], (npv[t] - 1) & 1, abort_flag, err, wlim)) { ok = false; break; }
              tc_fence_after();
              issue_s(t, s1);
              if (j + 1 == it.nkv - 1) umma_commit(q_empty);   // the item's last S
            }
          }
          if (!ok) break;
          umma_commit(&v_empty[s]);
          if (j + 1 < it.nkv) umma_commit(&k_empty[s1]);
        }
        g0 += it.nkv;
      }
      umma_commit(drain);
      for (uint32_t i = 0; i < (1u << 22) && !mbar_try_wait(drain, 0); ++i) {}
    }
  } else if (warp >= 4) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 224;\n" ::: "memory");
    // ---------------------------------------------------------- softmax
    const int tile = (warp - 4) >> 2;           // 0: A, 1: B
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_base + tile * 128;
    const uint32_t t_o = tmem + lane_base + 256 + tile * 128;
    const uint64_t sl2 = f2_pack(scale_log2, scale_log2);
    bool ok = true;
    uint32_t nblk = 0;   // S blocks consumed on this tile so far
    auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
      const bool got = mbar_wait_t<kFine>(bar, par, abort_flag, err, wlim);
      __syncwarp();
      return __all_sync(0xffffffffu, got);
    };
    for (int n = 0; ok; ++n) {
      if (!wait_all(q_full, n & 1)) { ok = false; break; }
      const int idx = item_ring[n & 3];
      __syncwarp();
      if (lane == 0) mbar_arrive(q_empty);   // this warp has the item number
      if (idx < 0) break;
      const FwdItem it = fwd_item(idx, nq, H, Hkv, kvs, wl);
      if (tile == 1 && !it.hasB) continue;
      const int qt = it.qtA + tile;
      const int q0 = qt * 128;
      const int q = q0 + r;
      const int nkv_t = tile ? it.nkvB : it.nkvA;
      float m_ref = -INFINITY, l = 0.f;   // reference max (log2 units) and row sum relative to it
      for (int j = 0; j < nkv_t && ok; ++j) {
        if (!wait_all(&s_full[tile], nblk & 1)) { ok = false; break; }
        ++nblk;
        tc_fence_after();
        // the whole S row at once
        uint32_t sr[128];
        {
          uint32_t (&r0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
          uint32_t (&r1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
          uint32_t (&r2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[64]);
          uint32_t (&r3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[96]);
          tmem_load32_async(t_s, r0);
          tmem_load32_async(t_s + 32, r1);
          tmem_load32_async(t_s + 64, r2);
          tmem_load32_async(t_s + 96, r3);
          tmem_wait_ld();
        }
        const int kbase = (it.j0 + j) * 128;
        const bool diag = it.j0 + j == qt, edge = (kbase + 128 > T) || (kbase < q0 + 127 - wl);
        if (diag && !edge) {
          // causal diagonal block: only the keys above the row are masked, so
          // per element in one 32-key chunk, whole chunks beyond it
          switch (quarter) {
            case 0: causal_mask_row<0>(sr, lane); break;
            case 1: causal_mask_row<1>(sr, lane); break;
            case 2: causal_mask_row<2>(sr, lane); break;
            default: causal_mask_row<3>(sr, lane); break;
          }
        } else if (diag || edge) {
          // ragged tail or window edge: masked scores become -inf
#pragma unroll
          for (int k = 0; k < 128; ++k) {
            const int key = kbase + k;
            if (key > q || key >= T || key < q - wl) sr[k] = __float_as_uint(-INFINITY);
          }
        }
        // block max of the raw scores (the scale is positive), eight independent
        // chains of three-input maxima (two new scores per instruction)
        float mx8[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) mx8[t] = fmaxf(__uint_as_float(sr[2 * t]), __uint_as_float(sr[2 * t + 1]));
#pragma unroll
        for (int k = 16; k < 128; k += 16) {
#pragma unroll
          for (int t = 0; t < 8; ++t)
            mx8[t] = fmax3(mx8[t], __uint_as_float(sr[k + 2 * t]), __uint_as_float(sr[k + 2 * t + 1]));
        }
        const float mraw = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
        const float mblk = mraw * scale_log2;
        const bool move = mblk > m_ref + TF_RESCALE;   // true on the first block with a visible key
        const float m_new = move ? mblk : m_ref;
        // 1 when the reference stays, 0 when it leaves -inf; a row that has seen
        // only masked scores (window edge) keeps -inf and offsets by 0 below
        const bool none = m_new == -INFINITY;
        const float factor = none ? 1.f : ex2_approx(m_ref - m_new);
        // O holds the products of blocks < j (S of this block was issued after
        // the last of them completed), so it may be rescaled now
        if (j >= 1 && __any_sync(0xffffffffu, move)) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t ra[32];
            tmem_load32_async(t_o + c * 32, ra);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) ra[k] = __float_as_uint(__uint_as_float(ra[k]) * factor);
            tmem_store32(t_o + c * 32, ra);
          }
        }
        // probabilities relative to the reference (masked scores give 0), row sum,
        // bf16 P over the first 64 columns of S
        const float m_off = none ? 0.f : m_new;
        const uint64_t nb2 = f2_pack(-m_off, -m_off);
        uint64_t rs2 = f2_pack(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[32];
#pragma unroll
          for (int k = 0; k < 64; k += 8) {
            float p[8];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              float x0, x1;
              f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[c * 64 + k + e]), __uint_as_float(sr[c * 64 + k + e + 1])),
                               sl2, nb2),
                        x0, x1);
              if (e < ((k & 8) ? GPT_FWD_MUFU_ODD : GPT_FWD_MUFU_EVEN)) {
                p[e] = ex2_approx(x0);
                p[e + 1] = ex2_approx(x1);
              } else {
                f2_unpack(f2_exp2_poly(f2_pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f))), p[e], p[e + 1]);
              }
            }
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              rs2 = f2_add(rs2, f2_pack(p[e], p[e + 1]));
              pk[(k + e) >> 1] = pack_bf16x2(p[e], p[e + 1]);
            }
          }
          tmem_store32(t_s + c * 32, pk);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        mbar_arrive(&p_full[tile]);
        float rs0, rs1;
        f2_unpack(rs2, rs0, rs1);
        l = l * factor + (rs0 + rs1);
        m_ref = m_new;
      }
      // epilogue: O / l once the last P V has landed
      if (ok) ok = wait_all(&pv_done[tile], (nblk - 1) & 1);
      if (ok) {
        tc_fence_after();
        const int b = it.bh / H, h = it.bh - (it.bh / H) * H;
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
        if (q < T) lse[static_cast<long long>(it.bh) * T + q] = (m_ref + log2f(l)) * 0.69314718055994531f;
        // O of this tile has been read: the next item's first P V may overwrite it
        tc_fence_before();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------ backward on tcgen05 / TMEM
//
// Persistent: one CTA per SM takes work units, key blocks j and nkb - 1 - j
// of one batch*kv head (equal work under the causal mask), until none are
// left.  Units are numbered head-major, the longest of a head first, so the
// CTAs running at one time read the Q and dO of a few heads from L2; a
// scheduler word hands them out in that order (an atomic counter, zeroed
// before the launch), else each CTA takes every gridDim.x-th unit.  Each
// key block of a unit is one item.  The TMA warp publishes each item number in a shared
// ring with the K/V barrier; every other warp acknowledges it on the barrier
// that frees K/V, so no barrier phase can run two ahead of a waiter.  For each key block
// the CTA loops over the query heads of the kv group and, for each, the query
// blocks i >= j that see those keys (up to the last one inside the window);
// dK and dV add up over the whole loop.  The barrier phases run on across
// key blocks, so the next block's Q and dO loads start while the previous
// block's last products run, and its K and V load as soon as those are done.
// 512 threads in four warp groups (the first and the last give registers to
// the softmax groups: 72 / 168 / 168 / 96 per thread):
//   warp 0      TMA: Q_i through a two-slot ring; dO_i; K_j and V_j once per
//               key block (after the previous block's last product).
//   warp 1      TMEM owner and MMA issuer.  TMEM columns: [0,128) S^T_i and
//               dQ_i in turn; [128,256) dP^T_i, then P^T_i as packed bf16
//               (queries 0..63 at 128.., 64..127 at 192..); [256,384) dV;
//               [384,512) dK.  Per query block i:
//                 dV += P^T dO   once P_i is in TMEM (A from TMEM; then
//                                dO_{i+1} may load)
//                 dK += dS^T Q   once dS_i is in shared memory (then Q_{i+2}
//                                may load)
//                 dQ = dS K into [0,128) once S^T_{i+1} has been read (A is
//                                dS^T in shared memory read MN-major, so
//                                the queries land in the TMEM lanes)
//                 dP^T_{i+1} = V dO_{i+1}^T into [128,256)
//                 S^T_{i+2} = K Q_{i+2}^T into [0,128) once dQ_i has been read
//   warps 2, 3  idle
//   warps 4..11 softmax, two warps per TMEM lane quarter, each on 64 of the
//               128 query columns of its key rows: when dP^T_i lands, P_i
//               (computed during the previous block) over the dP^T columns the
//               warp has read, then dS'_i = P_i (dP_i - D) to shared memory
//               while dV runs; then S^T_{i+1}
//               and P_{i+1} while the tensor cores run block i's products.
//               1/sqrt(d) of dS = dS' / sqrt(d) is applied to dK and dQ.
//               After a key block's last products they write its dK and dV.
//   warps 12..15 dQ: one warp per TMEM lane quarter (lane = query), each
//               thread staging its query's row of dQ_i, 64 dims at a time, as
//               fp32 [32 queries][32 dims] boxes (eight 16-byte stores per
//               row) in a 32 KB buffer, and adding them into the fp32 dq
//               buffer by TMA reduce-add, so the reduction runs beside the
//               other warps' work.  (Adding each row with 16-byte vector
//               reductions from registers measured 0.925 ms against 0.68 ms
//               at B 16, H 10, T 2048.)

// Row r, query columns 64*half .. 64*half+63 of a [128][128] bf16 tile kept as
// two 64-column halves of [128 rows][128 B] with the 128-byte swizzle (16-byte
// unit u of row r at u ^ (r & 7)); w holds the 64 values as packed pairs.
__device__ __forceinline__ void store_row_units(uint8_t* tile, const uint32_t (&w)[32], int half, int r) {
  uint8_t* row = tile + half * TF_TILE + r * 128;
#pragma unroll
  for (int u = 0; u < 8; ++u)
    *reinterpret_cast<uint4*>(row + ((u ^ (r & 7)) << 4)) = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
}

constexpr int TB_STAGE = 32768;   // dQ staging: 4 warps x two [32 queries][32 dims] fp32 boxes
constexpr int TB_SMEM = 6 * TF_BUF + TB_STAGE + 2048 + 256;

// Query-block loop of key block j: nb query blocks j .. (window end) for each
// of the G query heads of the group.
struct BwdBlock {
  int bkv, kvrow, j, k0, nb, n_it, b, hk, G;   // kvrow: the k/v row (batch rows of kvs heads)
  __device__ __forceinline__ int q_block(int it) const { return j + it % nb; }
  __device__ __forceinline__ int q_head(int it) const { return hk * G + it / nb; }   // within the batch row
};

// Item idx: kv head idx / nq, key block idx mod nq.
__device__ __forceinline__ BwdBlock bwd_block(int idx, int H, int Hkv, int kvs, int nq, int wl) {
  BwdBlock k;
  k.bkv = idx / nq;
  const int j = idx - k.bkv * nq;
  const int bkv = k.bkv;
  k.j = j;
  k.k0 = j * 128;
  k.b = bkv / Hkv;
  k.hk = bkv - k.b * Hkv;
  k.kvrow = k.b * kvs + k.hk;
  k.G = H / Hkv;
  k.nb = min(nq - 1, (k.k0 + 127 + wl) / 128) - j + 1;
  k.n_it = k.G * k.nb;
  return k;
}

template <bool kFine>
__global__ void __launch_bounds__(512, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                       const __grid_constant__ CUtensorMap tdq, const float* __restrict__ lse,
                       const float* __restrict__ Dv, bf16* __restrict__ dk, bf16* __restrict__ dv, int H, int Hkv,
                       int kvs, int T, int wl, float scale, int n_units, int* sched, int* err,
                       long long wait_cycles, const float* __restrict__ rk, const float2* __restrict__ rope,
                       bf16* __restrict__ dqkv) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the 128-byte-swizzled tiles need a 1024-byte-aligned base, which the
  // dynamic shared memory window provides; refuse to run otherwise
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0 && err) atomicOr(err, ERRF_SHAPE);
    return;
  }
  uint8_t* sm = smem_raw;
  uint8_t* sK = sm;
  uint8_t* sV = sm + TF_BUF;
  uint8_t* sQ = sm + 2 * TF_BUF;     // two slots
  uint8_t* sdO = sm + 4 * TF_BUF;
  uint8_t* sdSt = sm + 5 * TF_BUF;
  uint8_t* sStage = sm + 6 * TF_BUF;
  float* lse_s = reinterpret_cast<float*>(sm + 6 * TF_BUF + TB_STAGE);   // [2][128]: -lse * log2(e)
  float* dd_s = lse_s + 256;                                              // [2][128]: -D
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + 6 * TF_BUF + TB_STAGE + 2048);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;    // [2]
  uint64_t* q_empty = bars + 3;   // [2]
  uint64_t* do_full = bars + 5;
  uint64_t* do_empty = bars + 6;  // dV_i complete: dO_i and P_i are no longer read
  uint64_t* s_full = bars + 7;    // S^T_i in TMEM
  uint64_t* s_free = bars + 8;    // S^T_i read by the softmax warps
  uint64_t* dp_full = bars + 9;   // dP^T_i in TMEM
  uint64_t* p_ready = bars + 10;  // P_i in TMEM
  uint64_t* mm_done = bars + 11;  // dV, dK, dQ of block i complete
  uint64_t* dq_free = bars + 12;  // dQ_i read by the dQ warps
  uint64_t* drain = bars + 13;
  uint64_t* ds_ready = bars + 14; // dS_i in shared memory
  uint64_t* kv_empty = bars + 15; // an item's last products complete (K and V free) and every warp has its number
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* item_ring = reinterpret_cast<volatile int*>(tmem_holder + 2);   // [4]

  const int warp = warp_id(), lane = lane_id();
  const int nq = (T + 127) / 128;
  const long long wlim = wait_limit_or_default(wait_cycles);

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1 + 12);   // the MMA commit and one arrival per softmax and dQ warp
    for (int i = 0; i < 2; ++i) { mbar_init(&q_full[i], 1); mbar_init(&q_empty[i], 1); }
    mbar_init(do_full, 1);
    mbar_init(do_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(s_free, 256);
    mbar_init(dp_full, 1);
    mbar_init(p_ready, 256);
    mbar_init(ds_ready, 256);
    mbar_init(mm_done, 1);
    mbar_init(dq_free, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    tma_prefetch_desc(&tdo);
    tma_prefetch_desc(&tdq);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // registers: 72 for the TMA / MMA warp group, 96 for the dQ group, 168 for
  // the two softmax groups (4*72 + 4*96 + 8*168 = 2016 per lane of a warp,
  // within the 16 warps x 128 the block is launched with)
  if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 72;\n" ::: "memory");
  if (warp == 0) {
    if (lane == 0) {
      // -------------------------------------------------------------- TMA
      bool ok = true;
      int g = 0, nblk = 0;          // query blocks and items loaded so far
      int issued_q = 0, issued_do = 0;
      auto load_q_do = [&](const BwdBlock& kb, int it) -> bool {
        const int i = kb.q_block(it), h = kb.q_head(it), bh = kb.b * H + h;
        const int s = g & 1;
        if (!mbar_wait_t<kFine>(&q_empty[s], ((g >> 1) & 1) ^ 1u, abort_flag, err, wlim)) return false;
        mbar_arrive_expect_tx(&q_full[s], TF_BUF);
        tma_load_3d(sQ + s * TF_BUF, &tq, &q_full[s], 0, i * 128, bh);
        tma_load_3d(sQ + s * TF_BUF + TF_TILE, &tq, &q_full[s], 64, i * 128, bh);
        ++issued_q;
        if (!mbar_wait_t<kFine>(do_empty, (g & 1) ^ 1u, abort_flag, err, wlim)) return false;
        mbar_arrive_expect_tx(do_full, TF_BUF);
        tma_load_4d(sdO, &tdo, do_full, 0, h, i * 128, kb.b);
        tma_load_4d(sdO + TF_TILE, &tdo, do_full, 64, h, i * 128, kb.b);
        ++issued_do;
        ++g;
        return true;
      };
      // work is handed out in units of two key blocks, u and nkb - 1 - u of one
      // kv head (the same work under the causal mask), longest unit of a head
      // first; the unit's blocks become consecutive items
      const int nu = (nq + 1) / 2;
      int pending = -1, taken = 0;
      for (int n = 0; ok; ++n) {
        int idx = pending;
        pending = -1;
        if (idx < 0) {
          const int unit = sched ? atomicAdd(sched, 1) : taken * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x);
          ++taken;
          if (unit < n_units) {
            const int bkv = unit / nu, uu = nu - 1 - (unit - bkv * nu);
            idx = bkv * nq + uu;
            if (nq - 1 - uu != uu) pending = bkv * nq + nq - 1 - uu;
          }
        }
        item_ring[n & 3] = idx;
        if (idx < 0) {
          // end marker, once every warp has the previous item's number
          if (n > 0 && !mbar_wait_t<kFine>(kv_empty, (n - 1) & 1, abort_flag, err, wlim)) { ok = false; break; }
          mbar_arrive(kv_full);
          break;
        }
        const BwdBlock kb = bwd_block(idx, H, Hkv, kvs, nq, wl);
        // the first query block's Q and dO may load while the previous item
        // finishes; K and V (which publish the item number) once its last
        // products are done
        if (!load_q_do(kb, 0)) { ok = false; break; }
        if (n > 0 && !mbar_wait_t<kFine>(kv_empty, (n - 1) & 1, abort_flag, err, wlim)) { ok = false; break; }
        mbar_arrive_expect_tx(kv_full, 2 * TF_BUF);
        tma_load_3d(sK, &tk, kv_full, 0, kb.k0, kb.kvrow);
        tma_load_3d(sK + TF_TILE, &tk, kv_full, 64, kb.k0, kb.kvrow);
        tma_load_3d(sV, &tv, kv_full, 0, kb.k0, kb.kvrow);
        tma_load_3d(sV + TF_TILE, &tv, kv_full, 64, kb.k0, kb.kvrow);
        ++nblk;
        for (int it = 1; it < kb.n_it; ++it)
          if (!load_q_do(kb, it)) { ok = false; break; }
      }
      if (!ok) {
        // let the copies already started land before the CTA exits
        if (nblk > 0)
          for (uint32_t x = 0; x < (1u << 20) && !mbar_try_wait(kv_full, (nblk - 1) & 1); ++x) {}
        for (int it = (issued_q > 2 ? issued_q - 2 : 0); it < issued_q; ++it)
          for (uint32_t x = 0; x < (1u << 20) && !mbar_try_wait(&q_full[it & 1], (it >> 1) & 1); ++x) {}
        if (issued_do > 0)
          for (uint32_t x = 0; x < (1u << 20) && !mbar_try_wait(do_full, (issued_do - 1) & 1); ++x) {}
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // -------------------------------------------------------------- MMA
      constexpr uint32_t IDESC_KK = make_idesc(1, 128, false, false);   // S^T, dP^T
      constexpr uint32_t IDESC_KM = make_idesc(1, 128, false, true);    // dV (A in TMEM), dK
      constexpr uint32_t IDESC_MM = make_idesc(1, 128, true, true);     // dQ
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV), do_addr = smem_u32(sdO);
      const uint32_t dst_addr = smem_u32(sdSt);
      // X^T = A B^T over the 128 head dims, both operands K-major; the empty
      // asm keeps the descriptors from being hoisted into registers
      auto qk_product = [&](uint32_t d_tmem, uint32_t a_addr, uint32_t b_addr) {
        uint64_t da = smem_desc_sw128(a_addr, 16, 1024), db = smem_desc_sw128(b_addr, 16, 1024);
        asm volatile("" : "+l"(da), "+l"(db));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off16 = ((kk >> 2) * TF_TILE + (kk & 3) * 32) >> 4;
          umma_f16(d_tmem, da + off16, db + off16, IDESC_KK, kk > 0 ? 1u : 0u);
        }
      };
      bool ok = true;
      int g0 = 0;   // query blocks done so far
      for (int n = 0; ok; ++n) {
        if (!mbar_wait_t<kFine>(kv_full, n & 1, abort_flag, err, wlim)) { ok = false; break; }
        const int idx = item_ring[n & 3];
        if (idx < 0) break;
        {
          const BwdBlock kb = bwd_block(idx, H, Hkv, kvs, nq, wl);
          const int n_it = kb.n_it;
          // S^T of the first query block goes where the previous key block's
          // last dQ was (wait until the dQ warps have read it), dP^T where
          // its last P was (wait until that dV is done)
          ok = mbar_wait_t<kFine>(&q_full[g0 & 1], (g0 >> 1) & 1, abort_flag, err, wlim) &&
               (g0 == 0 || mbar_wait_t<kFine>(dq_free, (g0 - 1) & 1, abort_flag, err, wlim));
          if (!ok) break;
          tc_fence_after();
          qk_product(tmem, k_addr, smem_u32(sQ + (g0 & 1) * TF_BUF));   // S^T of the first block
          umma_commit(s_full);
          ok = mbar_wait_t<kFine>(do_full, g0 & 1, abort_flag, err, wlim) &&
               (g0 == 0 || mbar_wait_t<kFine>(do_empty, (g0 - 1) & 1, abort_flag, err, wlim));
          if (!ok) break;
          tc_fence_after();
          qk_product(tmem + 128, v_addr, do_addr);   // dP^T of the first block
          umma_commit(dp_full);
          if (n_it > 1) {
            ok = mbar_wait_t<kFine>(s_free, g0 & 1, abort_flag, err, wlim) &&
                 mbar_wait_t<kFine>(&q_full[(g0 + 1) & 1], ((g0 + 1) >> 1) & 1, abort_flag, err, wlim);
            if (!ok) break;
            tc_fence_after();
            qk_product(tmem, k_addr, smem_u32(sQ + ((g0 + 1) & 1) * TF_BUF));   // S^T of the second block
            umma_commit(s_full);
          }
          for (int it = 0; it < n_it && ok; ++it) {
            const int gi = g0 + it;
            const int s = gi & 1;
            if (!mbar_wait_t<kFine>(p_ready, gi & 1, abort_flag, err, wlim)) { ok = false; break; }
            tc_fence_after();
            const uint32_t q_addr = smem_u32(sQ + s * TF_BUF);
            // dV += P^T dO: A = P^T from TMEM, 16 queries = 8 packed columns per
            // step; queries 0..63 at columns 128.., 64..127 at columns 192..
            {
              uint64_t ddo = smem_desc_sw128(do_addr, TF_TILE, 1024);
              asm volatile("" : "+l"(ddo));
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                umma_f16_tmem_a(tmem + 256, tmem + 128 + (kk >> 2) * 64 + (kk & 3) * 8, ddo + ((kk * 2048) >> 4),
                                IDESC_KM, (it > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(do_empty);
            // dK and dQ once dS_i is in shared memory (the softmax warps compute it
            // while dV runs)
            if (!mbar_wait_t<kFine>(ds_ready, gi & 1, abort_flag, err, wlim)) { ok = false; break; }
            tc_fence_after();
            {
              uint64_t dsa = smem_desc_sw128(dst_addr, 16, 1024), dqb = smem_desc_sw128(q_addr, TF_TILE, 1024);
              asm volatile("" : "+l"(dsa), "+l"(dqb));
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint32_t aoff16 = ((kk >> 2) * TF_TILE + (kk & 3) * 32) >> 4;   // K-major A: 16 queries per step
                const uint32_t boff16 = (kk * 2048) >> 4;                            // MN-major B: 16 query rows per step
                umma_f16(tmem + 384, dsa + aoff16, dqb + boff16, IDESC_KM, (it > 0 || kk > 0) ? 1u : 0u);
              }
            }
            umma_commit(&q_empty[s]);
            // dQ_i goes to [0,128), which holds S^T_{i+1} (wait until the softmax
            // warps have read it) or, for the last block, dQ_{i-1} (wait until
            // the dQ warps have read it)
            if (it + 1 < n_it) {
              if (!mbar_wait_t<kFine>(s_free, (gi + 1) & 1, abort_flag, err, wlim)) { ok = false; break; }
            } else if (it > 0) {
              if (!mbar_wait_t<kFine>(dq_free, (gi - 1) & 1, abort_flag, err, wlim)) { ok = false; break; }
            }
            tc_fence_after();
            {
              uint64_t dka = smem_desc_sw128(k_addr, TF_TILE, 1024), dsb = smem_desc_sw128(dst_addr, TF_TILE, 1024);
              asm volatile("" : "+l"(dka), "+l"(dsb));
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off16 = (kk * 2048) >> 4;   // 16 keys per step, both operands MN-major
                umma_f16(tmem, dsb + off16, dka + off16, IDESC_MM, kk > 0 ? 1u : 0u);   // dQ = dS K
              }
            }
            umma_commit(mm_done);
            if (it + 1 == n_it) umma_commit(kv_empty);   // K and V of this key block are free
            if (it + 1 < n_it) {
              // dP^T_{i+1} overwrites P^T_i: dV_i must have completed
              if (!mbar_wait_t<kFine>(do_empty, gi & 1, abort_flag, err, wlim) ||
                  !mbar_wait_t<kFine>(do_full, (gi + 1) & 1, abort_flag, err, wlim)) { ok = false; break; }
              tc_fence_after();
              qk_product(tmem + 128, v_addr, do_addr);
              umma_commit(dp_full);
            }
            if (it + 2 < n_it) {
              if (!mbar_wait_t<kFine>(dq_free, gi & 1, abort_flag, err, wlim) ||
                  !mbar_wait_t<kFine>(&q_full[s], ((gi + 2) >> 1) & 1, abort_flag, err, wlim)) { ok = false; break; }
              tc_fence_after();
              qk_product(tmem, k_addr, q_addr);   // S^T_{i+2} (same Q slot as block i)
              umma_commit(s_full);
            }
          }
          g0 += n_it;
        }
      }
      umma_commit(drain);
      for (uint32_t x = 0; x < (1u << 22) && !mbar_try_wait(drain, 0); ++x) {}
    }
  } else if (warp >= 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 96;\n" ::: "memory");
    // ------------------------------------------------------------------ dQ
    const int quarter = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint64_t sc2 = f2_pack(scale, scale);
    bool ok = true;
    // dQ of one query block: this thread's query row (TMEM lane) of 128 dims,
    // staged 64 dims at a time as two [32 queries][32 dims] fp32 boxes (a row
    // is 128 bytes: eight 16-byte stores) and added into dq by TMA reduce-add
    uint8_t* box = sStage + quarter * 8192;
    int g = 0;
    for (int n = 0; ok; ++n) {
      {
        const bool got = mbar_wait_t<kFine>(kv_full, n & 1, abort_flag, err, wlim);
        __syncwarp();
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      }
      const int idx = item_ring[n & 3];
      __syncwarp();
      if (lane == 0) mbar_arrive(kv_empty);   // this warp has the item number
      if (idx < 0) break;
      {
        const BwdBlock kb = bwd_block(idx, H, Hkv, kvs, nq, wl);
        for (int it = 0; it < kb.n_it && ok; ++it, ++g) {
          const int q0 = kb.q_block(it) * 128 + quarter * 32, bh = kb.b * H + kb.q_head(it);
          const bool got = mbar_wait_t<kFine>(mm_done, g & 1, abort_flag, err, wlim);
          __syncwarp();
          if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t va[32], vb[32];
            tmem_load32_async(tmem + lane_base + hh * 64, va);
            tmem_load32_async(tmem + lane_base + hh * 64 + 32, vb);
            tmem_wait_ld();
            if (hh == 1) {
              tc_fence_before();
              mbar_arrive(dq_free);
            }
            if (lane == 0) bulk_wait_read_all();   // the boxes' previous contents have been read
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 64; j += 4) {
              const uint32_t (&v)[32] = j < 32 ? va : vb;
              const int e = j & 31;
              float a0, a1, a2, a3;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), sc2), a0, a1);
              f2_unpack(f2_mul(f2_pack(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])), sc2), a2, a3);
              *reinterpret_cast<float4*>(box + (j >> 5) * 4096 + lane * 128 + ((((e >> 2) ^ lane) & 7) << 4)) =
                  make_float4(a0, a1, a2, a3);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_reduce_add_3d(&tdq, box, hh * 64, q0, bh);
              tma_reduce_add_3d(&tdq, box + 4096, hh * 64 + 32, q0, bh);
              bulk_commit();
            }
          }
        }
      }
    }
    if (lane == 0) bulk_wait_all();
  } else if (warp >= 4) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 168;\n" ::: "memory");
    // ------------------------------------------------------- P, dS, dK, dV
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;        // which 64 query columns of the row
    const int r = quarter * 32 + lane;       // key row (TMEM lane)
    const int t256 = threadIdx.x - 128;      // 0..255
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const float scale_log2 = scale * 1.4426950408889634f;
    const uint64_t sl2 = f2_pack(scale_log2, scale_log2);
    bool ok = true;
    // Named barrier 1 over the 256 softmax threads, which also tells every
    // thread whether any of them failed its wait (so all leave the loop together)
    auto any_fail = [&](bool got) -> bool {
      __syncwarp();
      uint32_t f;
      asm volatile(
          "{\n\t.reg .pred pi, po;\n\tsetp.eq.u32 pi, %1, 0;\n\t"
          "bar.red.or.pred po, 1, 256, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
          : "=r"(f)
          : "r"(got ? 1u : 0u)
          : "memory");
      return f != 0;
    };
    // Every decision to leave a loop is taken by this vote, so the eight
    // warps always meet at the same named barriers: a warp that left on its
    // own would leave the others waiting at the next vote.
    int g0 = 0;
    for (int n = 0; ok; ++n) {
      {
        const bool got = mbar_wait_t<kFine>(kv_full, n & 1, abort_flag, err, wlim);
        if (any_fail(got)) { ok = false; break; }
      }
      const int idx = item_ring[n & 3];
      __syncwarp();
      // this warp has the item number; when dK goes through the QK-norm
      // backward, K stays until the item's epilogue has read its rows
      if (lane == 0 && (idx < 0 || !dqkv)) mbar_arrive(kv_empty);
      if (idx < 0) break;
      {
        const BwdBlock kb = bwd_block(idx, H, Hkv, kvs, nq, wl);
        const int n_it = kb.n_it, k0 = kb.k0, bkv = kb.kvrow;
        const int key = k0 + r;
        const bool key_ok = key < T;
        if (dqkv && key_ok) {
          // the epilogue's rotation table row and inverse RMS, on their way to L2
          asm volatile("prefetch.global.L2 [%0];" ::"l"(rope + static_cast<long long>(key) * 64 + 32 * half));
          asm volatile("prefetch.global.L2 [%0];" ::"l"(rope + static_cast<long long>(key) * 64 + 32 * half + 16));
          asm volatile("prefetch.global.L2 [%0];" ::"l"(rk + (static_cast<long long>(kb.b) * T + key) * H + kb.hk));
        }
        // this thread's share of a query block's -lse (log2 units; -inf past T so
        // P = 0) or -D, fetched a block ahead so the load latency hides
        auto fetch = [&](int it2) -> float {
          const int q0f = kb.q_block(it2) * 128;
          const long long bh = static_cast<long long>(kb.b) * H + kb.q_head(it2);
          if (t256 < 128) {
            const int qq = q0f + t256;
            return qq < T ? __ldg(lse + bh * T + qq) * -1.4426950408889634f : -INFINITY;
          }
          const int qq = q0f + t256 - 128;
          return qq < T ? -__ldg(Dv + bh * T + qq) : 0.f;
        };
        // block it2's values go to buffer (g0 + it2) & 1; a barrier publishes them
        auto publish = [&](int it2, float v) {
          float* base = (t256 < 128 ? lse_s : dd_s) + ((g0 + it2) & 1) * 128;
          base[t256 & 127] = v;
        };
        // P of block it2 for this thread's key row and 64 query columns, packed bf16
        uint32_t pk[32];
        auto compute_p = [&](int it2) {
          const bool diag = it2 % kb.nb == 0;
          const int q0 = kb.q_block(it2) * 128;
          // causal diagonal block, ragged key block, or a query block whose last
          // rows' windows start past this block's first key
          const bool edge = k0 + 128 > T || q0 + 127 - wl > k0;
          const bool masked = diag || edge;
          const float* nls = lse_s + ((g0 + it2) & 1) * 128;
          uint32_t sa[32], sb[32];
          tmem_load32_async(tmem + lane_base + (2 * half) * 32, sa);
          tmem_load32_async(tmem + lane_base + (2 * half + 1) * 32, sb);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(s_free);   // S^T of this block has been read
          // One 32-query chunk of the row in one of four forms, chosen per
          // chunk by a warp-uniform test: no mask, the causal diagonal's lane
          // mask (queries below the key row), all masked (P = 0), or the general
          // mask (ragged keys, window edge).  A per-element mask inside one loop
          // was if-converted into every block's path and cost more than the
          // exponentials.
          auto run_chunk = [&](auto kCC, auto kMode) {
            constexpr int cc = decltype(kCC)::value, mode = decltype(kMode)::value;
            const int c = 2 * half + cc;
            const uint32_t (&sr)[32] = cc == 0 ? sa : sb;
            if constexpr (mode == 3) {
#pragma unroll
              for (int x = 0; x < 16; ++x) pk[16 * cc + x] = 0u;
            } else {
#pragma unroll
              for (int kq = 0; kq < 32; kq += 8) {
                const float4 la = *reinterpret_cast<const float4*>(nls + c * 32 + kq);
                const float4 lb = *reinterpret_cast<const float4*>(nls + c * 32 + kq + 4);
                const float nl[8] = {la.x, la.y, la.z, la.w, lb.x, lb.y, lb.z, lb.w};   // -lse * log2(e)
                // P = 2^(S * scale * log2(e) - lse * log2(e)): GPT_BWD_MUFU of every
                // eight on the MUFU unit, the rest by the polynomial on the FMA pipe
                float p[8];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                  float x0, x1;
                  f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[kq + e]), __uint_as_float(sr[kq + e + 1])), sl2,
                                   f2_pack(nl[e], nl[e + 1])),
                            x0, x1);
                  if (e < GPT_BWD_MUFU) {
                    p[e] = ex2_approx(x0);
                    p[e + 1] = ex2_approx(x1);
                  } else {
                    f2_unpack(f2_exp2_poly(f2_pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f))), p[e], p[e + 1]);
                  }
                }
                if constexpr (mode == 1) {
#pragma unroll
                  for (int e = 0; e < 8; ++e)
                    if (kq + e < lane) p[e] = 0.f;
                } else if constexpr (mode == 2) {
#pragma unroll
                  for (int e = 0; e < 8; ++e)
                    if (!key_ok || (diag && key > q0 + c * 32 + kq + e) || key < q0 + c * 32 + kq + e - wl) p[e] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < 8; e += 2) pk[16 * cc + ((kq + e) >> 1)] = pack_bf16x2(p[e], p[e + 1]);
              }
            }
          };
          using M0 = std::integral_constant<int, 0>;
          using M1 = std::integral_constant<int, 1>;
          using M2 = std::integral_constant<int, 2>;
          using M3 = std::integral_constant<int, 3>;
          auto do_chunk = [&](auto kCC) {
            const int c = 2 * half + decltype(kCC)::value;
            if (diag && !edge) {
              if (c < quarter)
                run_chunk(kCC, M3{});
              else if (c == quarter)
                run_chunk(kCC, M1{});
              else
                run_chunk(kCC, M0{});
            } else if (masked) {
              run_chunk(kCC, M2{});
            } else {
              run_chunk(kCC, M0{});
            }
          };
          do_chunk(std::integral_constant<int, 0>{});
          do_chunk(std::integral_constant<int, 1>{});
        };

        publish(0, fetch(0));
        float staged = n_it > 1 ? fetch(1) : 0.f;
        // it = -1 only computes P of the first block
        for (int it = -1; it < n_it && ok; ++it) {
          const int gi = g0 + it;
          if (it >= 0) {
            // dS'_i = P_i (dP_i - D) once dP^T_i is in TMEM
            const bool got = mbar_wait_t<kFine>(dp_full, gi & 1, abort_flag, err, wlim);
            if (any_fail(got)) { ok = false; break; }
            // every thread is past block i-1's use of buffer (i+1) & 1
            if (it + 1 < n_it) publish(it + 1, staged);
            if (it + 2 < n_it) staged = fetch(it + 2);
            tc_fence_after();
            uint32_t da[32], db[32];
            tmem_load32_async(tmem + lane_base + 128 + (2 * half) * 32, da);
            tmem_load32_async(tmem + lane_base + 128 + (2 * half + 1) * 32, db);
            tmem_wait_ld();
            // P^T_i over the first 32 of the 64 dP^T columns this warp has just read
            tmem_store32(tmem + lane_base + 128 + 64 * half, pk);
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            tc_fence_before();
            mbar_arrive(p_ready);
            const float* nds = dd_s + (gi & 1) * 128;
            uint32_t dk2[32];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              const int c = 2 * half + cc;
              const uint32_t (&dr)[32] = cc == 0 ? da : db;
#pragma unroll
              for (int kq = 0; kq < 32; kq += 4) {
                const float4 d4 = *reinterpret_cast<const float4*>(nds + c * 32 + kq);
                const uint32_t w0 = pk[16 * cc + (kq >> 1)], w1 = pk[16 * cc + (kq >> 1) + 1];
                float a0, a1, a2, a3;
                f2_unpack(f2_mul(f2_pack(bf16_lo(w0), bf16_hi(w0)),
                                 f2_add(f2_pack(__uint_as_float(dr[kq]), __uint_as_float(dr[kq + 1])),
                                        f2_pack(d4.x, d4.y))),
                          a0, a1);
                f2_unpack(f2_mul(f2_pack(bf16_lo(w1), bf16_hi(w1)),
                                 f2_add(f2_pack(__uint_as_float(dr[kq + 2]), __uint_as_float(dr[kq + 3])),
                                        f2_pack(d4.z, d4.w))),
                          a2, a3);
                dk2[16 * cc + (kq >> 1)] = pack_bf16x2(a0, a1);
                dk2[16 * cc + (kq >> 1) + 1] = pack_bf16x2(a2, a3);
              }
            }
            store_row_units(sdSt, dk2, half, r);
            fence_proxy_async_smem();
            mbar_arrive(ds_ready);
          }
          // P_{i+1} while the tensor cores run this block's dV, dK, dQ
          if (it + 1 < n_it) {
            const bool got1 = mbar_wait_t<kFine>(s_full, (gi + 1) & 1, abort_flag, err, wlim);
            if (any_fail(got1)) { ok = false; break; }   // also publishes lse/D of block i+1
            tc_fence_after();
            compute_p(it + 1);
          }
        }
        // dK and dV of this key block, complete with the last block's products
        if (ok) {
          const bool got = mbar_wait_t<kFine>(mm_done, (g0 + n_it - 1) & 1, abort_flag, err, wlim);
          ok = !any_fail(got);
        }
        if (ok && dqkv) {
          // straight into the token-major q|k|v gradient rows: dV as it is, dK
          // through the backward of the QK RMS norm and of the rotation
          // (head dims i and 64 + i form a rotated pair; this thread takes the
          // pairs 32 * half .. 32 * half + 31, the other half's thread the rest
          // of the row, and the two add up the row's <dK, k> in shared memory)
          tc_fence_after();
          const long long m = static_cast<long long>(kb.b) * T + key;
          const int dqk = H * 128, kvd = Hkv * 128;
          bf16* orow = dqkv + m * (dqk + 2 * kvd) + dqk + kb.hk * 128;
          // the normalised rotated k of this row at the same dims, from the K
          // tile in shared memory (two 64-column halves of [128 rows][128 B],
          // 16-byte unit u of row r at u ^ (r & 7)); then K may be replaced
          uint4 yl[4], yh[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const int u = (4 * half + x) ^ (r & 7);
            yl[x] = *reinterpret_cast<const uint4*>(sK + r * 128 + u * 16);
            yh[x] = *reinterpret_cast<const uint4*>(sK + TF_TILE + r * 128 + u * 16);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(kv_empty);
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t vr[32];
            tmem_load32_async(tmem + lane_base + 256 + 64 * half + 32 * c, vr);
            tmem_wait_ld();
            if (key_ok) {
#pragma unroll
              for (int gg = 0; gg < 32; gg += 8) {
                uint4 wv;
                wv.x = pack_bf16x2(__uint_as_float(vr[gg]), __uint_as_float(vr[gg + 1]));
                wv.y = pack_bf16x2(__uint_as_float(vr[gg + 2]), __uint_as_float(vr[gg + 3]));
                wv.z = pack_bf16x2(__uint_as_float(vr[gg + 4]), __uint_as_float(vr[gg + 5]));
                wv.w = pack_bf16x2(__uint_as_float(vr[gg + 6]), __uint_as_float(vr[gg + 7]));
                *reinterpret_cast<uint4*>(orow + kvd + 64 * half + 32 * c + gg) = wv;
              }
            }
          }
          // <dK, k> over this thread's pairs, 16 at a time (dK read from TMEM
          // twice, here and for the result, to keep the registers down)
          float part = 0.f;
#pragma unroll
          for (int hq = 0; hq < 2; ++hq) {
            uint32_t gl[16], gh[16];
            tmem_load16_async(tmem + lane_base + 384 + 32 * half + 16 * hq, gl);
            tmem_load16_async(tmem + lane_base + 448 + 32 * half + 16 * hq, gh);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              const uint4 a = yl[2 * hq + x], bq = yh[2 * hq + x];
              const uint32_t wl4[4] = {a.x, a.y, a.z, a.w};
              const uint32_t wh4[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int i = 8 * x + 2 * e;
                part += __uint_as_float(gl[i]) * bf16_lo(wl4[e]) + __uint_as_float(gl[i + 1]) * bf16_hi(wl4[e]) +
                        __uint_as_float(gh[i]) * bf16_lo(wh4[e]) + __uint_as_float(gh[i + 1]) * bf16_hi(wh4[e]);
              }
            }
          }
          // the two halves of the row meet in the softmax warps' lse buffer,
          // which no thread reads again before the next item's first vote
          lse_s[half * 128 + r] = part;
          asm volatile("bar.sync 1, 256;" ::: "memory");
          // dK = scale * (the TMEM sums); <dK, k> / 128 over the whole row
          const float dot = (part + lse_s[(half ^ 1) * 128 + r]) * scale * (1.f / 128.f);
          const float rr = key_ok ? rk[m * H + kb.hk] : 0.f;
          const float4* e4 = reinterpret_cast<const float4*>(rope + static_cast<long long>(key_ok ? key : 0) * 64 +
                                                             32 * half);
#pragma unroll
          for (int hq = 0; hq < 2; ++hq) {
            uint32_t gl[16], gh[16];
            tmem_load16_async(tmem + lane_base + 384 + 32 * half + 16 * hq, gl);
            tmem_load16_async(tmem + lane_base + 448 + 32 * half + 16 * hq, gh);
            tmem_wait_ld();
            if (key_ok) {
#pragma unroll
              for (int x = 0; x < 2; ++x) {
                const uint4 a = yl[2 * hq + x], bq = yh[2 * hq + x];
                const uint32_t wl4[4] = {a.x, a.y, a.z, a.w};
                const uint32_t wh4[4] = {bq.x, bq.y, bq.z, bq.w};
                uint32_t ol[4], oh[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int i = 8 * x + 2 * e;
                  const float4 cs = __ldg(e4 + ((16 * hq + i) >> 1));   // (cos, sin) of pairs i and i + 1
                  // gradient w.r.t. the rotated vector, then the transposed rotation
                  const float rl0 = rr * (__uint_as_float(gl[i]) * scale - bf16_lo(wl4[e]) * dot);
                  const float rl1 = rr * (__uint_as_float(gl[i + 1]) * scale - bf16_hi(wl4[e]) * dot);
                  const float rh0 = rr * (__uint_as_float(gh[i]) * scale - bf16_lo(wh4[e]) * dot);
                  const float rh1 = rr * (__uint_as_float(gh[i + 1]) * scale - bf16_hi(wh4[e]) * dot);
                  ol[e] = pack_bf16x2(rl0 * cs.x + rh0 * cs.y, rl1 * cs.z + rh1 * cs.w);
                  oh[e] = pack_bf16x2(-rl0 * cs.y + rh0 * cs.x, -rl1 * cs.w + rh1 * cs.z);
                }
                const int col = 32 * half + 16 * hq + 8 * x;
                *reinterpret_cast<uint4*>(orow + col) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
                *reinterpret_cast<uint4*>(orow + 64 + col) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
              }
            }
          }
          // dK and dV have been read: the next key block's first products may
          // overwrite them (they follow this thread's next p_ready / ds_ready)
          tc_fence_before();
        } else if (ok) {
          tc_fence_after();
          bf16* dkrow = dk + (static_cast<long long>(bkv) * T + key) * 128;
          bf16* dvrow = dv + (static_cast<long long>(bkv) * T + key) * 128;
#pragma unroll 1
          for (int c = 2 * half; c < 2 * half + 2; ++c) {
            uint32_t vr[32], kr[32];
            tmem_load32_async(tmem + lane_base + 256 + c * 32, vr);
            tmem_load32_async(tmem + lane_base + 384 + c * 32, kr);
            tmem_wait_ld();
            if (key_ok) {
#pragma unroll
              for (int gg = 0; gg < 32; gg += 8) {
                uint4 wv, wk;
                wv.x = pack_bf16x2(__uint_as_float(vr[gg]), __uint_as_float(vr[gg + 1]));
                wv.y = pack_bf16x2(__uint_as_float(vr[gg + 2]), __uint_as_float(vr[gg + 3]));
                wv.z = pack_bf16x2(__uint_as_float(vr[gg + 4]), __uint_as_float(vr[gg + 5]));
                wv.w = pack_bf16x2(__uint_as_float(vr[gg + 6]), __uint_as_float(vr[gg + 7]));
                wk.x = pack_bf16x2(__uint_as_float(kr[gg]) * scale, __uint_as_float(kr[gg + 1]) * scale);
                wk.y = pack_bf16x2(__uint_as_float(kr[gg + 2]) * scale, __uint_as_float(kr[gg + 3]) * scale);
                wk.z = pack_bf16x2(__uint_as_float(kr[gg + 4]) * scale, __uint_as_float(kr[gg + 5]) * scale);
                wk.w = pack_bf16x2(__uint_as_float(kr[gg + 6]) * scale, __uint_as_float(kr[gg + 7]) * scale);
                *reinterpret_cast<uint4*>(dvrow + c * 32 + gg) = wv;
                *reinterpret_cast<uint4*>(dkrow + c * 32 + gg) = wk;
              }
            }
          }
          // dK and dV have been read: the next key block's first products may
          // overwrite them (they follow this thread's next p_ready / ds_ready)
          tc_fence_before();
        }
        g0 += n_it;
      }
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

}  // namespace

// Window in tokens as the kernels take it: keys t - wl .. t; "no window" is a
// bound no row reaches (kept small enough that k0 + 127 + wl fits in an int).
static int window_bound(int window, int T) { return window < 0 || window >= T ? (1 << 30) : window; }


// Scheduler words for callers that bring none: a ring of 64 library-owned
// counters, one per launch in turn, each zeroed on the launch's stream
// before use (so up to 64 such launches may be in flight at once).
__device__ int g_sched_ring[64];

static int* sched_word(int* sched, cudaStream_t s) {
  if (!sched) {
    static std::atomic<unsigned> next{0};
    int* base = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&base), g_sched_ring) != cudaSuccess) return nullptr;
    sched = base + (next++ & 63u);
  }
  cudaMemsetAsync(sched, 0, sizeof(int), s);
  return sched;
}

void launch_attn_fwd(const bf16* q, const bf16* k, const bf16* v, bf16* o, float* lse, int B, int H, int T,
                     cudaStream_t s, int* err, int Hkv, int window, int* sched, int kv_stride,
                     long long wait_cycles) {
  // a limit shorter than one blocking probe needs the finely polling build
  const bool fine = wait_limit_or_default(wait_cycles) < kShortWaitCycles;
  auto kern = fine ? attn_fwd_tc_kernel<true> : attn_fwd_tc_kernel<false>;
  static std::atomic<unsigned long long> configured[2] = {};
  if (set_smem_limit_once(kern, TF_SMEM, configured[fine ? 1 : 0]) != cudaSuccess) {
    if (err) cudaMemsetAsync(err, 0xff, sizeof(int), s);   // latched as a device error
    return;
  }
  if (Hkv <= 0) Hkv = H;
  if (kv_stride <= 0) kv_stride = Hkv;
  CUtensorMap mq, mk, mv;
  const long long bh = 1ll * B * H, bhkv = 1ll * B * kv_stride;
  if (H % Hkv || kv_stride < Hkv || !make_map(&mq, q, 2, HD, T, bh, HD, 1ll * T * HD, 64, 128) ||
      !make_map(&mk, k, 2, HD, T, bhkv, HD, 1ll * T * HD, 64, 128) ||
      !make_map(&mv, v, 2, HD, T, bhkv, HD, 1ll * T * HD, 64, 128)) {
    if (err) cudaMemsetAsync(err, 0xff, sizeof(int), s);   // latched as a device error
    return;
  }
  // persistent: one CTA per SM over the pairs of query tiles of every head
  const long long n_items = ((T + 127) / 128 + 1) / 2 * bh;
  const int grid = static_cast<int>(std::min<long long>(n_items, device_sm_count()));
  const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(HD));
  kern<<<grid, 384, TF_SMEM, s>>>(mq, mk, mv, o, lse, H, Hkv, kv_stride, T, window_bound(window, T),
                                                scale_log2,
                                                static_cast<int>(n_items), sched_word(sched, s), err, wait_cycles);
}

void launch_attn_bwd(const bf16* q, const bf16* k, const bf16* v, const bf16* o, const bf16* dout,
                     const float* lse, float* Dv, float* dq, bf16* dk, bf16* dv, int B, int H, int T,
                     cudaStream_t s, int* err, int Hkv, int window, int* sched, int kv_stride,
                     long long wait_cycles, const float* rk, const float2* rope, bf16* dqkv, bool d_ready) {
  const bool fine = wait_limit_or_default(wait_cycles) < kShortWaitCycles;
  auto kern = fine ? attn_bwd_tc_kernel<true> : attn_bwd_tc_kernel<false>;
  static std::atomic<unsigned long long> configured[2] = {};
  if (set_smem_limit_once(kern, TB_SMEM, configured[fine ? 1 : 0]) != cudaSuccess) {
    if (err) cudaMemsetAsync(err, 0xff, sizeof(int), s);   // latched as a device error
    return;
  }
  if (Hkv <= 0) Hkv = H;
  const long long rows = 1ll * B * H * T;
  if (!d_ready) attn_bwd_dot_kernel<<<static_cast<int>((rows + 7) / 8), 256, 0, s>>>(o, dout, Dv, B, H, T);
  cudaMemsetAsync(dq, 0, static_cast<size_t>(rows) * HD * sizeof(float), s);
  CUtensorMap mq, mk, mv, mdo, mdq;
  if (kv_stride <= 0) kv_stride = Hkv;
  const long long bh = 1ll * B * H, bhkv = 1ll * B * kv_stride;
  const long long dims[4] = {HD, H, T, B};
  const long long strides[3] = {HD * 2ll, 1ll * H * HD * 2, 1ll * T * H * HD * 2};
  const int box[4] = {64, 1, 128, 1};
  if (H % Hkv || kv_stride < Hkv || !make_map(&mq, q, 2, HD, T, bh, HD, 1ll * T * HD, 64, 128) ||
      !make_map(&mk, k, 2, HD, T, bhkv, HD, 1ll * T * HD, 64, 128) ||
      !make_map(&mv, v, 2, HD, T, bhkv, HD, 1ll * T * HD, 64, 128) || !make_map_4d(&mdo, dout, dims, strides, box) ||
      !make_map(&mdq, dq, 4, HD, T, bh, HD, 1ll * T * HD, 32, 32)) {
    if (err) cudaMemsetAsync(err, 0xff, sizeof(int), s);
    return;
  }
  // persistent: one CTA per SM over units of two key blocks of every kv head.
  // Without a window every unit costs the same and a fixed stride spreads
  // them evenly (measured ~3% faster than the counter, which claims each
  // CTA's next unit ahead of time); with one, unit costs differ and the
  // counter balances them.
  const long long n_units = 1ll * B * Hkv * (((T + 127) / 128 + 1) / 2);
  const int grid = static_cast<int>(std::min<long long>(n_units, device_sm_count()));
  const int wl = window_bound(window, T);
  int* word = wl >= T ? nullptr : sched_word(sched, s);
  kern<<<grid, 512, TB_SMEM, s>>>(mq, mk, mv, mdo, mdq, lse, Dv, dk, dv, H, Hkv, kv_stride, T, wl,
                                                1.f / sqrtf(static_cast<float>(HD)), static_cast<int>(n_units),
                                                word, err, wait_cycles, rk, rope, dqkv);
}

}  // namespace gpt
