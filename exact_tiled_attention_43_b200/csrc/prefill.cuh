// prefill.cuh -- fused exact attention forward (dense and packed/varlen) and HSTU pointwise attention, one
// kernel template for B200 (sm_100a): TMA tile loads, tcgen05 MMAs accumulating in tensor memory (TMEM),
// warp-specialised softmax, in-kernel causal mask with masked tiles skipped.
//
// What it computes:
//   softmax modes: O = softmax(scale * Q K^T [+ causal]) V and lse = ln sum_j exp(scale q_i.k_j), tile by
//     tile with an online softmax ("FlashAttention (TH)", sections "Tiling และการประมวลผลแบบบล็อก",
//     "การคำนวณ Softmax แบบออนไลน์", "การรวมการดำเนินการเป็น CUDA Kernel เดียว"; the ops-transformer page,
//     section "FlashAttention 的解法": per block update the running max, correct the earlier weights and
//     the partial output, write back only the final output).
//   HSTU mode: O = (silu(alpha Q K^T) * causal_mask * inv_n) V over packed sequences (the HSTU page,
//     sections "先搞懂：HSTU到底难在哪？", "绝杀优化二：内置Mask生成", "绝杀优化三：Jagged变长张量").
//
// Work decomposition: one CTA owns 256 query rows of one (batch, head) -- two 128-row Q tiles -- and
// streams the key/value tiles (128 rows each) its rows can see.  Causal tiles past the diagonal are never
// loaded (the "after the diagonal: all zero, skip" class of the HSTU page's in-kernel mask); only the
// diagonal tile and a ragged last tile evaluate a per-element mask.
//
// Roles (320 threads):
//   warp 0      TMA producer: Q0,Q1 once, then K_0, V_0, K_1, V_1, ... through an NST-stage ring.
//   warp 1      TMEM allocator + MMA issuer (one thread):  S_t = Q_t K_j^T (SS form) into TMEM,
//               O_t += P_t V_j (TS form: P read from TMEM, V from shared memory).
//   warps 2-5   softmax warpgroup for Q tile 0; warps 6-9 for Q tile 1.  Thread r of a group owns query
//               row r = TMEM lane r: it loads its S row from TMEM, applies the mask, updates the running
//               max/exp-sum, writes P (bf16) back into TMEM over the first 64 columns of S, rescales its
//               O row when the max moved, and finally normalises O and stores O and lse.
// The MMA thread interleaves the two tiles (PV_0, S_0', PV_1, S_1') so that one warpgroup's softmax runs
// while the tensor core works for the other.
//
// TMEM (512 columns x 128 lanes): S_0 [0,128), S_1 [128,256), O_0 [256,256+D), O_1 [256+D,256+2D);
// P_t aliases the first 64 columns of S_t, so S_t of the next key tile is issued only after the MMA that
// reads P_t has completed.
//
// Online-softmax rescale is conditional: the running max used for exponentiation is only raised when a
// row's block max exceeds it by more than 8 (log2 units).  The final O / l and lse use the same stale max
// consistently, so the result is exact (up to rounding) while most key tiles skip the O rescale.
#pragma once

#include <type_traits>

#include "ptx.cuh"

namespace eta {

constexpr int PF_BM = 128;            // query rows per Q tile (= TMEM lanes)
constexpr int PF_BN = 128;            // keys per K/V tile
constexpr int PF_SM_WARPS = 8;        // softmax warps: 2 Q tiles x 4 lane quarters (one thread per query row)
constexpr int PF_THREADS = 32 * (4 + PF_SM_WARPS);  // + control warpgroup: TMA, 2 MMA issuers, 1 spare
// Register split (setmaxnreg): the CTA launches with PF_LAUNCH_REGS per thread; the control warpgroup drops
// to PF_CTRL_REGS and the two softmax warpgroups grow to PF_SM_REGS.  The shares add up to the launch total
// exactly, and the host refuses to launch a build whose register count is not PF_LAUNCH_REGS (a larger
// request than the launch total would stall forever).
constexpr int PF_LAUNCH_REGS = 168, PF_CTRL_REGS = 56, PF_SM_REGS = 224;
static_assert(128 * PF_CTRL_REGS + 32 * PF_SM_WARPS * PF_SM_REGS == PF_THREADS * PF_LAUNCH_REGS, "register split");
constexpr float PF_RESCALE_THRESHOLD = 8.0f;  // log2 units

enum PrefillMode { MODE_DENSE = 0, MODE_VARLEN = 1, MODE_HSTU = 2 };

struct PrefillParams {
  void *o;                 // dense: [B,H,N,D]; packed: [T,H,D]; bf16 or fp32
  float *lse;              // dense: [B,H,N]; packed: [T,H]; may be null
  const int *cu_seqlens;   // packed modes: [S+1]
  int H, N, max_len;       // N: dense sequence length
  int causal, o_f32;
  float scale_log2;        // softmax: scale * log2(e)
  float hstu_half_alpha;   // HSTU: 0.5 * alpha      (tanh argument scale)
  float hstu_out;          // HSTU: 0.5 * alpha * inv_n
  long long wait_ns;
};

template <int D>
struct PfCfg {
  // TMEM (512 columns): S_t at 128 t, O_t at 256 + D t.  With D = 64 there is room for a separate P_t
  // (at 384 + 64 t), so the next key tile's S_t can be computed while the softmax still works on P_t.
  // With D = 128 TMEM is full and P_t overwrites the first 64 columns of S_t (S_t of the next key tile is
  // then issued only after the PV that reads P_t has completed).
  static constexpr bool ALIAS_P = (D == 128);
  static constexpr int KCH = D / 64;                     // 128-byte column chunks per row
  static constexpr int CHUNK_BYTES = PF_BM * 128;        // 128 rows x 128 B
  static constexpr int TILE_BYTES = KCH * CHUNK_BYTES;   // one 128 x D bf16 tile
  static constexpr int NST = (D == 64) ? 8 : 4;          // K/V ring depth (each stage holds one tile)
  // Of every 8 exp2 pairs, how many use the FMA-pipe polynomial instead of the MUFU.  Off: measured inside
  // this kernel it costs more (issue slots, dependency chains) than the MUFU time it saves.
  static constexpr int POLY_PAIRS = 0;
  // barriers: full/empty per stage, q, per tile {s_full, s_free, p_full, pv_done, mma_done}
  static constexpr int NBAR = 2 * NST + 1 + 2 * 5;
  static constexpr int SMEM_BYTES = 1024 /*alignment slack*/ + (2 + NST) * TILE_BYTES + NBAR * 8 + 16;
  static constexpr uint32_t TM_O = 256;                  // O_t at TM_O + D*t
  static constexpr uint32_t TM_P = 384;                  // P_t at TM_P + 64*t (D = 64); S_t's columns [0,64) (D = 128)
};

// Control warpgroup: warp 0 streams Q, K, V with TMA; warps 1 and 2 issue the MMAs of Q tiles 0 and 1;
// warp 3 has no role.
template <int D, int MODE>
__device__ __forceinline__ void prefill_control(const CUtensorMap &tmQ, const CUtensorMap &tmK,
                                                const CUtensorMap &tmV, const PrefillParams &p, uint8_t *smem,
                                                uint32_t tmem, int warp, int lane, int r0, int h, int bh,
                                                int seq_start, const int (&n_t)[2], int n_kv) {
  using C = PfCfg<D>;
  constexpr bool HSTU = (MODE == MODE_HSTU);
  constexpr bool PACKED = (MODE != MODE_DENSE);
  uint8_t *sQ = smem;
  uint8_t *sKV = smem + 2 * C::TILE_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sKV + C::NST * C::TILE_BYTES);
  uint64_t *full = bars;
  uint64_t *empty = bars + C::NST;
  uint64_t *q_full = bars + 2 * C::NST;
  uint64_t *s_full = q_full + 1;
  uint64_t *s_free = s_full + 2;
  uint64_t *p_full = s_free + 2;
  uint64_t *pv_done = p_full + 2;
  uint64_t *mma_done = pv_done + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  (void)sQ; (void)sKV; (void)full; (void)empty; (void)q_full; (void)s_full; (void)s_free;
  (void)p_full; (void)pv_done; (void)mma_done; (void)abort_flag; (void)HSTU; (void)PACKED;
  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, 2 * C::TILE_BYTES);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
#pragma unroll
        for (int c = 0; c < C::KCH; ++c) {
          uint8_t *dst = sQ + t * C::TILE_BYTES + c * C::CHUNK_BYTES;
          if constexpr (PACKED)
            tma_load_3d(dst, &tmQ, q_full, 64 * c, h, seq_start + r0 + t * PF_BM);
          else
            tma_load_3d(dst, &tmQ, q_full, 64 * c, r0 + t * PF_BM, bh);
        }
      }
      int item = 0;
      const int n_items = 2 * n_kv;
      for (; item < n_items; ++item) {
        const int st = item % C::NST;
        if (!mbar_wait(&empty[st], ((item / C::NST) & 1) ^ 1, abort_flag, p.wait_ns)) break;
        const int j = item >> 1;
        const CUtensorMap *m = (item & 1) ? &tmV : &tmK;
        mbar_arrive_expect_tx(&full[st], C::TILE_BYTES);
#pragma unroll
        for (int c = 0; c < C::KCH; ++c) {
          uint8_t *dst = sKV + st * C::TILE_BYTES + c * C::CHUNK_BYTES;
          if constexpr (PACKED)
            tma_load_3d(dst, m, &full[st], 64 * c, h, seq_start + j * PF_BN);
          else
            tma_load_3d(dst, m, &full[st], 64 * c, j * PF_BN, bh);
        }
      }
      if (item < n_items) {
        // Abandoned pipeline: let copies already in flight land before shared memory is released.
        mbar_wait(q_full, 0, nullptr, p.wait_ns);
        for (int i = max(0, item - C::NST); i < item; ++i)
          mbar_wait(&full[i % C::NST], (i / C::NST) & 1, nullptr, p.wait_ns);
      }
    }
  } else if (C::ALIAS_P && warp == 1) {
    // ================================================================ single MMA issuer (P aliased into S)
    // One thread issues both tiles' MMAs in the order PV_0(j), S_0(j+1), PV_1(j), S_1(j+1).  tcgen05.mma
    // operations issued by one thread execute in issue order, so S_t(j+1) -- which overwrites the columns
    // holding P_t(j) -- needs no wait for PV_t(j) to complete; its commit also tracks that PV, so a softmax
    // that has seen S_t(j+1) may rescale O_t.  The single ordered stream keeps the two softmax warpgroups
    // half a period apart.
    if (lane == 0) {
      constexpr uint32_t ID_QK = idesc_bf16_f32(PF_BM, PF_BN, false);
      constexpr uint32_t ID_PV = idesc_bf16_f32(PF_BM, D, true);
      const uint32_t sQa = smem_u32(sQ), sKVa = smem_u32(sKV);
      auto issue_s = [&](int t, int st) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * C::CHUNK_BYTES + (uint32_t)(kk & 3) * 32u;
          mma_ss(tmem + 128u * t, sdesc_sw128(sQa + t * C::TILE_BYTES + off, 16, 1024),
                 sdesc_sw128(sKVa + st * C::TILE_BYTES + off, 16, 1024), ID_QK, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, int st, bool acc) {
#pragma unroll
        for (int kk = 0; kk < PF_BN / 16; ++kk)
          mma_ts(tmem + C::TM_O + (uint32_t)(D * t), tmem + 128u * t + 8u * kk,
                 sdesc_sw128(sKVa + st * C::TILE_BYTES + kk * 2048, C::CHUNK_BYTES, 1024), ID_PV,
                 (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, p.wait_ns);
      if (ok && n_kv > 0) {
        ok = mbar_wait(&full[0], 0, abort_flag, p.wait_ns);
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int t = 0; t < 2; ++t)
            if (n_t[t] > 0) {
              issue_s(t, 0);
              mma_commit(&s_full[t]);
            }
          mma_commit(&empty[0]);
        }
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        const int iv = 2 * j + 1, sv = iv % C::NST;
        const int ik = 2 * j + 2, sk = ik % C::NST;
        ok = mbar_wait(&full[sv], (iv / C::NST) & 1, abort_flag, p.wait_ns);
        if (!ok) break;
        bool k_ready = false;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!ok || j >= n_t[t]) continue;
          ok = mbar_wait(&p_full[t], j & 1, abort_flag, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
          issue_pv(t, sv, j > 0);
          mma_commit(&pv_done[t]);
          if (j + 1 < n_t[t]) {
            if (!k_ready) {
              ok = mbar_wait(&full[sk], (ik / C::NST) & 1, abort_flag, p.wait_ns);
              if (!ok) break;
              k_ready = true;
            }
            issue_s(t, sk);
            mma_commit(&s_full[t]);
          }
        }
        if (!ok) break;
        mma_commit(&empty[sv]);
        if (k_ready) mma_commit(&empty[sk]);
      }
      mma_commit(&mma_done[0]);
      mbar_wait(&mma_done[0], 0, nullptr, p.wait_ns);
    }
    __syncwarp();
  } else if (!C::ALIAS_P && (warp == 1 || warp == 2)) {
    // ================================================================ MMA issuer for Q tile t
    const int t = warp - 1;
    if (lane == 0) {
      constexpr uint32_t ID_QK = idesc_bf16_f32(PF_BM, PF_BN, false);
      constexpr uint32_t ID_PV = idesc_bf16_f32(PF_BM, D, true);
      const uint32_t sQa = smem_u32(sQ) + t * C::TILE_BYTES, sKVa = smem_u32(sKV);
      const uint32_t tS = tmem + 128u * t, tO = tmem + C::TM_O + (uint32_t)(D * t);
      const uint32_t tP = C::ALIAS_P ? tS : tmem + C::TM_P + 64u * t;
      // S_t = Q_t K^T : K-steps of 16 elements = 32 bytes inside a 128-byte swizzled row.
      auto issue_s = [&](int st) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * C::CHUNK_BYTES + (uint32_t)(kk & 3) * 32u;
          mma_ss(tS, sdesc_sw128(sQa + off, 16, 1024), sdesc_sw128(sKVa + st * C::TILE_BYTES + off, 16, 1024), ID_QK,
                 kk > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t V : K-steps of 16 keys = 8 TMEM columns of packed bf16 P, 16 rows (2048 B) of V.
      auto issue_pv = [&](int st, bool acc) {
#pragma unroll
        for (int kk = 0; kk < PF_BN / 16; ++kk)
          mma_ts(tO, tP + 8u * kk, sdesc_sw128(sKVa + st * C::TILE_BYTES + kk * 2048, C::CHUNK_BYTES, 1024), ID_PV,
                 (acc || kk > 0) ? 1u : 0u);
      };
      const int nt = n_t[t];
      bool ok = mbar_wait(q_full, 0, abort_flag, p.wait_ns);
      if (ok && nt > 0) {
        ok = mbar_wait(&full[0], 0, abort_flag, p.wait_ns);
        if (ok) {
          tc_fence_after();
          issue_s(0);
          mma_commit(&s_full[t]);
          mma_commit(&empty[0]);
        }
      }
      for (int j = 0; ok && j < nt; ++j) {
        const int ik = 2 * j + 2, sk = ik % C::NST;
        const int iv = 2 * j + 1, sv = iv % C::NST;
        if constexpr (!C::ALIAS_P) {
          // Separate P: S_t of the next key tile as soon as the softmax has copied S_t to registers.
          if (j + 1 < nt) {
            ok = mbar_wait(&full[sk], (ik / C::NST) & 1, abort_flag, p.wait_ns) &&
                 mbar_wait(&s_free[t], j & 1, abort_flag, p.wait_ns);
            if (!ok) break;
            tc_fence_after();
            issue_s(sk);
            mma_commit(&s_full[t]);
            mma_commit(&empty[sk]);
          }
        }
        ok = mbar_wait(&full[sv], (iv / C::NST) & 1, abort_flag, p.wait_ns) &&
             mbar_wait(&p_full[t], j & 1, abort_flag, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        issue_pv(sv, j > 0);
        mma_commit(&pv_done[t]);
        mma_commit(&empty[sv]);
        if constexpr (C::ALIAS_P) {
          // P_t lives in S_t's columns: the PV just issued must finish reading it first.
          if (j + 1 < nt) {
            ok = mbar_wait(&full[sk], (ik / C::NST) & 1, abort_flag, p.wait_ns) &&
                 mbar_wait(&pv_done[t], j & 1, abort_flag, p.wait_ns);
            if (!ok) break;
            tc_fence_after();
            issue_s(sk);
            mma_commit(&s_full[t]);
            mma_commit(&empty[sk]);
          }
        }
      }
      // Key/value tiles this Q tile does not see (past its diagonal, or the whole tile past the end):
      // release them too, in order, once they have landed.
      for (int item = 2 * nt; ok && item < 2 * n_kv; ++item) {
        ok = mbar_wait(&full[item % C::NST], (item / C::NST) & 1, abort_flag, p.wait_ns);
        if (ok) mbar_arrive(&empty[item % C::NST]);
      }
      // Every MMA issued by this thread has completed before TMEM is released.
      mma_commit(&mma_done[t]);
      mbar_wait(&mma_done[t], 0, nullptr, p.wait_ns);
    }
    __syncwarp();
  }
}

// Softmax (or HSTU pointwise) warpgroups: warps 4-7 for Q tile 0, warps 8-11 for Q tile 1.  Thread
// (quarter, lane) owns query row 32 quarter + lane of its tile (= its TMEM lane): it loads the S row from
// TMEM, applies the mask, updates the running max and exp-sum, writes P (bf16) to TMEM, rescales its O row
// when the max moved, and finally normalises O and stores O and lse.
template <int D, int MODE>
__device__ __forceinline__ void prefill_softmax(const PrefillParams &p, uint8_t *smem, uint32_t tmem, int warp,
                                                int lane, int r0, int L, int h, int bh, int seq_start, bool causal,
                                                const int (&n_t)[2]) {
  using C = PfCfg<D>;
  constexpr bool HSTU = (MODE == MODE_HSTU);
  constexpr bool PACKED = (MODE != MODE_DENSE);
  uint8_t *sQ = smem;
  uint8_t *sKV = smem + 2 * C::TILE_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sKV + C::NST * C::TILE_BYTES);
  uint64_t *full = bars;
  uint64_t *empty = bars + C::NST;
  uint64_t *q_full = bars + 2 * C::NST;
  uint64_t *s_full = q_full + 1;
  uint64_t *s_free = s_full + 2;
  uint64_t *p_full = s_free + 2;
  uint64_t *pv_done = p_full + 2;
  uint64_t *mma_done = pv_done + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  (void)sQ; (void)sKV; (void)full; (void)empty; (void)q_full; (void)s_full; (void)s_free;
  (void)p_full; (void)pv_done; (void)mma_done; (void)abort_flag; (void)HSTU; (void)PACKED;
  const int t = (warp - 4) >> 2;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_addr + 128u * t;
  const uint32_t tO = tmem + lane_addr + C::TM_O + (uint32_t)(D * t);
  const uint32_t tP = C::ALIAS_P ? tS : tmem + lane_addr + C::TM_P + 64u * t;
  const int q_start = r0 + t * PF_BM;
  const int qpos = q_start + row;
  const int nt = n_t[t];
  float m_used = -INFINITY, l = 0.f;
  bool ok = true;
  for (int j = 0; j < nt; ++j) {
    ok = mbar_wait(&s_full[t], j & 1, abort_flag, p.wait_ns);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    tc_fence_after();
    uint32_t sr[128];
    ETA_TMEM_LD_X32(tS + 0u, (sr + 0));
    ETA_TMEM_LD_X32(tS + 32u, (sr + 32));
    ETA_TMEM_LD_X32(tS + 64u, (sr + 64));
    ETA_TMEM_LD_X32(tS + 96u, (sr + 96));
    tmem_wait_ld();
    if constexpr (!C::ALIAS_P) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[t]);  // S_t may now be overwritten by the next key tile's QK^T
    }
    const int k0 = j * PF_BN;
    const bool need_mask = (k0 + PF_BN > L) || (causal && k0 + PF_BN - 1 > q_start);
    const int kmax = causal ? min(L - 1, qpos) - k0 : L - 1 - k0;  // last visible key, tile-local
    uint32_t pk[64];
    bool resc = false;
    float f = 1.f, rowsum = 0.f, m_new = m_used;
    if constexpr (!HSTU) {
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > kmax) sr[c] = __float_as_uint(-INFINITY);
      }
      // row max: four independent 3-input max chains
      float mxa = -INFINITY, mxb = -INFINITY, mxc = -INFINITY, mxd = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; c += 8) {
        mxa = max3f(mxa, __uint_as_float(sr[c + 0]), __uint_as_float(sr[c + 1]));
        mxb = max3f(mxb, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
        mxc = max3f(mxc, __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
        mxd = max3f(mxd, __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
      }
      const float mx = max3f(mxa, mxb, fmaxf(mxc, mxd)) * p.scale_log2;
      if (mx > m_used + PF_RESCALE_THRESHOLD) {
        m_new = mx;
        resc = true;
      }
      const float msub = (m_new == -INFINITY) ? 0.f : m_new;
      const uint64_t cs2 = f2pack(p.scale_log2, p.scale_log2), nm2 = f2pack(-msub, -msub);
      uint64_t rs_a = f2pack(0.f, 0.f), rs_b = f2pack(0.f, 0.f);
      // p = 2^(s * scale_log2 - m): pairs with (i % 8) < POLY_PAIRS go to the FMA-pipe polynomial on
      // unmasked tiles, the rest (and every element of a masked tile) to the MUFU.
      auto exp_row = [&](auto use_poly) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const uint64_t x2 =
              fma_x2(f2pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), cs2, nm2);
          float x0, x1, p0, p1;
          f2unpack(x2, x0, x1);
          if (decltype(use_poly)::value && (i % 8) < C::POLY_PAIRS) {
            exp2_poly_x2(x0, x1, p0, p1);
          } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          if (i & 1) rs_b = add_x2(rs_b, f2pack(p0, p1));
          else rs_a = add_x2(rs_a, f2pack(p0, p1));
          pk[i] = pack_bf16x2(p0, p1);
        }
      };
      if (need_mask) exp_row(std::false_type{});
      else exp_row(std::true_type{});
      float r0a, r1a, r2a, r3a;
      f2unpack(rs_a, r0a, r1a);
      f2unpack(rs_b, r2a, r3a);
      rowsum = (r0a + r1a) + (r2a + r3a);
      f = resc ? ex2_approx(m_used - msub) : 1.f;  // 0 on the first tile
    } else {
      // HSTU: p = inv_n * silu(alpha s) = h + h * tanh(alpha s / 2),  h = (alpha * inv_n / 2) s
      const uint64_t ha2 = f2pack(p.hstu_half_alpha, p.hstu_half_alpha), ho2 = f2pack(p.hstu_out, p.hstu_out);
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const int c0 = 2 * i;
        const uint64_t s2 = f2pack(__uint_as_float(sr[c0]), __uint_as_float(sr[c0 + 1]));
        float y0, y1;
        f2unpack(mul_x2(s2, ha2), y0, y1);
        const uint64_t h2 = mul_x2(s2, ho2);
        float p0, p1;
        f2unpack(fma_x2(h2, f2pack(tanh_approx(y0), tanh_approx(y1)), h2), p0, p1);
        if (need_mask) {
          p0 = (c0 > kmax) ? 0.f : p0;
          p1 = (c0 + 1 > kmax) ? 0.f : p1;
        }
        pk[i] = pack_bf16x2(p0, p1);
      }
    }
    if constexpr (!C::ALIAS_P) {
      // P_t's buffer (and O_t) are free once the previous key tile's PV has completed.  (With P aliased into
      // S_t this is implied: S_t of this key tile was issued only after that PV completed.)
      if (j > 0) {
        ok = mbar_wait(&pv_done[t], (j - 1) & 1, abort_flag, p.wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
      }
    }
    ETA_TMEM_ST_X32(tP + 0u, (pk + 0));
    ETA_TMEM_ST_X32(tP + 32u, (pk + 32));
    if constexpr (!HSTU) {
      if (__any_sync(0xffffffffu, resc && j > 0)) {
        const uint64_t f2 = f2pack(f, f);
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t orr[32];
          ETA_TMEM_LD_X32(tO + 32u * cc, orr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float a, b;
            f2unpack(mul_x2(f2pack(__uint_as_float(orr[2 * i]), __uint_as_float(orr[2 * i + 1])), f2), a, b);
            orr[2 * i] = __float_as_uint(a);
            orr[2 * i + 1] = __float_as_uint(b);
          }
          ETA_TMEM_ST_X32(tO + 32u * cc, orr);
        }
      }
      l = l * f + rowsum;
      m_used = m_new;
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&p_full[t]);
  }
  // ---------------------------------------------------------------- epilogue
  if (ok && nt > 0) {
    ok = mbar_wait(&pv_done[t], (nt - 1) & 1, abort_flag, p.wait_ns);
    ok = __all_sync(0xffffffffu, ok);
  }
  if (ok && nt > 0) {
    tc_fence_after();
    const float inv_l = HSTU ? 1.f : ((l > 0.f) ? 1.f / l : 0.f);
    const bool valid = qpos < L;
    const size_t orow = PACKED ? ((size_t)(seq_start + qpos) * p.H + h) : ((size_t)bh * p.N + qpos);
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t orr[32];
      ETA_TMEM_LD_X32(tO + 32u * cc, orr);
      tmem_wait_ld();
      if (valid) {
        if (p.o_f32) {
          float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.o) + orow * D + 32 * cc);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(orr[4 * i]) * inv_l, __uint_as_float(orr[4 * i + 1]) * inv_l,
                                 __uint_as_float(orr[4 * i + 2]) * inv_l, __uint_as_float(orr[4 * i + 3]) * inv_l);
        } else {
          uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) + orow * D + 32 * cc);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(orr[8 * i + 0]) * inv_l, __uint_as_float(orr[8 * i + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(orr[8 * i + 2]) * inv_l, __uint_as_float(orr[8 * i + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(orr[8 * i + 4]) * inv_l, __uint_as_float(orr[8 * i + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(orr[8 * i + 6]) * inv_l, __uint_as_float(orr[8 * i + 7]) * inv_l);
            dst[i] = w;
          }
        }
      }
    }
    if constexpr (!HSTU) {
      if (valid && p.lse != nullptr)
        p.lse[orow] = (l > 0.f) ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }
}

template <int D, int MODE>
__global__ void __launch_bounds__(PF_THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = PfCfg<D>;
  constexpr bool HSTU = (MODE == MODE_HSTU);
  constexpr bool PACKED = (MODE != MODE_DENSE);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;                                        // 2 tiles
  uint8_t *sKV = smem + 2 * C::TILE_BYTES;                   // NST tiles
  uint64_t *bars = reinterpret_cast<uint64_t *>(sKV + C::NST * C::TILE_BYTES);
  uint64_t *full = bars;                 // [NST] TMA -> MMA issuers
  uint64_t *empty = bars + C::NST;       // [NST] both MMA issuers -> TMA (count 2)
  uint64_t *q_full = bars + 2 * C::NST;  // Q tiles landed
  uint64_t *s_full = q_full + 1;         // [2] S_t ready in TMEM              (MMA t -> softmax t)
  uint64_t *s_free = s_full + 2;         // [2] S_t copied to registers        (softmax t -> MMA t; D = 64)
  uint64_t *p_full = s_free + 2;         // [2] P_t written, O_t rescaled      (softmax t -> MMA t)
  uint64_t *pv_done = p_full + 2;        // [2] O_t += P_t V complete           (MMA t -> softmax t, MMA t)
  uint64_t *mma_done = pv_done + 2;      // [2] every MMA of issuer t complete
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ------------------------------------------------------------------ work item
  // Heaviest (latest) row blocks are launched first: dense grid (B*H, blocks), packed grid (H, S, blocks).
  const int blk = PACKED ? (int)(gridDim.z - 1 - blockIdx.z) : (int)(gridDim.y - 1 - blockIdx.y);
  int L, seq_start = 0, bh = 0, h = 0;
  if constexpr (PACKED) {
    h = blockIdx.x;
    const int s = blockIdx.y;
    seq_start = p.cu_seqlens[s];
    L = p.cu_seqlens[s + 1] - seq_start;
    if (L < 0 || L > p.max_len) {
      if (threadIdx.x == 0 && blk == 0) record_status(3 /* ETA_DEV_BAD_CUSEQ */);
      return;
    }
  } else {
    bh = blockIdx.x;
    L = p.N;
  }
  const int r0 = blk * 2 * PF_BM;
  if (r0 >= L) return;  // uniform over the CTA
  const bool causal = HSTU ? true : (p.causal != 0);
  int n_t[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qs = r0 + t * PF_BM;
    const int kv_end = (qs >= L) ? 0 : (causal ? min(L, qs + PF_BM) : L);
    n_t[t] = (kv_end + PF_BN - 1) / PF_BN;
  }
  const int n_kv = max(n_t[0], n_t[1]);

  // ------------------------------------------------------------------ setup
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::ALIAS_P ? 1 : 2);  // released by each MMA issuer
    }
    mbar_init(q_full, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&s_free[t], 4);   // one elected arrive per softmax warp of the tile
      mbar_init(&p_full[t], 4);
      mbar_init(&pv_done[t], 1);
      mbar_init(&mma_done[t], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Each role runs to its own end; the teardown barrier (id 1, every thread of the CTA) is reached from
  // both sides.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(PF_CTRL_REGS));
    prefill_control<D, MODE>(tmQ, tmK, tmV, p, smem, tmem, warp, lane, r0, h, bh, seq_start, n_t, n_kv);
    tc_fence_before();
    asm volatile("bar.sync 1, %0;" ::"n"(PF_THREADS) : "memory");
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(PF_SM_REGS));
    prefill_softmax<D, MODE>(p, smem, tmem, warp, lane, r0, L, h, bh, seq_start, causal, n_t);
    tc_fence_before();
    asm volatile("bar.sync 1, %0;" ::"n"(PF_THREADS) : "memory");
  }
}

}  // namespace eta
