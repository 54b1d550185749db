// prefill_wide.cuh -- exact attention forward for head dimension 256 (dense and packed/varlen), a persistent
// tcgen05 kernel beside the d = 64 / 128 one in prefill.cuh.
//
// What it computes: the same O = softmax(scale * Q K^T [+ causal]) V and lse as prefill.cuh, tile by tile with
// an online softmax ("FlashAttention (TH)", sections "การคำนวณ Softmax แบบออนไลน์" and "FlashAttention-2": the
// second version extends head-size support to 256).
//
// Why a kernel of its own: a 128-row O accumulator of 256 fp32 columns takes half of TMEM, so a CTA holds one
// Q tile, not two.  Layout per CTA:
//   TMEM   S_0 [0,128), S_1 [128,256) (double-buffered 128 x 128 scores; P of a key tile is written over the
//          first 64 columns of its S buffer), O [256,512).
//   SMEM   Q (128 x 256 bf16, 64 KB) + a ring of five 32 KB slots.  A key tile (128 keys) is K in two slots
//          (two 64-column chunks each) and V in two slots (64 keys with all four column chunks each), so a
//          QK^T is 16 MMAs of N = 128 and a PV 8 of N = 256, and each slot is handed back to the producer as
//          soon as the MMAs that read it are complete: the loads of the next tile start while the current
//          one is still being multiplied.
//   warps  0: work fetcher + TMA producer; 1: MMA issuer (one thread); 2-3: no role; 4-7: softmax (thread r
//          owns query row r = TMEM lane r).
// The issuer runs PV(j) then QK^T(j+2) into the buffer PV(j) has just read, with no wait between them
// (tcgen05.mma operations issued by one thread execute in issue order), so the softmax always finds the next
// S ready while the tensor core works on the key tile after it.  Work items are 128 query rows of one
// (batch|sequence, head), handed out heaviest-first from the same device counters as prefill.cuh.
#pragma once

#include "prefill.cuh"

namespace eta {

struct WideCfg {
  static constexpr int D = 256;
  static constexpr int BN = 128;                         // keys per key tile
  static constexpr int KCH = D / 64;                     // 128-byte column chunks per row
  static constexpr int Q_CHUNK = PF_BM * 128;            // 128 rows x 128 B
  static constexpr int Q_TILE = KCH * Q_CHUNK;           // 64 KB
  static constexpr int K_CHUNK = BN * 128;               // one column chunk of a K tile: 128 keys x 128 B
  // The K/V ring is made of equal slots.  A K slot holds KC_PER_SLOT column chunks of one key tile (all 128
  // keys); a V slot holds V_ROWS keys of one key tile with every column chunk (V_CHUNK bytes each), so the
  // QK^T k-steps and the PV k-steps each consume their slots in order and release them one by one.  (16 KB
  // slots -- ten of them -- measured 16 % slower: twice the barrier waits and commits on the issuer thread.)
  static constexpr int KC_PER_SLOT = 2;
  static constexpr int SLOT = KC_PER_SLOT * K_CHUNK;
  static constexpr int V_ROWS = SLOT / (KCH * 128);      // 64 keys
  static constexpr int V_CHUNK = V_ROWS * 128;
  static constexpr int K_SLOTS = KCH / KC_PER_SLOT;      // slots per K tile
  static constexpr int V_SLOTS = BN / V_ROWS;            // slots per V tile
  static constexpr int NSLOT = 5;                        // 160 KB of ring
  static constexpr int NSB = 2;                          // S buffers
  static constexpr uint32_t TM_O = 256;
  static constexpr int THREADS = 256;
  // barriers: full/empty per slot; q_full, q_empty; item_full[2], item_empty[2]; s_full, p_full and pv_done
  // per S buffer; o_free; mma_done.  The S, P and PV barriers are per buffer because with two S buffers the
  // softmax runs up to a key tile ahead of the tensor core: one shared barrier could then be two phases from
  // its waiter, and a parity wait cannot tell that from being done.  Per buffer, the previous phase of each
  // barrier is always complete when it is waited on (a key tile's QK^T is issued after the PV two tiles back).
  static constexpr int NBAR = 2 * NSLOT + 2 + 4 + 3 * NSB + 2;
  static constexpr int SMEM_BYTES = 1024 + Q_TILE + NSLOT * SLOT + NBAR * 8 + 2 * (int)sizeof(PfItem) + 16;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
  static_assert(K_SLOTS * KC_PER_SLOT == KCH && V_SLOTS * V_ROWS == BN && V_ROWS % 16 == 0, "slot shapes");
};

struct WideSmem {
  using C = WideCfg;
  static constexpr int OFF_KV = C::Q_TILE;
  static constexpr int OFF_BAR = OFF_KV + C::NSLOT * C::SLOT;
  static constexpr int B_FULL = 0, B_EMPTY = C::NSLOT, B_QFULL = 2 * C::NSLOT, B_QEMPTY = B_QFULL + 1,
                       B_ITEM_FULL = B_QEMPTY + 1, B_ITEM_EMPTY = B_ITEM_FULL + 2, B_S_FULL = B_ITEM_EMPTY + 2,
                       B_P_FULL = B_S_FULL + C::NSB, B_PV_DONE = B_P_FULL + C::NSB, B_O_FREE = B_PV_DONE + C::NSB,
                       B_MMA_DONE = B_O_FREE + 1, B_END = B_MMA_DONE + 1;
  static_assert(B_END == C::NBAR, "barrier count");
  static constexpr int OFF_ITEMS = OFF_BAR + C::NBAR * 8;
  static constexpr int OFF_TMEM_SLOT = OFF_ITEMS + 2 * (int)sizeof(PfItem);
  static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 4;
  uint8_t *base;
  __device__ explicit WideSmem(uint8_t *smem) : base(smem) {}
  __device__ __forceinline__ uint64_t *bar(int i) const { return reinterpret_cast<uint64_t *>(base + OFF_BAR) + i; }
  __device__ __forceinline__ uint8_t *sQ() const { return base; }
  __device__ __forceinline__ uint8_t *sKV() const { return base + OFF_KV; }
  __device__ __forceinline__ uint64_t *full(int i) const { return bar(B_FULL + i); }
  __device__ __forceinline__ uint64_t *empty(int i) const { return bar(B_EMPTY + i); }
  __device__ __forceinline__ uint64_t *q_full() const { return bar(B_QFULL); }
  __device__ __forceinline__ uint64_t *q_empty() const { return bar(B_QEMPTY); }
  __device__ __forceinline__ uint64_t *item_full(int i) const { return bar(B_ITEM_FULL + i); }
  __device__ __forceinline__ uint64_t *item_empty(int i) const { return bar(B_ITEM_EMPTY + i); }
  __device__ __forceinline__ uint64_t *s_full(int b) const { return bar(B_S_FULL + b); }  // S buffer b ready
  __device__ __forceinline__ uint64_t *p_full(int b) const { return bar(B_P_FULL + b); }  // P_b written, O rescaled
  __device__ __forceinline__ uint64_t *pv_done(int b) const { return bar(B_PV_DONE + b); }  // O += P_b V done
  __device__ __forceinline__ uint64_t *o_free() const { return bar(B_O_FREE); }           // epilogue read O
  __device__ __forceinline__ uint64_t *mma_done() const { return bar(B_MMA_DONE); }
  __device__ __forceinline__ PfItem *items() const { return reinterpret_cast<PfItem *>(base + OFF_ITEMS); }
  __device__ __forceinline__ uint32_t *tmem_slot() const {
    return reinterpret_cast<uint32_t *>(base + OFF_TMEM_SLOT);
  }
  __device__ __forceinline__ volatile int *abort_flag() const {
    return reinterpret_cast<volatile int *>(base + OFF_ABORT);
  }
};

// Work item `idx` (128-row blocks; packed: the latest block of every (sequence, head) first; dense: units
// in L2-sized groups, heaviest block first inside a group -- the order of decode_item).  n0 = key tiles the
// block sees.
template <int MODE>
__device__ __forceinline__ PfItem wide_decode_item(const PrefillParams &p, int idx) {
  PfItem it{};
  int blk;
  if constexpr (MODE != MODE_DENSE) {
    const int per = p.S * p.H;
    blk = p.nblk - 1 - idx / per;
    const int rem = idx - (idx / per) * per;
    const int s = rem / p.H;
    it.h = rem - s * p.H;
    packed_sequence(p, s, blk == 0 && it.h == 0, it.seq_start, it.L);
  } else {
    dense_unit_block(p, idx, it.bh, blk);
    it.L = p.N;
  }
  it.r0 = blk * PF_BM;
  const int e = (it.r0 >= it.L) ? 0 : (p.causal ? min(it.L, it.r0 + PF_BM) : it.L);
  it.n0 = (e + WideCfg::BN - 1) / WideCfg::BN;
  it.n1 = 0;
  it.split = 0;
  it.stop = 0;
  return it;
}

template <int MODE>
__device__ __forceinline__ void wide_control(const CUtensorMap &tmQ, const CUtensorMap &tmK, const CUtensorMap &tmV,
                                             const PrefillParams &p, uint8_t *smem, uint32_t tmem, int warp,
                                             int lane) {
  using C = WideCfg;
  constexpr bool PACKED = (MODE != MODE_DENSE);
  WideSmem sm(smem);
  if (warp == 0) {
    // ================================================================ work fetcher + TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      bool retired = false;
      auto retire = [&]() {
        retired = true;
        __threadfence();
        if (atomicAdd(&g_pf_sched[p.sched_slot][1], 1u) == gridDim.x - 1) {
          __threadfence();
          atomicExch(&g_pf_sched[p.sched_slot][0], 0u);
          atomicExch(&g_pf_sched[p.sched_slot][1], 0u);
        }
      };
      int kv_issued = 0, q_issued = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        PfItem it;
        for (bool first = (k == 0);; first = false) {
          const unsigned int idx = first ? blockIdx.x : gridDim.x + atomicAdd(&g_pf_sched[p.sched_slot][0], 1u);
          if (idx >= (unsigned int)p.n_items) {
            it = PfItem{};
            it.stop = 1;
            retire();
            break;
          }
          it = wide_decode_item<MODE>(p, (int)idx);
          if (it.r0 < it.L) break;
        }
        ok = mbar_wait(sm.item_empty(k & 1), ((k >> 1) & 1) ^ 1, sm.abort_flag(), p.wait_ns);
        if (!ok) break;
        sm.items()[k & 1] = it;
        mbar_arrive(sm.item_full(k & 1));
        if (it.stop) break;
        if (k > 0) {
          ok = mbar_wait(sm.q_empty(), (k - 1) & 1, sm.abort_flag(), p.wait_ns);
          if (!ok) break;
        }
        mbar_arrive_expect_tx(sm.q_full(), C::Q_TILE);
#pragma unroll
        for (int c = 0; c < C::KCH; ++c) {
          uint8_t *dst = sm.sQ() + c * C::Q_CHUNK;
          if constexpr (PACKED)
            tma_load_3d(dst, &tmQ, sm.q_full(), 64 * c, it.h, it.seq_start + it.r0);
          else
            tma_load_3d(dst, &tmQ, sm.q_full(), 64 * c, it.r0, it.bh);
        }
        ++q_issued;
        // Slots in the order the issuer consumes them: K_0, K_1, then V_j, K_{j+2} for each key tile j.
        auto acquire = [&]() {
          const int st = kv_issued % C::NSLOT;
          if (!mbar_wait(sm.empty(st), ((kv_issued / C::NSLOT) & 1) ^ 1, sm.abort_flag(), p.wait_ns)) return -1;
          mbar_arrive_expect_tx(sm.full(st), C::SLOT);
          return st;
        };
        auto load_k = [&](int j) {
          for (int s = 0; s < C::K_SLOTS; ++s) {
            const int st = acquire();
            if (st < 0) return false;
#pragma unroll
            for (int c2 = 0; c2 < C::KC_PER_SLOT; ++c2) {
              uint8_t *dst = sm.sKV() + st * C::SLOT + c2 * C::K_CHUNK;
              const int x = 64 * (s * C::KC_PER_SLOT + c2);
              if constexpr (PACKED)
                tma_load_3d(dst, &tmK, sm.full(st), x, it.h, it.seq_start + j * C::BN);
              else
                tma_load_3d(dst, &tmK, sm.full(st), x, j * C::BN, it.bh);
            }
            ++kv_issued;
          }
          return true;
        };
        auto load_v = [&](int j) {
          for (int s = 0; s < C::V_SLOTS; ++s) {
            const int st = acquire();
            if (st < 0) return false;
            const int r = j * C::BN + s * C::V_ROWS;
#pragma unroll
            for (int c = 0; c < C::KCH; ++c) {
              uint8_t *dst = sm.sKV() + st * C::SLOT + c * C::V_CHUNK;
              if constexpr (PACKED)
                tma_load_3d(dst, &tmV, sm.full(st), 64 * c, it.h, it.seq_start + r);
              else
                tma_load_3d(dst, &tmV, sm.full(st), 64 * c, r, it.bh);
            }
            ++kv_issued;
          }
          return true;
        };
        const int n = it.n0;
        ok = load_k(0) && (n < 2 || load_k(1));
        for (int j = 0; ok && j < n; ++j) ok = load_v(j) && (j + 2 >= n || load_k(j + 2));
      }
      if (!retired) retire();
      if (!ok) {
        if (q_issued > 0) mbar_wait(sm.q_full(), (q_issued - 1) & 1, nullptr, p.wait_ns);
        for (int i = max(0, kv_issued - C::NSLOT); i < kv_issued; ++i)
          mbar_wait(sm.full(i % C::NSLOT), (i / C::NSLOT) & 1, nullptr, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_QK = idesc_bf16_f32(PF_BM, C::BN, false);
      constexpr uint32_t ID_PV = idesc_bf16_f32(PF_BM, C::D, true);
      const uint32_t sQa = smem_u32(sm.sQ()), sKVa = smem_u32(sm.sKV());
      const uint64_t dQ = sdesc_sw128(sQa, 16, 1024), dK = sdesc_sw128(sKVa, 16, 1024);
      const uint64_t dV = sdesc_sw128(sKVa, C::V_CHUNK, 1024);
      int g = 0;  // ring slots consumed, over all items
      bool ok = true;
      auto slot_wait = [&]() {
        ok = ok && mbar_wait(sm.full(g % C::NSLOT), (g / C::NSLOT) & 1, sm.abort_flag(), p.wait_ns);
        if (ok) tc_fence_after();
        return (uint64_t)(((g % C::NSLOT) * C::SLOT) >> 4);
      };
      auto slot_release = [&]() {
        mma_commit(sm.empty(g % C::NSLOT));
        ++g;
      };
      // S_b = Q K^T : 16 k-steps of 16 head-dim elements (32 bytes inside a 128-byte swizzled row), N = 128;
      // each K slot is released once the k-steps that read it are complete.
      auto issue_s = [&](int b) {
        const uint32_t dt = tmem + (uint32_t)(C::BN * b);
        eta_static_for<C::K_SLOTS>([&](auto s_c) {
          constexpr int s = decltype(s_c)::value;
          const uint64_t so = slot_wait();
          if (!ok) return;
          const uint64_t db = dK + so;
          eta_static_for<4 * C::KC_PER_SLOT>([&](auto i_c) {
            constexpr int kk = s * 4 * C::KC_PER_SLOT + decltype(i_c)::value;
            constexpr uint32_t a_off = ((uint32_t)(kk >> 2) * C::Q_CHUNK + (uint32_t)(kk & 3) * 32u) >> 4;
            constexpr uint32_t b_off =
                ((uint32_t)((kk >> 2) % C::KC_PER_SLOT) * C::K_CHUNK + (uint32_t)(kk & 3) * 32u) >> 4;
            mma_ss_off<a_off, b_off>(dt, dQ, db, ID_QK, kk > 0 ? 1u : 0u);
          });
          slot_release();
        });
        if (ok) mma_commit(sm.s_full(b));
        return ok;
      };
      // O += P_b V : 8 k-steps of 16 keys (8 TMEM columns of packed bf16 P; 16 rows = 2048 B of each column
      // chunk of a V slot), N = 256
      auto issue_pv = [&](int b, bool acc) {
        const uint32_t tP = tmem + (uint32_t)(C::BN * b);
        const uint32_t acc0 = acc ? 1u : 0u;
        eta_static_for<C::V_SLOTS>([&](auto s_c) {
          constexpr int s = decltype(s_c)::value;
          const uint64_t so = slot_wait();
          if (!ok) return;
          const uint64_t db = dV + so;
          eta_static_for<C::V_ROWS / 16>([&](auto i_c) {
            constexpr int ki = decltype(i_c)::value;
            constexpr int kk = s * (C::V_ROWS / 16) + ki;
            constexpr uint32_t ta_off = 8u * kk, b_off = (2048u * ki) / 16u;
            mma_ts_off<ta_off, b_off>(tmem + C::TM_O, tP, db, ID_PV, kk > 0 ? 1u : acc0);
          });
          slot_release();
        });
        return ok;
      };
      int gs = 0, gp = 0, go = 0;  // S issued, PV issued, items done (over all items)
      for (int k = 0; ok; ++k) {
        ok = mbar_wait(sm.item_full(k & 1), (k >> 1) & 1, sm.abort_flag(), p.wait_ns);
        if (!ok) break;
        const PfItem it = sm.items()[k & 1];
        mbar_arrive(sm.item_empty(k & 1));
        if (it.stop) break;
        const int n = it.n0;  // >= 1
        ok = mbar_wait(sm.q_full(), k & 1, sm.abort_flag(), p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        // S(j) goes to buffer (gs of that S) % NSB.  The first two of an item follow the previous item's last
        // PVs in issue order, which is all the buffers need.
        auto s_step = [&](int j) {
          if (!issue_s(gs % C::NSB)) return false;
          ++gs;
          if (j == n - 1) mma_commit(sm.q_empty());  // every QK^T of this item is issued
          return true;
        };
        ok = s_step(0) && (n < 2 || s_step(1));
        for (int j = 0; ok && j < n; ++j) {
          ok = mbar_wait(sm.p_full(gp % C::NSB), (gp / C::NSB) & 1, sm.abort_flag(), p.wait_ns) &&
               (j > 0 || go == 0 || mbar_wait(sm.o_free(), (go - 1) & 1, sm.abort_flag(), p.wait_ns));
          if (!ok) break;
          tc_fence_after();
          if (!issue_pv(gp % C::NSB, j > 0)) break;
          mma_commit(sm.pv_done(gp % C::NSB));
          ++gp;
          if (j + 2 < n) ok = s_step(j + 2);  // into the buffer PV(j) has just read, in issue order after it
        }
        ++go;
      }
      mma_commit(sm.mma_done());
      mbar_wait(sm.mma_done(), 0, nullptr, p.wait_ns);
    }
    __syncwarp();
  }
}

// Softmax warpgroup (warps 4-7): thread (quarter, lane) owns query row 32 quarter + lane.
template <int MODE>
__device__ __forceinline__ void wide_softmax(const PrefillParams &p, uint8_t *smem, uint32_t tmem, int warp,
                                             int lane) {
  using C = WideCfg;
  constexpr int BN = C::BN, D = C::D;
  constexpr bool PACKED = (MODE != MODE_DENSE);
  WideSmem sm(smem);
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
  const uint32_t tO = tmem + lane_addr + C::TM_O;
  const bool causal = (p.causal != 0);
  int gj = 0;  // key tiles processed over all items: S buffer gj % NSB, phases of s_full / p_full / pv_done
  bool ok = true;
  for (int k = 0; ok; ++k) {
    ok = mbar_wait(sm.item_full(k & 1), (k >> 1) & 1, sm.abort_flag(), p.wait_ns);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    const PfItem it = sm.items()[k & 1];
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.item_empty(k & 1));
    if (it.stop) break;
    const int L = it.L, q_start = it.r0, qpos = q_start + row, n = it.n0;
    const size_t orow = PACKED ? ((size_t)(it.seq_start + qpos) * p.H + it.h) : ((size_t)it.bh * p.N + qpos);
    float m_used = -INFINITY, l = 0.f;
    for (int j = 0; j < n; ++j, ++gj) {
      const int b = gj % C::NSB;
      const uint32_t tS = tmem + lane_addr + (uint32_t)(BN * b);
      ok = mbar_wait(sm.s_full(b), (gj / C::NSB) & 1, sm.abort_flag(), p.wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[BN];
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) ETA_TMEM_LD_X32(tS + 32u * cc, (sr + 32 * cc));
      tmem_wait_ld();
      const int k0 = j * BN;
      const bool need_mask = (k0 + BN > L) || (causal && k0 + BN - 1 > q_start);
      const int kmax = causal ? min(L - 1, qpos) - k0 : L - 1 - k0;
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c > kmax) sr[c] = __float_as_uint(-INFINITY);
      }
      float mxa = -INFINITY, mxb = -INFINITY, mxc = -INFINITY, mxd = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN; c += 8) {
        mxa = max3f(mxa, __uint_as_float(sr[c + 0]), __uint_as_float(sr[c + 1]));
        mxb = max3f(mxb, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
        mxc = max3f(mxc, __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
        mxd = max3f(mxd, __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
      }
      const float mx = max3f(mxa, mxb, fmaxf(mxc, mxd)) * p.scale_log2;
      bool resc = false;
      float m_new = m_used;
      if (mx > m_used + PF_RESCALE_THRESHOLD) {
        m_new = mx;
        resc = true;
      }
      const float msub = (m_new == -INFINITY) ? 0.f : m_new;
      const uint64_t cs2 = f2pack(p.scale_log2, p.scale_log2), nm2 = f2pack(-msub, -msub);
      uint64_t rs_a = f2pack(0.f, 0.f), rs_b = f2pack(0.f, 0.f);
      uint32_t pk[BN / 2];
#pragma unroll
      for (int i = 0; i < BN / 2; ++i) {
        const uint64_t x2 = fma_x2(f2pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), cs2, nm2);
        float x0, x1;
        f2unpack(x2, x0, x1);
        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
        if (i & 1) rs_b = add_x2(rs_b, f2pack(p0, p1));
        else rs_a = add_x2(rs_a, f2pack(p0, p1));
        pk[i] = pack_bf16x2(p0, p1);
      }
      float r0a, r1a, r2a, r3a;
      f2unpack(rs_a, r0a, r1a);
      f2unpack(rs_b, r2a, r3a);
      const float f = resc ? ex2_approx(m_used - msub) : 1.f;
      // The previous key tile's PV must be complete before this tile's P is written (this S was issued
      // before that PV, so nothing else orders them).  Letting the softmax run a tile ahead of it -- P
      // written, and the next PV issued, while the previous PV into O was still executing behind a QK^T --
      // produced wrong O columns when tried.
      if (gj > 0) {
        ok = mbar_wait(sm.pv_done((gj - 1) % C::NSB), ((gj - 1) / C::NSB) & 1, sm.abort_flag(), p.wait_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
      }
      // P over the first BN/2 columns of this S buffer (read just above)
#pragma unroll
      for (int cc = 0; cc < BN / 64; ++cc) ETA_TMEM_ST_X32(tS + 32u * cc, (pk + 32 * cc));
      if (__any_sync(0xffffffffu, resc && j > 0)) {
        const uint64_t f2 = f2pack(f, f);
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t orr[32];
          ETA_TMEM_LD_X32(tO + 32u * cc, orr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float a, c;
            f2unpack(mul_x2(f2pack(__uint_as_float(orr[2 * i]), __uint_as_float(orr[2 * i + 1])), f2), a, c);
            orr[2 * i] = __float_as_uint(a);
            orr[2 * i + 1] = __float_as_uint(c);
          }
          ETA_TMEM_ST_X32(tO + 32u * cc, orr);
        }
      }
      l = l * f + ((r0a + r1a) + (r2a + r3a));
      m_used = m_new;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.p_full(b));
    }
    if (!ok) break;
    // ---------------------------------------------------------------- epilogue of the item
    // (the last PV accumulates after all earlier ones, so its completion covers them)
    ok = mbar_wait(sm.pv_done((gj - 1) % C::NSB), ((gj - 1) / C::NSB) & 1, sm.abort_flag(), p.wait_ns);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    tc_fence_after();
    const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
    const bool valid = qpos < L;
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t orr[32];
      ETA_TMEM_LD_X32(tO + 32u * cc, orr);
      tmem_wait_ld();
      if (cc == D / 32 - 1) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sm.o_free());
      }
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
    if (valid && p.lse != nullptr)
      p.lse[orow] = (l > 0.f) ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
  }
}

template <int MODE>
__global__ void __launch_bounds__(WideCfg::THREADS, 1)
    prefill_wide_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = WideCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  WideSmem sm(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(sm.full(i), 1);
      mbar_init(sm.empty(i), 1);
    }
    mbar_init(sm.q_full(), 1);
    mbar_init(sm.q_empty(), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(sm.item_full(i), 1);
      mbar_init(sm.item_empty(i), 1 + 4);  // the issuer and the four softmax warps read each item
    }
    for (int b = 0; b < C::NSB; ++b) mbar_init(sm.s_full(b), 1);
    for (int b = 0; b < C::NSB; ++b) mbar_init(sm.p_full(b), 4);
    for (int b = 0; b < C::NSB; ++b) mbar_init(sm.pv_done(b), 1);
    mbar_init(sm.o_free(), 4);
    mbar_init(sm.mma_done(), 1);
    *sm.abort_flag() = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sm.tmem_slot(), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot();
  if (warp < 4) wide_control<MODE>(tmQ, tmK, tmV, p, smem, tmem, warp, lane);
  else wide_softmax<MODE>(p, smem, tmem, warp, lane);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace eta
