// prefill.cuh -- fused exact attention forward (dense and packed/varlen) and HSTU pointwise attention, one
// persistent kernel template for B200 (sm_100a): TMA tile loads, tcgen05 MMAs accumulating in tensor
// memory (TMEM), warp-specialised softmax, in-kernel causal mask with masked tiles skipped.
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
// Work decomposition: a work item is 256 query rows of one (batch, head) or (sequence, head) -- two 128-row
// Q tiles -- streaming the key/value tiles (128 rows each) its rows can see.  Causal tiles past the
// diagonal are never loaded (the "after the diagonal: all zero, skip" class of the HSTU page's in-kernel
// mask); only the diagonal tile and a ragged last tile evaluate a per-element mask.  The grid is persistent
// (at most one CTA per SM): CTAs take items from a device counter -- dense launches unit group by unit group
// (so a group's K/V stay in L2), heaviest row block first inside a group -- and keep their pipeline running
// across items, so the next item's Q, K/V and first QK^T overlap the current item's epilogue.  Split items
// (one 128-row Q tile whose key range is halved between the two softmax warpgroups, the halves merged inside
// the CTA: exact, the same rescale identity as the online softmax) serve two cases the host decides: the
// last wave of a non-causal launch when at most half full, and every item of a launch too small to fill
// the GPU.
//
// Roles (12 warps):
//   warp 0      work fetcher + TMA producer: publishes each item to the other roles through a 2-deep ring,
//               then loads its Q0, Q1 and K_0, V_0, K_1, V_1, ... through an NST-stage ring.
//   warps 1, 2  MMA issuers (one thread each; warp 1 also owns TMEM):  S_t = Q_t K_j^T (SS form) into
//               TMEM, O_t += P_t V_j (TS form: P read from TMEM, V from shared memory).
//   warp 3      no role.
//   warps 4-11  two softmax warpgroups, one per Q tile; thread r owns query row r = TMEM lane r.
//
// TMEM (512 columns x 128 lanes): S_0 [0,128), S_1 [128,256), O_t at 256 + t * O_COLS (O_COLS = D rounded up
// to whole 64-column chunks: 64 for D = 64, 128 for D = 96 and 128).
//   D = 64: P_t has its own columns [384+64t, 448+64t); issuer 1+t serves Q tile t and issues the next
//           S_t as soon as the softmax has copied S_t to registers.  Two Q slots in shared memory: the
//           next item's Q tiles load while the current item runs.
//   D = 96: 96-key tiles, so S_t uses 96 of its 128 columns and O_t 96 of its 128; P_t (48 columns) lives
//           in those spare columns (keys [0, 64) after S_t, keys [64, 96) after O_t) and the D = 64 flow
//           applies: one issuer per tile, the next S_t issued as soon as S_t has been read.
//   D = 128 (and e4m3): TMEM is full; P_t overwrites the first columns of S_t and one issuer (warp 1) runs
//           PV_0(j), S_0(j+1), PV_1(j), S_1(j+1) with no wait between a PV and the next QK^T: tcgen05.mma
//           operations issued by one thread execute in issue order, so the QK^T's writes follow the PV's
//           reads of P, and the QK^T's commit also covers the PV (a softmax that has seen the new S may
//           rescale O).  The single ordered stream keeps the two softmax warpgroups half a period apart.
//
// Online-softmax rescale is conditional: the running max used for exponentiation is only raised when a
// row's block max exceeds it by more than 8 (log2 units).  The final O / l and lse use the same stale max
// consistently, so the result is exact (up to rounding) while most key tiles skip the O rescale.
#pragma once

#include <type_traits>
#include <utility>

#include "ptx.cuh"

namespace eta {

// Calls f(std::integral_constant<int, i>) for i = 0 .. N-1 (a loop whose index is a compile-time constant).
template <int N, typename F, int... I>
__device__ __forceinline__ void eta_static_for_impl(F &&f, std::integer_sequence<int, I...>) {
  (f(std::integral_constant<int, I>{}), ...);
}
template <int N, typename F>
__device__ __forceinline__ void eta_static_for(F &&f) {
  eta_static_for_impl<N>(f, std::make_integer_sequence<int, N>{});
}

constexpr int PF_BM = 128;            // query rows per Q tile (= TMEM lanes)
constexpr int PF_SM_WARPS = 8;        // softmax warps: 2 Q tiles x 4 lane quarters (one thread per query row)
constexpr int PF_THREADS = 32 * (4 + PF_SM_WARPS);  // + control warpgroup: TMA, 2 MMA issuers, 1 spare
// Register split (setmaxnreg): the CTA launches with PF_LAUNCH_REGS per thread; the control warpgroup drops
// to PF_CTRL_REGS and the two softmax warpgroups grow to PF_SM_REGS.  The shares add up to the launch total
// exactly, and the host refuses to launch a build whose register count is not PF_LAUNCH_REGS (a larger
// request than the launch total would stall forever).
constexpr int PF_LAUNCH_REGS = 168, PF_CTRL_REGS = 56, PF_SM_REGS = 224;
static_assert(128 * PF_CTRL_REGS + 32 * PF_SM_WARPS * PF_SM_REGS == PF_THREADS * PF_LAUNCH_REGS, "register split");
constexpr float PF_RESCALE_THRESHOLD = 8.0f;  // log2 units
// Work counters of the persistent scheduler, one pair per launch in flight, handed out round-robin by the
// host: [slot][0] = next item, [slot][1] = CTAs that took their last item.  The last CTA of a launch to take
// its last item resets the pair to zero for the launch that reuses the slot.
constexpr int PF_SCHED_SLOTS = 256;
__device__ unsigned int g_pf_sched[PF_SCHED_SLOTS][2];

enum PrefillMode { MODE_DENSE = 0, MODE_VARLEN = 1, MODE_HSTU = 2 };

struct PrefillParams {
  void *o;                 // dense: [B,H,N,D]; packed: [T,H,D]; bf16 or fp32
  float *lse;              // dense: [B,H,N]; packed: [T,H]; may be null
  const int *cu_seqlens;   // packed modes: [S+1]
  int H, N, max_len;       // N: dense sequence length
  int BH, S;               // dense: B*H; packed: number of sequences
  int T_total;             // packed: rows of q/k/v/o (the last offset the host was given)
  int grp;                 // dense: (batch, head) units per scheduling group (see decode_item)
  int nblk;                // 256-row blocks per (batch|sequence, head)
  int n_items;             // work indices: n_whole whole items, then two split halves per remaining item
  int n_whole;             // items (in heaviest-first order) processed whole; the rest are split
  int sched_slot;
  int causal, o_f32;
  float scale_log2;        // softmax: scale * log2(e)
  float hstu_half_alpha;   // HSTU: 0.5 * alpha      (tanh argument scale)
  float hstu_inv_n;        // HSTU: inv_n (applied to O at the end of an item)
  float o_scale;           // multiplies O / l (1; the V descale factor for e4m3 inputs)
  long long wait_ns;
};

// One work item as the producer publishes it to the other roles.
struct PfItem {
  int bh, h, seq_start, L;  // dense: bh; packed: head and first packed row of the sequence; rows L
  int r0;                   // first query row of the item (whole: tile t starts at r0 + 128 t)
  int n0, n1;               // whole: key tiles seen by Q tile 0 / 1; split: key tiles [0,n0) / [n0,n0+n1)
  int split;                // one Q tile at r0, its keys halved between the two softmax warpgroups
  int stop;                 // no more work
};

// Item-local position of a K (v = 0) or V (v = 1) tile load in the K/V ring.  Whole items load K_0, V_0,
// K_1, V_1, ... (each shared by both Q tiles).  Split items load, per step j, K_j, K_{n0+j}, V_j, V_{n0+j}
// (the second warpgroup's pair only while j < n1).
__device__ __forceinline__ int kv_pos(const PfItem &it, int t, int j, int v) {
  if (!it.split) return 2 * j + v;
  const int g = 2 * j + 2 * min(j, it.n1);
  return g + (v ? (j < it.n1 ? 2 : 1) : 0) + t;
}
// Loads of the item in the ring.
__device__ __forceinline__ int kv_loads(const PfItem &it) {
  return it.split ? 2 * (it.n0 + it.n1) : 2 * max(it.n0, it.n1);
}
// Whether ring position `pos` of the item is read by Q tile (warpgroup) t.
__device__ __forceinline__ bool kv_owned(const PfItem &it, int t, int pos) {
  if (!it.split) return pos < 2 * (t ? it.n1 : it.n0);
  return pos < 4 * it.n1 ? ((pos & 1) == t) : (t == 0);
}

// F8: Q, K, V are e4m3 (one byte per element), P is rounded to e4m3 for the PV MMA (kind::f8f6f4).
template <int D, bool F8 = false>
struct PfCfg {
  static constexpr int ELT = F8 ? 1 : 2;                 // bytes per input element
  static constexpr int ROW_BYTES = D * ELT;
  // Keys per K/V tile.  (At d = 128, 64-key tiles would leave TMEM room for a separate P -- 2 S + 2 O + 2 P =
  // 128 + 256 + 64 columns -- so that the next QK^T need not follow the PV that reads P; measured, the
  // halved tiles cost more in per-tile overhead and MMA latency than that saves: 11 % slower.)
  // (d = 96: 96-key tiles, so that a separate P fits in TMEM; see P_IN_HOLES.)
  static constexpr int BN = (D == 96 && !F8) ? 96 : 128;
  static constexpr int P_COLS = BN * ELT / 4;            // TMEM columns of one tile's P (bf16 or e4m3, packed)
  // 128-byte column chunks per row.  A row that is not a whole number of chunks (d = 96: 192 bytes) has its
  // last chunk half filled by the TMA's zero fill past the tensor's inner extent; the MMAs never read the
  // zeros (Q K^T stops at ROW_BYTES, P V has N = D).
  static constexpr int KCH = (ROW_BYTES + 127) / 128;
  // TMEM columns reserved per O tile: the head dim rounded up to whole chunks (d = 96 keeps 128).
  static constexpr int O_COLS = KCH * 128 / ELT;
  // S_t takes 128 columns from S_STRIDE * t (BN of them used).  d = 96: P_t goes into the spare columns, keys
  // [0, 64) into S_t's [96, 128) and keys [64, 96) into O_t's [96, 112), so that every tile has its own P
  // (no PV -> next QK^T chain) while S and O keep 128-column slots.  Otherwise P overwrites S's first columns
  // when S, O and P of both tiles do not fit in 512 TMEM columns.
  static constexpr int S_STRIDE = 128;
  static constexpr bool P_IN_HOLES = (D == 96 && !F8);
  static constexpr bool ALIAS_P = !P_IN_HOLES && (2 * BN + 2 * O_COLS + 2 * P_COLS) > 512;
  static constexpr int N_ISSUERS = ALIAS_P ? 1 : 2;
  static constexpr int Q_CHUNK = PF_BM * 128;            // 128 rows x 128 B
  static constexpr int Q_TILE = KCH * Q_CHUNK;           // one 128 x D Q tile
  static constexpr int KV_CHUNK = BN * 128;              // BN rows x 128 B
  static constexpr int KV_TILE = KCH * KV_CHUNK;         // one BN x D K or V tile
  static constexpr int QK_STEPS = ROW_BYTES / 32;        // K-steps of Q K^T: 32 bytes (16 bf16 or 32 e4m3) each
  static constexpr int PV_KEYS = 32 / ELT;               // keys per K-step of P V (8 TMEM columns of P)
  // K/V ring depth (each stage holds one tile).  d = 96 takes six 24 KB stages and one Q slot (four stages
  // and two Q slots measured 6 % slower at B8 H32 N4096 causal, 8 % non-causal).
  static constexpr int NST = (KV_TILE <= 16384) ? 8 : (P_IN_HOLES ? 6 : 4);
  // HSTU: of every 8 tanh pairs, how many go to the FMA-pipe polynomial (when in range) instead of the MUFU.
  // With a separate P (d = 64, 96) both softmax warpgroups run at once and share the MUFU; moving 3 of 8
  // measured +10 % (jagged) and +13 % (dense) over 0, 2 or 4 of 8 at d = 64.  With P aliased into S (d = 128)
  // the warpgroups take turns and the MUFU is not the shared resource, so all stay on it.
  static constexpr int TANH_FMA_PAIRS = ALIAS_P ? 0 : 3;
  // barriers: full/empty per stage; q_full[2], q_empty[2]; item_full[2], item_empty[2];
  // per tile {s_full, s_free, p_full, pv_done, o_free, mma_done}
  static constexpr int NBAR = 2 * NST + 4 + 4 + 2 * 6;
  static constexpr int SMEM_FIXED = 1024 /*alignment slack*/ + NST * KV_TILE + NBAR * 8 +
                                    2 * (int)sizeof(PfItem) + PF_BM * 8 /*split merge*/ + 16;
  // Slots for the two Q tiles of an item: two where they fit (d = 64, e4m3), so that the next item's Q is
  // loaded while the current item still runs and its first QK^T is ready when the softmax gets to it.
  static constexpr int QSLOTS = (SMEM_FIXED + 4 * Q_TILE <= 227 * 1024) ? 2 : 1;
  static constexpr int SMEM_BYTES = SMEM_FIXED + QSLOTS * 2 * Q_TILE;
  // TMEM columns: S_t at S_STRIDE*t, O_t at TM_O + O_COLS*t, P_t at TM_P + P_COLS*t (S_t's first columns if
  // ALIAS_P; S_t's and O_t's spare columns if P_IN_HOLES)
  static constexpr uint32_t TM_O = 2 * S_STRIDE;
  static constexpr uint32_t TM_P = 2 * S_STRIDE + 2 * O_COLS;
  static_assert(BN <= S_STRIDE && TM_P + ((ALIAS_P || P_IN_HOLES) ? 0 : 2 * P_COLS) <= 512, "TMEM columns");
  static_assert(!P_IN_HOLES || (BN == 96 && O_COLS == 128 && P_COLS == 48), "d = 96 P layout");
  static_assert(ROW_BYTES % 32 == 0 && D % 32 == 0 && D <= O_COLS, "head dim: whole K-steps and TMEM loads");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
};

// Shared-memory carve-up, common to every role.  Every member is the base address plus a compile-time
// offset, computed where it is used (nothing but the base stays live in registers).
template <int D, bool F8 = false>
struct PfSmem {
  using C = PfCfg<D, F8>;
  static constexpr int OFF_KV = C::QSLOTS * 2 * C::Q_TILE;
  static constexpr int OFF_BAR = OFF_KV + C::NST * C::KV_TILE;
  static constexpr int B_FULL = 0, B_EMPTY = C::NST, B_QFULL = 2 * C::NST, B_QEMPTY = B_QFULL + 2,
                       B_ITEM_FULL = B_QEMPTY + 2, B_ITEM_EMPTY = B_ITEM_FULL + 2, B_S_FULL = B_ITEM_EMPTY + 2,
                       B_S_FREE = B_S_FULL + 2, B_P_FULL = B_S_FREE + 2, B_PV_DONE = B_P_FULL + 2,
                       B_O_FREE = B_PV_DONE + 2, B_MMA_DONE = B_O_FREE + 2, B_END = B_MMA_DONE + 2;
  static_assert(B_END == C::NBAR, "barrier count");
  static constexpr int OFF_ITEMS = OFF_BAR + C::NBAR * 8;
  static constexpr int OFF_XCH = OFF_ITEMS + 2 * (int)sizeof(PfItem);
  static constexpr int OFF_TMEM_SLOT = OFF_XCH + PF_BM * 8;
  static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 4;
  uint8_t *base;
  __device__ explicit PfSmem(uint8_t *smem) : base(smem) {}
  __device__ __forceinline__ uint64_t *bar(int i) const { return reinterpret_cast<uint64_t *>(base + OFF_BAR) + i; }
  __device__ __forceinline__ uint8_t *sQ(int slot) const { return base + slot * 2 * C::Q_TILE; }
  __device__ __forceinline__ uint8_t *sKV() const { return base + OFF_KV; }
  __device__ __forceinline__ uint64_t *full(int i) const { return bar(B_FULL + i); }          // TMA -> MMA
  __device__ __forceinline__ uint64_t *empty(int i) const { return bar(B_EMPTY + i); }        // MMA -> TMA
  // Q slot: the item's Q tiles landed / every QK^T of the item completed (the slot may be overwritten)
  __device__ __forceinline__ uint64_t *q_full(int slot) const { return bar(B_QFULL + slot); }
  __device__ __forceinline__ uint64_t *q_empty(int slot) const { return bar(B_QEMPTY + slot); }
  // item ring: published by the producer / read by every consumer warp
  __device__ __forceinline__ uint64_t *item_full(int i) const { return bar(B_ITEM_FULL + i); }
  __device__ __forceinline__ uint64_t *item_empty(int i) const { return bar(B_ITEM_EMPTY + i); }
  // per Q tile t: S_t ready in TMEM (MMA -> softmax) / S_t copied to registers (softmax -> MMA; D = 64)
  __device__ __forceinline__ uint64_t *s_full(int t) const { return bar(B_S_FULL + t); }
  __device__ __forceinline__ uint64_t *s_free(int t) const { return bar(B_S_FREE + t); }
  // P_t written, O_t rescaled (softmax -> MMA) / O_t += P_t V complete (MMA -> softmax)
  __device__ __forceinline__ uint64_t *p_full(int t) const { return bar(B_P_FULL + t); }
  __device__ __forceinline__ uint64_t *pv_done(int t) const { return bar(B_PV_DONE + t); }
  // epilogue has read O_t (softmax -> MMA) / every MMA of issuer 1+t complete
  __device__ __forceinline__ uint64_t *o_free(int t) const { return bar(B_O_FREE + t); }
  __device__ __forceinline__ uint64_t *mma_done(int t) const { return bar(B_MMA_DONE + t); }
  __device__ __forceinline__ PfItem *items() const { return reinterpret_cast<PfItem *>(base + OFF_ITEMS); }
  // split items: (running max, exp-sum) of each query row of the second warpgroup's key half
  __device__ __forceinline__ float2 *xch() const { return reinterpret_cast<float2 *>(base + OFF_XCH); }
  __device__ __forceinline__ uint32_t *tmem_slot() const { return reinterpret_cast<uint32_t *>(base + OFF_TMEM_SLOT); }
  __device__ __forceinline__ volatile int *abort_flag() const {
    return reinterpret_cast<volatile int *>(base + OFF_ABORT);
  }
};

// Sequence s of a packed launch: its first row and length, checked against the launch's contract.  A
// sequence whose rows would leave [0, T_total) (a negative or decreasing offset, a length above max_len, an
// end past T_total) gets length 0 and is skipped, so no load or store of it happens; every breach of the
// contract (also a first offset other than 0 or a last one other than T_total, which stay in bounds) records
// ETA_DEV_BAD_CUSEQ once, from the sequence's block-0, head-0 item.
__device__ __forceinline__ void packed_sequence(const PrefillParams &p, int s, bool report, int &start, int &L) {
  const int a = p.cu_seqlens[s], b = p.cu_seqlens[s + 1];
  const bool unsafe = a < 0 || b < a || b - a > p.max_len || b > p.T_total;
  const bool off_contract = (s == 0 && a != 0) || (s == p.S - 1 && b != p.T_total);
  if ((unsafe || off_contract) && report) record_status(3 /* ETA_DEV_BAD_CUSEQ */);
  start = unsafe ? 0 : a;
  L = unsafe ? 0 : b - a;
}

// Dense work item `idx` -> (unit, row block).  Units ((batch, head) pairs) are taken in groups of p.grp,
// sized on the host so that one group's K and V stay resident in L2; inside a group the latest (heaviest,
// when causal) row block of every unit comes first.  The K/V tiles of a unit are then read from HBM about
// once, shared through L2 by its row blocks, instead of once per row block when all units run each level
// together.  The last group's light blocks still end the launch (heaviest-first tail).
__device__ __forceinline__ void dense_unit_block(const PrefillParams &p, int idx, int &unit, int &blk) {
  const int per_grp = p.grp * p.nblk;
  const int g = idx / per_grp;
  const int u0 = g * p.grp;
  const int gsz = min(p.grp, p.BH - u0);
  const int rem = idx - g * per_grp;
  blk = p.nblk - 1 - rem / gsz;
  unit = u0 + (rem - (rem / gsz) * gsz);
}

// Work item `idx`: packed launches take the latest row block of every (sequence, head) first; dense ones go
// group by group (dense_unit_block).
template <int D, int MODE, bool F8>
__device__ __forceinline__ PfItem decode_item(const PrefillParams &p, int idx) {
  constexpr int BN = PfCfg<D, F8>::BN;  // the key-tile size of the kernel instance that runs the item
  PfItem it{};
  int half = -1;
  if (idx >= p.n_whole) {  // split halves (only softmax launches with rows > 128 have any)
    half = (idx - p.n_whole) & 1;
    idx = p.n_whole + ((idx - p.n_whole) >> 1);
  }
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
  it.r0 = blk * 2 * PF_BM;
  const bool causal = (MODE == MODE_HSTU) ? true : (p.causal != 0);
  const int qs0 = it.r0, qs1 = it.r0 + PF_BM;
  const int e0 = (qs0 >= it.L) ? 0 : (causal ? min(it.L, qs0 + PF_BM) : it.L);
  const int e1 = (qs1 >= it.L) ? 0 : (causal ? min(it.L, qs1 + PF_BM) : it.L);
  it.n0 = (e0 + BN - 1) / BN;
  it.n1 = (e1 + BN - 1) / BN;
  it.split = 0;
  it.stop = 0;
  if (half >= 0) {
    // One Q tile (rows r0 + 128 half) whose key tiles are halved between the warpgroups.  Causal: the keys up
    // to the tile's diagonal; a tile that sees a single key tile stays whole (its second tile empty).
    it.r0 += half * PF_BM;
    const int n = ((causal ? min(it.L, it.r0 + PF_BM) : it.L) + BN - 1) / BN;
    it.split = (n >= 2) ? 1 : 0;
    it.n0 = (n + it.split) >> it.split;  // (n + 1) / 2 when split, else n
    it.n1 = n - it.n0;
  }
  return it;
}

// Control warpgroup: warp 0 fetches items and streams Q, K, V with TMA; warps 1-2 issue MMAs; warp 3 idles.
template <int D, int MODE, bool F8 = false>
__device__ __forceinline__ void prefill_control(const CUtensorMap &tmQ, const CUtensorMap &tmK,
                                                const CUtensorMap &tmV, const PrefillParams &p, uint8_t *smem,
                                                uint32_t tmem, int warp, int lane) {
  using C = PfCfg<D, F8>;
  constexpr bool PACKED = (MODE != MODE_DENSE);
  PfSmem<D, F8> sm(smem);
  if (warp == 0) {
    // ================================================================ work fetcher + TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      // Once this CTA takes no more items it counts itself finished; the last CTA of the launch to do so
      // returns the slot's counters to zero (no CTA touches them after its final fetch).
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
      int kv_issued = 0;  // K/V ring loads issued, over all items
      int q_issued = 0;   // items whose Q tiles were loaded
      bool ok = true;
      for (int k = 0; ok; ++k) {
        PfItem it;
        for (bool first = (k == 0);; first = false) {
          // The first item of every CTA is its block index; later ones come from the shared counter.
          const unsigned int idx = first ? blockIdx.x : gridDim.x + atomicAdd(&g_pf_sched[p.sched_slot][0], 1u);
          if (idx >= (unsigned int)p.n_items) {
            it = PfItem{};
            it.stop = 1;
            retire();
            break;
          }
          it = decode_item<D, MODE, F8>(p, (int)idx);
          if (it.r0 < it.L) break;  // row blocks past the end of their sequence have no work
        }
        ok = mbar_wait(sm.item_empty(k & 1), ((k >> 1) & 1) ^ 1, sm.abort_flag(), p.wait_ns);
        if (!ok) break;
        sm.items()[k & 1] = it;
        mbar_arrive(sm.item_full(k & 1));  // release semantics: the item is visible to its readers
        if (it.stop) break;
        // Q tiles into slot k % QSLOTS: every QK^T of the item that used the slot before must have finished.
        const int qs = k % C::QSLOTS;
        if (k >= C::QSLOTS) {
          ok = mbar_wait(sm.q_empty(qs), (k / C::QSLOTS - 1) & 1, sm.abort_flag(), p.wait_ns);
          if (!ok) break;
        }
        mbar_arrive_expect_tx(sm.q_full(qs), 2 * C::Q_TILE);
        // Q tile t: rows r0 + 128 t (whole item), or the item's one Q tile in both slots (split item).
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int qrow = it.r0 + (it.split ? 0 : t * PF_BM);
#pragma unroll
          for (int c = 0; c < C::KCH; ++c) {
            uint8_t *dst = sm.sQ(qs) + t * C::Q_TILE + c * C::Q_CHUNK;
            if constexpr (PACKED)
              tma_load_3d(dst, &tmQ, sm.q_full(qs), 64 * c, it.h, it.seq_start + qrow);
            else
              tma_load_3d(dst, &tmQ, sm.q_full(qs), 64 * c, qrow, it.bh);
          }
        }
        ++q_issued;
        // K/V tiles in ring order (the order kv_pos numbers them).
        auto load_kv = [&](const CUtensorMap *m, int jt) {
          const int st = kv_issued % C::NST;
          if (!mbar_wait(sm.empty(st), ((kv_issued / C::NST) & 1) ^ 1, sm.abort_flag(), p.wait_ns)) return false;
          mbar_arrive_expect_tx(sm.full(st), C::KV_TILE);
#pragma unroll
          for (int c = 0; c < C::KCH; ++c) {
            uint8_t *dst = sm.sKV() + st * C::KV_TILE + c * C::KV_CHUNK;
            if constexpr (PACKED)
              tma_load_3d(dst, m, sm.full(st), 64 * c, it.h, it.seq_start + jt * C::BN);
            else
              tma_load_3d(dst, m, sm.full(st), 64 * c, jt * C::BN, it.bh);
          }
          ++kv_issued;
          return true;
        };
        if (!it.split) {
          const int n_kv = max(it.n0, it.n1);
          for (int j = 0; ok && j < n_kv; ++j) ok = load_kv(&tmK, j) && load_kv(&tmV, j);
        } else {
          for (int j = 0; ok && j < it.n0; ++j) {
            const bool both = j < it.n1;
            ok = load_kv(&tmK, j) && (!both || load_kv(&tmK, it.n0 + j)) && load_kv(&tmV, j) &&
                 (!both || load_kv(&tmV, it.n0 + j));
          }
        }
      }
      if (!retired) retire();  // abandoned before the work ran out
      if (!ok) {
        // Abandoned pipeline: let copies already in flight land before shared memory is released.
        for (int i = max(0, q_issued - C::QSLOTS); i < q_issued; ++i)
          mbar_wait(sm.q_full(i % C::QSLOTS), (i / C::QSLOTS) & 1, nullptr, p.wait_ns);
        for (int i = max(0, kv_issued - C::NST); i < kv_issued; ++i)
          mbar_wait(sm.full(i % C::NST), (i / C::NST) & 1, nullptr, p.wait_ns);
      }
    }
  } else if (warp == 1 || (!C::ALIAS_P && warp == 2)) {
    // ================================================================ MMA issuer(s)
    if (lane == 0) {
      constexpr uint32_t ID_QK = F8 ? idesc_e4m3_f32(PF_BM, C::BN, false) : idesc_bf16_f32(PF_BM, C::BN, false);
      constexpr uint32_t ID_PV = F8 ? idesc_e4m3_f32(PF_BM, D, true) : idesc_bf16_f32(PF_BM, D, true);
      const uint32_t sQa = smem_u32(sm.sQ(0)), sKVa = smem_u32(sm.sKV());
      uint32_t q_off = 0;  // byte offset of the current item's Q slot
      // S_t = Q_t K^T : K-steps of 16 elements = 32 bytes inside a 128-byte swizzled row.
      const uint64_t dQ = sdesc_sw128(sQa, 16, 1024), dKV = sdesc_sw128(sKVa, 16, 1024);
      const uint64_t dV = sdesc_sw128(sKVa, C::KV_CHUNK, 1024);
      auto issue_s = [&](int t, int st) {
        const uint64_t da = dQ + (uint64_t)((q_off + (uint32_t)(t * C::Q_TILE)) >> 4);
        const uint64_t db = dKV + (uint64_t)((st * C::KV_TILE) >> 4);
        const uint32_t dt = tmem + (uint32_t)(C::S_STRIDE * t);
        eta_static_for<C::QK_STEPS>([&](auto kk_c) {
          constexpr int kk = decltype(kk_c)::value;
          constexpr uint32_t a_off = ((uint32_t)(kk >> 2) * C::Q_CHUNK + (uint32_t)(kk & 3) * 32u) >> 4;
          constexpr uint32_t b_off = ((uint32_t)(kk >> 2) * C::KV_CHUNK + (uint32_t)(kk & 3) * 32u) >> 4;
          if constexpr (F8)
            mma_ss_off_f8<a_off, b_off>(dt, da, db, ID_QK, kk > 0 ? 1u : 0u);
          else
            mma_ss_off<a_off, b_off>(dt, da, db, ID_QK, kk > 0 ? 1u : 0u);
        });
      };
      // O_t += P_t V : K-steps of 16 keys = 8 TMEM columns of packed bf16 P, 16 rows (2048 B) of V.
      auto issue_pv = [&](int t, int st, bool acc) {
        const uint32_t tP = C::ALIAS_P      ? tmem + (uint32_t)(C::S_STRIDE * t)
                            : C::P_IN_HOLES ? tmem + (uint32_t)(C::S_STRIDE * t + C::BN)
                                            : tmem + C::TM_P + (uint32_t)(C::P_COLS * t);
        const uint64_t db = dV + (uint64_t)((st * C::KV_TILE) >> 4);
        const uint32_t dt = tmem + C::TM_O + (uint32_t)(C::O_COLS * t);
        const uint32_t tP2 = dt + (uint32_t)D;  // (P_IN_HOLES) keys [64, 96): O_t's spare columns
        const uint32_t acc0 = acc ? 1u : 0u;
        // K-step kk: PV_KEYS keys = 8 TMEM columns of P, PV_KEYS rows (PV_KEYS * 128 B) of V
        eta_static_for<C::BN / C::PV_KEYS>([&](auto kk_c) {
          constexpr int kk = decltype(kk_c)::value;
          constexpr uint32_t b_off = (uint32_t)(C::PV_KEYS * 128 * kk) / 16u;
          if constexpr (F8) {
            mma_ts_off_f8<8u * kk, b_off>(dt, tP, db, ID_PV, kk > 0 ? 1u : acc0);
          } else if constexpr (C::P_IN_HOLES && kk >= 4) {
            mma_ts_off<8u * (kk - 4), b_off>(dt, tP2, db, ID_PV, 1u);
          } else {
            mma_ts_off<8u * kk, b_off>(dt, tP, db, ID_PV, kk > 0 ? 1u : acc0);
          }
        });
      };
      // Counts over all items; each gives the phase of the barrier it tracks.  With one issuer per tile
      // only slot 0 is used (for the issuer's own tile).
      int gs[2] = {0, 0};  // QK^T issued for tile t           (s_full / s_free completions)
      int gp[2] = {0, 0};  // PV issued for tile t             (p_full / pv_done completions)
      int go[2] = {0, 0};  // items with rows in tile t        (o_free completions)
      int kv_base = 0;     // ring index of the current item's K_0
      bool ok = true;
      for (int k = 0; ok; ++k) {
        ok = mbar_wait(sm.item_full(k & 1), (k >> 1) & 1, sm.abort_flag(), p.wait_ns);
        if (!ok) break;
        const PfItem it = sm.items()[k & 1];
        mbar_arrive(sm.item_empty(k & 1));
        if (it.stop) break;
        const int n_t[2] = {it.n0, it.n1};
        const int qs = k % C::QSLOTS;
        q_off = (uint32_t)(qs * 2 * C::Q_TILE);
        ok = mbar_wait(sm.q_full(qs), (k / C::QSLOTS) & 1, sm.abort_flag(), p.wait_ns);
        if (!ok) break;
        auto kv_wait = [&](int i) {  // item-local ring position i (numbered by kv_pos)
          const int g = kv_base + i;
          return mbar_wait(sm.full(g % C::NST), (g / C::NST) & 1, sm.abort_flag(), p.wait_ns);
        };
        auto kv_stage = [&](int i) { return (kv_base + i) % C::NST; };
        // Before the first PV of an item overwrites O_t, the previous item's epilogue must have read it.
        // (c: the counter slot of tile t -- t itself with one issuer, 0 for a per-tile issuer.)
        auto o_wait = [&](int t, int c) {
          return go[c] == 0 || mbar_wait(sm.o_free(t), (go[c] - 1) & 1, sm.abort_flag(), p.wait_ns);
        };
        if constexpr (!C::ALIAS_P) {
          // ---------------- issuer 1+t serves Q tile t; the next S_t as soon as S_t is free
          const int t = warp - 1;
          const int nt = (t == 0) ? it.n0 : it.n1;
          if (MODE == MODE_HSTU || !it.split) {
            const int n_kv = max(it.n0, it.n1);
            if (nt > 0) {
              ok = kv_wait(0) && (gs[0] == 0 || mbar_wait(sm.s_free(t), (gs[0] - 1) & 1, sm.abort_flag(), p.wait_ns));
              if (!ok) break;
              tc_fence_after();
              issue_s(t, kv_stage(0));
              mma_commit(sm.s_full(t));
              mma_commit(sm.empty(kv_stage(0)));
              ++gs[0];
            }
            if (nt <= 1) mma_commit(sm.q_empty(qs));  // every QK^T of this item is issued
            for (int j = 0; ok && j < nt; ++j) {
              if (j + 1 < nt) {
                ok = kv_wait(2 * j + 2) && mbar_wait(sm.s_free(t), (gs[0] - 1) & 1, sm.abort_flag(), p.wait_ns);
                if (!ok) break;
                tc_fence_after();
                issue_s(t, kv_stage(2 * j + 2));
                mma_commit(sm.s_full(t));
                mma_commit(sm.empty(kv_stage(2 * j + 2)));
                ++gs[0];
                if (j + 2 == nt) mma_commit(sm.q_empty(qs));
              }
              ok = kv_wait(2 * j + 1) && mbar_wait(sm.p_full(t), gp[0] & 1, sm.abort_flag(), p.wait_ns) &&
                   (j > 0 || o_wait(t, 0));
              if (!ok) break;
              tc_fence_after();
              issue_pv(t, kv_stage(2 * j + 1), j > 0);
              mma_commit(sm.pv_done(t));
              mma_commit(sm.empty(kv_stage(2 * j + 1)));
              ++gp[0];
            }
            // Key/value tiles of this item that tile t does not see: release them once they landed.
            for (int i = 2 * nt; ok && i < 2 * n_kv; ++i) {
              ok = kv_wait(i);
              if (ok) mbar_arrive(sm.empty(kv_stage(i)));
            }
          } else {
            // Ring positions this tile does not read are released (arrive on their empty barrier) in order.
            // Arriving for position r is in the right phase once the producer has issued load r.  Below a
            // position of its own that this issuer has just seen land, that holds with no further wait (and
            // the producer never needs a release at or above that position to issue it: a split item's own
            // positions are at most 4 apart, a whole item's are a prefix).  Past its last own position the
            // issuer waits for each position before releasing it.
            int rel = 0;  // positions below rel are accounted for
            auto release_below = [&](int pos) {
              for (; rel < pos; ++rel)
                if (!kv_owned(it, t, rel)) mbar_arrive(sm.empty(kv_stage(rel)));
            };
            if (nt > 0) {
              const int pk = kv_pos(it, t, 0, 0);
              ok = kv_wait(pk);
              if (!ok) break;
              release_below(pk);
              ok = gs[0] == 0 || mbar_wait(sm.s_free(t), (gs[0] - 1) & 1, sm.abort_flag(), p.wait_ns);
              if (!ok) break;
              tc_fence_after();
              issue_s(t, kv_stage(pk));
              mma_commit(sm.s_full(t));
              mma_commit(sm.empty(kv_stage(pk)));
              ++gs[0];
            }
            if (nt <= 1) mma_commit(sm.q_empty(qs));  // every QK^T of this item is issued
            for (int j = 0; ok && j < nt; ++j) {
              if (j + 1 < nt) {
                const int pk = kv_pos(it, t, j + 1, 0);
                ok = kv_wait(pk);
                if (!ok) break;
                release_below(pk);
                ok = mbar_wait(sm.s_free(t), (gs[0] - 1) & 1, sm.abort_flag(), p.wait_ns);
                if (!ok) break;
                tc_fence_after();
                issue_s(t, kv_stage(pk));
                mma_commit(sm.s_full(t));
                mma_commit(sm.empty(kv_stage(pk)));
                ++gs[0];
                if (j + 2 == nt) mma_commit(sm.q_empty(qs));
              }
              const int pv = kv_pos(it, t, j, 1);
              ok = kv_wait(pv);
              if (!ok) break;
              release_below(pv);
              ok = mbar_wait(sm.p_full(t), gp[0] & 1, sm.abort_flag(), p.wait_ns) && (j > 0 || o_wait(t, 0));
              if (!ok) break;
              tc_fence_after();
              issue_pv(t, kv_stage(pv), j > 0);
              mma_commit(sm.pv_done(t));
              mma_commit(sm.empty(kv_stage(pv)));
              ++gp[0];
            }
            for (const int tot = kv_loads(it); ok && rel < tot; ++rel) {
              if (kv_owned(it, t, rel)) continue;
              ok = kv_wait(rel);
              if (ok) mbar_arrive(sm.empty(kv_stage(rel)));
            }
          }
          if (nt > 0) ++go[0];
        } else {
          // ---------------- one issuer for both tiles; P aliased into S; issue order PV_t(j), S_t(j+1).
          // A whole item's K_j / V_j serve both tiles (released after both); a split item's each serve one.
          const int n_kv = max(it.n0, it.n1);  // >= 1: an item has at least one row
          if (MODE == MODE_HSTU || !it.split) {
            ok = kv_wait(0);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int t = 0; t < 2; ++t)
              if (n_t[t] > 0) {
                issue_s(t, kv_stage(0));
                mma_commit(sm.s_full(t));
                ++gs[t];
              }
            mma_commit(sm.empty(kv_stage(0)));
            if (n_kv == 1) mma_commit(sm.q_empty(qs));
            for (int j = 0; ok && j < n_kv; ++j) {
              ok = kv_wait(2 * j + 1);
              if (!ok) break;
              bool k_ready = false;
#pragma unroll
              for (int t = 0; t < 2; ++t) {
                if (!ok || j >= n_t[t]) continue;
                ok = mbar_wait(sm.p_full(t), gp[t] & 1, sm.abort_flag(), p.wait_ns) && (j > 0 || o_wait(t, t));
                if (!ok) break;
                tc_fence_after();
                issue_pv(t, kv_stage(2 * j + 1), j > 0);
                mma_commit(sm.pv_done(t));
                ++gp[t];
                if (j + 1 < n_t[t]) {
                  if (!k_ready) {
                    ok = kv_wait(2 * j + 2);
                    if (!ok) break;
                    k_ready = true;
                  }
                  issue_s(t, kv_stage(2 * j + 2));
                  mma_commit(sm.s_full(t));
                  ++gs[t];
                }
              }
              if (!ok) break;
              mma_commit(sm.empty(kv_stage(2 * j + 1)));
              if (k_ready) mma_commit(sm.empty(kv_stage(2 * j + 2)));
              if (j + 2 == n_kv) mma_commit(sm.q_empty(qs));
            }
          } else {
            // Split item: every ring position serves one tile (both tiles have key tiles).
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              const int pk = kv_pos(it, t, 0, 0);
              ok = ok && kv_wait(pk);
              if (!ok) break;
              tc_fence_after();
              issue_s(t, kv_stage(pk));
              mma_commit(sm.s_full(t));
              mma_commit(sm.empty(kv_stage(pk)));
              ++gs[t];
            }
            if (!ok) break;
            if (n_kv == 1) mma_commit(sm.q_empty(qs));
            for (int j = 0; ok && j < n_kv; ++j) {
#pragma unroll
              for (int t = 0; t < 2; ++t) {
                if (!ok || j >= n_t[t]) continue;
                const int pv = kv_pos(it, t, j, 1);
                ok = kv_wait(pv) && mbar_wait(sm.p_full(t), gp[t] & 1, sm.abort_flag(), p.wait_ns) &&
                     (j > 0 || o_wait(t, t));
                if (!ok) break;
                tc_fence_after();
                issue_pv(t, kv_stage(pv), j > 0);
                mma_commit(sm.pv_done(t));
                mma_commit(sm.empty(kv_stage(pv)));
                ++gp[t];
                if (j + 1 < n_t[t]) {
                  const int pk = kv_pos(it, t, j + 1, 0);
                  ok = kv_wait(pk);
                  if (!ok) break;
                  issue_s(t, kv_stage(pk));
                  mma_commit(sm.s_full(t));
                  mma_commit(sm.empty(kv_stage(pk)));
                  ++gs[t];
                }
              }
              if (!ok) break;
              if (j + 2 == n_kv) mma_commit(sm.q_empty(qs));
            }
          }
#pragma unroll
          for (int t = 0; t < 2; ++t)
            if (n_t[t] > 0) ++go[t];
        }
        kv_base += kv_loads(it);
      }
      // Every MMA issued by this thread has completed before TMEM is released.
      mma_commit(sm.mma_done(warp - 1));
      mbar_wait(sm.mma_done(warp - 1), 0, nullptr, p.wait_ns);
    }
    __syncwarp();
  }
}

// Softmax (or HSTU pointwise) warpgroups: warps 4-7 for Q tile 0, warps 8-11 for Q tile 1.  Thread
// (quarter, lane) owns query row 32 quarter + lane of its tile (= its TMEM lane): per key tile it loads the
// S row from TMEM, applies the mask, updates the running max and exp-sum, writes P (bf16) to TMEM and
// rescales its O row when the max moved; per item it finally normalises O and stores O and lse.
template <int D, int MODE, bool F8 = false>
__device__ __forceinline__ void prefill_softmax(const PrefillParams &p, uint8_t *smem, uint32_t tmem, int warp,
                                                int lane) {
  using C = PfCfg<D, F8>;
  constexpr bool HSTU = (MODE == MODE_HSTU);
  constexpr bool PACKED = (MODE != MODE_DENSE);
  PfSmem<D, F8> sm(smem);
  const int t = (warp - 4) >> 2;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
  constexpr int BN = C::BN;
  const uint32_t tS = tmem + lane_addr + (uint32_t)(C::S_STRIDE * t);
  const uint32_t tO = tmem + lane_addr + C::TM_O + (uint32_t)(C::O_COLS * t);
  const uint32_t tP = C::ALIAS_P      ? tS
                      : C::P_IN_HOLES ? tS + (uint32_t)BN  // (and O_t's spare columns for keys [64, 96))
                                      : tmem + lane_addr + C::TM_P + (uint32_t)(C::P_COLS * t);
  const bool causal = HSTU ? true : (p.causal != 0);
  int gj = 0;  // key tiles of Q tile t processed, over all items (phases of s_full, p_full, pv_done)
  bool ok = true;
  for (int k = 0; ok; ++k) {
    ok = mbar_wait(sm.item_full(k & 1), (k >> 1) & 1, sm.abort_flag(), p.wait_ns);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    const PfItem it = sm.items()[k & 1];
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.item_empty(k & 1));
    if (it.stop) break;
    const int L = it.L;
    const int q_start = it.r0 + (it.split ? 0 : t * PF_BM);
    const int qpos = q_start + row;
    const int nt = (t == 0) ? it.n0 : it.n1;
    const int kv_lo = (it.split && t == 1) ? it.n0 : 0;  // first key tile of this warpgroup
    const size_t orow = PACKED ? ((size_t)(it.seq_start + qpos) * p.H + it.h) : ((size_t)it.bh * p.N + qpos);
    float m_used = -INFINITY, l = 0.f;
    for (int j = 0; j < nt; ++j, ++gj) {
      ok = mbar_wait(sm.s_full(t), gj & 1, sm.abort_flag(), p.wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[BN];
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) ETA_TMEM_LD_X32(tS + 32u * cc, (sr + 32 * cc));
      tmem_wait_ld();
      if constexpr (!C::ALIAS_P) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sm.s_free(t));  // S_t may now be overwritten by the next QK^T
      }
      const int k0 = (kv_lo + j) * BN;
      const bool need_mask = (k0 + BN > L) || (causal && k0 + BN - 1 > q_start);
      const int kmax = causal ? min(L - 1, qpos) - k0 : L - 1 - k0;  // last visible key, tile-local
      uint32_t pk[C::P_COLS];
      bool resc = false;
      float f = 1.f, rowsum = 0.f, m_new = m_used;
      if constexpr (!HSTU) {
        if (need_mask) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c > kmax) sr[c] = __float_as_uint(-INFINITY);
        }
        // row max: four independent 3-input max chains
        float mxa = -INFINITY, mxb = -INFINITY, mxc = -INFINITY, mxd = -INFINITY;
#pragma unroll
        for (int c = 0; c < BN; c += 8) {
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
        float q0 = 0.f, q1 = 0.f;  // (F8) the previous pair, packed with the next one
        // p = 2^(s * scale_log2 - m) on the MUFU; P packed to bf16 (or e4m3), the row sum kept in fp32
#pragma unroll
        for (int i = 0; i < BN / 2; ++i) {
          const uint64_t x2 = fma_x2(f2pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), cs2, nm2);
          float x0, x1;
          f2unpack(x2, x0, x1);
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          if (i & 1) rs_b = add_x2(rs_b, f2pack(p0, p1));
          else rs_a = add_x2(rs_a, f2pack(p0, p1));
          if constexpr (F8) {
            // four keys per TMEM column: pairs 2m and 2m+1 go to column m
            if (i & 1) pk[i >> 1] = pack_e4m3x4(q0, q1, p0, p1);
            q0 = p0;
            q1 = p1;
          } else {
            pk[i] = pack_bf16x2(p0, p1);
          }
        }
        float r0a, r1a, r2a, r3a;
        f2unpack(rs_a, r0a, r1a);
        f2unpack(rs_b, r2a, r3a);
        rowsum = (r0a + r1a) + (r2a + r3a);
        f = resc ? ex2_approx(m_used - msub) : 1.f;  // 0 on the first tile
      } else {
        // HSTU: p = inv_n * silu(alpha s) = inv_n (y + y tanh(y)),  y = alpha s / 2.  P holds y + y tanh(y)
        // and the factor inv_n is applied to O at the end of the item (one multiply a row instead of one a
        // score).  Masked keys get s = 0 first, which gives p = 0 exactly (y = 0), so the pointwise loop is
        // the same straight-line code for every tile.
        if (need_mask) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c > kmax) sr[c] = 0u;
        }
        const uint64_t ha2 = f2pack(p.hstu_half_alpha, p.hstu_half_alpha);
        // tanh on the MUFU for every pair, or (TANH_FMA_PAIRS of every 8 pairs) on the FMA pipe by the degree-7
        // polynomial, so that the two pipes share the work.  The polynomial holds for |alpha s / 2| <= 1: a
        // warp takes the mixed loop only when every row's polynomial pairs are in that range.
        bool mixed = false;
        if constexpr (C::TANH_FMA_PAIRS > 0) {
          float amax = 0.f;
#pragma unroll
          for (int i = 0; i < BN / 2; ++i)
            if ((i % 8) < C::TANH_FMA_PAIRS)
              amax = max3f(amax, fabsf(__uint_as_float(sr[2 * i])), fabsf(__uint_as_float(sr[2 * i + 1])));
          mixed = __all_sync(0xffffffffu, amax * fabsf(p.hstu_half_alpha) <= 1.f);
        }
        auto pointwise = [&](auto with_poly) {
#pragma unroll
          for (int i = 0; i < BN / 2; ++i) {
            const uint64_t s2 = f2pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]));
            const uint64_t y2 = mul_x2(s2, ha2);
            uint64_t t2;
            if (decltype(with_poly)::value && (i % 8) < C::TANH_FMA_PAIRS) {
              t2 = tanh_poly_x2(y2);
            } else {
              float y0, y1;
              f2unpack(y2, y0, y1);
              t2 = f2pack(tanh_approx(y0), tanh_approx(y1));
            }
            float p0, p1;
            f2unpack(fma_x2(y2, t2, y2), p0, p1);
            pk[i] = pack_bf16x2(p0, p1);
          }
        };
        if (mixed) pointwise(std::true_type{});
        else pointwise(std::false_type{});
      }
      if constexpr (!C::ALIAS_P) {
        // P_t's columns (and O_t) are free once the previous PV of this tile -- possibly the previous
        // item's last -- has completed.  (With P aliased into S_t this is implied: the S_t just read was
        // issued after that PV, and its commit covers it.)
        if (gj > 0) {
          ok = mbar_wait(sm.pv_done(t), (gj - 1) & 1, sm.abort_flag(), p.wait_ns);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
        }
      }
      if constexpr (C::P_IN_HOLES) {
        ETA_TMEM_ST_X32(tP, pk);                           // keys [0, 64): S_t's spare columns
        ETA_TMEM_ST_X16(tO + (uint32_t)D, (pk + 32));      // keys [64, 96): O_t's spare columns
      } else {
#pragma unroll
        for (int cc = 0; cc < C::P_COLS / 32; ++cc) ETA_TMEM_ST_X32(tP + 32u * cc, (pk + 32 * cc));
      }
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
      if (lane == 0) mbar_arrive(sm.p_full(t));
    }
    if (!ok) break;
    if (nt == 0) continue;
    // ---------------------------------------------------------------- epilogue of the item
    ok = mbar_wait(sm.pv_done(t), (gj - 1) & 1, sm.abort_flag(), p.wait_ns);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    tc_fence_after();
    // Final row statistics; with a split item the first warpgroup merges the two key halves:
    //   m = max(m0, m1),  l = l0 2^(m0-m) + l1 2^(m1-m),  O = (O_0 2^(m0-m) + O_1 2^(m1-m)) / l.
    float m_fin = m_used, l_fin = l, a0 = 1.f, a1 = 0.f;
    bool merge = false;
    if constexpr (MODE != MODE_HSTU) {
      if (it.split) {
        if (t == 1) {
          // Hand this row's (m, l) to the first warpgroup, which reads O_1 from TMEM and stores the row.
          sm.xch()[row] = make_float2(m_used, l);
          tc_fence_before();
          asm volatile("bar.arrive 2, %0;" ::"n"(2 * 128) : "memory");
          continue;
        }
        asm volatile("bar.sync 2, %0;" ::"n"(2 * 128) : "memory");
        tc_fence_after();
        const float2 x = sm.xch()[row];
        m_fin = fmaxf(m_used, x.x);
        const float msub = (m_fin == -INFINITY) ? 0.f : m_fin;
        a0 = (m_used == -INFINITY) ? 0.f : ex2_approx(m_used - msub);
        a1 = (x.x == -INFINITY) ? 0.f : ex2_approx(x.x - msub);
        l_fin = l * a0 + x.y * a1;
        merge = true;
      }
    }
    const float inv_l = HSTU ? p.hstu_inv_n : ((l_fin > 0.f) ? p.o_scale / l_fin : 0.f);
    const float w0 = a0 * inv_l, w1 = a1 * inv_l;
    const bool valid = qpos < L;
    const uint32_t tO1 = tmem + lane_addr + C::TM_O + (uint32_t)C::O_COLS;  // O_1 (read here only when merging)
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      float ov[32];
      {
        uint32_t orr[32];
        ETA_TMEM_LD_X32(tO + 32u * cc, orr);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] = __uint_as_float(orr[i]) * w0;
      }
      if (merge) {
        uint32_t orr[32];
        ETA_TMEM_LD_X32(tO1 + 32u * cc, orr);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] = fmaf(__uint_as_float(orr[i]), w1, ov[i]);
      }
      if (cc == D / 32 - 1) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(sm.o_free(t));  // the next item's first PV may overwrite O_t
          if (merge) mbar_arrive(sm.o_free(1));
        }
      }
      if (valid) {
        if (p.o_f32) {
          float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.o) + orow * D + 32 * cc);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_float4(ov[4 * i], ov[4 * i + 1], ov[4 * i + 2], ov[4 * i + 3]);
        } else {
          uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) + orow * D + 32 * cc);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = pack_bf16x2(ov[8 * i + 0], ov[8 * i + 1]);
            w.y = pack_bf16x2(ov[8 * i + 2], ov[8 * i + 3]);
            w.z = pack_bf16x2(ov[8 * i + 4], ov[8 * i + 5]);
            w.w = pack_bf16x2(ov[8 * i + 6], ov[8 * i + 7]);
            dst[i] = w;
          }
        }
      }
    }
    if (valid) {
      if constexpr (!HSTU) {
        if (p.lse != nullptr)
          p.lse[orow] = (l_fin > 0.f) ? (m_fin + log2f(l_fin)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }
}

template <int D, int MODE, bool F8 = false>
__global__ void __launch_bounds__(PF_THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = PfCfg<D, F8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  PfSmem<D, F8> sm(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ------------------------------------------------------------------ setup
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(sm.full(i), 1);
      mbar_init(sm.empty(i), C::N_ISSUERS);  // released by each MMA issuer
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(sm.q_full(i), 1);
      mbar_init(sm.q_empty(i), C::N_ISSUERS);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(sm.item_full(i), 1);
      mbar_init(sm.item_empty(i), C::N_ISSUERS + PF_SM_WARPS);  // every consumer warp reads the item
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(sm.s_full(t), 1);
      mbar_init(sm.s_free(t), 4);  // one elected arrive per softmax warp of the tile
      mbar_init(sm.p_full(t), 4);
      mbar_init(sm.pv_done(t), 1);
      mbar_init(sm.o_free(t), 4);
      mbar_init(sm.mma_done(t), 1);
    }
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
  // Each role runs to its own end; the teardown barrier (id 1, every thread of the CTA) is reached from
  // both sides.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(PF_CTRL_REGS));
    prefill_control<D, MODE, F8>(tmQ, tmK, tmV, p, smem, tmem, warp, lane);
    tc_fence_before();
    asm volatile("bar.sync 1, %0;" ::"n"(PF_THREADS) : "memory");
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(PF_SM_REGS));
    prefill_softmax<D, MODE, F8>(p, smem, tmem, warp, lane);
    tc_fence_before();
    asm volatile("bar.sync 1, %0;" ::"n"(PF_THREADS) : "memory");
  }
}

}  // namespace eta
