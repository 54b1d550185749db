// decode_paged.cuh -- one decode step with grouped query heads (GQA; MQA when there is one KV head) over a
// paged KV cache, split along the sequence (split-KV).
//
// What it computes: the decode step of "AI attention complexity ledger", section "带宽账：decode 阶段的真正
// 瓶颈" (one new query per head against every cached key, s_j = scale q.k_j, o = sum_j softmax(s)_j v_j),
// with the two cache-side changes the pages name: query heads share key/value heads (the same section: GQA
// is one of the routes that shrink the KV cache; "FlashAttention (TH)", section "FlashAttention-2": MQA),
// and the cache lives in fixed-size pages addressed through a per-sequence page table (the ops-transformer
// page, section on the repository's other operators: KV-cache management, the PagedAttention of inference).
// Query head hq reads key/value head hq / G, G = Hq / Hkv.
//
// Design (B200):
//  * grid (split, kv head, b): split i owns cache rows [i*chunk, min((i+1)*chunk, L_b)) of sequence b; the
//    CTA serves the G query heads of one KV head, so every K/V byte is read once for all G of them.
//  * one producer thread reads the split's page numbers, then streams 32-row K and V stages with TMA
//    (3-D tensor map over [page * Hkv + kv head, row in page, d], 128-byte swizzle) through a
//    4-deep ring.  A stage is one 32-row slice of a page, or two 16-row pages.
//  * two consumer warps take alternate stages.  The G queries (padded to 16 rows) stay in registers as
//    warp-MMA A fragments; S = Q K^T, the online softmax and O += P V run on 16 x 32 register tiles
//    (mma.sync m16n8k16, bf16 in, fp32 out; K and V fragments by ldmatrix from the swizzled stage).  The
//    step is HBM-bound (about 2G flops per K/V byte): per 32 rows a warp issues ~150 instructions against
//    ~680 cycles of HBM time per SM, so the register-level MMA -- no TMEM round trip, no 64-row minimum --
//    is the lighter tool than tcgen05 here.
//  * the warps' states are merged in shared memory and each query head's partial (o, lse) is written;
//    decode_combine_kernel merges the splits with logsumexp weights (exact).
#pragma once

#include "decode.cuh"
#include "ptx.cuh"

namespace eta {

constexpr int DPG_ROWS = 32;                       // cache rows per stage
constexpr int DPG_STAGES = 4;
constexpr int DPG_CWARPS = 2;                      // consumer warps (alternate stages)
constexpr int DPG_THREADS = 32 * (1 + DPG_CWARPS);
constexpr int DPG_MAX_G = 16;                      // query heads per KV head (one 16-row MMA tile)
constexpr int DPG_MAX_SPLIT_PAGES = 1024 / 16 + 1; // pages a split can touch (chunk <= 1024, page >= 16)
constexpr float DPG_RESCALE_THRESHOLD = 8.0f;     // log2 units (as the prefill softmax)

struct PagedDecodeParams {
  const __nv_bfloat16 *q;   // [B, Hq, D]
  const int *block_table;   // [B, max_pages]
  const int *kv_lens;       // [B]
  float *part_o;            // [B, Hq, max_splits, D]
  float *part_lse;          // [B, Hq, max_splits]
  int B, Hq, Hkv, G, num_pages, page_size, max_pages, Lmax, chunk, max_splits;
  float scale_log2;         // scale * log2(e)
  long long wait_ns;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// c (16x8 fp32) += a (16x16 bf16, row) * b (16x8 bf16, col)
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of (row r, 16-byte column group cg) in a stage tile stored as 64-column chunks of 32 rows x
// 128 B with the 128-byte swizzle (group g of row r sits at g ^ (r % 8)).
__device__ __forceinline__ uint32_t dpg_off(int r, int cg) {
  return (uint32_t)((cg >> 3) * (DPG_ROWS * 128) + r * 128 + (((cg & 7) ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(DPG_THREADS) decode_paged_split_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                         const __grid_constant__ CUtensorMap tmV,
                                                                         const PagedDecodeParams p) {
  constexpr int TILE_BYTES = DPG_ROWS * D * 2;  // one 32-row stage of K (or V)
  constexpr int NT_D = D / 8;                   // 8-wide column tiles of O
  constexpr int KS_D = D / 16;                  // 16-deep k-steps of Q K^T
  extern __shared__ uint8_t dsm_raw[];
  uint8_t *dsm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sK = dsm;                                // [DPG_STAGES][TILE_BYTES]
  uint8_t *sV = dsm + DPG_STAGES * TILE_BYTES;      // [DPG_STAGES][TILE_BYTES]
  __shared__ __align__(8) uint64_t full[DPG_STAGES], empty[DPG_STAGES];
  __shared__ int pages[DPG_MAX_SPLIT_PAGES];
  __shared__ float wm[DPG_CWARPS][16], wl[DPG_CWARPS][16];
  __shared__ int abort_flag;

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  int L = p.kv_lens[b];
  if (L < 0 || L > p.Lmax) {
    if (split == 0 && kvh == 0 && threadIdx.x == 0) record_status(2 /* ETA_DEV_BAD_KVLEN */);
    L = L < 0 ? 0 : p.Lmax;
  }
  const int s0 = split * p.chunk;
  if (s0 >= L) return;  // no rows in this split (uniform over the CTA)
  const int nrows = min(L, s0 + p.chunk) - s0;
  const int nst = (nrows + DPG_ROWS - 1) / DPG_ROWS;
  const int first_page = s0 / p.page_size;
  const int n_pages = (s0 + nrows - 1) / p.page_size - first_page + 1;
  const int box_rows = min(p.page_size, DPG_ROWS);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < DPG_STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);  // one consumer warp per stage
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    // The split's page numbers, checked against the page pool (an out-of-range entry reads page 0 and
    // sets ETA_DEV_BAD_PAGE).
    for (int i = lane; i < n_pages; i += 32) {
      int pg = p.block_table[(size_t)b * p.max_pages + first_page + i];
      if (pg < 0 || pg >= p.num_pages) {
        record_status(4 /* ETA_DEV_BAD_PAGE */);
        pg = 0;
      }
      pages[i] = pg;
    }
  }
  __syncthreads();

  if (warp == 0) {
    // ---------------- producer: one thread streams K and V stages ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int it = 0;
      for (; it < nst; ++it) {
        const int st = it % DPG_STAGES;
        if (!mbar_wait(&empty[st], ((it / DPG_STAGES) & 1) ^ 1, &abort_flag, p.wait_ns)) break;
        // boxes of this stage that hold rows of the sequence (a box never straddles a page)
        const int r0 = s0 + it * DPG_ROWS;
        const int nbox = min(DPG_ROWS, (s0 + nrows) - r0 + box_rows - 1) / box_rows;
        mbar_arrive_expect_tx(&full[st], (uint32_t)(2 * nbox * box_rows * D * 2));
        for (int bx = 0; bx < nbox; ++bx) {
          const int lr = r0 + bx * box_rows;
          const int pg = pages[lr / p.page_size - first_page];
          const int off = lr % p.page_size;
          const int z = pg * p.Hkv + kvh;
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            const uint32_t dst = (uint32_t)(c * DPG_ROWS * 128 + bx * box_rows * 128);
            tma_load_3d(sK + st * TILE_BYTES + dst, &tmK, &full[st], 64 * c, off, z);
            tma_load_3d(sV + st * TILE_BYTES + dst, &tmV, &full[st], 64 * c, off, z);
          }
        }
      }
      if (it < nst) {
        // Abandoned: let the copies already issued land before the CTA's shared memory goes away.
        for (int j = max(0, it - DPG_STAGES); j < it; ++j)
          mbar_wait(&full[j % DPG_STAGES], (j / DPG_STAGES) & 1, nullptr, p.wait_ns);
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int cw = warp - 1;
  const int qr = lane >> 2, qc = (lane & 3) * 2;  // fragment row (and row + 8), column pair
  const float cl = p.scale_log2;
  // Q as A fragments: rows = the G query heads of this KV head (rows >= G are zero), k = head dim.
  uint32_t qa[KS_D][4];
  {
    const size_t qbase = ((size_t)b * p.Hq + (size_t)kvh * p.G) * D;
#pragma unroll
    for (int ks = 0; ks < KS_D; ++ks) {
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const int row = qr + ((h & 1) ? 8 : 0), col = ks * 16 + qc + ((h & 2) ? 8 : 0);
        qa[ks][h] = (row < p.G) ? *reinterpret_cast<const uint32_t *>(p.q + qbase + (size_t)row * D + col) : 0u;
      }
    }
  }
  float oc[NT_D][4];
#pragma unroll
  for (int j = 0; j < NT_D; ++j) oc[j][0] = oc[j][1] = oc[j][2] = oc[j][3] = 0.f;
  float m_used[2] = {-INFINITY, -INFINITY}, lp[2] = {0.f, 0.f};  // rows qr, qr + 8 (log2 units)

  bool ok = true;
  for (int it = cw; it < nst; it += DPG_CWARPS) {
    const int st = it % DPG_STAGES;
    ok = mbar_wait(&full[st], (it / DPG_STAGES) & 1, &abort_flag, p.wait_ns);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    const int rows = min(DPG_ROWS, nrows - it * DPG_ROWS);
    const uint32_t kb = smem_u32(sK + st * TILE_BYTES), vb = smem_u32(sV + st * TILE_BYTES);
    if (rows < DPG_ROWS) {
      // Rows past the sequence end (not loaded, or garbage in the last page): zero V so that P = 0
      // multiplies zeros, never stale or non-finite values.
      uint8_t *vt = sV + st * TILE_BYTES;
      for (int i = lane; i < (DPG_ROWS - rows) * (D / 8); i += 32) {
        const int r = rows + i / (D / 8), cg = i % (D / 8);
        *reinterpret_cast<uint4 *>(vt + dpg_off(r, cg)) = make_uint4(0u, 0u, 0u, 0u);
      }
      __syncwarp();
    }
    // S = Q K^T : 4 key tiles of 8.  ldmatrix.x4 of 8 keys x 32 head-dim columns gives two k-steps of B.
    float sc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
      for (int kp = 0; kp < KS_D / 2; ++kp) {
        uint32_t bk[4];
        ldsm_x4(kb + dpg_off(8 * j + (lane & 7), 4 * kp + (lane >> 3)), bk);
        mma_16816(sc[j], qa[2 * kp], bk[0], bk[1]);
        mma_16816(sc[j], qa[2 * kp + 1], bk[2], bk[3]);
      }
    }
    // mask keys past the end, row max (rows qr and qr + 8; a row's 4 threads share it)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = 8 * j + qc + (e & 1);
        if (key >= rows) sc[j][e] = -INFINITY;
        mx[e >> 1] = fmaxf(mx[e >> 1], sc[j][e]);
      }
    }
    float f[2];
    bool resc = false;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2)) * cl;
      // conditional rescale: raise the running max only when the block max exceeds it by more than 8
      f[h] = 1.f;
      if (mx[h] > m_used[h] + DPG_RESCALE_THRESHOLD) {
        f[h] = ex2_approx(m_used[h] - mx[h]);  // 0 on the first block
        m_used[h] = mx[h];
        resc = true;
      }
    }
    if (__any_sync(0xffffffffu, resc)) {
      lp[0] *= f[0];
      lp[1] *= f[1];
#pragma unroll
      for (int j = 0; j < NT_D; ++j) {
        oc[j][0] *= f[0];
        oc[j][1] *= f[0];
        oc[j][2] *= f[1];
        oc[j][3] *= f[1];
      }
    }
    // P = 2^(s * scale_log2 - m), as bf16 A fragments (two 16-key k-steps)
    uint32_t pa[2][4];
    const float ms0 = (m_used[0] == -INFINITY) ? 0.f : m_used[0];
    const float ms1 = (m_used[1] == -INFINITY) ? 0.f : m_used[1];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float p0 = ex2_approx(fmaf(sc[j][0], cl, -ms0)), p1 = ex2_approx(fmaf(sc[j][1], cl, -ms0));
      const float p2 = ex2_approx(fmaf(sc[j][2], cl, -ms1)), p3 = ex2_approx(fmaf(sc[j][3], cl, -ms1));
      lp[0] += p0 + p1;
      lp[1] += p2 + p3;
      pa[j >> 1][(j & 1) * 2 + 0] = pack_bf16x2(p0, p1);
      pa[j >> 1][(j & 1) * 2 + 1] = pack_bf16x2(p2, p3);
    }
    // O += P V : ldmatrix.x4.trans of 16 keys x 16 head-dim columns gives B for two column tiles.
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
#pragma unroll
      for (int jp = 0; jp < NT_D / 2; ++jp) {
        uint32_t bv[4];
        ldsm_x4_trans(vb + dpg_off(16 * ks + 8 * ((lane >> 3) & 1) + (lane & 7), 2 * jp + (lane >> 4)), bv);
        mma_16816(oc[2 * jp], pa[ks], bv[0], bv[1]);
        mma_16816(oc[2 * jp + 1], pa[ks], bv[2], bv[3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }

  // ---------------- merge the consumer warps' states; write one partial per query head ----------------
  lp[0] += __shfl_xor_sync(0xffffffffu, lp[0], 1);
  lp[0] += __shfl_xor_sync(0xffffffffu, lp[0], 2);
  lp[1] += __shfl_xor_sync(0xffffffffu, lp[1], 1);
  lp[1] += __shfl_xor_sync(0xffffffffu, lp[1], 2);
  // every stage has been consumed (or the pipeline abandoned), so the K ring is free for the exchange
  asm volatile("bar.sync 1, %0;" ::"n"(32 * DPG_CWARPS) : "memory");
  float *wo = reinterpret_cast<float *>(sK);  // [DPG_CWARPS][16][D]
  if ((lane & 3) == 0) {
    wm[cw][qr] = ok ? m_used[0] : -INFINITY;
    wm[cw][qr + 8] = ok ? m_used[1] : -INFINITY;
    wl[cw][qr] = ok ? lp[0] : 0.f;
    wl[cw][qr + 8] = ok ? lp[1] : 0.f;
  }
#pragma unroll
  for (int j = 0; j < NT_D; ++j) {
    float *r0 = wo + ((size_t)cw * 16 + qr) * D + 8 * j + qc;
    float *r1 = wo + ((size_t)cw * 16 + qr + 8) * D + 8 * j + qc;
    r0[0] = ok ? oc[j][0] : 0.f;
    r0[1] = ok ? oc[j][1] : 0.f;
    r1[0] = ok ? oc[j][2] : 0.f;
    r1[1] = ok ? oc[j][3] : 0.f;
  }
  asm volatile("bar.sync 1, %0;" ::"n"(32 * DPG_CWARPS) : "memory");
  const int t = threadIdx.x - 32;  // consumer thread index
  for (int r = 0; r < p.G; ++r) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < DPG_CWARPS; ++w) M = fmaxf(M, wm[w][r]);
    const float Msub = (M == -INFINITY) ? 0.f : M;
    float wgt[DPG_CWARPS], Lsum = 0.f;
#pragma unroll
    for (int w = 0; w < DPG_CWARPS; ++w) {
      wgt[w] = (wm[w][r] == -INFINITY) ? 0.f : ex2_approx(wm[w][r] - Msub);
      Lsum += wl[w][r] * wgt[w];
    }
    const size_t pidx = ((size_t)b * p.Hq + (size_t)kvh * p.G + r) * p.max_splits + split;
    for (int e = t; e < D; e += 32 * DPG_CWARPS) {
      float o = 0.f;
#pragma unroll
      for (int w = 0; w < DPG_CWARPS; ++w) o += wo[((size_t)w * 16 + r) * D + e] * wgt[w];
      p.part_o[pidx * D + e] = (Lsum > 0.f) ? o / Lsum : 0.f;
    }
    if (t == 0) p.part_lse[pidx] = (Lsum > 0.f) ? (Msub + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
  }
}

}  // namespace eta
