// decode.cuh -- single-query decode step over a long KV cache, split along the sequence (split-KV).
//
// What it computes ("AI attention complexity ledger", section "带宽账：decode 阶段的真正瓶颈"): for each
// (b, h) the one new query attends to every cached key, s_j = scale * q . k_j for j < L_b, and returns
// o = sum_j softmax(s)_j v_j.  The page's point is that this step does O(L d) arithmetic on O(L d) bytes,
// so it is bound by HBM bandwidth: the kernel's job is to stream K and V once at full bandwidth.
//
// Design (B200):
//  * grid (split, h, b); split i owns cache rows [i*chunk, min((i+1)*chunk, L_b)).  Splits past L_b exit.
//  * one producer thread streams the split's K and V rows with 1-D bulk copies (cp.async.bulk) into
//    a DEC_STAGES-deep shared-memory ring of DEC_ROWS-row stages; each stage's K and V
//    rows are contiguous in HBM because the cache is [B, H, Lmax, d].
//  * eight consumer warps take 4 rows of each stage; lane l holds d/32 consecutive elements of q, k and v,
//    so a row's dot product is d/32 FMAs per lane plus a 5-step xor-shuffle reduction.  Each warp keeps
//    its own online-softmax state (running max m in log2 units, exp-sum l, fp32 output accumulator).
//  * the warp states are merged in shared memory, normalised, and written as one partial (o, lse).
//  * a second kernel merges the splits of each (b, h) with logsumexp weights (exact) and writes o, lse.
#pragma once

#include "ptx.cuh"

namespace eta {

constexpr int DEC_ROWS = 32;          // cache rows per pipeline stage
constexpr int DEC_STAGES = 4;         // pipeline depth
constexpr int DEC_CWARPS = 8;         // consumer warps (4 were compute-bound: 5.3 TB/s vs 7.3 with 8)
constexpr int DEC_THREADS = 32 * (1 + DEC_CWARPS);

// Rows per split: about Lmax/16, a multiple of the stage size, at most 1024 rows (512 KB of K+V at d=128).
__host__ __device__ inline int decode_chunk(int Lmax) {
  int c = (Lmax + 15) / 16;
  c = (c + DEC_ROWS - 1) / DEC_ROWS * DEC_ROWS;
  if (c < DEC_ROWS) c = DEC_ROWS;
  if (c > 1024) c = 1024;
  return c;
}
__host__ __device__ inline int decode_max_splits(int Lmax) {
  const int c = decode_chunk(Lmax);
  return (Lmax + c - 1) / c;
}

struct DecodeParams {
  const __nv_bfloat16 *q;   // [B, H, D]
  const __nv_bfloat16 *kc;  // [B, H, Lmax, D]
  const __nv_bfloat16 *vc;  // [B, H, Lmax, D]
  const int *kv_lens;       // [B]
  __nv_bfloat16 *o;         // [B, H, D]
  float *lse;               // [B, H] or null
  float *part_o;            // [B, H, max_splits, D]
  float *part_lse;          // [B, H, max_splits]
  int B, H, Lmax, chunk, max_splits;
  float scale_log2;         // scale * log2(e)
  long long wait_ns;
};

__device__ __forceinline__ int clamped_len(const DecodeParams &p, int b) {
  int L = p.kv_lens[b];
  if (L < 0 || L > p.Lmax) {
    record_status(2 /* ETA_DEV_BAD_KVLEN */);
    L = L < 0 ? 0 : p.Lmax;
  }
  return L;
}

template <int D>
__global__ void __launch_bounds__(DEC_THREADS) decode_split_kernel(const DecodeParams p) {
  constexpr int EPL = D / 32;                    // elements per lane
  constexpr int ROW_BYTES = D * 2;
  constexpr int STAGE_BYTES = DEC_ROWS * ROW_BYTES;
  extern __shared__ __align__(128) uint8_t dsmem[];
  uint8_t *sK = dsmem;                                     // [DEC_STAGES][DEC_ROWS][D]
  uint8_t *sV = dsmem + DEC_STAGES * STAGE_BYTES;          // [DEC_STAGES][DEC_ROWS][D]
  __shared__ __align__(8) uint64_t full[DEC_STAGES], empty[DEC_STAGES];
  __shared__ float wm[DEC_CWARPS], wl[DEC_CWARPS];
  __shared__ float wacc[DEC_CWARPS][D];
  __shared__ int abort_flag;

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int L = clamped_len(p, b);
  const int s0 = split * p.chunk;
  if (s0 >= L) return;  // no rows in this split (uniform over the CTA)
  const int nrows = min(L, s0 + p.chunk) - s0;
  const int nst = (nrows + DEC_ROWS - 1) / DEC_ROWS;
  const size_t head = (size_t)b * p.H + h;
  const __nv_bfloat16 *kbase = p.kc + (head * p.Lmax + s0) * D;
  const __nv_bfloat16 *vbase = p.vc + (head * p.Lmax + s0) * D;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < DEC_STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], DEC_CWARPS);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ---------------- producer: one thread streams K and V rows ----------------
    if (lane == 0) {
      int it = 0;
      for (; it < nst; ++it) {
        const int st = it % DEC_STAGES;
        if (!mbar_wait(&empty[st], ((it / DEC_STAGES) & 1) ^ 1, &abort_flag, p.wait_ns)) break;
        const int rows = min(DEC_ROWS, nrows - it * DEC_ROWS);
        const uint32_t bytes = (uint32_t)rows * ROW_BYTES;
        mbar_arrive_expect_tx(&full[st], 2 * bytes);
        bulk_load(sK + st * STAGE_BYTES, kbase + (size_t)it * DEC_ROWS * D, bytes, &full[st]);
        bulk_load(sV + st * STAGE_BYTES, vbase + (size_t)it * DEC_ROWS * D, bytes, &full[st]);
      }
      if (it < nst) {
        // Abandoned: let the copies already issued land before the CTA's shared memory goes away.
        for (int j = max(0, it - DEC_STAGES); j < it; ++j)
          mbar_wait(&full[j % DEC_STAGES], (j / DEC_STAGES) & 1, nullptr, p.wait_ns);
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int cw = warp - 1;
  float qf[EPL];
  {
    const __nv_bfloat16 *qp = p.q + head * D + lane * EPL;
#pragma unroll
    for (int e = 0; e < EPL; ++e) qf[e] = __bfloat162float(qp[e]) * p.scale_log2;
  }
  float m = -INFINITY, l = 0.f, acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;

  constexpr int RPW = DEC_ROWS / DEC_CWARPS;  // rows per warp per stage
  bool ok = true;
  for (int it = 0; it < nst; ++it) {
    const int st = it % DEC_STAGES;
    ok = mbar_wait(&full[st], (it / DEC_STAGES) & 1, &abort_flag, p.wait_ns);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    const int rows = min(DEC_ROWS, nrows - it * DEC_ROWS);
    const __nv_bfloat16 *ks = reinterpret_cast<const __nv_bfloat16 *>(sK + st * STAGE_BYTES);
    const __nv_bfloat16 *vs = reinterpret_cast<const __nv_bfloat16 *>(sV + st * STAGE_BYTES);
    float s[RPW];
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
      const int r = cw * RPW + i;
      float part = 0.f;
      if (r < rows) {
        const __nv_bfloat16 *kr = ks + r * D + lane * EPL;
        if constexpr (EPL == 4) {
          const uint2 raw = *reinterpret_cast<const uint2 *>(kr);
          const __nv_bfloat162 k01 = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
          const __nv_bfloat162 k23 = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
          part = qf[0] * __low2float(k01) + qf[1] * __high2float(k01) + qf[2] * __low2float(k23) +
                 qf[3] * __high2float(k23);
        } else {
          const __nv_bfloat162 k01 = *reinterpret_cast<const __nv_bfloat162 *>(kr);
          part = qf[0] * __low2float(k01) + qf[1] * __high2float(k01);
        }
      }
      s[i] = part;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
      for (int i = 0; i < RPW; ++i) s[i] += __shfl_xor_sync(0xffffffffu, s[i], off);
    }
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
      if (cw * RPW + i >= rows) s[i] = -INFINITY;
      mx = fmaxf(mx, s[i]);
    }
    const float m_new = fmaxf(m, mx);
    const float msub = (m_new == -INFINITY) ? 0.f : m_new;
    const float corr = ex2_approx(m - msub);  // 0 when m = -inf
    l *= corr;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] *= corr;
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
      const int r = cw * RPW + i;
      if (r < rows) {
        const float pr = ex2_approx(s[i] - msub);
        l += pr;
        const __nv_bfloat16 *vr = vs + r * D + lane * EPL;
        if constexpr (EPL == 4) {
          const uint2 raw = *reinterpret_cast<const uint2 *>(vr);
          const __nv_bfloat162 v01 = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
          const __nv_bfloat162 v23 = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
          acc[0] += pr * __low2float(v01);
          acc[1] += pr * __high2float(v01);
          acc[2] += pr * __low2float(v23);
          acc[3] += pr * __high2float(v23);
        } else {
          const __nv_bfloat162 v01 = *reinterpret_cast<const __nv_bfloat162 *>(vr);
          acc[0] += pr * __low2float(v01);
          acc[1] += pr * __high2float(v01);
        }
      }
    }
    m = m_new;
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }

  // merge the consumer warps' states, normalise, write this split's partial
  if (lane == 0) {
    wm[cw] = ok ? m : -INFINITY;
    wl[cw] = ok ? l : 0.f;
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) wacc[cw][lane * EPL + e] = ok ? acc[e] : 0.f;
  asm volatile("bar.sync 1, %0;" ::"r"(32 * DEC_CWARPS) : "memory");
  const int t = threadIdx.x - 32;  // consumer thread index
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < DEC_CWARPS; ++w) M = fmaxf(M, wm[w]);
  const float Msub = (M == -INFINITY) ? 0.f : M;
  float Lsum = 0.f;
  float wgt[DEC_CWARPS];
#pragma unroll
  for (int w = 0; w < DEC_CWARPS; ++w) {
    wgt[w] = ex2_approx(wm[w] - Msub);
    Lsum += wl[w] * wgt[w];
  }
  const size_t pidx = head * p.max_splits + split;
  for (int e = t; e < D; e += 32 * DEC_CWARPS) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < DEC_CWARPS; ++w) o += wacc[w][e] * wgt[w];
    p.part_o[pidx * D + e] = (Lsum > 0.f) ? o / Lsum : 0.f;
  }
  if (t == 0) p.part_lse[pidx] = (Lsum > 0.f) ? (Msub + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
}

// Merges the splits of one (b, h): lse = ln sum_i e^{lse_i}, o = sum_i e^{lse_i - lse} o_i.
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecodeParams p) {
  const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
  const int L = clamped_len(p, b);
  const int n = (L + p.chunk - 1) / p.chunk;
  const size_t head = (size_t)b * p.H + h;
  const float *pl = p.part_lse + head * p.max_splits;
  const float *po = p.part_o + head * p.max_splits * D;
  float M = -INFINITY;
  for (int i = 0; i < n; ++i) M = fmaxf(M, pl[i]);
  float o = 0.f, z = 0.f;
  if (M != -INFINITY) {
    for (int i = 0; i < n; ++i) {
      const float w = expf(pl[i] - M);
      z += w;
      o += w * po[(size_t)i * D + t];
    }
    o /= z;
  }
  p.o[head * D + t] = __float2bfloat16_rn(o);
  if (t == 0 && p.lse != nullptr) p.lse[head] = (M == -INFINITY) ? -INFINITY : M + logf(z);
}

}  // namespace eta
