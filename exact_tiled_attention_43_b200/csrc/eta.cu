// eta.cu -- the C ABI of libeta.so (declared in include/eta.h): argument validation, TMA tensor-map
// encoding, kernel launches and the device status word.  The kernels themselves live in prefill.cuh and
// decode.cuh and are compiled into this one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "eta.h"
#include "decode.cuh"
#include "decode_paged.cuh"
#include "prefill.cuh"
#include "prefill_wide.cuh"

namespace {

constexpr long long kDefaultWaitNs = 2000000000LL;  // 2 s
long long g_wait_ns = kDefaultWaitNs;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The current device must be sm_100 (B200 class).  Cached per device ordinal.
int check_device() {
  static int cache[64];  // 0 unknown, 1 ok, -1 bad
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ETA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return ETA_ERR_DEVICE;
  if (cache[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return ETA_ERR_CUDA;
    cache[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  return cache[dev] == 1 ? ETA_OK : ETA_ERR_DEVICE;
}

// Number of SMs of the current device (the persistent prefill grid), cached per device ordinal.
int sm_count(int *out) {
  static int cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ETA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return ETA_ERR_DEVICE;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      return ETA_ERR_CUDA;
    cache[dev] = n;
  }
  *out = cache[dev];
  return ETA_OK;
}

// Work-counter slot of the next prefill launch (round-robin over eta::PF_SCHED_SLOTS; a launch's last CTA
// returns its slot to zero, so a slot is reusable once the launch that held it has finished).
int next_sched_slot() {
  static std::atomic<unsigned int> next{0};
  return (int)(next.fetch_add(1u, std::memory_order_relaxed) % (unsigned int)eta::PF_SCHED_SLOTS);
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (no -lcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// The last few tensor maps this host thread encoded, keyed by everything that goes into one.  A call with
// the same buffers and shapes as a recent one (the usual case in a loop) reuses the map instead of encoding
// it again: the map holds only the address, sizes, strides, box and layout, so equal keys give equal maps.
struct MapKey {
  const void *base;
  long long n1, n2;
  int d, rows, elt, kind;  // kind: 0 dense, 1 packed, 2 page pool
  bool operator==(const MapKey &o) const {
    return base == o.base && n1 == o.n1 && n2 == o.n2 && d == o.d && rows == o.rows && elt == o.elt &&
           kind == o.kind;
  }
};
struct MapCache {
  static constexpr int N = 16;
  MapKey key[N];
  CUtensorMap map[N];
  bool used[N] = {};
  int next = 0;
  const CUtensorMap *find(const MapKey &k) const {
    for (int i = 0; i < N; ++i)
      if (used[i] && key[i] == k) return &map[i];
    return nullptr;
  }
  void put(const MapKey &k, const CUtensorMap &m) {
    key[next] = k;
    map[next] = m;
    used[next] = true;
    next = (next + 1) % N;
  }
};
thread_local MapCache t_maps;

// bf16 rows of `d` elements; box = 64 elements (128 B, one swizzle span) x `rows` rows.
// dense  : tensor [BH][N][d]      -> dims {d, N, BH},  box {64, rows, 1}
// packed : tensor [T][H][d]       -> dims {d, H, T},   box {64, 1, rows}
// `elt` bytes per element: 2 (bf16) or 1 (e4m3, mapped as bytes); the box always spans 128 bytes of a row.
int encode_map(CUtensorMap *m, const void *base, bool packed, long long n1, long long n2, int d, int rows,
               int elt = 2) {
  const MapKey key{base, n1, n2, d, rows, elt, packed ? 1 : 0};
  if (const CUtensorMap *hit = t_maps.find(key)) {
    *m = *hit;
    return ETA_OK;
  }
  EncodeTiledFn enc = get_encode();
  if (!enc) return ETA_ERR_CUDA;
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3], estr[3] = {1, 1, 1};
  dims[0] = (cuuint64_t)d;
  if (packed) {  // n1 = H, n2 = T
    dims[1] = (cuuint64_t)n1;
    dims[2] = (cuuint64_t)n2;
    strides[0] = (cuuint64_t)d * elt;
    strides[1] = (cuuint64_t)n1 * d * elt;
    box[0] = (cuuint32_t)(128 / elt); box[1] = 1; box[2] = (cuuint32_t)rows;
  } else {       // n1 = N, n2 = BH
    dims[1] = (cuuint64_t)n1;
    dims[2] = (cuuint64_t)n2;
    strides[0] = (cuuint64_t)d * elt;
    strides[1] = (cuuint64_t)n1 * d * elt;
    box[0] = (cuuint32_t)(128 / elt); box[1] = (cuuint32_t)rows; box[2] = 1;
  }
  CUresult r = enc(m, (elt == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16), 3, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return ETA_ERR_CUDA;
  t_maps.put(key, *m);
  return ETA_OK;
}

// Per-device, per-kernel launch set-up done once: the dynamic shared-memory limit and (for kernels that split
// their registers between warpgroups) the check of the build's register count.  `state` is the calling
// launcher's own table (one per kernel instance).
template <typename Kern>
int kernel_setup_once(std::atomic<int> (&state)[64], Kern kern, int smem, int want_regs) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ETA_ERR_CUDA;
  if (state[dev].load(std::memory_order_acquire) == 1) return ETA_OK;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return ETA_ERR_CUDA;
  if (want_regs > 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || fa.numRegs != want_regs) return ETA_ERR_CUDA;
  }
  state[dev].store(1, std::memory_order_release);  // a racing first call repeats the same set-up
  return ETA_OK;
}

template <int MODE>
int launch_prefill_wide(const void *q, const void *k, const void *v, bool packed, long long n1, long long n2,
                        dim3 grid, const eta::PrefillParams &p, cudaStream_t stream) {
  constexpr int D = eta::WideCfg::D;
  CUtensorMap mq, mk, mv;
  int rc;
  if ((rc = encode_map(&mq, q, packed, n1, n2, D, eta::PF_BM)) != ETA_OK) return rc;
  if ((rc = encode_map(&mk, k, packed, n1, n2, D, eta::WideCfg::BN)) != ETA_OK) return rc;
  if ((rc = encode_map(&mv, v, packed, n1, n2, D, eta::WideCfg::V_ROWS)) != ETA_OK) return rc;
  auto kern = eta::prefill_wide_kernel<MODE>;
  constexpr int smem = eta::WideCfg::SMEM_BYTES;
  static std::atomic<int> ready[64];
  if ((rc = kernel_setup_once(ready, kern, smem, 0)) != ETA_OK) return rc;
  kern<<<grid, eta::WideCfg::THREADS, smem, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? ETA_OK : ETA_ERR_CUDA;
}

template <int D, int MODE, bool F8 = false>
int launch_prefill(const void *q, const void *k, const void *v, bool packed, long long n1, long long n2, dim3 grid,
                   const eta::PrefillParams &p, cudaStream_t stream) {
  using C = eta::PfCfg<D, F8>;
  CUtensorMap mq, mk, mv;
  int rc;
  // Q tiles are 128 rows; K/V tiles are BN rows.
  if ((rc = encode_map(&mq, q, packed, n1, n2, D, eta::PF_BM, C::ELT)) != ETA_OK) return rc;
  if ((rc = encode_map(&mk, k, packed, n1, n2, D, C::BN, C::ELT)) != ETA_OK) return rc;
  if ((rc = encode_map(&mv, v, packed, n1, n2, D, C::BN, C::ELT)) != ETA_OK) return rc;
  auto kern = eta::prefill_kernel<D, MODE, F8>;
  constexpr int smem = C::SMEM_BYTES;
  // The kernel re-splits its registers between warpgroups (setmaxnreg); the split only adds up when the
  // build uses exactly PF_LAUNCH_REGS registers per thread, so refuse any other build.
  static std::atomic<int> ready[64];
  if ((rc = kernel_setup_once(ready, kern, smem, eta::PF_LAUNCH_REGS)) != ETA_OK) return rc;
  kern<<<grid, eta::PF_THREADS, smem, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? ETA_OK : ETA_ERR_CUDA;
}

bool finite_pos(float x) { return std::isfinite(x) && x > 0.f; }

// Work decomposition of a prefill launch: `units` (batch, head) or (sequence, head) pairs of `rows` query
// rows (N, or max_len for packed launches) -> work items, how many stay whole, and the persistent grid.
struct PrefillPlan {
  long long nblk = 0, items = 0, whole = 0, split_items = 0;
  int ctas = 0;
};

// Dense launches take their (batch, head) units in groups whose K and V (2 * rows * d * elt bytes per unit)
// fit in this many bytes, a quarter of the B200's L2, so that the row blocks of a unit find its K/V tiles
// in L2 (the kernels' decode_item order).
constexpr long long kSchedGroupBytes = 32ll << 20;
long long sched_group(long long units, long long rows, int d, int elt) {
  const long long kv = 2 * rows * (long long)d * elt;
  const long long g = kv > 0 ? kSchedGroupBytes / kv : units;
  return std::max<long long>(1, std::min<long long>(g, units));
}
int plan_prefill(int mode, long long units, long long rows, int d, int causal, int sms, PrefillPlan *pl) {
  if (d != 64 && d != 96 && d != 128 && !(d == 256 && mode != eta::MODE_HSTU)) return ETA_ERR_HEAD_DIM;
  if (units <= 0 || rows <= 0 || sms <= 0) return ETA_ERR_SHAPE;
  if (causal != 0 && causal != 1) return ETA_ERR_ARG;
  const long long rows_per_item = (d == 256) ? eta::PF_BM : 2 * eta::PF_BM;  // one or two 128-row Q tiles
  pl->nblk = (rows + rows_per_item - 1) / rows_per_item;
  if (pl->nblk > 65535) return ETA_ERR_SHAPE;
  pl->items = units * pl->nblk;
  // The work counter may run past the work count by one per CTA: keep it far from 2^32.
  if (pl->items > (long long)INT_MAX / 4) return ETA_ERR_SHAPE;
  const long long G = std::min<long long>(pl->items, sms);  // CTAs the unsplit items would occupy
  // Split items (softmax modes): one Q tile each, its key tiles halved between the CTA's two softmax
  // warpgroups and merged in the CTA (needs at least two key tiles: more than 128 rows).  Non-causal dense
  // items all cost the same: when their count leaves a last wave at most half full, those last items are
  // split, so the last wave takes about half an item's time.  Launches too small to fill the GPU split every
  // item: causal ones (whose heaviest item sets the time of a single partial wave) with no more items than
  // SMs, non-causal ones with at most half as many (B1 H8 N2048 d128: causal 196 -> 290 TFLOP/s,
  // non-causal 357 -> 524).  Packed (varlen) launches follow the same rules on their item count.
  pl->whole = pl->items;
  if (mode != eta::MODE_HSTU && d <= 128 && rows > 128) {
    if (causal == 0 && pl->items > G) {
      const long long R = pl->items % G;
      if (R > 0 && 2 * R <= G) pl->whole = pl->items - R;
    } else if ((causal != 0 && pl->items <= sms) || (causal == 0 && 2 * pl->items <= sms)) {
      pl->whole = 0;
    }
  }
  pl->split_items = pl->whole + 2 * (pl->items - pl->whole);
  // persistent: at most one CTA per SM, and no more CTAs than (split) items
  pl->ctas = (int)std::min<long long>(pl->split_items, sms);
  return ETA_OK;
}

int prefill_common(int mode, const void *q, const void *k, const void *v, void *o, float *lse,
                   const int *cu_seqlens, int B, int S, int N, int max_len, int T_total, int H, int d,
                   float scale, int causal, int o_dtype, float alpha, float inv_n, void *stream, bool f8 = false,
                   float qk_descale = 1.f, float v_descale = 1.f) {
  if (!q || !k || !v || !o) return ETA_ERR_NULL;
  if (mode != eta::MODE_DENSE && !cu_seqlens) return ETA_ERR_NULL;
  if (f8 && d != 128) return ETA_ERR_HEAD_DIM;  // e4m3: one 128-byte swizzle span per row
  if (f8 && (!finite_pos(qk_descale) || !finite_pos(v_descale))) return ETA_ERR_ARG;
  // head dims 64, 96 and 128 (two 128-row Q tiles per work item); 256 for softmax attention (one Q tile per item)
  if (d != 64 && d != 96 && d != 128 && !(d == 256 && mode != eta::MODE_HSTU)) return ETA_ERR_HEAD_DIM;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ETA_ERR_ALIGN;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ETA_ERR_ALIGN;
  if (o_dtype != ETA_OUT_BF16 && o_dtype != ETA_OUT_F32) return ETA_ERR_ARG;
  if (causal != 0 && causal != 1) return ETA_ERR_ARG;
  if (H <= 0 || H > 65535) return ETA_ERR_SHAPE;
  eta::PrefillParams p{};
  long long n1, n2, units, rows;
  if (mode == eta::MODE_DENSE) {
    if (B <= 0 || N <= 0) return ETA_ERR_SHAPE;
    units = (long long)B * H;
    if (units > INT_MAX) return ETA_ERR_SHAPE;
    rows = N;
    n1 = N;
    n2 = units;
    p.N = N;
    p.BH = (int)units;
    p.grp = (int)sched_group(units, rows, d, f8 ? 1 : 2);
  } else {
    if (S <= 0 || max_len <= 0 || T_total < 0 || S > 65535) return ETA_ERR_SHAPE;
    if (T_total == 0) return ETA_OK;  // nothing to compute
    units = (long long)S * H;
    rows = max_len;
    n1 = H;
    n2 = T_total;
    p.max_len = max_len;
    p.S = S;
    p.T_total = T_total;
  }
  if (mode == eta::MODE_HSTU) {
    if (!std::isfinite(alpha) || !finite_pos(inv_n)) return ETA_ERR_ARG;
    if (o_dtype != ETA_OUT_BF16) return ETA_ERR_ARG;
  } else if (!finite_pos(scale)) {
    return ETA_ERR_ARG;
  }
  PrefillPlan pl;
  int rc = plan_prefill(mode, units, rows, d, causal, 1, &pl);  // shape checks before any device query
  if (rc != ETA_OK) return rc;
  if ((rc = check_device()) != ETA_OK) return rc;
  int sms = 0;
  if ((rc = sm_count(&sms)) != ETA_OK) return rc;
  if ((rc = plan_prefill(mode, units, rows, d, causal, sms, &pl)) != ETA_OK) return rc;
  p.nblk = (int)pl.nblk;
  p.n_whole = (int)pl.whole;
  p.n_items = (int)pl.split_items;
  const dim3 grid((unsigned)pl.ctas, 1, 1);
  p.sched_slot = next_sched_slot();
  p.o = o;
  p.lse = (mode == eta::MODE_HSTU) ? nullptr : lse;
  p.cu_seqlens = cu_seqlens;
  p.H = H;
  p.causal = causal;
  p.o_f32 = (o_dtype == ETA_OUT_F32);
  p.scale_log2 = scale * qk_descale * 1.4426950408889634f;
  p.hstu_half_alpha = 0.5f * alpha;
  p.hstu_inv_n = inv_n;
  p.o_scale = v_descale;
  p.wait_ns = g_wait_ns;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool packed = (mode != eta::MODE_DENSE);
  if (f8) return launch_prefill<128, eta::MODE_DENSE, true>(q, k, v, packed, n1, n2, grid, p, st);
  if (d == 256) {
    if (mode == eta::MODE_DENSE) return launch_prefill_wide<eta::MODE_DENSE>(q, k, v, packed, n1, n2, grid, p, st);
    return launch_prefill_wide<eta::MODE_VARLEN>(q, k, v, packed, n1, n2, grid, p, st);
  }
  if (d == 64) {
    if (mode == eta::MODE_DENSE) return launch_prefill<64, eta::MODE_DENSE>(q, k, v, packed, n1, n2, grid, p, st);
    if (mode == eta::MODE_VARLEN) return launch_prefill<64, eta::MODE_VARLEN>(q, k, v, packed, n1, n2, grid, p, st);
    return launch_prefill<64, eta::MODE_HSTU>(q, k, v, packed, n1, n2, grid, p, st);
  }
  if (d == 96) {
    if (mode == eta::MODE_DENSE) return launch_prefill<96, eta::MODE_DENSE>(q, k, v, packed, n1, n2, grid, p, st);
    if (mode == eta::MODE_VARLEN) return launch_prefill<96, eta::MODE_VARLEN>(q, k, v, packed, n1, n2, grid, p, st);
    return launch_prefill<96, eta::MODE_HSTU>(q, k, v, packed, n1, n2, grid, p, st);
  }
  if (mode == eta::MODE_DENSE) return launch_prefill<128, eta::MODE_DENSE>(q, k, v, packed, n1, n2, grid, p, st);
  if (mode == eta::MODE_VARLEN) return launch_prefill<128, eta::MODE_VARLEN>(q, k, v, packed, n1, n2, grid, p, st);
  return launch_prefill<128, eta::MODE_HSTU>(q, k, v, packed, n1, n2, grid, p, st);
}

template <int D>
int launch_decode(const eta::DecodeParams &p, cudaStream_t st) {
  constexpr int smem = 2 * eta::DEC_STAGES * eta::DEC_ROWS * D * 2;
  auto ks = eta::decode_split_kernel<D>;
  static std::atomic<int> ready[64];
  int rc;
  if ((rc = kernel_setup_once(ready, ks, smem, 0)) != ETA_OK) return rc;
  ks<<<dim3(p.max_splits, p.H, p.B), eta::DEC_THREADS, smem, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return ETA_ERR_CUDA;
  eta::decode_combine_kernel<D><<<dim3(p.H, p.B), D, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? ETA_OK : ETA_ERR_CUDA;
}

size_t decode_ws_bytes(int B, int H, int Lmax, int d) {
  const size_t n = (size_t)B * H * eta::decode_max_splits(Lmax);
  const size_t o_bytes = (n * d * sizeof(float) + 255) & ~size_t(255);
  return o_bytes + n * sizeof(float);
}

// Page pool [num_pages, Hkv, page_size, d] bf16 viewed as a 3-D tensor {d, page_size, num_pages * Hkv}; box =
// 64 elements (128 B, one swizzle span) x min(page_size, 32) rows x 1.
int encode_paged_map(CUtensorMap *m, const void *base, int num_pages, int Hkv, int page_size, int d) {
  const MapKey key{base, num_pages, Hkv, d, page_size, 2, 2};
  if (const CUtensorMap *hit = t_maps.find(key)) {
    *m = *hit;
    return ETA_OK;
  }
  EncodeTiledFn enc = get_encode();
  if (!enc) return ETA_ERR_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)page_size, (cuuint64_t)num_pages * Hkv};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)page_size * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)std::min(page_size, eta::DPG_ROWS), 1}, estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return ETA_ERR_CUDA;
  t_maps.put(key, *m);
  return ETA_OK;
}

template <int D>
int launch_decode_paged(const void *k_pages, const void *v_pages, const eta::PagedDecodeParams &p,
                        const eta::DecodeParams &cp, cudaStream_t st) {
  CUtensorMap mk, mv;
  int rc;
  if ((rc = encode_paged_map(&mk, k_pages, p.num_pages, p.Hkv, p.page_size, D)) != ETA_OK) return rc;
  if ((rc = encode_paged_map(&mv, v_pages, p.num_pages, p.Hkv, p.page_size, D)) != ETA_OK) return rc;
  constexpr int smem = 1024 /*alignment slack*/ + 2 * eta::DPG_STAGES * eta::DPG_ROWS * D * 2;
  auto ks = eta::decode_paged_split_kernel<D>;
  static std::atomic<int> ready[64];
  if ((rc = kernel_setup_once(ready, ks, smem, 0)) != ETA_OK) return rc;
  ks<<<dim3(p.max_splits, p.Hkv, p.B), eta::DPG_THREADS, smem, st>>>(mk, mv, p);
  if (cudaGetLastError() != cudaSuccess) return ETA_ERR_CUDA;
  eta::decode_combine_kernel<D><<<dim3(cp.H, cp.B), D, 0, st>>>(cp);
  return cudaGetLastError() == cudaSuccess ? ETA_OK : ETA_ERR_CUDA;
}

bool valid_page_size(int ps) { return ps == 16 || ps == 32 || ps == 64 || ps == 128 || ps == 256; }

__global__ void selftest_wait_kernel(long long wait_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    eta::mbar_init(&bar, 1);  // nothing ever arrives
    abort_flag = 0;
    eta::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) eta::mbar_wait(&bar, 0, &abort_flag, wait_ns);
}

}  // namespace

extern "C" {

int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int N, int d,
             float scale, int causal, int o_dtype, void *stream) {
  return prefill_common(eta::MODE_DENSE, q, k, v, o, lse, nullptr, B, 0, N, 0, 0, H, d, scale, causal, o_dtype, 0.f,
                        1.f, stream);
}

int attn_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse, const int *cu_seqlens, int S,
                    int max_len, int T_total, int H, int d, float scale, int causal, int o_dtype, void *stream) {
  return prefill_common(eta::MODE_VARLEN, q, k, v, o, lse, cu_seqlens, 0, S, 0, max_len, T_total, H, d, scale, causal,
                        o_dtype, 0.f, 1.f, stream);
}

int attn_fwd_fp8(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int N, int d,
                 float scale, float q_descale, float k_descale, float v_descale, int causal, int o_dtype,
                 void *stream) {
  if (!finite_pos(q_descale) || !finite_pos(k_descale)) return ETA_ERR_ARG;
  return prefill_common(eta::MODE_DENSE, q, k, v, o, lse, nullptr, B, 0, N, 0, 0, H, d, scale, causal, o_dtype, 0.f,
                        1.f, stream, true, q_descale * k_descale, v_descale);
}

int hstu_fwd_jagged(const void *q, const void *k, const void *v, void *o, const int *cu_seqlens, int S, int max_len,
                    int T_total, int H, int d, float alpha, float inv_n, void *stream) {
  return prefill_common(eta::MODE_HSTU, q, k, v, o, nullptr, cu_seqlens, 0, S, 0, max_len, T_total, H, d, 1.f, 1,
                        ETA_OUT_BF16, alpha, inv_n, stream);
}

size_t attn_decode_workspace_size(int B, int H, int Lmax, int d) {
  if (B <= 0 || H <= 0 || Lmax <= 0 || (d != 64 && d != 128)) return 0;
  return decode_ws_bytes(B, H, Lmax, d);
}

int attn_decode(const void *q, const void *kcache, const void *vcache, const int *kv_lens, void *o, float *lse, int B,
                int H, int Lmax, int d, float scale, void *workspace, size_t workspace_bytes, void *stream) {
  if (!q || !kcache || !vcache || !kv_lens || !o || !workspace) return ETA_ERR_NULL;
  if (d != 64 && d != 128) return ETA_ERR_HEAD_DIM;
  if (B <= 0 || H <= 0 || Lmax <= 0 || B > 65535 || H > 65535) return ETA_ERR_SHAPE;
  if ((long long)B * H * Lmax * d >= (1LL << 40)) return ETA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(o) || !aligned16(workspace))
    return ETA_ERR_ALIGN;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ETA_ERR_ALIGN;
  if (!finite_pos(scale)) return ETA_ERR_ARG;
  if (workspace_bytes < decode_ws_bytes(B, H, Lmax, d)) return ETA_ERR_WORKSPACE;
  int rc = check_device();
  if (rc != ETA_OK) return rc;
  eta::DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.kc = static_cast<const __nv_bfloat16 *>(kcache);
  p.vc = static_cast<const __nv_bfloat16 *>(vcache);
  p.kv_lens = kv_lens;
  p.o = static_cast<__nv_bfloat16 *>(o);
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Lmax = Lmax;
  p.chunk = eta::decode_chunk(Lmax);
  p.max_splits = eta::decode_max_splits(Lmax);
  const size_t n = (size_t)B * H * p.max_splits;
  p.part_o = static_cast<float *>(workspace);
  p.part_lse = reinterpret_cast<float *>(static_cast<char *>(workspace) + ((n * d * sizeof(float) + 255) & ~size_t(255)));
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_ns = g_wait_ns;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 64 ? launch_decode<64>(p, st) : launch_decode<128>(p, st);
}

size_t attn_decode_paged_workspace_size(int B, int Hq, int max_pages, int page_size, int d) {
  if (B <= 0 || Hq <= 0 || max_pages <= 0 || !valid_page_size(page_size) || (d != 64 && d != 128)) return 0;
  if ((long long)max_pages * page_size > INT_MAX) return 0;
  return decode_ws_bytes(B, Hq, max_pages * page_size, d);
}

int attn_decode_paged(const void *q, const void *k_pages, const void *v_pages, const int *block_table,
                      const int *kv_lens, void *o, float *lse, int B, int Hq, int Hkv, int num_pages, int page_size,
                      int max_pages, int d, float scale, void *workspace, size_t workspace_bytes, void *stream) {
  if (!q || !k_pages || !v_pages || !block_table || !kv_lens || !o || !workspace) return ETA_ERR_NULL;
  if (d != 64 && d != 128) return ETA_ERR_HEAD_DIM;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || num_pages <= 0 || max_pages <= 0 || B > 65535 || Hkv > 65535)
    return ETA_ERR_SHAPE;
  if (Hq % Hkv != 0 || Hq / Hkv > eta::DPG_MAX_G) return ETA_ERR_SHAPE;
  if (!valid_page_size(page_size)) return ETA_ERR_SHAPE;
  if ((long long)num_pages * Hkv > INT_MAX || (long long)max_pages * page_size > INT_MAX ||
      (long long)B * max_pages > INT_MAX)
    return ETA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o) || !aligned16(workspace))
    return ETA_ERR_ALIGN;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ETA_ERR_ALIGN;
  if (!finite_pos(scale)) return ETA_ERR_ARG;
  const int Lmax = max_pages * page_size;
  if (workspace_bytes < decode_ws_bytes(B, Hq, Lmax, d)) return ETA_ERR_WORKSPACE;
  int rc = check_device();
  if (rc != ETA_OK) return rc;
  eta::PagedDecodeParams p{};
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.block_table = block_table;
  p.kv_lens = kv_lens;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.num_pages = num_pages;
  p.page_size = page_size;
  p.max_pages = max_pages;
  p.Lmax = Lmax;
  p.chunk = eta::decode_chunk(Lmax);
  p.max_splits = eta::decode_max_splits(Lmax);
  const size_t n = (size_t)B * Hq * p.max_splits;
  p.part_o = static_cast<float *>(workspace);
  p.part_lse = reinterpret_cast<float *>(static_cast<char *>(workspace) + ((n * d * sizeof(float) + 255) & ~size_t(255)));
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_ns = g_wait_ns;
  // the split merge is the contiguous decode's combine step over the Hq query heads
  eta::DecodeParams cp{};
  cp.kv_lens = kv_lens;
  cp.o = static_cast<__nv_bfloat16 *>(o);
  cp.lse = lse;
  cp.part_o = p.part_o;
  cp.part_lse = p.part_lse;
  cp.B = B;
  cp.H = Hq;
  cp.Lmax = Lmax;
  cp.chunk = p.chunk;
  cp.max_splits = p.max_splits;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 64 ? launch_decode_paged<64>(k_pages, v_pages, p, cp, st)
                 : launch_decode_paged<128>(k_pages, v_pages, p, cp, st);
}

int eta_status(void *stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return ETA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, eta::g_status, sizeof(int)) != cudaSuccess) return ETA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(eta::g_status, &zero, sizeof(int)) != cudaSuccess) return ETA_ERR_CUDA;
  return v;
}

const char *eta_strerror(int code) {
  switch (code) {
    case ETA_OK: return "ok";
    case ETA_ERR_NULL: return "a required pointer is NULL";
    case ETA_ERR_HEAD_DIM:
      return "unsupported head dimension (attn_fwd, attn_fwd_varlen: 64, 96, 128, 256; hstu_fwd_jagged: 64, 96, 128; "
             "attn_fwd_fp8: 128; attn_decode, attn_decode_paged: 64, 128)";
    case ETA_ERR_SHAPE: return "a size is out of range or inconsistent";
    case ETA_ERR_ALIGN: return "a tensor pointer is not 16-byte aligned";
    case ETA_ERR_WORKSPACE: return "workspace is smaller than attn_decode_workspace_size()";
    case ETA_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case ETA_ERR_ARG: return "a flag or scalar argument is out of range";
    case ETA_ERR_DEVICE: return "the current device is not an sm_100 GPU";
    case ETA_DEV_TIMEOUT: return "device: a bounded pipeline wait expired";
    case ETA_DEV_BAD_KVLEN: return "device: kv_lens entry outside [0, Lmax]";
    case ETA_DEV_BAD_CUSEQ:
      return "device: cu_seqlens not a valid offset table for the call (negative or decreasing, a sequence longer "
             "than max_len, first offset not 0 or last offset not T_total)";
    case ETA_DEV_BAD_PAGE: return "device: a block_table entry outside [0, num_pages)";
    default: return "unknown code";
  }
}

void eta_set_wait_timeout_ns(long long ns) { g_wait_ns = ns > 0 ? ns : kDefaultWaitNs; }

int eta_selftest_wait_timeout(void *stream) {
  int rc = check_device();
  if (rc != ETA_OK) return rc;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(g_wait_ns);
  return cudaGetLastError() == cudaSuccess ? ETA_OK : ETA_ERR_CUDA;
}

long long eta_prefill_sched_group(long long units, long long rows, int d, int elt_bytes) {
  if (units <= 0 || rows <= 0 || d <= 0 || (elt_bytes != 1 && elt_bytes != 2)) return ETA_ERR_SHAPE;
  return sched_group(units, rows, d, elt_bytes);
}

int eta_prefill_plan(int kind, long long units, long long rows, int d, int causal, int sms, long long *items,
                     long long *whole, int *ctas) {
  if (kind < eta::MODE_DENSE || kind > eta::MODE_HSTU) return ETA_ERR_ARG;
  if (kind == eta::MODE_HSTU) causal = 1;
  PrefillPlan pl;
  const int rc = plan_prefill(kind, units, rows, d, causal, sms, &pl);
  if (rc != ETA_OK) return rc;
  if (items) *items = pl.items;
  if (whole) *whole = pl.whole;
  if (ctas) *ctas = pl.ctas;
  return ETA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------
// Allocation-free decode: the split-KV partials live in a fixed file-scope device array instead of a
// caller-provided workspace.  Same kernels as attn_decode.
// ------------------------------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[ETA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch per device ordinal, looked up once with that device current.  In
// host code the array's name is only a host-side stand-in; kernels must be given this address.
void *noalloc_scratch_ptr(int *rc) {
  static void *ptrs[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *rc = ETA_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      *rc = ETA_ERR_CUDA;
      return nullptr;
    }
    ptrs[dev] = p;
  }
  *rc = ETA_OK;
  return ptrs[dev];
}

}  // namespace

extern "C" int attn_decode_noalloc(const void *q, const void *kcache, const void *vcache, const int *kv_lens,
                                   void *o, float *lse, int B, int H, int Lmax, int d, float scale, void *stream) {
  if (B > 0 && H > 0 && Lmax > 0 && (d == 64 || d == 128) &&
      decode_ws_bytes(B, H, Lmax, d) > (size_t)ETA_NOALLOC_SCRATCH_BYTES)
    return ETA_ERR_WORKSPACE;
  // Argument checks that need no device come first (same order as attn_decode).
  if (!q || !kcache || !vcache || !kv_lens || !o) return ETA_ERR_NULL;
  if (d != 64 && d != 128) return ETA_ERR_HEAD_DIM;
  if (B <= 0 || H <= 0 || Lmax <= 0) return ETA_ERR_SHAPE;
  int rc = check_device();
  if (rc != ETA_OK) return rc;
  void *scratch = noalloc_scratch_ptr(&rc);
  if (rc != ETA_OK) return rc;
  return attn_decode(q, kcache, vcache, kv_lens, o, lse, B, H, Lmax, d, scale, scratch,
                     (size_t)ETA_NOALLOC_SCRATCH_BYTES, stream);
}

