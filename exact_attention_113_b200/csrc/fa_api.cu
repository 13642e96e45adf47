// fa_api.cu -- the C ABI declared in include/fa.h: argument checks, TMA
// tensor-map encoding, kernel selection and launch, device status.
//
// Operator statement followed ("FlashAttention算法原理与性能优化实战" section
// 2.2): 4-D [B, H, S, D] query/key/value, an output shaped like the query,
// fp32 softmax statistics of shape [B, H, S]; scale, pre_tokens and
// next_tokens as attributes.  The statistics here are one log-sum-exp per row
// (Triton FA2 walkthrough: the logsumexp kept for the backward pass).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "fa.h"
#include "fa_fwd_kernel.cuh"
#include "fa_bwd_kernel.cuh"
#include "fa_decode_kernel.cuh"

namespace fa {
namespace {

constexpr int kVersion = 10000;  // 1.0.0
constexpr int kMaxSeq = 1 << 30;
constexpr int kMaxSplits = 64;

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A rank-3 tensor map over a contiguous [n_heads, L, D] array with a box of
// [box_heads, box_rows, box_cols] and the swizzle that matches `box_cols`
// 16-bit elements.  box_heads * box_rows = 128 (one tile of rows).
bool encode_map(CUtensorMap *map, const void *base, int dtype, int n_heads, int L, int D,
                int box_cols, int box_rows = kBM, int box_heads = 1) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  // dtype 0 fp16, 1 bf16, 2 fp8 e4m3 (moved as bytes)
  const CUtensorMapDataType dt = dtype == FA_F16    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                 : dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const cuuint64_t es = dtype == 2 ? 1 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L),
                        static_cast<cuuint64_t>(n_heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * es,
                           static_cast<cuuint64_t>(L) * D * es};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows),
                       static_cast<cuuint32_t>(box_heads)};
  cuuint32_t estr[3] = {1, 1, 1};
  const int sw_bytes = box_cols * static_cast<int>(es);
  const CUtensorMapSwizzle sw = sw_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : sw_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                 : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = enc(map, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A rank-3 fp32 tensor map over a contiguous [n_heads, L, D] array with a
// box of [1, 128, box_cols] (box_cols 32: 128-byte swizzle; 16: 64-byte).
bool encode_map_f32(CUtensorMap *map, const void *base, int n_heads, int L, int D,
                    int box_cols) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L),
                        static_cast<cuuint64_t>(n_heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 4,
                           static_cast<cuuint64_t>(L) * D * 4};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(kBM), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw =
      box_cols * 4 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Head dims of the 16-bit forward: every multiple of 16 up to 128 (rows of
// 32..256 bytes, swizzled in 128-, 64- or 32-byte atoms).
bool valid_fwd_d(int D) { return D >= 16 && D <= 128 && D % 16 == 0; }

// The swizzle span (bytes) of a row of D elements of `es` bytes.
int sw_span(int D, int es) {
  const int rb = D * es;
  return rb % 128 == 0 ? 128 : (rb % 64 == 0 ? 64 : 32);
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

__global__ void fill_kernel(float *p, size_t n, float value) {
  size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (; i < n; i += stride) p[i] = value;
}

template <int D, int DT, bool kMask, bool kDual = false>
int launch_kernel(const FwdParams &prm, int B, int H, cudaStream_t stream) {
  using G = Geo<D, DT == 2 ? 1 : 2>;
  auto kern = fa_fwd_kernel<D, DT, kMask, kDual>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  static bool configured[64] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return FA_ERR_CUDA;
    if (!configured[dev]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               G::kSmemBytes) != cudaSuccess)
        return FA_ERR_CUDA;
      configured[dev] = true;
    }
  }
  const unsigned items = static_cast<unsigned>(B) * (prm.packed ? prm.H_kv : H);
  if (prm.bal) {
    // balanced one-wave schedule: clusters of two CTAs, all resident at once
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2u * items * static_cast<unsigned>(prm.bal_cpi), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = G::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    static int max_clusters[64] = {};   // per device: pairs resident at once (0: not known)
    int mc = 0;
    {
      std::lock_guard<std::mutex> lock(mu);
      if (max_clusters[dev] == 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
          cudaGetLastError();
          n = -1;
        }
        max_clusters[dev] = n;
      }
      mc = max_clusters[dev];
    }
    if (mc >= static_cast<int>(items) * prm.bal_cpi) {
      if (cudaLaunchKernelEx(&cfg, kern, prm) != cudaSuccess) return FA_ERR_CUDA;
      return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
    }
    FwdParams plain = prm;                // the pairs would not all fit: plain grid
    plain.bal = 0;
    dim3 grid(static_cast<unsigned>(plain.n_qpairs) * items, 1, 1);
    kern<<<grid, kThreads, G::kSmemBytes, stream>>>(plain);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
  }
  dim3 grid(static_cast<unsigned>(prm.n_qpairs) * items * static_cast<unsigned>(prm.n_splits),
            1, 1);
  kern<<<grid, kThreads, G::kSmemBytes, stream>>>(prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// One query tile per CTA: the dual softmax (the tile's keys split between
// both softmax warpgroups); two tiles: the kernel's default for its head dim.
template <int D, int DT, bool kMask>
int launch(const FwdParams &prm, int B, int H, cudaStream_t stream) {
  if (prm.tiles == 1) return launch_kernel<D, DT, kMask, true>(prm, B, H, stream);
  return launch_kernel<D, DT, kMask, false>(prm, B, H, stream);
}

// Split-KV workspace: partial O [n_splits][rows][D] fp32, then (m, l)
// [n_splits][rows] as float2, starting at a 256-byte boundary.
size_t ws_o_bytes(int64_t rows, int D, int n_splits) {
  return static_cast<size_t>(n_splits) * rows * D * sizeof(float);
}
size_t ws_ml_offset(int64_t rows, int D, int n_splits) {
  return (ws_o_bytes(rows, D, n_splits) + 255) & ~static_cast<size_t>(255);
}
size_t ws_total_bytes(int64_t rows, int D, int n_splits) {
  return ws_ml_offset(rows, D, n_splits) + static_cast<size_t>(n_splits) * rows * sizeof(float2);
}

// Merge the key slices of every row: m = max_s m_s, w_s = 2^(m_s - m),
// O = oscale * sum_s w_s O_s / sum_s w_s l_s, lse = (m + log2 l) ln 2.  One
// warp per row; the slices' partial sums are exact softmax pieces of the
// same row (online-softmax merge of "FlashAttention算法原理与性能优化实战"
// §1.2.2).  DT: 0 fp16 / 1 bf16 output, 2 (fp8 inputs) bf16 output; oscale
// is descale_v for fp8 inputs, else 1.
template <int D, int DT>
__global__ void __launch_bounds__(256) fa_combine_kernel(const float *ws_o, const float2 *ws_ml,
                                                         void *out, float *lse, int n_splits,
                                                         long long rows_total, float oscale) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows_total) return;
  float m = -INFINITY;
  for (int sp = 0; sp < n_splits; ++sp) m = fmaxf(m, ws_ml[sp * rows_total + row].x);
  constexpr int kPer = (D + 31) / 32;   // elements per lane
  float acc[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) acc[u] = 0.0f;
  float l = 0.0f;
  if (m != -INFINITY) {
    for (int sp = 0; sp < n_splits; ++sp) {
      const float2 ml = ws_ml[sp * rows_total + row];
      if (ml.x == -INFINITY) continue;
      const float w = exp2f(ml.x - m);
      l += w * ml.y;
      const float *o = ws_o + (static_cast<size_t>(sp) * rows_total + row) * D;
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int d = lane + 32 * u;
        if (d < D) acc[u] += w * o[d];
      }
    }
  }
  const float inv_l = l > 0.0f ? oscale / l : 0.0f;
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int d = lane + 32 * u;
    if (d >= D) continue;
    const float val = acc[u] * inv_l;
    if constexpr (DT == 0)
      reinterpret_cast<__half *>(out)[row * D + d] = __float2half_rn(val);
    else
      reinterpret_cast<__nv_bfloat16 *>(out)[row * D + d] = __float2bfloat16_rn(val);
  }
  if (lse != nullptr && lane == 0)
    lse[row] = l > 0.0f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
}

template <int D, int DT>
int launch_combine(const float *ws_o, const float2 *ws_ml, void *out, float *lse, int n_splits,
                   long long rows_total, cudaStream_t stream, float oscale = 1.0f) {
  const unsigned blocks = static_cast<unsigned>((rows_total + 7) / 8);
  fa_combine_kernel<D, DT><<<blocks, 256, 0, stream>>>(ws_o, ws_ml, out, lse, n_splits,
                                                       rows_total, oscale);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// ---------------------------------------------------------------- decoding
// Problems with at most kDecMaxRows query rows per K/V head (decoding: one
// new token per head, or a GQA group's few heads, against a long cache) run
// on the CUDA-core decode kernel (fa_decode_kernel.cuh) instead of the
// tensor-core kernel, whose 128-row tiles would hold one real row.
constexpr int kDecMaxRows = 2;

bool decode_eligible(int D, int dtype, int64_t rows_per_kv_head) {
  if (rows_per_kv_head < 1 || rows_per_kv_head > kDecMaxRows) return false;
  if (dtype == 2) return D == 32 || D == 64 || D == 128;
  return D == 16 || D == 32 || D == 64 || D == 128;
}

int sm_count() {
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
    return sms;
  cudaGetLastError();
  return 148;
}

template <int D, int DT, int R>
int launch_decode_kernel(const DecParams &prm, unsigned grid, cudaStream_t stream) {
  auto kern = fa_decode_kernel<D, DT, R>;
  const int smem = DecSmem<D, DT, R>::kBytes;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  static bool configured[64] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return FA_ERR_CUDA;
    if (!configured[dev]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess)
        return FA_ERR_CUDA;
      configured[dev] = true;
    }
  }
  kern<<<grid, kDecThreads, smem, stream>>>(prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D, int DT>
int launch_decode(const DecParams &prm, unsigned grid, cudaStream_t stream) {
  if (prm.rows <= 1) return launch_decode_kernel<D, DT, 1>(prm, grid, stream);
  return launch_decode_kernel<D, DT, 2>(prm, grid, stream);
}

// Keys a CTA of the decode kernel should get at least, so that its fixed
// work (set-up, the first copies' latency, the merge) stays small.
constexpr int64_t kDecMinKeysPerCta = 256;

// Grid of the decode kernel.  One slot per row: one CTA per K/V head (at
// most one per SM; heads taken with a stride).  n_splits >= 2 slots: the
// flattened (head, key) space of U = heads * key_span keys in G equal
// ranges, each at least ceil(key_span / (n_splits - 1)) keys long (and at
// least kDecMinKeysPerCta), so that one head's key_span keys meet at most
// (n_splits - 1) + 1 ranges: no head needs more slots than it has.
unsigned decode_grid(int64_t heads, int64_t key_span, int n_splits, int sms) {
  if (n_splits <= 1) return static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(heads, sms)));
  const int64_t per_min = std::max<int64_t>((key_span + n_splits - 2) / (n_splits - 1),
                                            kDecMinKeysPerCta);
  const int64_t g = std::min<int64_t>(sms, heads * key_span / per_min);
  return static_cast<unsigned>(std::max<int64_t>(g, 1));
}

// Slots for the decode kernel: enough that every SM gets an equal share of
// the keys (decode_grid then uses one CTA per SM when there are enough).
int decode_auto_splits(int64_t kv_heads, int64_t key_span, int sms) {
  const int64_t g = std::min<int64_t>(sms, kv_heads * key_span / kDecMinKeysPerCta);
  // with at least three K/V heads per four SMs, whole heads (one slot, no
  // merge launch) measured faster than equal ranges over every SM
  if (g <= 1 || 4 * kv_heads >= 3 * static_cast<int64_t>(sms)) return 1;
  const int64_t need = (g + kv_heads - 1) / kv_heads + 2;
  return static_cast<int>(std::min<int64_t>(kMaxSplits, need));
}

// Optional inputs / outputs beyond fa_fwd's: the mask and softmax
// statistics of fa_fwd_ex, the value descale of fa_fwd_fp8.
struct FwdExtras {
  const void *mask = nullptr;
  int type = FA_MASK_NONE;         // FA_MASK_*
  long long sb = 0, sh = 0, sq = 0;   // element strides
  float *smax = nullptr, *ssum = nullptr;
  float descale_v = 1.0f;
};

constexpr int kE4M3 = 2;           // internal dtype code of fp8 e4m3 inputs

// The split-KV merge for any head dim / dtype (oscale: descale_v of fp8).
int launch_combine_any(int D, int dtype, const float *ws_o, const float2 *ws_ml, void *out,
                       float *lse, int n_splits, long long rows_total, cudaStream_t stream,
                       float oscale);

// Shared body of fa_fwd, fa_fwd_ex and fa_fwd_splitkv (n_splits == 0: plain
// forward; mx == nullptr: no mask, no statistics).
int fwd_impl(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H,
             int H_kv, int L_q, int L_k, int D, float scale, int causal, int window_left,
             int window_right, int dtype, int n_splits, void *workspace,
             size_t workspace_bytes, const FwdExtras *mx, cudaStream_t stream);

}  // namespace
}  // namespace fa

using namespace fa;

namespace fa {
namespace {
int fwd_impl(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H,
             int H_kv, int L_q, int L_k, int D, float scale, int causal, int window_left,
             int window_right, int dtype, int n_splits, void *workspace,
             size_t workspace_bytes, const FwdExtras *mx, cudaStream_t stream) {
  // ---------------------------------------------------------------- checks
  if (B < 1 || H < 1 || H_kv < 1 || L_q < 0 || L_k < 0) return FA_ERR_SHAPE;
  // a pointer may be NULL only when its tensor has no elements
  if ((L_q > 0 && (!q || !out)) || (L_k > 0 && (!k || !v))) return FA_ERR_NULL;
  if (H % H_kv != 0) return FA_ERR_SHAPE;
  if (L_q > kMaxSeq || L_k > kMaxSeq) return FA_ERR_SHAPE;
  if (static_cast<int64_t>(B) * H * ((static_cast<int64_t>(L_q) + 127) / 128) >
      (1ll << 31) - 1)
    return FA_ERR_SHAPE;                   // at most one CTA per (head, 128 query rows)
  if (!valid_fwd_d(D)) return FA_ERR_HEADDIM;
  if (dtype != FA_F16 && dtype != FA_BF16 && dtype != kE4M3) return FA_ERR_DTYPE;
  if (dtype == kE4M3 && D != 32 && D != 64 && D != 128) return FA_ERR_HEADDIM;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
    return FA_ERR_ALIGN;
  if (lse && !aligned(lse, 4)) return FA_ERR_ALIGN;
  if (!std::isfinite(scale) || scale < 0.0f) return FA_ERR_ARG;
  const bool masked = mx != nullptr && mx->type != FA_MASK_NONE;
  if (mx != nullptr) {
    if (mx->type < FA_MASK_NONE || mx->type > FA_MASK_F32) return FA_ERR_ARG;
    if (mx->sb < 0 || mx->sh < 0 || mx->sq < 0) return FA_ERR_ARG;
    if (masked && L_q > 0 && L_k > 0 && !mx->mask) return FA_ERR_NULL;
    if ((mx->smax == nullptr) != (mx->ssum == nullptr)) return FA_ERR_NULL;
    if (L_q > 0 && (!aligned(mx->smax, 4) || !aligned(mx->ssum, 4))) return FA_ERR_ALIGN;
  }
  const int64_t rows_total = static_cast<int64_t>(B) * H * L_q;
  if (n_splits != 0) {
    if (n_splits < 1 || n_splits > kMaxSplits) return FA_ERR_ARG;
    if (L_q > 0 && L_k > 0) {
      if (!workspace) return FA_ERR_NULL;
      if (!aligned(workspace, 256)) return FA_ERR_ALIGN;
      if (workspace_bytes < ws_total_bytes(rows_total, D, n_splits)) return FA_ERR_WORKSPACE;
    }
  }

  // ---------------------------------------------------------------- edges
  if (L_q == 0) return FA_OK;
  if (L_k == 0) {
    // no key is visible: O = 0, lse = -inf
    const size_t n_out = static_cast<size_t>(B) * H * L_q * D * 2;
    if (cudaMemsetAsync(out, 0, n_out, stream) != cudaSuccess) return FA_ERR_CUDA;
    const size_t n = static_cast<size_t>(B) * H * L_q;
    if (lse) {
      fill_kernel<<<148, 256, 0, stream>>>(lse, n, -INFINITY);
      if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    }
    if (mx != nullptr && mx->smax != nullptr) {
      fill_kernel<<<148, 256, 0, stream>>>(mx->smax, n, -INFINITY);
      fill_kernel<<<148, 256, 0, stream>>>(mx->ssum, n, 0.0f);
      if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    }
    return FA_OK;
  }

  // ---------------------------------------------------------------- params
  FwdParams prm;
  std::memset(&prm, 0, sizeof(prm));
  int wl = window_left < 0 ? -1 : window_left;
  int wr = window_right < 0 ? -1 : window_right;
  if (causal) wr = 0;                      // causal => wr := min(wr, 0)
  if (wl >= L_q) wl = -1;                  // no constraint left of row 0
  if (wr >= L_k) wr = -1;                  // no constraint right of L_k - 1

  // decoding shapes: the CUDA-core kernel (no mask, no softmax statistics)
  if (!masked && (mx == nullptr || mx->smax == nullptr) &&
      decode_eligible(D, dtype, static_cast<int64_t>(L_q) * (H / H_kv))) {
    DecParams dp;
    std::memset(&dp, 0, sizeof(dp));
    dp.q = static_cast<const uint8_t *>(q);
    dp.k = static_cast<const uint8_t *>(k);
    dp.v = static_cast<const uint8_t *>(v);
    dp.out = out;
    dp.lse = lse;
    dp.H = H;
    dp.H_kv = H_kv;
    dp.L_q = L_q;
    dp.L_k = L_k;
    dp.group = H / H_kv;
    dp.rows = L_q * (H / H_kv);
    dp.wl = wl;
    dp.wr = wr;
    dp.n_splits = n_splits > 0 ? n_splits : 1;
    // visible keys of the rows 0 .. L_q-1 of a head: [0, key_hi]
    dp.key_span = (wr < 0 ? L_k - 1 : std::min(L_k - 1, L_q - 1 + wr)) + 1;
    dp.heads = static_cast<long long>(B) * H_kv;
    dp.rows_total = rows_total;
    const unsigned grid = decode_grid(dp.heads, dp.key_span, dp.n_splits, sm_count());
    {
      const float sl2 = scale * 1.4426950408889634f;
      dp.scale_log2 = sl2 < 1e-30f ? 1e-30f : sl2;
    }
    dp.oscale = mx != nullptr ? mx->descale_v : 1.0f;
    if (n_splits > 1) {   // one slot: whole heads write their rows directly
      dp.ws_o = static_cast<float *>(workspace);
      dp.ws_ml = reinterpret_cast<float2 *>(static_cast<char *>(workspace) +
                                            ws_ml_offset(rows_total, D, n_splits));
    }
    int st = FA_ERR_HEADDIM;
    switch (D * 2 + dtype) {
#ifndef FA_TEST_HOOKS
      case 32: st = launch_decode<16, 0>(dp, grid, stream); break;
      case 33: st = launch_decode<16, 1>(dp, grid, stream); break;
      case 64: st = launch_decode<32, 0>(dp, grid, stream); break;
      case 65: st = launch_decode<32, 1>(dp, grid, stream); break;
      case 128: st = launch_decode<64, 0>(dp, grid, stream); break;
      case 129: st = launch_decode<64, 1>(dp, grid, stream); break;
      case 256: st = launch_decode<128, 0>(dp, grid, stream); break;
      case 257: st = launch_decode<128, 1>(dp, grid, stream); break;
      case 66: st = launch_decode<32, kE4M3>(dp, grid, stream); break;
      case 130: st = launch_decode<64, kE4M3>(dp, grid, stream); break;
      case 258: st = launch_decode<128, kE4M3>(dp, grid, stream); break;
#else
    // the watchdog test library (FA_TEST_HOOKS): fp16 head dims 64 and 128 only
      case 128: st = launch_decode<64, 0>(dp, grid, stream); break;
      case 256: st = launch_decode<128, 0>(dp, grid, stream); break;
#endif
    }
    if (st != FA_OK || n_splits <= 1) return st;
    return launch_combine_any(D, dtype, dp.ws_o, dp.ws_ml, out, lse, n_splits, rows_total,
                              stream, dp.oscale);
  }
  prm.lse = lse;
  prm.H = H;
  prm.H_kv = H_kv;
  prm.L_q = L_q;
  prm.L_k = L_k;
  prm.group = H / H_kv;
  // GQA packing for short query ranges: the group's heads share a tile, so
  // a K/V head is streamed once per group instead of once per query head.
  {
    const int g = prm.group;
    const bool pow2 = g >= 2 && g <= kBM && (g & (g - 1)) == 0;
    prm.packed = (pow2 && L_q < kBM) ? 1 : 0;
    prm.tile_q = prm.packed ? kBM / g : kBM;
    int sh = 0;
    while ((1 << sh) < prm.tile_q) ++sh;
    prm.tile_q_shift = sh;
  }
  const int64_t q_tiles = (L_q + prm.tile_q - 1) / prm.tile_q;      // per work item
  const int64_t items = static_cast<int64_t>(B) * (prm.packed ? H_kv : H);
  // Two query tiles per CTA keep the tensor pipe busy (ping-pong); when that
  // leaves SMs idle (few heads, short sequences), one tile per CTA doubles
  // the number of CTAs.
  {
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    prm.tiles = (items * q_tiles <= static_cast<int64_t>(sms)) ? 1 : 2;
  }
  prm.n_qpairs = static_cast<int>((q_tiles + prm.tiles - 1) / prm.tiles);
  if (items * prm.n_qpairs * (n_splits > 0 ? n_splits : 1) > 0x7fffffffll)
    return FA_ERR_SHAPE;                   // grid.x limit
  prm.wl = wl;
  prm.wr = wr;
  prm.reverse = (wr >= 0) ? 1 : 0;         // later query tiles see more keys
  // Balanced one-wave schedule: with one tile per CTA (a single wave) and
  // uneven key ranges (causal, windows), the kernel time is the longest
  // tile's.  Tiles with more than half the longest range's key blocks are
  // then split between the two CTAs of a cluster pair, which merge their
  // (m, l, O) in shared memory; the other tiles run alone, two to a
  // cluster.  Only when every CTA still fits in one wave.
  if (prm.tiles == 1 && n_splits <= 0 && !prm.packed && dtype != kE4M3) {
    const int n_t = static_cast<int>(q_tiles);
    int nb[kBalMaxEntries * 2];
    int nb_max = 0;
    if (n_t <= kBalMaxEntries * 2) {
      for (int tq = 0; tq < n_t; ++tq) {
        const int first = tq * kBM, last = std::min(L_q, first + kBM) - 1;
        const int klo = wl < 0 ? 0 : std::max(0, first - wl);
        const int khi = wr < 0 ? L_k - 1 : std::min(L_k - 1, last + wr);
        nb[tq] = khi < klo ? 0 : khi / kBN - klo / kBN + 1;
        nb_max = std::max(nb_max, nb[tq]);
      }
    }
    // (at most 1024 blocks: the pair's hand-off waits are bounded by the
    // device wait limit, far above the time such a slice takes)
    if (nb_max >= 4 && nb_max <= 1024) {
      int heavy[kBalMaxEntries * 2], light[kBalMaxEntries * 2];
      int n_heavy = 0, n_light = 0;
      for (int tq = 0; tq < n_t; ++tq) {
        if (2 * nb[tq] > nb_max + 1)
          heavy[n_heavy++] = tq;
        else
          light[n_light++] = tq;
      }
      const int cpi = n_heavy + (n_light + 1) / 2;
      // only uneven ranges: with every tile as long as the longest, the
      // pair's hand-off costs about what the halved range saves
      if (n_heavy > 0 && n_light > 0 && cpi <= kBalMaxEntries &&
          2 * items * cpi <= sm_count()) {
        int e = 0;
        for (int h = n_heavy - 1; h >= 0; --h)     // heaviest first
          prm.bal_desc[e++] = static_cast<uint32_t>(heavy[h]) | (0xffu << 8) | (1u << 16);
        for (int i2 = 0; i2 < n_light; i2 += 2)
          prm.bal_desc[e++] = static_cast<uint32_t>(light[i2]) |
                              (static_cast<uint32_t>(i2 + 1 < n_light ? light[i2 + 1] : 0xff) << 8);
        prm.bal = 1;
        prm.bal_cpi = cpi;
      }
    }
  }
  {
    float sl2 = scale * 1.4426950408889634f;
    prm.scale_log2 = sl2 < 1e-30f ? 1e-30f : sl2;
  }
  if (mx != nullptr) {
    prm.smax = mx->smax;
    prm.ssum = mx->ssum;
    if (masked) {
      const long long esz = mx->type == FA_MASK_BOOL ? 1 : (mx->type == FA_MASK_F16 ? 2 : 4);
      prm.mask = mx->mask;
      prm.mask_type = mx->type;
      prm.mask_sb = mx->sb;
      prm.mask_sh = mx->sh;
      prm.mask_sq = mx->sq;
      prm.mask_vec = aligned(mx->mask, 16) && (mx->sb * esz) % 16 == 0 &&
                     (mx->sh * esz) % 16 == 0 && (mx->sq * esz) % 16 == 0;
    }
  }
  prm.out_ptr = out;
  prm.descale_v = mx != nullptr ? mx->descale_v : 1.0f;
  prm.n_splits = n_splits > 0 ? n_splits : 1;
  prm.rows_total = rows_total;
  if (n_splits > 0) {
    prm.ws_o = static_cast<float *>(workspace);
    prm.ws_ml = reinterpret_cast<float2 *>(static_cast<char *>(workspace) +
                                           ws_ml_offset(rows_total, D, n_splits));
  }
  const int esz = dtype == kE4M3 ? 1 : 2;
  const int box_cols = sw_span(D, esz) / esz;
  const int q_box_heads = prm.packed ? prm.group : 1;
  if (!encode_map(&prm.tm_q, q, dtype, B * H, L_q, D, box_cols, prm.tile_q, q_box_heads) ||
      !encode_map(&prm.tm_k, k, dtype, B * H_kv, L_k, D, box_cols) ||
      !encode_map(&prm.tm_v, v, dtype, B * H_kv, L_k, D, box_cols) ||
      !encode_map(&prm.tm_o, out, dtype == kE4M3 ? FA_BF16 : dtype, B * H, L_q, D,
                  sw_span(D, 2) / 2, prm.tile_q, q_box_heads))
    return FA_ERR_CUDA;

  int st = FA_ERR_HEADDIM;
  switch (D * 2 + dtype + (masked ? 1000 : 0)) {
#ifndef FA_TEST_HOOKS
    case 32: st = launch<16, 0, false>(prm, B, H, stream); break;
    case 33: st = launch<16, 1, false>(prm, B, H, stream); break;
    case 64: st = launch<32, 0, false>(prm, B, H, stream); break;
    case 65: st = launch<32, 1, false>(prm, B, H, stream); break;
    case 128: st = launch<64, 0, false>(prm, B, H, stream); break;
    case 129: st = launch<64, 1, false>(prm, B, H, stream); break;
    case 256: st = launch<128, 0, false>(prm, B, H, stream); break;
    case 257: st = launch<128, 1, false>(prm, B, H, stream); break;
    case 96: st = launch<48, 0, false>(prm, B, H, stream); break;
    case 97: st = launch<48, 1, false>(prm, B, H, stream); break;
    case 160: st = launch<80, 0, false>(prm, B, H, stream); break;
    case 161: st = launch<80, 1, false>(prm, B, H, stream); break;
    case 192: st = launch<96, 0, false>(prm, B, H, stream); break;
    case 193: st = launch<96, 1, false>(prm, B, H, stream); break;
    case 224: st = launch<112, 0, false>(prm, B, H, stream); break;
    case 225: st = launch<112, 1, false>(prm, B, H, stream); break;
    case 1032: st = launch<16, 0, true>(prm, B, H, stream); break;
    case 1033: st = launch<16, 1, true>(prm, B, H, stream); break;
    case 1064: st = launch<32, 0, true>(prm, B, H, stream); break;
    case 1065: st = launch<32, 1, true>(prm, B, H, stream); break;
    case 1128: st = launch<64, 0, true>(prm, B, H, stream); break;
    case 1129: st = launch<64, 1, true>(prm, B, H, stream); break;
    case 1256: st = launch<128, 0, true>(prm, B, H, stream); break;
    case 1257: st = launch<128, 1, true>(prm, B, H, stream); break;
    case 1096: st = launch<48, 0, true>(prm, B, H, stream); break;
    case 1097: st = launch<48, 1, true>(prm, B, H, stream); break;
    case 1160: st = launch<80, 0, true>(prm, B, H, stream); break;
    case 1161: st = launch<80, 1, true>(prm, B, H, stream); break;
    case 1192: st = launch<96, 0, true>(prm, B, H, stream); break;
    case 1193: st = launch<96, 1, true>(prm, B, H, stream); break;
    case 1224: st = launch<112, 0, true>(prm, B, H, stream); break;
    case 1225: st = launch<112, 1, true>(prm, B, H, stream); break;
    case 66: st = launch<32, kE4M3, false>(prm, B, H, stream); break;
    case 130: st = launch<64, kE4M3, false>(prm, B, H, stream); break;
    case 258: st = launch<128, kE4M3, false>(prm, B, H, stream); break;
    case 1066: st = launch<32, kE4M3, true>(prm, B, H, stream); break;
    case 1130: st = launch<64, kE4M3, true>(prm, B, H, stream); break;
    case 1258: st = launch<128, kE4M3, true>(prm, B, H, stream); break;
#else
    // the watchdog test library (FA_TEST_HOOKS): fp16 head dims 64 and 128 only
    case 128: st = launch<64, 0, false>(prm, B, H, stream); break;
    case 256: st = launch<128, 0, false>(prm, B, H, stream); break;
#endif
  }
  if (st != FA_OK || n_splits == 0) return st;
  return launch_combine_any(D, dtype, prm.ws_o, prm.ws_ml, out, lse, n_splits, rows_total,
                            stream, prm.descale_v);
}

int launch_combine_any(int D, int dtype, const float *ws_o, const float2 *ws_ml, void *out,
                       float *lse, int n_splits, long long rows_total, cudaStream_t stream,
                       float oscale) {
  switch (D * 2 + dtype) {
#ifndef FA_TEST_HOOKS
    case 32: return launch_combine<16, 0>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 33: return launch_combine<16, 1>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 64: return launch_combine<32, 0>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 65: return launch_combine<32, 1>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 128: return launch_combine<64, 0>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 129: return launch_combine<64, 1>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 256: return launch_combine<128, 0>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 257: return launch_combine<128, 1>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 96: return launch_combine<48, 0>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 97: return launch_combine<48, 1>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 160: return launch_combine<80, 0>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 161: return launch_combine<80, 1>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 192: return launch_combine<96, 0>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 193: return launch_combine<96, 1>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 224: return launch_combine<112, 0>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 225: return launch_combine<112, 1>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 66: return launch_combine<32, kE4M3>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream, oscale);
    case 130: return launch_combine<64, kE4M3>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream, oscale);
    case 258: return launch_combine<128, kE4M3>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream, oscale);
#else
    // the watchdog test library (FA_TEST_HOOKS): fp16 head dims 64 and 128 only
    case 128: return launch_combine<64, 0>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
    case 256: return launch_combine<128, 0>(ws_o, ws_ml, out, lse, n_splits, rows_total, stream);
#endif
  }
  return FA_ERR_HEADDIM;
}
}  // namespace
}  // namespace fa

extern "C" int fa_fwd(const void *q, const void *k, const void *v, void *out, float *lse,
                      int B, int H, int H_kv, int L_q, int L_k, int D, float scale,
                      int causal, int window_left, int window_right, int dtype,
                      cudaStream_t stream) {
  if (dtype != FA_F16 && dtype != FA_BF16) return FA_ERR_DTYPE;
  return fwd_impl(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, scale, causal, window_left,
                  window_right, dtype, 0, nullptr, 0, nullptr, stream);
}

extern "C" int fa_fwd_ex(const void *q, const void *k, const void *v, void *out, float *lse,
                         float *softmax_max, float *softmax_sum, const void *mask,
                         int mask_type, long long mask_stride_b, long long mask_stride_h,
                         long long mask_stride_q, int B, int H, int H_kv, int L_q, int L_k,
                         int D, float scale, int causal, int window_left, int window_right,
                         int dtype, cudaStream_t stream) {
  if (dtype != FA_F16 && dtype != FA_BF16) return FA_ERR_DTYPE;
  fa::FwdExtras mx;
  mx.mask = mask;
  mx.type = mask_type;
  mx.sb = mask_stride_b;
  mx.sh = mask_stride_h;
  mx.sq = mask_stride_q;
  mx.smax = softmax_max;
  mx.ssum = softmax_sum;
  return fwd_impl(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, scale, causal, window_left,
                  window_right, dtype, 0, nullptr, 0, &mx, stream);
}

namespace fa {
namespace {
// fp8 entries: descales checked and folded (q, k into the scores' scale; v
// into the extras); `ex` carries fa_fwd_fp8_ex's mask and statistics.
int fp8_impl(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H,
             int H_kv, int L_q, int L_k, int D, float scale, float descale_q, float descale_k,
             float descale_v, int causal, int window_left, int window_right, int n_splits,
             void *workspace, size_t workspace_bytes, FwdExtras ex, cudaStream_t stream) {
  for (float d : {descale_q, descale_k, descale_v})
    if (!std::isfinite(d) || d < 0.0f) return FA_ERR_ARG;
  if (!std::isfinite(scale) || scale < 0.0f) return FA_ERR_ARG;
  const float s = scale * descale_q * descale_k;   // the scores' full scale
  if (!std::isfinite(s)) return FA_ERR_ARG;
  ex.descale_v = descale_v;
  return fwd_impl(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, s, causal, window_left,
                  window_right, kE4M3, n_splits, workspace, workspace_bytes, &ex, stream);
}
}  // namespace
}  // namespace fa

extern "C" int fa_fwd_fp8(const void *q, const void *k, const void *v, void *out, float *lse,
                          int B, int H, int H_kv, int L_q, int L_k, int D, float scale,
                          float descale_q, float descale_k, float descale_v, int causal,
                          int window_left, int window_right, cudaStream_t stream) {
  return fa::fp8_impl(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, scale, descale_q, descale_k,
                      descale_v, causal, window_left, window_right, 0, nullptr, 0,
                      fa::FwdExtras{}, stream);
}

extern "C" int fa_fwd_fp8_ex(const void *q, const void *k, const void *v, void *out,
                             float *lse, float *softmax_max, float *softmax_sum,
                             const void *mask, int mask_type, long long mask_stride_b,
                             long long mask_stride_h, long long mask_stride_q, int B, int H,
                             int H_kv, int L_q, int L_k, int D, float scale, float descale_q,
                             float descale_k, float descale_v, int causal, int window_left,
                             int window_right, cudaStream_t stream) {
  fa::FwdExtras mx;
  mx.mask = mask;
  mx.type = mask_type;
  mx.sb = mask_stride_b;
  mx.sh = mask_stride_h;
  mx.sq = mask_stride_q;
  mx.smax = softmax_max;
  mx.ssum = softmax_sum;
  return fa::fp8_impl(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, scale, descale_q, descale_k,
                      descale_v, causal, window_left, window_right, 0, nullptr, 0, mx, stream);
}

extern "C" int fa_fwd_fp8_splitkv(const void *q, const void *k, const void *v, void *out,
                                  float *lse, int B, int H, int H_kv, int L_q, int L_k, int D,
                                  float scale, float descale_q, float descale_k,
                                  float descale_v, int causal, int window_left,
                                  int window_right, int n_splits, void *workspace,
                                  size_t workspace_bytes, cudaStream_t stream) {
  if (n_splits < 1 || n_splits > kMaxSplits) return FA_ERR_ARG;
  return fa::fp8_impl(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, scale, descale_q, descale_k,
                      descale_v, causal, window_left, window_right, n_splits, workspace,
                      workspace_bytes, fa::FwdExtras{}, stream);
}

extern "C" int fa_splitkv_auto_splits(int B, int H, int H_kv, int L_q, int L_k, int D,
                                      int dtype) {
  if (B < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || L_q < 1 || L_k < 1) return 1;
  const int sms = fa::sm_count();
  const int64_t rows_kv = static_cast<int64_t>(L_q) * (H / H_kv);
  if (fa::decode_eligible(D, dtype == FA_F16 || dtype == FA_BF16 ? dtype : 2, rows_kv))
    return fa::decode_auto_splits(static_cast<int64_t>(B) * H_kv, L_k, sms);   // upper bound
  // tensor-core kernel: query tiles (GQA-packed when the group is a power of
  // two and L_q < 128) x slices in waves of one CTA per SM; a CTA costs about
  // 4.5 key blocks of fixed work (set-up, pipeline fill, epilogue) plus its
  // blocks (a fit to decode timings on B200)
  const int g = H / H_kv;
  const bool packed = g >= 2 && g <= 128 && (g & (g - 1)) == 0 && L_q < 128;
  const int64_t tile_q = packed ? 128 / g : 128;
  const int64_t tiles = static_cast<int64_t>(B) * (packed ? H_kv : H) * ((L_q + tile_q - 1) / tile_q);
  const int64_t blocks = std::max<int64_t>(1, (static_cast<int64_t>(L_k) + 127) / 128);
  int best = 1;
  double best_cost = 0.0;
  for (int sp = 1; sp <= fa::kMaxSplits; ++sp) {
    const int64_t per = (blocks + sp - 1) / sp;
    if (sp > 1 && per < 2) break;
    const double cost = static_cast<double>((tiles * sp + sms - 1) / sms) * (4.5 + per);
    if (sp == 1 || cost < best_cost) {
      best = sp;
      best_cost = cost;
    }
  }
  return best;
}

extern "C" size_t fa_splitkv_workspace_bytes(int B, int H, int L_q, int D, int n_splits) {
  if (B < 1 || H < 1 || L_q < 0 || n_splits < 1 || n_splits > kMaxSplits) return 0;
  if (!valid_fwd_d(D)) return 0;
  return ws_total_bytes(static_cast<int64_t>(B) * H * L_q, D, n_splits);
}

extern "C" int fa_fwd_splitkv(const void *q, const void *k, const void *v, void *out,
                              float *lse, int B, int H, int H_kv, int L_q, int L_k, int D,
                              float scale, int causal, int window_left, int window_right,
                              int dtype, int n_splits, void *workspace, size_t workspace_bytes,
                              cudaStream_t stream) {
  if (n_splits < 1 || n_splits > kMaxSplits) return FA_ERR_ARG;
  if (dtype != FA_F16 && dtype != FA_BF16) return FA_ERR_DTYPE;
  return fwd_impl(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, scale, causal, window_left,
                  window_right, dtype, n_splits, workspace, workspace_bytes, nullptr, stream);
}

// ---------------------------------------------------------------------------
// Forward on host buffers, pipelined: the K/V-head groups are cut into
// n_chunks contiguous ranges (whole GQA groups: a range of K/V heads is a
// contiguous range of query heads); chunk c's inputs are copied in on one
// stream, computed on the caller's stream and copied out on a third, into
// and out of two device slots taken from the caller's workspace, so that
// the copies of neighbouring chunks overlap the kernel.
namespace fa {
namespace {
struct HostPlan {
  int64_t groups, per;              // K/V-head groups, groups per chunk
  size_t q_b, kv_b, o_b, lse_b;     // bytes of one slot's buffers
  size_t slot_b;
};
HostPlan host_plan(int B, int H, int H_kv, int L_q, int L_k, int D, int n_chunks) {
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  HostPlan hp;
  hp.groups = static_cast<int64_t>(B) * H_kv;
  hp.per = (hp.groups + n_chunks - 1) / n_chunks;
  const int64_t g = H / H_kv;
  hp.q_b = up(static_cast<size_t>(hp.per * g) * L_q * D * 2);
  hp.kv_b = up(static_cast<size_t>(hp.per) * L_k * D * 2);
  hp.o_b = hp.q_b;
  hp.lse_b = up(static_cast<size_t>(hp.per * g) * L_q * sizeof(float));
  hp.slot_b = hp.q_b + 2 * hp.kv_b + hp.o_b + hp.lse_b;
  return hp;
}

// Per device: the copy streams and the events that order the pipeline.
struct HostPipe {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t in_ready[2], comp_done[2], out_done[2];
  bool ready = false;
};
std::mutex g_pipe_mu;
HostPipe g_pipe[64];

int host_pipe(HostPipe **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe &hp = g_pipe[dev];
  if (!hp.ready) {
    if (cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) != cudaSuccess)
      return FA_ERR_CUDA;
    for (int i = 0; i < 2; ++i)
      if (cudaEventCreateWithFlags(&hp.in_ready[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&hp.comp_done[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&hp.out_done[i], cudaEventDisableTiming) != cudaSuccess)
        return FA_ERR_CUDA;
    hp.ready = true;
  }
  *out = &hp;
  return FA_OK;
}
}  // namespace
}  // namespace fa

extern "C" size_t fa_fwd_host_workspace_bytes(int B, int H, int H_kv, int L_q, int L_k, int D,
                                              int n_chunks) {
  if (B < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || L_q < 0 || L_k < 0 ||
      L_q > fa::kMaxSeq || L_k > fa::kMaxSeq || n_chunks < 1 || !fa::valid_fwd_d(D))
    return 0;
  return 2 * fa::host_plan(B, H, H_kv, L_q, L_k, D, n_chunks).slot_b;
}

extern "C" int fa_fwd_host(const void *q, const void *k, const void *v, void *out, float *lse,
                           int B, int H, int H_kv, int L_q, int L_k, int D, float scale,
                           int causal, int window_left, int window_right, int dtype,
                           void *workspace, size_t workspace_bytes, int n_chunks,
                           cudaStream_t stream) {
  using namespace fa;
  if (B < 1 || H < 1 || H_kv < 1 || L_q < 0 || L_k < 0 || H % H_kv != 0) return FA_ERR_SHAPE;
  if (L_q > kMaxSeq || L_k > kMaxSeq) return FA_ERR_SHAPE;
  if (!valid_fwd_d(D)) return FA_ERR_HEADDIM;
  if (dtype != FA_F16 && dtype != FA_BF16) return FA_ERR_DTYPE;
  if (n_chunks < 1) return FA_ERR_ARG;
  if (!std::isfinite(scale) || scale < 0.0f) return FA_ERR_ARG;
  if (L_q == 0) return FA_OK;
  if (!q || !out || (L_k > 0 && (!k || !v)) || !workspace) return FA_ERR_NULL;
  if (!aligned(workspace, 256)) return FA_ERR_ALIGN;
  const HostPlan hp = host_plan(B, H, H_kv, L_q, L_k, D, n_chunks);
  if (workspace_bytes < 2 * hp.slot_b) return FA_ERR_WORKSPACE;
  HostPipe *pp = nullptr;
  int st = host_pipe(&pp);
  if (st != FA_OK) return st;
  const int64_t g = H / H_kv;
  const size_t qrow = static_cast<size_t>(L_q) * D * 2, kvrow = static_cast<size_t>(L_k) * D * 2;
  const size_t lrow = static_cast<size_t>(L_q) * sizeof(float);
  // the first chunk's copies wait for work the caller queued before this call
  if (cudaEventRecord(pp->comp_done[0], stream) != cudaSuccess ||
      cudaStreamWaitEvent(pp->h2d, pp->comp_done[0], 0) != cudaSuccess)
    return FA_ERR_CUDA;
  int n_used = 0;
  for (int64_t g0 = 0; g0 < hp.groups; g0 += hp.per, ++n_used) {
    const int slot = n_used & 1;
    const int64_t ng = std::min(hp.per, hp.groups - g0);   // K/V heads in this chunk
    char *base = static_cast<char *>(workspace) + slot * hp.slot_b;
    char *dq = base, *dk = dq + hp.q_b, *dv = dk + hp.kv_b, *dout = dv + hp.kv_b;
    float *dlse = reinterpret_cast<float *>(dout + hp.o_b);
    bool ok = true;
    // inputs in (after the slot's previous chunk has been copied out)
    if (n_used >= 2) ok = ok && cudaStreamWaitEvent(pp->h2d, pp->out_done[slot], 0) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(dq, static_cast<const char *>(q) + g0 * g * qrow, ng * g * qrow,
                               cudaMemcpyHostToDevice, pp->h2d) == cudaSuccess;
    if (L_k > 0) {
      ok = ok && cudaMemcpyAsync(dk, static_cast<const char *>(k) + g0 * kvrow, ng * kvrow,
                                 cudaMemcpyHostToDevice, pp->h2d) == cudaSuccess;
      ok = ok && cudaMemcpyAsync(dv, static_cast<const char *>(v) + g0 * kvrow, ng * kvrow,
                                 cudaMemcpyHostToDevice, pp->h2d) == cudaSuccess;
    }
    ok = ok && cudaEventRecord(pp->in_ready[slot], pp->h2d) == cudaSuccess;
    // compute on the caller's stream: the chunk is one batch of ng*g heads
    ok = ok && cudaStreamWaitEvent(stream, pp->in_ready[slot], 0) == cudaSuccess;
    if (!ok) return FA_ERR_CUDA;
    st = fwd_impl(dq, dk, dv, dout, lse ? dlse : nullptr, 1, static_cast<int>(ng * g),
                  static_cast<int>(ng), L_q, L_k, D, scale, causal, window_left, window_right,
                  dtype, 0, nullptr, 0, nullptr, stream);
    if (st != FA_OK) return st;
    ok = cudaEventRecord(pp->comp_done[slot], stream) == cudaSuccess;
    // results out
    ok = ok && cudaStreamWaitEvent(pp->d2h, pp->comp_done[slot], 0) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(static_cast<char *>(out) + g0 * g * qrow, dout, ng * g * qrow,
                               cudaMemcpyDeviceToHost, pp->d2h) == cudaSuccess;
    if (lse)
      ok = ok && cudaMemcpyAsync(reinterpret_cast<char *>(lse) + g0 * g * lrow, dlse,
                                 ng * g * lrow, cudaMemcpyDeviceToHost, pp->d2h) == cudaSuccess;
    ok = ok && cudaEventRecord(pp->out_done[slot], pp->d2h) == cudaSuccess;
    if (!ok) return FA_ERR_CUDA;
  }
  // the caller's stream sees the whole call: wait for the last copies out
  for (int i = 0; i < std::min(n_used, 2); ++i)
    if (cudaStreamWaitEvent(stream, pp->out_done[(n_used - 1 - i) & 1], 0) != cudaSuccess)
      return FA_ERR_CUDA;
  return FA_OK;
}

// ---------------------------------------------------------------------------
// Backward.  Workspace: dQ accumulator [B*H][L_q][D] fp32, then lse2 and
// delta [B*H][L_q_pad] fp32 (L_q_pad = L_q rounded up to 128), each part at
// a 256-byte boundary.
namespace fa {
namespace {
struct BwdWs {
  size_t dq_off, lse2_off, delta_off, total;
};
BwdWs bwd_ws(int64_t BH, int64_t L_q, int D) {
  const int64_t L_q_pad = (L_q + kBM - 1) / kBM * kBM;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  BwdWs w;
  w.dq_off = 0;
  w.lse2_off = up(static_cast<size_t>(BH) * L_q * D * sizeof(float));
  w.delta_off = w.lse2_off + up(static_cast<size_t>(BH) * L_q_pad * sizeof(float));
  w.total = w.delta_off + up(static_cast<size_t>(BH) * L_q_pad * sizeof(float));
  return w;
}

template <int D, int DT, bool kMask>
int launch_bwd(const BwdParams &prm, const void *out, const void *dout, const float *lse,
               void *dq, int B, int H, cudaStream_t stream) {
  using BG = BwdGeo<D>;
  auto kern = fa_bwd_kernel<D, DT, kMask>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  static bool configured[64] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return FA_ERR_CUDA;
    if (!configured[dev]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               BG::kSmemBytes) != cudaSuccess)
        return FA_ERR_CUDA;
      // the warpgroups' setmaxnreg budgets add up to exactly the launch
      // allocation the kernel was built with; any other count would leave
      // the drain's increase waiting for registers that never come free
      cudaFuncAttributes fa_attr{};
      if (cudaFuncGetAttributes(&fa_attr, kern) != cudaSuccess ||
          fa_attr.numRegs != static_cast<int>(BwdCfg<D>::kLaunchRegs))
        return FA_ERR_CUDA;
      configured[dev] = true;
    }
  }
  const long long rows_pad = static_cast<long long>(B) * H * prm.L_q_pad;
  fa_bwd_prep_kernel<D, DT><<<static_cast<unsigned>((rows_pad + 7) / 8), 256, 0, stream>>>(
      out, dout, lse, const_cast<float *>(prm.lse2), const_cast<float *>(prm.delta),
      prm.dq_acc, prm.L_q, prm.L_q_pad, rows_pad);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(B) * prm.H_kv * prm.n_kblocks;
  kern<<<grid, BwdCfg<D>::kThreads, BG::kSmemBytes, stream>>>(prm);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  const size_t n = static_cast<size_t>(B) * H * prm.L_q * D;
  const unsigned cblocks = static_cast<unsigned>(std::min<size_t>((n / 4 + 255) / 256, 148 * 16));
  fa_bwd_dq_kernel<DT><<<cblocks, 256, 0, stream>>>(prm.dq_acc, dq, n);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
}  // namespace
}  // namespace fa

extern "C" size_t fa_bwd_workspace_bytes(int B, int H, int L_q, int D) {
  if (B < 1 || H < 1 || L_q < 0 || L_q > fa::kMaxSeq) return 0;
  if (!fa::valid_fwd_d(D)) return 0;
  return fa::bwd_ws(static_cast<int64_t>(B) * H, L_q, D).total;
}

namespace fa {
namespace {
// Shared body of fa_bwd and fa_bwd_ex (mask == nullptr: no mask).
int bwd_impl(const void *q, const void *k, const void *v, const void *out, const void *dout,
             const float *lse, void *dq, void *dk, void *dv, int B, int H, int H_kv, int L_q,
             int L_k, int D, float scale, int causal, int window_left, int window_right,
             int dtype, const FwdExtras *mx, void *workspace, size_t workspace_bytes,
             cudaStream_t stream) {
  if (B < 1 || H < 1 || H_kv < 1 || L_q < 0 || L_k < 0) return FA_ERR_SHAPE;
  if (H % H_kv != 0) return FA_ERR_SHAPE;
  if (L_q > kMaxSeq || L_k > kMaxSeq) return FA_ERR_SHAPE;
  if (static_cast<int64_t>(B) * H_kv * ((static_cast<int64_t>(L_k) + 127) / 128) >
      (1ll << 31) - 1)
    return FA_ERR_SHAPE;
  if (!valid_fwd_d(D)) return FA_ERR_HEADDIM;
  if (dtype != FA_F16 && dtype != FA_BF16) return FA_ERR_DTYPE;
  const bool nq = L_q > 0, nk = L_k > 0;
  if ((nq && (!q || !out || !dout || !dq)) || (nk && (!k || !v || !dk || !dv)) ||
      (nq && nk && (!lse || !workspace)))
    return FA_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
      !aligned(lse, 4) || !aligned(workspace, 256))
    return FA_ERR_ALIGN;
  if (!std::isfinite(scale) || scale < 0.0f) return FA_ERR_ARG;
  const bool masked = mx != nullptr && mx->type != FA_MASK_NONE;
  if (mx != nullptr) {
    if (mx->type < FA_MASK_NONE || mx->type > FA_MASK_F32) return FA_ERR_ARG;
    if (mx->sb < 0 || mx->sh < 0 || mx->sq < 0) return FA_ERR_ARG;
    if (masked && nq && nk && !mx->mask) return FA_ERR_NULL;
  }
  const int64_t BH = static_cast<int64_t>(B) * H;
  const BwdWs ws = bwd_ws(BH, L_q, D);
  if (nq && nk && workspace_bytes < ws.total) return FA_ERR_WORKSPACE;

  // ---------------------------------------------------------------- edges
  if (!nq && !nk) return FA_OK;
  if (!nq) {   // no query: no gradient reaches K or V
    const size_t bytes = static_cast<size_t>(B) * H_kv * L_k * D * 2;
    if (cudaMemsetAsync(dk, 0, bytes, stream) != cudaSuccess ||
        cudaMemsetAsync(dv, 0, bytes, stream) != cudaSuccess)
      return FA_ERR_CUDA;
    return FA_OK;
  }
  if (!nk) {   // no key: O = 0 does not depend on Q
    if (cudaMemsetAsync(dq, 0, static_cast<size_t>(BH) * L_q * D * 2, stream) != cudaSuccess)
      return FA_ERR_CUDA;
    return FA_OK;
  }

  // ---------------------------------------------------------------- params
  BwdParams prm;
  std::memset(&prm, 0, sizeof(prm));
  int wl = window_left < 0 ? -1 : window_left;
  int wr = window_right < 0 ? -1 : window_right;
  if (causal) wr = 0;
  if (wl >= L_q) wl = -1;
  if (wr >= L_k) wr = -1;
  prm.H = H;
  prm.H_kv = H_kv;
  prm.L_q = L_q;
  prm.L_k = L_k;
  prm.L_q_pad = static_cast<int>((static_cast<int64_t>(L_q) + kBM - 1) / kBM * kBM);
  prm.group = H / H_kv;
  prm.n_kblocks = (L_k + kBN - 1) / kBN;
  prm.wl = wl;
  prm.wr = wr;
  {
    float sl2 = scale * 1.4426950408889634f;
    prm.scale_log2 = sl2 < 1e-30f ? 1e-30f : sl2;
  }
  prm.scale = scale;
  char *wsb = static_cast<char *>(workspace);
  prm.dq_acc = reinterpret_cast<float *>(wsb + ws.dq_off);
  prm.lse2 = reinterpret_cast<const float *>(wsb + ws.lse2_off);
  prm.delta = reinterpret_cast<const float *>(wsb + ws.delta_off);
  prm.dk = dk;
  prm.dv = dv;
  if (masked) {
    prm.mask = mx->mask;
    prm.mask_type = mx->type;
    prm.mask_sb = mx->sb;
    prm.mask_sh = mx->sh;
    prm.mask_sq = mx->sq;
  }
  const int box_cols = sw_span(D, 2) / 2;
  if (!encode_map(&prm.tm_q, q, dtype, B * H, L_q, D, box_cols) ||
      !encode_map(&prm.tm_k, k, dtype, B * H_kv, L_k, D, box_cols) ||
      !encode_map(&prm.tm_v, v, dtype, B * H_kv, L_k, D, box_cols) ||
      !encode_map(&prm.tm_do, dout, dtype, B * H, L_q, D, box_cols) ||
      !encode_map_f32(&prm.tm_dq, prm.dq_acc, B * H, L_q, D, D % 32 == 0 ? 32 : 16))
    return FA_ERR_CUDA;
  switch (D * 2 + dtype + (masked ? 1000 : 0)) {
#ifndef FA_TEST_HOOKS
    case 32: return launch_bwd<16, 0, false>(prm, out, dout, lse, dq, B, H, stream);
    case 33: return launch_bwd<16, 1, false>(prm, out, dout, lse, dq, B, H, stream);
    case 64: return launch_bwd<32, 0, false>(prm, out, dout, lse, dq, B, H, stream);
    case 65: return launch_bwd<32, 1, false>(prm, out, dout, lse, dq, B, H, stream);
    case 128: return launch_bwd<64, 0, false>(prm, out, dout, lse, dq, B, H, stream);
    case 129: return launch_bwd<64, 1, false>(prm, out, dout, lse, dq, B, H, stream);
    case 256: return launch_bwd<128, 0, false>(prm, out, dout, lse, dq, B, H, stream);
    case 257: return launch_bwd<128, 1, false>(prm, out, dout, lse, dq, B, H, stream);
    case 96: return launch_bwd<48, 0, false>(prm, out, dout, lse, dq, B, H, stream);
    case 97: return launch_bwd<48, 1, false>(prm, out, dout, lse, dq, B, H, stream);
    case 160: return launch_bwd<80, 0, false>(prm, out, dout, lse, dq, B, H, stream);
    case 161: return launch_bwd<80, 1, false>(prm, out, dout, lse, dq, B, H, stream);
    case 192: return launch_bwd<96, 0, false>(prm, out, dout, lse, dq, B, H, stream);
    case 193: return launch_bwd<96, 1, false>(prm, out, dout, lse, dq, B, H, stream);
    case 224: return launch_bwd<112, 0, false>(prm, out, dout, lse, dq, B, H, stream);
    case 225: return launch_bwd<112, 1, false>(prm, out, dout, lse, dq, B, H, stream);
    case 1032: return launch_bwd<16, 0, true>(prm, out, dout, lse, dq, B, H, stream);
    case 1033: return launch_bwd<16, 1, true>(prm, out, dout, lse, dq, B, H, stream);
    case 1064: return launch_bwd<32, 0, true>(prm, out, dout, lse, dq, B, H, stream);
    case 1065: return launch_bwd<32, 1, true>(prm, out, dout, lse, dq, B, H, stream);
    case 1128: return launch_bwd<64, 0, true>(prm, out, dout, lse, dq, B, H, stream);
    case 1129: return launch_bwd<64, 1, true>(prm, out, dout, lse, dq, B, H, stream);
    case 1256: return launch_bwd<128, 0, true>(prm, out, dout, lse, dq, B, H, stream);
    case 1257: return launch_bwd<128, 1, true>(prm, out, dout, lse, dq, B, H, stream);
    case 1096: return launch_bwd<48, 0, true>(prm, out, dout, lse, dq, B, H, stream);
    case 1097: return launch_bwd<48, 1, true>(prm, out, dout, lse, dq, B, H, stream);
    case 1160: return launch_bwd<80, 0, true>(prm, out, dout, lse, dq, B, H, stream);
    case 1161: return launch_bwd<80, 1, true>(prm, out, dout, lse, dq, B, H, stream);
    case 1192: return launch_bwd<96, 0, true>(prm, out, dout, lse, dq, B, H, stream);
    case 1193: return launch_bwd<96, 1, true>(prm, out, dout, lse, dq, B, H, stream);
    case 1224: return launch_bwd<112, 0, true>(prm, out, dout, lse, dq, B, H, stream);
    case 1225: return launch_bwd<112, 1, true>(prm, out, dout, lse, dq, B, H, stream);
#else
    // the watchdog test library (FA_TEST_HOOKS): fp16 head dims 64 and 128 only
    case 128: return launch_bwd<64, 0, false>(prm, out, dout, lse, dq, B, H, stream);
    case 256: return launch_bwd<128, 0, false>(prm, out, dout, lse, dq, B, H, stream);
#endif
  }
  return FA_ERR_HEADDIM;
}
}  // namespace
}  // namespace fa

extern "C" int fa_bwd(const void *q, const void *k, const void *v, const void *out,
                      const void *dout, const float *lse, void *dq, void *dk, void *dv, int B,
                      int H, int H_kv, int L_q, int L_k, int D, float scale, int causal,
                      int window_left, int window_right, int dtype, void *workspace,
                      size_t workspace_bytes, cudaStream_t stream) {
  return fa::bwd_impl(q, k, v, out, dout, lse, dq, dk, dv, B, H, H_kv, L_q, L_k, D, scale,
                      causal, window_left, window_right, dtype, nullptr, workspace,
                      workspace_bytes, stream);
}

extern "C" int fa_bwd_ex(const void *q, const void *k, const void *v, const void *out,
                         const void *dout, const float *lse, void *dq, void *dk, void *dv,
                         const void *mask, int mask_type, long long mask_stride_b,
                         long long mask_stride_h, long long mask_stride_q, int B, int H,
                         int H_kv, int L_q, int L_k, int D, float scale, int causal,
                         int window_left, int window_right, int dtype, void *workspace,
                         size_t workspace_bytes, cudaStream_t stream) {
  fa::FwdExtras mx;
  mx.mask = mask;
  mx.type = mask_type;
  mx.sb = mask_stride_b;
  mx.sh = mask_stride_h;
  mx.sq = mask_stride_q;
  return fa::bwd_impl(q, k, v, out, dout, lse, dq, dk, dv, B, H, H_kv, L_q, L_k, D, scale,
                      causal, window_left, window_right, dtype, &mx, workspace,
                      workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
// No-allocation variant of the split-KV forward.  Its partials live in this
// file-scope array (module memory: it exists once per device as soon as the
// library's module is loaded there, no call allocates it).  The pages have
// no counterpart; it serves callers that may not call cudaMalloc while they
// run attention (see fa.h).
static __device__ __align__(256) unsigned char g_fa_static_scratch[FA_STATIC_SCRATCH_BYTES];

namespace fa {
namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
// The cached address belongs to the context the module was loaded in: a
// device whose primary context is destroyed and made again (cudaDeviceReset)
// reloads the module, possibly elsewhere, so the cache is keyed on the
// context's unique id as well as the device.
struct ScratchSlot {
  unsigned long long ctx_id;
  void *addr;
};
ScratchSlot g_scratch[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// Unique id of the calling thread's current context, 0 if there is none or
// the driver does not say.
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch in the current device's context: looked
// up with cudaGetSymbolAddress on the first call there (and again after the
// context has been made anew), then cached.
int static_scratch(void **addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const unsigned long long id = current_ctx_id();
  if (id == 0 || g_scratch[dev].addr == nullptr || g_scratch[dev].ctx_id != id) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fa_static_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();   // leave no error behind for the caller's next check
      return FA_ERR_CUDA;
    }
    // the lookup made the primary context current if none was: key on it
    g_scratch[dev].ctx_id = current_ctx_id();
    g_scratch[dev].addr = p;
  }
  *addr = g_scratch[dev].addr;
  return FA_OK;
}
}  // namespace
}  // namespace fa

extern "C" int fa_fwd_splitkv_static(const void *q, const void *k, const void *v, void *out,
                                     float *lse, int B, int H, int H_kv, int L_q, int L_k,
                                     int D, float scale, int causal, int window_left,
                                     int window_right, int dtype, int n_splits,
                                     cudaStream_t stream) {
  if (n_splits < 1 || n_splits > fa::kMaxSplits) return FA_ERR_ARG;
  if (dtype != FA_F16 && dtype != FA_BF16) return FA_ERR_DTYPE;
  // the size limit first, so that an oversized problem never reaches the GPU
  // (sizes fwd_impl would reject fall through to its own error codes)
  if (B >= 1 && H >= 1 && L_q >= 0 && L_q <= fa::kMaxSeq &&
      fa::valid_fwd_d(D) &&
      fa::ws_total_bytes(static_cast<int64_t>(B) * H * L_q, D, n_splits) >
          FA_STATIC_SCRATCH_BYTES)
    return FA_ERR_SCRATCH;
  void *scratch = nullptr;
  const int st = fa::static_scratch(&scratch);
  if (st != FA_OK) return st;
  return fwd_impl(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, scale, causal, window_left,
                  window_right, dtype, n_splits, scratch, FA_STATIC_SCRATCH_BYTES, nullptr,
                  stream);
}

namespace fa {
// Watchdog self-test: the library's bounded waits (sm100.cuh) on a phase
// that completes and on one that nothing completes; see the header.
__global__ void __launch_bounds__(64, 1) wait_selftest_kernel(int *result) {
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar[0]), 1);
    mbar_init(smem_u32(&bar[1]), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int *flag = &abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (warp == 0) {
    if (elect_one()) mbar_arrive(smem_u32(&bar[0]));
    __syncwarp();
    const bool done = mbar_wait_warp(smem_u32(&bar[0]), 0, flag);
    const unsigned long long t0 = globaltimer_ns();
    const bool never = mbar_wait_warp(smem_u32(&bar[1]), 0, flag);
    const unsigned long long t1 = globaltimer_ns();
    if (lane == 0) {
      result[0] = done ? 1 : 0;
      result[1] = never ? 1 : 0;
      result[2] = *flag;
      result[3] = static_cast<int>((t1 - t0) / 1000000ull);
    }
  } else {
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < kWaitLimitNs / 2) __nanosleep(1000);
    const unsigned long long t1 = globaltimer_ns();
    const bool never = mbar_wait_warp(smem_u32(&bar[1]), 0, flag);
    const unsigned long long t2 = globaltimer_ns();
    if (lane == 0) {
      result[4] = never ? 1 : 0;
      result[5] = static_cast<int>((t2 - t1) / 1000000ull);
    }
  }
}
}  // namespace fa

extern "C" int fa_selftest_wait_timeout(int *result, cudaStream_t stream) {
  if (result == nullptr) return FA_ERR_NULL;
  fa::wait_selftest_kernel<<<1, 64, 0, stream>>>(result);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

#ifdef FA_TEST_HOOKS
// Watchdog test library only (include/fa_test_hooks.h): the key block whose
// copy the K producer of CTA 0 withholds in the forward kernel (-1: none).
extern "C" int fa_test_set_withhold(int block) {
  if (cudaMemcpyToSymbol(fa::g_fa_test_withhold_block, &block, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  return FA_OK;
}
#endif

extern "C" int fa_get_device_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return FA_ERR_CUDA;
  unsigned int st = 0;
  if (cudaMemcpyFromSymbol(&st, g_fa_status, sizeof(st)) != cudaSuccess) return FA_ERR_CUDA;
  if (st != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_fa_status, &zero, sizeof(zero)) != cudaSuccess)
      return FA_ERR_CUDA;
    return FA_ERR_TIMEOUT;
  }
  return FA_OK;
}

extern "C" const char *fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_NULL: return "FA_ERR_NULL: a required pointer is NULL";
    case FA_ERR_SHAPE: return "FA_ERR_SHAPE: bad sizes (B,H,H_kv>=1, L>=0, H%H_kv==0)";
    case FA_ERR_HEADDIM: return "FA_ERR_HEADDIM: unsupported head dim D (see fa.h)";
    case FA_ERR_DTYPE: return "FA_ERR_DTYPE: dtype must be FA_F16 or FA_BF16";
    case FA_ERR_ALIGN: return "FA_ERR_ALIGN: q/k/v/out need 16-byte, lse 4-byte alignment";
    case FA_ERR_ARG: return "FA_ERR_ARG: scale must be finite and >= 0";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: a CUDA call failed";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a device-side wait gave up";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE: workspace smaller than fa_splitkv_workspace_bytes()";
    case FA_ERR_SCRATCH: return "FA_ERR_SCRATCH: problem needs more than FA_STATIC_SCRATCH_BYTES of scratch";
  }
  return "unknown fa status";
}

extern "C" int fa_version(void) { return kVersion; }
