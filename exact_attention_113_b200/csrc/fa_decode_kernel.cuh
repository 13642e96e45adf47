// fa_decode_kernel.cuh -- exact attention for decoding shapes on the CUDA
// cores: at most R query rows per key/value head (one new token per head in
// multi-head attention, or a GQA group's few heads), a long key/value cache.
//
// There S = Q K^T is a matrix-vector product per head: one multiply-add per
// byte of K read, far below what the tensor cores are for, so the work is
// bounded by how fast the cache streams out of HBM.  The kernel therefore
// keeps every SM pulling bytes with as few instructions per key as it can:
//   - a persistent grid of at most one CTA per SM walks "segments" (a K/V
//     head and a range of its visible keys).  With a single partial slot per
//     row (fa_fwd: no workspace) a segment is a whole head and CTAs take
//     heads with a stride; with n_splits slots the (head, key) space is cut
//     into equal contiguous ranges, one per CTA (the ranges cross head
//     boundaries), so every SM gets the same number of keys and a head is
//     covered by at most n_splits CTAs, each writing its slice's partial;
//   - one producer warp streams chunks of keys of K and of V (each a
//     contiguous run of rows) into a ring of shared-memory stages with
//     untiled bulk copies, completion counted on mbarriers;
//   - eight compute warps: a lane holds one key (two or four lanes for long
//     rows) and HD of its dimensions, so the dot products and the V
//     accumulation are plain per-lane multiply-adds with no shuffles; lane
//     k reads the 16-byte units of its row starting at unit k (mod the row's
//     units), so a warp's shared-memory reads never share a bank more than
//     the 512 bytes they move require; the query slice and the output slice
//     of a lane are kept in that same rotated order;
//   - the online softmax ("Flash Attention是怎么做到又快又省显存的？":
//     running maximum, normaliser rescaled when the maximum grows; here
//     conditionally, the reference maximum moves only when a chunk exceeds
//     it by 2^8) runs per row with a warp-wide reference; the weights stay
//     fp32;
//   - at the end of a segment the lanes' partial outputs are summed (first
//     across lanes that share a rotation, then through shared memory) and
//     the warps' partials are merged as key slices of one row (the merge of
//     "FlashAttention算法原理与性能优化实战" section 1.2.2), then written
//     either as the final row (O / l, lse) or as the slice's unnormalised
//     partial (O, m, l) for the split-KV merge kernel.
// Every wait is bounded (sm100.cuh): a wait that gives up sets the abort
// flag and the device status word, and the CTA leaves after its copies in
// flight have landed.
#pragma once

#include "sm100.cuh"

namespace fa {

constexpr int kDecWarps = 8;            // compute warps
constexpr int kDecThreads = 32 * (kDecWarps + 1);
constexpr int kDecRingBytes = 192 * 1024;

struct DecParams {
  const uint8_t *q;       // [B*H,    L_q, D] elements of ES bytes
  const uint8_t *k;       // [B*H_kv, L_k, D]
  const uint8_t *v;
  void *out;              // [B*H, L_q, D] fp16 / bf16 (bf16 for fp8 inputs); single slot
  float *lse;             // [B*H, L_q] or nullptr; single slot
  float *ws_o;            // [n_splits][rows_total][D] partials, or nullptr
  float2 *ws_ml;          // [n_splits][rows_total] (m in log2 units, l)
  int H, H_kv, L_q, L_k, group;
  int rows;               // query rows per K/V head: group * L_q (<= R)
  int wl, wr;             // visible iff i - wl <= j <= i + wr; -1 = unbounded
  int n_splits;           // partial slots per row (1: whole heads, final rows)
  int key_span;           // visible keys of a head: [0, key_span)
  long long heads;        // B * H_kv
  long long rows_total;   // B * H * L_q
  float scale_log2;       // scale (* descale_q * descale_k) * log2(e)
  float oscale;           // descale_v for fp8 inputs, else 1
};

// Named barrier that also returns the OR of `pred` over the participating
// threads (the same value in every one of them).
__device__ __forceinline__ bool named_barrier_or(uint32_t id, uint32_t nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Geometry for head dim D, ES-byte elements and R query rows.
template <int D, int ES, int R>
struct DecGeo {
  static constexpr int kHD = D < 64 / R ? D : 64 / R;     // dimensions a lane holds
  static constexpr int kLPK = D / kHD;                    // lanes per key
  static constexpr int kKPW = 32 / kLPK;                  // keys per warp per chunk
  static constexpr int kChunk = kDecWarps * kKPW;         // keys per stage
  static constexpr int kEPU = 16 / ES;                    // elements per 16-byte unit
  static constexpr int kU = kHD * ES / 16;                // units a lane reads per row
  static constexpr int kRowBytes = D * ES;
  static constexpr int kTileBytes = kChunk * kRowBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;      // K and V
  static constexpr int kStages = kDecRingBytes / kStageBytes < 8 ? kDecRingBytes / kStageBytes : 8;
  // lanes that hold the same rotation of their units: one group per
  // rotation after the sum across lanes kU keys apart
  static constexpr int kRot = kU < kKPW ? kU : kKPW;
  static_assert(kHD * kLPK == D && kU >= 1 && kU * 16 == kHD * ES, "lane slices of 16-byte units");
  static_assert((kU & (kU - 1)) == 0 && (kLPK & (kLPK - 1)) == 0, "powers of two");
  static_assert(kStages >= 2, "ring depth");
};

// The segments of one CTA, in order: a segment is (head, keys [a, b), slot).
// Single slot: heads blockIdx.x + i * gridDim.x, whole.  Several slots: the
// CTA's equal share [x0, x1) of the flattened (head, key) space, cut at head
// boundaries; the slot of a segment is its CTA's index among the CTAs that
// cover its head, and the CTA that covers a head's last key also clears the
// head's unused slots.
struct DecSegment {
  long long head;
  int a, b, slot;
  bool last;              // this CTA covers the head's last visible key
};

struct DecWalk {
  long long x1;           // end of this CTA's flattened key range (several slots)
  long long next;         // next head (single slot) or next flattened key
  bool single;
  __device__ explicit DecWalk(const DecParams &p) {
    single = p.n_splits == 1;
    const long long U = p.heads * p.key_span;
    x1 = U * (blockIdx.x + 1) / gridDim.x;
    next = single ? static_cast<long long>(blockIdx.x) : U * blockIdx.x / gridDim.x;
  }
  // CTA whose range holds flattened key x: the largest c with U*c/G <= x
  __device__ static long long cta_of(long long x, long long U, long long G) {
    return ((x + 1) * G - 1) / U;
  }
  __device__ bool advance(const DecParams &p, DecSegment &s) {
    if (single) {
      if (next >= p.heads) return false;
      s.head = next;
      s.a = 0;
      s.b = p.key_span;
      s.slot = 0;
      s.last = true;
      next += gridDim.x;
      return true;
    }
    if (next >= x1) return false;
    const long long U = p.heads * p.key_span;
    s.head = next / p.key_span;
    const long long hstart = s.head * p.key_span;
    s.a = static_cast<int>(next - hstart);
    const long long end = min(x1, hstart + p.key_span);
    s.b = static_cast<int>(end - hstart);
    s.slot = static_cast<int>(blockIdx.x - cta_of(hstart, U, gridDim.x));
    s.last = end == hstart + p.key_span;
    next = end;
    return true;
  }
};

// Untiled bulk copy global -> shared (as bulk_load_1d) with an L2 policy:
// the cache is streamed once, so its lines are marked evict-first.
__device__ __forceinline__ void bulk_load_1d_hint(uint32_t dst, const void *src, uint32_t bytes,
                                                  uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

// One 16-byte unit -> its elements as floats.
template <int DT>
__device__ __forceinline__ void dec_unpack(const uint4 &w, float (&x)[16 / (DT == 2 ? 1 : 2)]) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  if constexpr (DT == 0) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&ws[u]));
      x[2 * u] = f.x;
      x[2 * u + 1] = f.y;
    }
  } else if constexpr (DT == 1) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ws[u]));
      x[2 * u] = f.x;
      x[2 * u + 1] = f.y;
    }
  } else {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t h2;
        const uint16_t pair = static_cast<uint16_t>(ws[u] >> (16 * hh));
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h2));
        x[4 * u + 2 * hh] = f.x;
        x[4 * u + 2 * hh + 1] = f.y;
      }
    }
  }
}

// Shared memory of one instance: the ring, then the warps' partial outputs
// (one per rotation group), then (m, l) per warp and row, then barriers.
template <int D, int DT, int R>
struct DecSmem {
  using G = DecGeo<D, DT == 2 ? 1 : 2, R>;
  static constexpr int kOffXo = G::kStages * G::kStageBytes;
  static constexpr int kXoFloats = kDecWarps * G::kRot * R * D;
  static constexpr int kOffXml = kOffXo + kXoFloats * 4;
  static constexpr int kOffBar = kOffXml + kDecWarps * R * 2 * 4;
  static constexpr int kBytes = kOffBar + 2 * G::kStages * 8 + 16;
  static_assert(kOffBar % 8 == 0, "barrier alignment");
  static_assert(kBytes <= 232448, "shared memory budget");
};

// DT: 0 fp16, 1 bf16, 2 fp8 e4m3 (bf16 output).  R: most query rows per
// K/V head.
template <int D, int DT, int R>
__global__ void __launch_bounds__(kDecThreads, 1) fa_decode_kernel(const __grid_constant__ DecParams p) {
  constexpr int ES = DT == 2 ? 1 : 2;
  using G = DecGeo<D, ES, R>;
  using SM = DecSmem<D, DT, R>;
  constexpr int HD = G::kHD, LPK = G::kLPK, KPW = G::kKPW, CH = G::kChunk;
  constexpr int EPU = G::kEPU, U = G::kU, NS = G::kStages, ROT = G::kRot;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t *ring = smem_raw;                                          // NS x (K, V)
  float *xo = reinterpret_cast<float *>(smem_raw + SM::kOffXo);      // [warps][ROT][R][D]
  float *xml = reinterpret_cast<float *>(smem_raw + SM::kOffXml);    // [warps][R][2]
  uint64_t *full = reinterpret_cast<uint64_t *>(smem_raw + SM::kOffBar);
  uint64_t *empty = full + NS;
  int *abort_i = reinterpret_cast<int *>(empty + NS);
  volatile int *abort_flag = abort_i;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), kDecWarps);
    }
    *abort_i = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kDecWarps) {
    // ============================================= producer
    int q = 0;           // chunks issued by this CTA so far (ring position)
    bool ok = true;
    const uint64_t pol = policy_evict_first();
    DecWalk walk(p);
    DecSegment sg;
    while (ok && walk.advance(p, sg)) {
      for (int j0 = sg.a; j0 < sg.b; j0 += CH, ++q) {
        const int s = q % NS;
        if (q >= NS) {
          ok = mbar_wait_warp(smem_u32(&empty[s]), ((q / NS) - 1) & 1, abort_flag);
          if (!ok) break;
        }
        const int n = min(CH, sg.b - j0);
        const uint32_t bytes = static_cast<uint32_t>(n) * G::kRowBytes;
        const size_t off = (static_cast<size_t>(sg.head) * p.L_k + j0) * G::kRowBytes;
        if (elect_one()) {
          const uint32_t bar = smem_u32(&full[s]);
          mbar_arrive_expect_tx(bar, 2 * bytes);
          bulk_load_1d_hint(smem_u32(ring + s * G::kStageBytes), p.k + off, bytes, bar, pol);
          bulk_load_1d_hint(smem_u32(ring + s * G::kStageBytes + G::kTileBytes), p.v + off, bytes,
                            bar, pol);
        }
        __syncwarp();
      }
    }
    if (!ok) {
      // let the copies already issued land before the CTA exits
      for (int k = max(0, q - NS); k < q; ++k)
        mbar_wait_slow(smem_u32(&full[k % NS]), (k / NS) & 1, abort_flag, false);
    }
  } else {
    // ============================================= compute warps
    const int kl = lane / LPK;             // key of this lane within the warp's keys
    const int part = lane % LPK;           // which HD-slice of the row
    const int rot = kl % U;                // this lane reads unit (u + rot) % U at step u
    const int kk = warp * KPW + kl;        // key within the chunk
    const uint32_t row_off = kk * G::kRowBytes + part * HD * ES;
    int q = 0;
    bool ok = true;
    DecWalk walk(p);
    DecSegment sg;
    while (walk.advance(p, sg)) {
      const int b = static_cast<int>(sg.head / p.H_kv);
      const int hk = static_cast<int>(sg.head - static_cast<long long>(b) * p.H_kv);

      // this lane's slice of every query row, units in rotated order
      float qv[R][U][EPU];
      int qpos[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int rr = r < p.rows ? r : 0;
        const int g = rr / p.L_q, i = rr - g * p.L_q;
        qpos[r] = r < p.rows ? i : -1;
        const long long row = (static_cast<long long>(b) * p.H + hk * p.group + g) * p.L_q + i;
        const uint8_t *qrow = p.q + row * G::kRowBytes + part * HD * ES;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const uint4 w = *reinterpret_cast<const uint4 *>(qrow + ((u + rot) % U) * 16);
          dec_unpack<DT>(w, qv[r][u]);
        }
      }
      float m_ref[R], l[R], o[R][U][EPU];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        m_ref[r] = -INFINITY;
        l[r] = 0.0f;
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int e = 0; e < EPU; ++e) o[r][u][e] = 0.0f;
      }

      for (int j0 = sg.a; j0 < sg.b && ok; j0 += CH, ++q) {
        const int s = q % NS;
        ok = mbar_wait_warp(smem_u32(&full[s]), (q / NS) & 1, abort_flag);
        if (!ok) break;
        const uint8_t *kt = ring + s * G::kStageBytes + row_off;
        const uint8_t *vt = kt + G::kTileBytes;
        const int j = j0 + kk;                 // this lane's key
        // S for this lane's key: per-lane multiply-adds over its slice
        float acc[R];
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r] = 0.0f;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const uint4 w = *reinterpret_cast<const uint4 *>(kt + ((u + rot) % U) * 16);
          float kx[EPU];
          dec_unpack<DT>(w, kx);
#pragma unroll
          for (int r = 0; r < R; ++r)
#pragma unroll
            for (int e = 0; e < EPU; ++e) acc[r] = fmaf(qv[r][u][e], kx[e], acc[r]);
        }
        float sc[R], cmax[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
#pragma unroll
          for (int off = LPK / 2; off > 0; off >>= 1)
            acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], off);
          const bool vis = j < sg.b && qpos[r] >= 0 && (p.wl < 0 || j >= qpos[r] - p.wl) &&
                           (p.wr < 0 || j <= qpos[r] + p.wr);
          sc[r] = vis ? acc[r] * p.scale_log2 : -INFINITY;
          // warp-wide maximum of the chunk; conditional rescale
          cmax[r] = sc[r];
#pragma unroll
          for (int off = 16; off >= LPK; off >>= 1)
            cmax[r] = fmaxf(cmax[r], __shfl_xor_sync(0xffffffffu, cmax[r], off));
          if (cmax[r] > m_ref[r] + kRescaleThreshold) {
            const float a = (m_ref[r] == -INFINITY) ? 1.0f : ex2(m_ref[r] - cmax[r]);
            m_ref[r] = cmax[r];
            l[r] *= a;
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
              for (int e = 0; e < EPU; ++e) o[r][u][e] *= a;
          }
        }
        // P and O += P V
        float pr[R];
        bool any = false;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          pr[r] = (sc[r] == -INFINITY) ? 0.0f : ex2(sc[r] - m_ref[r]);
          l[r] += pr[r];
          any = any || pr[r] != 0.0f;
        }
        if (any) {   // masked keys (and rows past the segment's end) add nothing
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const uint4 w = *reinterpret_cast<const uint4 *>(vt + ((u + rot) % U) * 16);
            float vx[EPU];
            dec_unpack<DT>(w, vx);
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
              for (int e = 0; e < EPU; ++e) o[r][u][e] = fmaf(pr[r], vx[e], o[r][u][e]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
      }

      // ---- the segment's row results.  l: the sum over the warp's keys (each
      // key counted by one lane of its group).  O: first summed across the
      // lanes that share a rotation (keys U apart), then each rotation group
      // writes its slice, un-rotated, for the merge below.
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (part != 0) l[r] = 0.0f;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) l[r] += __shfl_xor_sync(0xffffffffu, l[r], off);
#pragma unroll
        for (int off = 16; off >= LPK * ROT; off >>= 1)
#pragma unroll
          for (int u = 0; u < U; ++u)
#pragma unroll
            for (int e = 0; e < EPU; ++e)
              o[r][u][e] += __shfl_xor_sync(0xffffffffu, o[r][u][e], off);
      }
      if (kl < ROT) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int u = 0; u < U; ++u)
#pragma unroll
            for (int e = 0; e < EPU; ++e)
              xo[((warp * ROT + kl) * R + r) * D + part * HD + ((u + rot) % U) * EPU + e] =
                  o[r][u][e];
      }
      if (lane == 0) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          xml[(warp * R + r) * 2] = m_ref[r];
          xml[(warp * R + r) * 2 + 1] = l[r];
        }
      }
      named_barrier_sync(1, 32 * kDecWarps);
      for (int idx = threadIdx.x; idx < p.rows * D; idx += 32 * kDecWarps) {
        const int r = idx / D, d = idx - r * D;
        float m = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) m = fmaxf(m, xml[(w * R + r) * 2]);
        float lt = 0.0f, ot = 0.0f;
        if (m != -INFINITY) {
#pragma unroll
          for (int w = 0; w < kDecWarps; ++w) {
            const float mw = xml[(w * R + r) * 2];
            if (mw == -INFINITY) continue;
            const float a = ex2(mw - m);
            lt += a * xml[(w * R + r) * 2 + 1];
            float os = 0.0f;
#pragma unroll
            for (int g = 0; g < ROT; ++g) os += xo[((w * ROT + g) * R + r) * D + d];
            ot += a * os;
          }
        }
        const int g = r / p.L_q, i = r - g * p.L_q;
        const long long row = (static_cast<long long>(b) * p.H + hk * p.group + g) * p.L_q + i;
        if (p.ws_o != nullptr) {
          if (sg.slot >= p.n_splits) continue;   // never: the host sizes the grid for the slots
          const size_t prow = static_cast<size_t>(sg.slot) * p.rows_total + row;
          p.ws_o[prow * D + d] = ot;
          if (d == 0) p.ws_ml[prow] = make_float2(lt > 0.0f ? m : -INFINITY, lt);
          if (sg.last) {
            // the head's slots after this one hold nothing
            for (int sl = sg.slot + 1; sl < p.n_splits; ++sl) {
              const size_t erow = static_cast<size_t>(sl) * p.rows_total + row;
              p.ws_o[erow * D + d] = 0.0f;
              if (d == 0) p.ws_ml[erow] = make_float2(-INFINITY, 0.0f);
            }
          }
        } else {
          const float val = lt > 0.0f ? ot * (p.oscale / lt) : 0.0f;
          if constexpr (DT == 0)
            reinterpret_cast<__half *>(p.out)[row * D + d] = __float2half_rn(val);
          else
            reinterpret_cast<__nv_bfloat16 *>(p.out)[row * D + d] = __float2bfloat16_rn(val);
          if (d == 0 && p.lse != nullptr)
            p.lse[row] = lt > 0.0f ? (m + __log2f(lt)) * 0.6931471805599453f : -INFINITY;
        }
      }
      // the exchange area is reused by the next segment; the compute warps
      // leave together when any of them gave up a wait or saw the abort flag
      if (named_barrier_or(1, 32 * kDecWarps, !ok || *abort_flag)) break;
    }
  }
}

}  // namespace fa
