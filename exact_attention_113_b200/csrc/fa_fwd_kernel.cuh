// fa_fwd_kernel.cuh -- exact attention forward for sm_100a.
//
// What it computes (per (batch, head), query row i):
//   O_i = sum_j softmax_j(scale * q_i . k_j | visible) v_j,
//   lse_i = ln sum_j exp(scale * q_i . k_j) over visible j,
// with the online softmax of "Flash Attention是怎么做到又快又省显存的？"
// (running max m and normaliser d', rescaled when the max grows), in the FA2
// loop order of the Triton FA2 walkthrough (outer loop over query tiles, one
// per CTA slot; inner loop over K/V blocks; division by the normaliser moved
// to the end) and never writing the score matrix to global memory.
//
// CTA layout (384 threads = 3 warpgroups, one CTA per SM):
//   warps 0-3   softmax warpgroup for query tile 0 (rows q0 .. q0+127)
//   warps 4-7   softmax warpgroup for query tile 1 (rows q0+128 .. q0+255)
//   warp  8     MMA issuer (one elected thread) and TMEM owner
//   warp  9     TMA producer of K (one elected thread; thread 0 requests the Q
//               tiles and the first K block during setup)
//   warp  10    TMA producer of V (one elected thread)
//   warp  11    idle
// Each softmax thread owns one query row, which is one TMEM lane.
// Registers: launched at kLaunchRegs per thread; the third warpgroup gives
// back down to RegSplit::kSmall and the two softmax warpgroups grow to
// RegSplit::kBig: 2*128*kBig + 128*kSmall = 384*kLaunchRegs (64512).
//
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D),
// O1 [256+D, 256+2D).  P_t (fp16/bf16, two per 32-bit column) is read by the
// PV MMA straight from TMEM.
//
// D > 64, two query tiles (TMEM full): P_t is written over the first 64
// columns of S_t, and the two tiles ping-pong.  MMA issue order per K/V
// block j:
//   S0(j), PV1(j-1), S1(j), PV0(j)
// so that while softmax warpgroup 0 works on S0(j), the tensor pipe runs
// PV1(j-1) and S1(j), and the other way round.  S_t(j+1) is issued after
// PV_t(j), which reads P_t from the same TMEM columns; tcgen05 MMAs issued by
// one thread execute in issue order.
//
// One query tile, any D (kDual): the second softmax
// warpgroup would be idle, so the two warpgroups split every block's keys:
// warpgroup h takes keys [64h, 64h + 64) of S0 with its own running max and
// sum, its own P_h (columns [128 + 64h, 160 + 64h), S1's unused slot) and
// its own O_h (the O0 / O1 slots); the MMA issuer runs S(j) once both hold
// S(j-1), then PV_0(j-1) and PV_1(j-1) over the two key halves.  The
// epilogue merges the two (m, l, O) like two key slices.
//
// D <= 64 (room to spare): P_t has its own columns [384 + 64t, 448 + 64t).
// The softmax frees S_t as soon as it holds the row in registers and its
// maximum (barrier s_free), so S_t(j+1) is computed while block j's
// exponentials run, and both tiles' softmax warps run at the same time (two
// warps per SM sub-partition on its exp unit).  Issue order per block j:
//   S0(j), S1(j), PV0(j-1), PV1(j-1).
//
// Shared memory: Q tile 0, Q tile 1, a ring of kSlotsK K tiles and a ring of
// kSlotsV V tiles.  K_j is needed half a block before V_j, so K gets the
// deeper ring; each ring has its own producer warp so that neither waits
// behind the other's free slot.  Tiles are stored as TMA writes
// them (rows of `kSwBytes`, swizzled), which is the canonical K-major layout
// for Q and K and the canonical MN-major layout for V.
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace fa {

constexpr int kBM = 128;        // query rows per tile = TMEM lanes
constexpr int kBN = 128;        // keys per K/V block
constexpr int kThreads = 384;
constexpr uint32_t kLaunchRegs = 168;   // 65536 / 384, rounded down to 8
// Softmax / other-warpgroup register split.
struct RegSplit {
  static constexpr uint32_t kBig = 224;
  static constexpr uint32_t kSmall = (kThreads * kLaunchRegs - 2 * 128 * kBig) / 128;
  static_assert(kSmall % 8 == 0 && kSmall >= 24, "setmaxnreg takes multiples of 8");
  static_assert(2 * 128 * kBig + 128 * kSmall <= kThreads * kLaunchRegs,
                "register split must fit in the launch allocation");
};
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;     // Q and K
constexpr int kLoadWarpV = 10;   // V
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays <= 2^8
constexpr int kBalMaxEntries = 74;         // cluster pairs per item: at most 148 CTAs

#ifdef FA_TEST_HOOKS
// Watchdog test library only (never in libfa.so): the K producer of CTA 0
// skips the copy of this key block (-1: none), so that the MMA warp's
// bounded wait for it runs out and the abort path of every role runs.
__device__ int g_fa_test_withhold_block = -1;
#endif

struct FwdParams {
  CUtensorMap tm_q;   // [B*H,    L_q, D]
  CUtensorMap tm_k;   // [B*H_kv, L_k, D]
  CUtensorMap tm_v;   // [B*H_kv, L_k, D]
  CUtensorMap tm_o;   // [B*H,    L_q, D]
  float *lse;         // [B*H, L_q] or nullptr
  int H, H_kv, L_q, L_k;
  int group;          // H / H_kv
  int n_qpairs;       // query-tile groups per work item: ceil(ceil(L_q / tile_q) / tiles)
  // GQA packing (packed == 1, short query ranges): a 128-row tile holds
  // tile_q = 128 / group query rows of each of the group's heads, row
  // r = g * tile_q + i_local, so that one pass over a K/V head serves the
  // whole group.  The Q / O tensor maps then have a box of [group, tile_q,
  // cols] and a work item is one (batch, K/V head).
  int packed;
  int tile_q;         // query positions per tile: 128, or 128 / group when packed
  int tile_q_shift;   // log2(tile_q) when packed
  int tiles;          // query tiles per CTA: 2 (ping-pong) or 1 (small problems)
  int wl, wr;         // visible iff i - wl <= j <= i + wr; -1 = unbounded
  int reverse;        // process query pairs last-first (causal: heavy first)
  float scale_log2;   // scale * log2(e), clamped to >= 1e-30
  // split-KV mode (ws_o != nullptr): each CTA covers one of n_splits
  // contiguous slices of the key blocks and writes its unnormalised partial
  // O (fp32) and (m, l) per row; a combine kernel merges the slices.
  int n_splits;       // 1 outside split-KV mode
  long long rows_total;   // B * H * L_q
  float *ws_o;        // [n_splits][rows_total][D] or nullptr
  float2 *ws_ml;      // [n_splits][rows_total]: (m in log2 units, l)
  // optional attention mask (instances with kMask): element (b, h, i, j) at
  // mask + b*mask_sb + h*mask_sh + i*mask_sq + j; type 1 bool (nonzero
  // hides the key), 2 fp16 / 3 fp32 added to the scaled score
  const void *mask;
  int mask_type;
  int mask_vec;       // base and strides 16-byte aligned: 16-byte loads
  long long mask_sb, mask_sh, mask_sq;
  // fp8 inputs (DT = 2): bf16 output written straight from registers to
  // out_ptr [B*H, L_q, D], O scaled by descale_v
  void *out_ptr;
  float descale_v;
  // optional softmax statistics [B*H, L_q] (natural-log units): the row max
  // of the scaled, masked scores and sum_j e^{s_j - max}; nullptr = skip
  float *smax;
  float *ssum;
  // balanced one-wave schedule (bal != 0, one tile per CTA, launched as
  // clusters of two CTAs): cluster c serves item c / bal_cpi with entry
  // bal_desc[c % bal_cpi] = tile A (bits 0-7) | tile B (bits 8-15, 0xff:
  // none) | bit 16 when the pair splits tile A's key blocks (rank 0 the
  // first half, rank 1 the second, which rank 1 hands to rank 0 through
  // shared memory); otherwise rank 0 takes tile A and rank 1 tile B alone
  int bal;
  int bal_cpi;
  uint32_t bal_desc[kBalMaxEntries];
};

// Tile geometry for head dim D and element size ES bytes (2: fp16 / bf16,
// 1: fp8 e4m3).
template <int D, int ES = 2>
struct Geo {
  static constexpr int kRowBytes = D * ES;
  // swizzle span: the largest of 128 / 64 / 32 bytes dividing the row
  static constexpr int kSwBytes = kRowBytes % 128 == 0 ? 128 : (kRowBytes % 64 == 0 ? 64 : 32);
  static constexpr int kBoxCols = kSwBytes / ES;                      // elements per box row
  static constexpr int kNumBox = kRowBytes / kSwBytes;                 // column boxes per tile
  static constexpr int kBoxBytes = kBM * kSwBytes;
  static constexpr int kTileBytes = kBM * kRowBytes;
  static_assert(kSwBytes >= 32, "rows of at least 32 bytes (a swizzle span)");
  static_assert(kRowBytes % kSwBytes == 0, "whole swizzle atoms per row");
  // ring depth: the tuned values for D = 16..128 powers of two; otherwise as
  // many slots (up to 8) as the 224 KB shared-memory budget leaves beside Q
  static constexpr bool kPow2 = (D & (D - 1)) == 0;
  static constexpr int kFitSlots = (224 * 1024) / kTileBytes - 2 < 8
                                       ? (224 * 1024) / kTileBytes - 2 : 8;
  static constexpr int kSlotsK = kPow2 ? (kTileBytes >= 32768 ? 3 : (kTileBytes >= 16384 ? 4 : 8))
                                       : (kFitSlots + 1) / 2;
  static constexpr int kSlotsV = kPow2 ? (kTileBytes >= 32768 ? 2 : (kTileBytes >= 16384 ? 4 : 8))
                                       : kFitSlots / 2;
  static constexpr int kSlots = kSlotsK + kSlotsV;
  static constexpr uint32_t kLayout = kSwBytes == 128 ? 2u : (kSwBytes == 64 ? 4u : 6u);
  static constexpr int kUnitsPerBoxRow = kSwBytes / 16;
  // P in its own TMEM columns (decoupled from S) when there is room
  static constexpr bool kSplitP = D <= 64;
  // In unmasked blocks one column pair in kPolyPeriod takes 2^x from the FMA
  // pipe (exp2_poly2) instead of MUFU: the MUFU rate (16/clk/SM) alone needs
  // as many cycles per block as the D=128 tensor work.
  static constexpr int kPolyPeriod = 1 << 20;  // off; the kernel picks kPoly
  // shared memory map (offsets from a 1024-byte aligned base)
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = 2 * kTileBytes;
  static constexpr int kOffBar = kOffRing + kSlots * kTileBytes;
  static constexpr int kBarBytes = 512;
  // balanced split pairs: the sender's slice (128 fp32 O rows and a
  // (m, l, max, ok) quadruple per row) lands in a buffer of its own where
  // the budget leaves room (D <= 64), else in the receiver's K/V ring once
  // that is idle
  static constexpr int kPartnerBytes = kBM * (D * 4 + 16);
  static constexpr int kOffPartner = kOffBar + kBarBytes;
  static constexpr bool kPartnerOwn = kOffPartner + kPartnerBytes + 1024 <= 232448;
  static constexpr int kUsed = kOffPartner + (kPartnerOwn ? kPartnerBytes : 0);
  // at least ~116 KB so that only one CTA (and one 512-column TMEM
  // allocation) fits on an SM
  static constexpr int kSmemBytes = (kUsed + 1024 > 118 * 1024) ? kUsed + 1024 : 118 * 1024;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(256 + 2 * D <= 512, "TMEM budget");
};

// Barrier block inside shared memory.
template <int kSlots>
struct Bars {
  uint64_t q_full[2];
  uint64_t full[kSlots];
  uint64_t empty[kSlots];
  uint64_t s_full[2];     // S_t complete
  uint64_t s_free[2];     // softmax holds S_t in registers
  uint64_t p_full[2];
  uint64_t pv_done[2];
  uint64_t mma_done;
  uint64_t recv_ready;    // balanced pairs, sender: the receiver's ring is free (remote arrival)
  uint64_t partner_full;  // balanced pairs, receiver: the sender's rows have landed (bytes)
  uint64_t partner_ack;   // balanced pairs, sender: its copy has landed (remote arrival)
  uint32_t tmem_base;
  int abort_flag;
};

// Key range [lo, hi) in blocks for query rows [first, last] of one tile.
struct BlockRange {
  int lo, hi;
};

__device__ __forceinline__ BlockRange tile_block_range(int first, int last, int L_k, int wl,
                                                       int wr) {
  int klo = wl < 0 ? 0 : max(0, first - wl);
  int khi = wr < 0 ? L_k - 1 : min(L_k - 1, last + wr);
  BlockRange r;
  if (khi < klo) {
    r.lo = 0;
    r.hi = 0;
  } else {
    r.lo = klo / kBN;
    r.hi = khi / kBN + 1;
  }
  return r;
}

// Adds the mask of key block j to a row of raw scores and applies the scale:
// t_c = s_c * scale * log2(e) + mask_c * log2(e) (-inf where hidden), so
// that the rest of the softmax runs in log2 units with a unit scale.
// `base` is the row's first mask element; `n_cols` the valid keys of the
// block (the rest are already -inf); `row_ok` false: scale only.
__device__ __forceinline__ float mask_bias_f16(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}
template <int kBNc>
__device__ __forceinline__ void apply_mask(float (&sv)[kBNc], const FwdParams &p, long long base,
                                           int n_cols, bool row_ok, float sl2) {
  constexpr float kLog2e = 1.4426950408889634f;
  if (!row_ok) {
#pragma unroll
    for (int c = 0; c < kBNc; ++c) sv[c] *= sl2;
    return;
  }
  const bool vec = p.mask_vec && n_cols >= kBNc;
  if (p.mask_type == 1) {
    const uint8_t *m = static_cast<const uint8_t *>(p.mask) + base;
    if (vec) {
#pragma unroll
      for (int c0 = 0; c0 < kBNc; c0 += 16) {
        const uint4 w = __ldg(reinterpret_cast<const uint4 *>(m + c0));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int u = 0; u < 16; ++u)
          sv[c0 + u] = ((ws[u >> 2] >> (8 * (u & 3))) & 0xffu) ? -INFINITY : sv[c0 + u] * sl2;
      }
    } else {
#pragma unroll
      for (int c = 0; c < kBNc; ++c)
        sv[c] = (c < n_cols && m[c] != 0) ? -INFINITY : sv[c] * sl2;
    }
  } else if (p.mask_type == 2) {
    const uint16_t *m = static_cast<const uint16_t *>(p.mask) + base;
    if (vec) {
#pragma unroll
      for (int c0 = 0; c0 < kBNc; c0 += 8) {
        const uint4 w = __ldg(reinterpret_cast<const uint4 *>(m + c0));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int u = 0; u < 8; ++u)
          sv[c0 + u] = fmaf(sv[c0 + u], sl2,
                            mask_bias_f16(static_cast<uint16_t>(ws[u >> 1] >> (16 * (u & 1)))) *
                                kLog2e);
      }
    } else {
#pragma unroll
      for (int c = 0; c < kBNc; ++c)
        sv[c] = fmaf(sv[c], sl2, c < n_cols ? mask_bias_f16(m[c]) * kLog2e : 0.0f);
    }
  } else {
    const float *m = static_cast<const float *>(p.mask) + base;
    if (vec) {
#pragma unroll
      for (int c0 = 0; c0 < kBNc; c0 += 4) {
        const float4 w = __ldg(reinterpret_cast<const float4 *>(m + c0));
        sv[c0] = fmaf(sv[c0], sl2, w.x * kLog2e);
        sv[c0 + 1] = fmaf(sv[c0 + 1], sl2, w.y * kLog2e);
        sv[c0 + 2] = fmaf(sv[c0 + 2], sl2, w.z * kLog2e);
        sv[c0 + 3] = fmaf(sv[c0 + 3], sl2, w.w * kLog2e);
      }
    } else {
#pragma unroll
      for (int c = 0; c < kBNc; ++c)
        sv[c] = fmaf(sv[c], sl2, c < n_cols ? m[c] * kLog2e : 0.0f);
    }
  }
}

// Visit the D TMEM columns of an O row in chunks of 32 (a 16-wide tail when
// D is an odd multiple of 16): f(first column, width as an integral
// constant).
template <int D, typename F>
__device__ __forceinline__ void for_o_chunks(F &&f) {
#pragma unroll
  for (int c = 0; c < D; c += 32) {
    if (c + 32 <= D)
      f(c, std::integral_constant<int, 32>{});
    else
      f(c, std::integral_constant<int, 16>{});
  }
}

// O row *= alpha in TMEM.
template <int D>
__device__ __forceinline__ void scale_o_row(uint32_t tO, float alpha) {
  for_o_chunks<D>([&](int c, auto w) {
    constexpr int W = decltype(w)::value;
    uint32_t o[W];
    tmem_ld_cols<W>(tO + c, o);
    tmem_wait_ld();
    reg_dep(o);
#pragma unroll
    for (int u = 0; u < W; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * alpha);
    tmem_st_cols<W>(tO + c, o);
  });
}

// P of one half-row (64 keys) into 32-bit TMEM words: two 16-bit values a
// word, or four E4M3 codes a word (fp8 inputs); pair index p = key / 2.
template <int DT>
__device__ __forceinline__ void put_p(uint32_t (&pk)[32], int p, float a, float b) {
  if constexpr (DT == 2) {
    const uint32_t h = pack_e4m3x2(a, b);
    pk[p >> 1] = (p & 1) ? (pk[p >> 1] | (h << 16)) : h;
  } else {
    pk[p] = pack2<DT>(a, b);
  }
}
// Store a half-row of P at TMEM columns base + half * (32 or 16).
template <int DT>
__device__ __forceinline__ void store_p_half(uint32_t base, int half, const uint32_t (&pk)[32]) {
  if constexpr (DT == 2)
    tmem_st_x16(base + 16u * half, *reinterpret_cast<const uint32_t(*)[16]>(pk));
  else
    tmem_st_x32(base + 32u * half, pk);
}

template <int D, int DT, bool kMask, bool kDual = false>
__global__ void __launch_bounds__(kThreads, 1) fa_fwd_kernel(const __grid_constant__ FwdParams p) {
  // DT: 0 fp16, 1 bf16, 2 fp8 e4m3 inputs (bf16 output).  kDual: one query
  // tile, its keys split between the two softmax warpgroups (D <= 64).
  constexpr bool kF8 = DT == 2;
  constexpr int kES = kF8 ? 1 : 2;
  constexpr int kKStep = 32 / kES;             // K of one MMA instruction (32 bytes)
  using G = Geo<D, kES>;
  // One column pair in kPoly takes 2^x from the FMA pipe (unmasked blocks).
  // Measured: +4 % for fp8 at D = 128, where the tensor work per block halves
  // and MUFU becomes the limit; 10-25 % slower at D <= 64, whose softmax
  // threads are bound by their own instruction stream; neutral otherwise.
  constexpr int kPoly = (kF8 && D == 128) ? 8 : G::kPolyPeriod;
  constexpr int kSlots = G::kSlots;
  static_assert(sizeof(Bars<kSlots>) <= G::kBarBytes, "barrier block");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Bars<kSlots> *bars = reinterpret_cast<Bars<kSlots> *>(smem + G::kOffBar);
  volatile int *abort_flag = &bars->abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // ---- work item: (batch*head, pair of query tiles, key slice);
  // consecutive CTAs take consecutive query pairs of one head, so a head's
  // K/V stays hot in L2.
  int item, split, qpair;
  int bal_role = 0;   // balanced split pair: 1 receives the partner's slice, 2 sends its own
  if (kDual && p.bal) {   // (the host sets bal only with one tile per CTA)
    const int c = static_cast<int>(blockIdx.x) >> 1;
    item = c / p.bal_cpi;
    const uint32_t e = p.bal_desc[c - item * p.bal_cpi];
    const uint32_t rank = cluster_rank();
    const bool pair_split = (e >> 16) & 1u;
    int tile = static_cast<int>(pair_split || rank == 0 ? (e & 0xffu) : ((e >> 8) & 0xffu));
    if (tile == 0xff) tile = p.n_qpairs;   // no tile: rows past L_q, nothing to do
    qpair = tile;
    split = 0;
    if (pair_split) bal_role = rank == 0 ? 1 : 2;
  } else {
    const int per_item = p.n_qpairs * p.n_splits;
    item = static_cast<int>(blockIdx.x) / per_item;
    const int rem = static_cast<int>(blockIdx.x) - item * per_item;
    const int qp_idx = rem / p.n_splits;
    split = rem - qp_idx * p.n_splits;
    qpair = p.reverse ? (p.n_qpairs - 1 - qp_idx) : qp_idx;
  }
  // bh: (first) query head of the tile in [B*H]; bh_kv: its K/V head
  int bh, bh_kv;
  if (p.packed) {
    const int b = item / p.H_kv;
    const int hk = item - b * p.H_kv;
    bh = b * p.H + hk * p.group;
    bh_kv = item;
  } else {
    const int b = item / p.H;
    const int h = item - b * p.H;
    bh = item;
    bh_kv = b * p.H_kv + h / p.group;   // GQA: contiguous head groups
  }

  int q0[2], rows[2];   // first query position and query positions per head
  BlockRange rng[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    q0[t] = (qpair * p.tiles + t) * p.tile_q;
    rows[t] = t < p.tiles ? max(0, min(p.tile_q, p.L_q - q0[t])) : 0;
    if (rows[t] > 0) {
      rng[t] = tile_block_range(q0[t], q0[t] + rows[t] - 1, p.L_k, p.wl, p.wr);
    } else {
      rng[t].lo = 0;
      rng[t].hi = 0;
    }
  }
  if (p.n_splits > 1) {
    // this CTA's slice of the union of the tiles' key-block ranges
    const bool a0 = rng[0].hi > rng[0].lo, a1 = rng[1].hi > rng[1].lo;
    const int ulo = a0 ? (a1 ? min(rng[0].lo, rng[1].lo) : rng[0].lo) : rng[1].lo;
    const int uhi = a0 ? (a1 ? max(rng[0].hi, rng[1].hi) : rng[0].hi) : rng[1].hi;
    const int cs = (uhi - ulo + p.n_splits - 1) / p.n_splits;
    const int clo = ulo + split * cs, chi = min(uhi, clo + cs);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      rng[t].lo = max(rng[t].lo, clo);
      rng[t].hi = min(rng[t].hi, chi);
      if (rng[t].hi <= rng[t].lo) rng[t].lo = rng[t].hi = 0;
    }
  }
  if (bal_role != 0) {
    // the pair's shares of the tile's key blocks (the host splits only tiles
    // with at least three): halves, or, when the sender's rows have a buffer
    // of their own and their hand-off overlaps the receiver's last blocks,
    // one more block for the receiver
    const int nb = rng[0].hi - rng[0].lo;
    const int mid = rng[0].lo + (G::kPartnerOwn ? (nb + 2) / 2 : (nb + 1) / 2);
    if (bal_role == 1)
      rng[0].hi = mid;
    else
      rng[0].lo = mid;
  }
  const bool act0 = rng[0].hi > rng[0].lo, act1 = rng[1].hi > rng[1].lo;
  const int lo = act0 ? (act1 ? min(rng[0].lo, rng[1].lo) : rng[0].lo) : rng[1].lo;
  const int hi = act0 ? (act1 ? max(rng[0].hi, rng[1].hi) : rng[0].hi) : rng[1].hi;
  const bool any_work = act0 || act1;

  // ---- setup
  if (tid == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(&bars->q_full[t]), 1);
      mbar_init(smem_u32(&bars->s_full[t]), 1);
      mbar_init(smem_u32(&bars->s_free[t]), (kDual && t == 0) ? 2 * kBM : kBM);
      mbar_init(smem_u32(&bars->p_full[t]), kBM);
      mbar_init(smem_u32(&bars->pv_done[t]), 1);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 1);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->mma_done), 1);
    mbar_init(smem_u32(&bars->recv_ready), 1);
    mbar_init(smem_u32(&bars->partner_full), 1);
    mbar_init(smem_u32(&bars->partner_ack), 1);
    bars->abort_flag = 0;
    fence_mbar_init();
    // a receiver with its own buffer expects the sender's bytes from the start
    if (kDual && G::kPartnerOwn && bal_role == 1)
      mbar_arrive_expect_tx(smem_u32(&bars->partner_full), G::kPartnerBytes);
    // The Q tiles and the first K block are requested right here, so that
    // their latency overlaps the TMEM allocation and the block-wide barrier
    // (the K producer starts at the second block).
    if (any_work) {
      const uint32_t sQ0 = smem_u32(smem + G::kOffQ);
      const uint64_t pol_stream = policy_evict_first();
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (rng[t].hi <= rng[t].lo) continue;
        const uint32_t bar = smem_u32(&bars->q_full[t]);
        mbar_arrive_expect_tx(bar, G::kTileBytes);
#pragma unroll
        for (int bx = 0; bx < G::kNumBox; ++bx)
          tma_load_3d(sQ0 + t * G::kTileBytes + bx * G::kBoxBytes, &p.tm_q, bar,
                      bx * G::kBoxCols, q0[t], bh, pol_stream);
      }
#ifdef FA_TEST_HOOKS
      const bool withhold_first = blockIdx.x == 0 && g_fa_test_withhold_block == lo;
#else
      constexpr bool withhold_first = false;
#endif
      if (!withhold_first) {
        const uint32_t bar = smem_u32(&bars->full[0]);
        mbar_arrive_expect_tx(bar, G::kTileBytes);
#pragma unroll
        for (int bx = 0; bx < G::kNumBox; ++bx)
          tma_load_3d(smem_u32(smem + G::kOffRing) + bx * G::kBoxBytes, &p.tm_k, bar,
                      bx * G::kBoxCols, lo * kBN, bh_kv, policy_evict_last());
      }
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    prefetch_tensormap(&p.tm_v);
    prefetch_tensormap(&p.tm_o);
  }
  tc_fence_before_sync();
  if (kDual && p.bal)
    cluster_sync_all();   // both CTAs' barriers are initialised before any remote use
  else
    __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  const uint32_t sQ = smem_u32(smem + G::kOffQ);
  const uint32_t sRing = smem_u32(smem + G::kOffRing);

  if (warp >= 8) {
  // ===================================================== warpgroup 2
  regs_dec<RegSplit::kSmall>();
  if (warp == kLoadWarp || warp == kLoadWarpV) {
    // =================================================== TMA producers
    // Warp 9 loads the K ring (from its second block), warp 10 the V ring.
    // The whole warp walks the schedule (its operands stay warp-uniform);
    // one elected lane issues each copy.
    if (any_work) {
      const bool is_k = warp == kLoadWarp;
      const uint64_t pol_keep = policy_evict_last();
      const int nslot = is_k ? G::kSlotsK : G::kSlotsV;
      const int base = is_k ? 0 : G::kSlotsK;           // first slot of this ring
      const CUtensorMap *map = is_k ? &p.tm_k : &p.tm_v;
      int q = 0;
      bool ok = true;
#ifdef FA_TEST_HOOKS
      const int withheld = (is_k && blockIdx.x == 0) ? g_fa_test_withhold_block : -1;
#else
      constexpr int withheld = -1;
#endif
      for (int j = lo; j < hi; ++j, ++q) {
        if (is_k && q == 0) continue;   // the first K block: requested at setup
        const int slot = base + q % nslot;
        if (q >= nslot) {
          ok = mbar_wait_warp(smem_u32(&bars->empty[slot]), ((q / nslot) - 1) & 1, abort_flag);
          if (!ok) break;
        }
        const uint32_t bar = smem_u32(&bars->full[slot]);
        if (j == withheld) continue;   // test library only: this fill never arrives
        if (elect_one()) {
          mbar_arrive_expect_tx(bar, G::kTileBytes);
#pragma unroll
          for (int bx = 0; bx < G::kNumBox; ++bx)
            tma_load_3d(sRing + slot * G::kTileBytes + bx * G::kBoxBytes, map, bar,
                        bx * G::kBoxCols, j * kBN, bh_kv, pol_keep);
        }
        __syncwarp();
      }
      if (!ok) {
        // drain: let the copies already issued land before the CTA exits
        // (Q tiles first: nothing else may have waited for them)
        if (is_k) {
          for (int t = 0; t < 2; ++t)
            if (rng[t].hi > rng[t].lo)
              mbar_wait_slow(smem_u32(&bars->q_full[t]), 0, abort_flag, false);
        }
        for (int k = max(0, q - nslot); k < q; ++k)
          if (lo + k != withheld)
            mbar_wait_slow(smem_u32(&bars->full[base + k % nslot]), (k / nslot) & 1,
                           abort_flag, false);
      }
    }
  } else if (warp == kMmaWarp) {
    // =================================================== MMA issuer
    // The whole warp runs the loop; one elected lane (always the same one,
    // so that its commits track its own MMAs) issues the tcgen05 ops.
    constexpr uint32_t kIdescS =
        kF8 ? make_idesc_e4m3(kBM, kBN, 0, 0) : make_idesc_f16(kBM, kBN, DT, 0, 0);
    constexpr uint32_t kIdescPV =
        kF8 ? make_idesc_e4m3(kBM, D, 0, 1) : make_idesc_f16(kBM, D, DT, 0, 1);
    constexpr uint32_t kHi = desc_hi(8 * G::kSwBytes, G::kLayout);   // K- and MN-major
    if (any_work) {
      bool ok = true;
      if (act0) ok = mbar_wait_warp(smem_u32(&bars->q_full[0]), 0, abort_flag);
      if (act1 && ok) ok = mbar_wait_warp(smem_u32(&bars->q_full[1]), 0, abort_flag);
      int npv0 = 0, npv1 = 0;
      const uint32_t q_lo0 = desc_lo(sQ, 16), q_lo1 = desc_lo(sQ + G::kTileBytes, 16);

      auto issue_s = [&](int t, int slot) {
        const uint32_t qlo = t ? q_lo1 : q_lo0;
        const uint32_t klo = desc_lo(sRing + slot * G::kTileBytes, 16);
        const uint32_t d_tmem = tmem + (t ? 128u : 0u);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / kKStep; ++kk) {
            const int byte = kk * 32;
            const uint32_t off = ((byte / G::kSwBytes) * G::kBoxBytes + (byte % G::kSwBytes)) >> 4;
            mma_ss_t<kF8>(d_tmem, desc_join(qlo + off, kHi), desc_join(klo + off, kHi), kIdescS,
                          kk > 0 ? 1u : 0u);
          }
          tc_commit(smem_u32(&bars->s_full[t]));
        }
        __syncwarp();
      };
      auto issue_pv = [&](int t, int slot) {
        const uint32_t vlo = desc_lo(sRing + slot * G::kTileBytes, G::kBoxBytes);
        // P_t: own columns (D <= 64) or S_t columns [0, 64) (ping-pong)
        const uint32_t a_tmem = tmem + (G::kSplitP ? 384u + (t ? 64u : 0u) : (t ? 128u : 0u));
        const uint32_t d_tmem = tmem + 256u + (t ? D : 0u);
        const bool first = (t ? npv1 : npv0) == 0;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kBN / kKStep; ++kk)
            mma_ts_t<kF8>(d_tmem, a_tmem + kk * 8,
                          desc_join(vlo + ((kk * kKStep * G::kSwBytes) >> 4), kHi), kIdescPV,
                          (!first || kk > 0) ? 1u : 0u);
          tc_commit(smem_u32(&bars->pv_done[t]));
        }
        __syncwarp();
        if (t) ++npv1; else ++npv0;
      };
      auto commit = [&](uint32_t bar) {
        if (elect_one()) tc_commit(bar);
        __syncwarp();
      };
      auto in = [&](int t, int j) { return j >= rng[t].lo && j < rng[t].hi; };
      // ring slots of K_j / V_j (q = j - lo) and the parity of their fill
      auto kslot = [&](int q) { return q % G::kSlotsK; };
      auto vslot = [&](int q) { return G::kSlotsK + q % G::kSlotsV; };
      auto kpar = [&](int q) { return static_cast<uint32_t>((q / G::kSlotsK) & 1); };
      auto vpar = [&](int q) { return static_cast<uint32_t>((q / G::kSlotsV) & 1); };

      if constexpr (kDual) {
        // One query tile, two softmax warpgroups: S(j) once both hold
        // S(j-1) in registers (s_free, 256 arrivals); then, once P_h(j-1)
        // of half h (keys [64h, 64h + 64)) is in TMEM, O_h += P_h V_h into
        // that half's own accumulator.
        int ns = 0;
        auto issue_pv_h = [&](int h, int slot) {
          const uint32_t vlo = desc_lo(sRing + slot * G::kTileBytes, G::kBoxBytes);
          const uint32_t a_tmem = tmem + 128u + (h ? 64u : 0u);   // P_h: S1's free slot
          const uint32_t d_tmem = tmem + 256u + (h ? D : 0u);
          const bool first = (h ? npv1 : npv0) == 0;
          constexpr int kHalfSteps = kBN / kKStep / 2;
          if (elect_one()) {
#pragma unroll
            for (int u = 0; u < kHalfSteps; ++u) {
              const int kk = h * kHalfSteps + u;
              mma_ts_t<kF8>(d_tmem, a_tmem + u * 8,
                            desc_join(vlo + ((kk * kKStep * G::kSwBytes) >> 4), kHi), kIdescPV,
                            (!first || u > 0) ? 1u : 0u);
            }
            tc_commit(smem_u32(&bars->pv_done[h]));
          }
          __syncwarp();
          if (h) ++npv1; else ++npv0;
        };
        for (int j = lo; j <= hi && ok; ++j) {
          const int q = j - lo;
          if (j < hi) {
            if (ns > 0) {
              const uint32_t b2[2] = {smem_u32(&bars->full[kslot(q)]), smem_u32(&bars->s_free[0])};
              const uint32_t p2[2] = {kpar(q), static_cast<uint32_t>((ns - 1) & 1)};
              ok = mbar_wait_all(b2, p2, abort_flag);
            } else {
              ok = mbar_wait_warp(smem_u32(&bars->full[kslot(q)]), kpar(q), abort_flag);
            }
            if (!ok) break;
            tc_fence_after_sync();
            issue_s(0, kslot(q));
            ++ns;
            commit(smem_u32(&bars->empty[kslot(q)]));
          }
          if (j > lo) {
            // V(j-1) and both halves' P(j-1): the two halves finish within a
            // few tens of cycles of each other, so one wait covers both
            const uint32_t b3[3] = {smem_u32(&bars->full[vslot(q - 1)]),
                                    smem_u32(&bars->p_full[0]), smem_u32(&bars->p_full[1])};
            const uint32_t p3[3] = {vpar(q - 1), static_cast<uint32_t>(npv0 & 1),
                                    static_cast<uint32_t>(npv1 & 1)};
            ok = mbar_wait_all(b3, p3, abort_flag);
            if (!ok) break;
            tc_fence_after_sync();
            issue_pv_h(0, vslot(q - 1));
            issue_pv_h(1, vslot(q - 1));
            commit(smem_u32(&bars->empty[vslot(q - 1)]));
          }
        }
      } else if constexpr (G::kSplitP) {
        // S0(j), S1(j), PV0(j-1), PV1(j-1): S_t(j) waits only until the
        // softmax of tile t holds S_t(j-1) in registers (s_free)
        int ns0 = 0, ns1 = 0;
        auto issue_s_free = [&](int t, int slot) -> bool {
          const int ns = t ? ns1 : ns0;
          if (ns > 0 &&
              !mbar_wait_warp(smem_u32(&bars->s_free[t]), (ns - 1) & 1, abort_flag))
            return false;
          tc_fence_after_sync();
          issue_s(t, slot);
          if (t) ++ns1; else ++ns0;
          return true;
        };
        auto issue_pv_ready = [&](int t, int qv) -> bool {
          const bool r = mbar_wait_warp(smem_u32(&bars->full[vslot(qv)]), vpar(qv), abort_flag) &&
                         mbar_wait_warp(smem_u32(&bars->p_full[t]), (t ? npv1 : npv0) & 1,
                                        abort_flag);
          if (!r) return false;
          tc_fence_after_sync();
          issue_pv(t, vslot(qv));
          return true;
        };
        for (int j = lo; j <= hi && ok; ++j) {
          const int q = j - lo;
          if (j < hi) {
            ok = mbar_wait_warp(smem_u32(&bars->full[kslot(q)]), kpar(q), abort_flag);
            if (!ok) break;
            tc_fence_after_sync();
            if (in(0, j)) ok = issue_s_free(0, kslot(q));
            if (ok && in(1, j)) ok = issue_s_free(1, kslot(q));
            if (!ok) break;
            commit(smem_u32(&bars->empty[kslot(q)]));
          }
          if (j > lo) {
            if (in(0, j - 1)) ok = issue_pv_ready(0, q - 1);
            if (ok && in(1, j - 1)) ok = issue_pv_ready(1, q - 1);
            if (!ok) break;
            commit(smem_u32(&bars->empty[vslot(q - 1)]));
          }
        }
      } else {
      // D > 64, two tiles: ping-pong
      // The fills of K(j+1) and V(j) are waited for at the end of block j,
      // before the wait for P0(j) (the one that really waits), so that
      // PV0(j) and S0(j+1) issue back to back and PV1(j) waits only for P1.
      ok = mbar_wait_warp(smem_u32(&bars->full[kslot(0)]), kpar(0), abort_flag);
      if (ok) tc_fence_after_sync();
      for (int j = lo; j < hi && ok; ++j) {
        const int q = j - lo;
        if (in(0, j)) issue_s(0, kslot(q));
        if (j > lo) {
          if (in(1, j - 1)) {
            ok = mbar_wait_warp(smem_u32(&bars->p_full[1]), npv1 & 1, abort_flag);
            if (!ok) break;
            tc_fence_after_sync();
            issue_pv(1, vslot(q - 1));
          }
          commit(smem_u32(&bars->empty[vslot(q - 1)]));
        }
        if (in(1, j)) issue_s(1, kslot(q));
        commit(smem_u32(&bars->empty[kslot(q)]));
        ok = mbar_wait_warp(smem_u32(&bars->full[vslot(q)]), vpar(q), abort_flag) &&
             (j + 1 >= hi ||
              mbar_wait_warp(smem_u32(&bars->full[kslot(q + 1)]), kpar(q + 1), abort_flag));
        if (!ok) break;
        if (in(0, j)) {
          ok = mbar_wait_warp(smem_u32(&bars->p_full[0]), npv0 & 1, abort_flag);
          if (!ok) break;
          tc_fence_after_sync();
          issue_pv(0, vslot(q));
        } else {
          tc_fence_after_sync();
        }
      }
      if (ok) {
        const int q = hi - 1 - lo;
        if (in(1, hi - 1)) {
          ok = mbar_wait_warp(smem_u32(&bars->p_full[1]), npv1 & 1, abort_flag);
          if (ok) {
            tc_fence_after_sync();
            issue_pv(1, vslot(q));
          }
        }
        commit(smem_u32(&bars->empty[vslot(q)]));
      }
      }   // ping-pong schedule
    }
    if (elect_one()) tc_commit(smem_u32(&bars->mma_done));
    __syncwarp();
  } else if (kDual && G::kPartnerOwn && bal_role == 1) {
    // =================================================== balanced receiver, warp 11
    // The sender's rows land in this CTA's own buffer whenever the sender
    // finishes its slice, whatever this CTA is doing; this otherwise idle
    // warp acknowledges them at once (so that the sender, which waits for
    // that before leaving, never waits on a CTA that has gone) and holds
    // this CTA until they have landed.  Bounded by three wait limits: the
    // sender copies even after its own waits gave up.
    if (lane == 0) {
      bool landed = false;
      for (int k = 0; k < 3 && !landed; ++k)
        landed = mbar_wait_cluster(smem_u32(&bars->partner_full), 0, abort_flag, false);
      if (landed) mbar_arrive_cluster(cluster_map(smem_u32(&bars->partner_ack), 1));
    }
    __syncwarp();
  }
  } else {
    // =================================================== softmax / epilogue
    regs_inc<RegSplit::kBig>();
    // warpgroup t: the softmax of query tile t, or (kDual) of keys
    // [64t, 64t + 64) of every block of tile 0
    const int t = warp >> 2;
    const int tt = kDual ? 0 : t;        // query tile of this warpgroup
    const int r = tid & 127;             // row within the tile = TMEM lane
    // this tile's scalars (selected, so that nothing is indexed at run time)
    const int tq0 = tt ? q0[1] : q0[0];
    const int trows = tt ? rows[1] : rows[0];
    const int tlo = tt ? rng[1].lo : rng[0].lo;
    const int n_blocks = tt ? rng[1].hi - rng[1].lo : rng[0].hi - rng[0].lo;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    // S columns this warpgroup reads; O_t and P_t are its own (kDual: the
    // second tile's slots hold the second key half's)
    const uint32_t tS = tmem + lane_base + (kDual ? 64u * t : t * 128u);
    const uint32_t tO = tmem + lane_base + 256u + t * D;
    // split-P: P_t columns; kDual: P_t of its key half in S1's free slot
    const uint32_t tPs = tmem + lane_base + (kDual ? 128u : 384u) + t * 64u;
    // packed tiles: row r is query position r % tile_q of head bh + r / tile_q
    const int r_loc = p.packed ? (r & (p.tile_q - 1)) : r;
    const int row_head = p.packed ? bh + (r >> p.tile_q_shift) : bh;
    const int i = tq0 + r_loc;           // query index of this row
    // One-tile schedules: a warp none of whose rows is a real query (short
    // query ranges: decoding) skips its loads, exponentials and P stores but
    // keeps every wait and arrival, so the barrier phases stay in step.
    // Its P rows are never written; PV then fills O rows that no one stores.
    const bool idle_warp = kDual && !__any_sync(0xffffffffu, r_loc < trows);
    const int row_lo = p.wl < 0 ? 0 : i - p.wl;
    const int row_hi = p.wr < 0 ? p.L_k - 1 : min(p.L_k - 1, i + p.wr);
    const int first = tq0, last = tq0 + trows - 1;
    const int full_lo = p.wl < 0 ? 0 : last - p.wl;               // block start bound
    const int full_hi = p.wr < 0 ? p.L_k - 1 : min(p.L_k - 1, first + p.wr);
    // with a mask the scores are scaled (and biased) as they are loaded and
    // the softmax below runs with a unit scale
    const float sl2 = kMask ? 1.0f : p.scale_log2;
    long long mask_row = 0;
    if constexpr (kMask) {
      const int mb = row_head / p.H, mh = row_head - (row_head / p.H) * p.H;
      mask_row = mb * p.mask_sb + mh * p.mask_sh + static_cast<long long>(i) * p.mask_sq;
    }

    float m_use = -INFINITY;   // running max (log2 units of scaled scores)
    float m_true = -INFINITY;  // exact running max, for the softmax statistics
    float l = 0.0f;            // running normaliser, relative to m_use
    bool ok = true;

    if (trows > 0) {
      for (int n = 0; n < n_blocks; ++n) {
        const int j = tlo + n;
        ok = mbar_wait_warp(
            smem_u32(&bars->s_full[tt]), n & 1, abort_flag);
        if (!ok) break;
        tc_fence_after_sync();

        const bool full = (j * kBN >= full_lo) && (j * kBN + kBN - 1 <= full_hi);
        // S row of this block -> registers (masked entries -> -inf)
        auto load_s = [&](float (&sv)[kBN]) {
          uint32_t sr[4][32];
          tmem_ld_x32(tS + 0, sr[0]);
          tmem_ld_x32(tS + 32, sr[1]);
          tmem_ld_x32(tS + 64, sr[2]);
          tmem_ld_x32(tS + 96, sr[3]);
          tmem_wait_ld();
          reg_dep(sr[0]);
          reg_dep(sr[1]);
          reg_dep(sr[2]);
          reg_dep(sr[3]);
#pragma unroll
          for (int c = 0; c < kBN; ++c) sv[c] = __uint_as_float(sr[c >> 5][c & 31]);
          if (!full) {
            const int lo_c = row_lo - j * kBN;
            const int hi_c = row_hi - j * kBN;
#pragma unroll
            for (int c = 0; c < kBN; ++c)
              if (c < lo_c || c > hi_c) sv[c] = -INFINITY;
          }
          if constexpr (kMask)
            apply_mask(sv, p, mask_row + static_cast<long long>(j) * kBN,
                       min(kBN, p.L_k - j * kBN), r_loc < trows, p.scale_log2);
        };
        const float2 sl2v = make_float2(sl2, sl2);

        // 64-key helpers of the dual schedule
        float alpha = 1.0f;
        bool rescaled = false;
        float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        // 64 keys of the row from TMEM address taddr, key k0 first
        auto load64 = [&](uint32_t taddr, int k0, float (&sv)[kBN / 2]) {
          uint32_t sr[2][32];
          tmem_ld_x32(taddr, sr[0]);
          tmem_ld_x32(taddr + 32, sr[1]);
          tmem_wait_ld();
          reg_dep(sr[0]);
          reg_dep(sr[1]);
#pragma unroll
          for (int c = 0; c < kBN / 2; ++c) sv[c] = __uint_as_float(sr[c >> 5][c & 31]);
          if (!full) {
            const int lo_c = row_lo - k0;
            const int hi_c = row_hi - k0;
#pragma unroll
            for (int c = 0; c < kBN / 2; ++c)
              if (c < lo_c || c > hi_c) sv[c] = -INFINITY;
          }
          if constexpr (kMask)
            apply_mask(sv, p, mask_row + static_cast<long long>(k0), min(kBN / 2, p.L_k - k0),
                       r_loc < trows, p.scale_log2);
        };
        // half maximum (four chains of 3-input maxima), in scaled log2 units
        auto half_max = [&](const float (&sv)[kBN / 2]) -> float {
          float mx[4] = {sv[0], sv[1], sv[2], sv[3]};
#pragma unroll
          for (int c = 4; c < kBN / 2 - 4; c += 8)
#pragma unroll
            for (int u = 0; u < 4; ++u) mx[u] = fmax3(mx[u], sv[c + 2 * u], sv[c + 2 * u + 1]);
          const float m = fmax3(fmax3(mx[0], mx[1], sv[kBN / 2 - 4]),
                                fmax3(mx[2], mx[3], sv[kBN / 2 - 3]),
                                fmaxf(sv[kBN / 2 - 2], sv[kBN / 2 - 1]));
          return m == -INFINITY ? -INFINITY : m * sl2;
        };
        // conditional rescale against a half's maximum; true if this warp
        // moved its reference
        auto raise = [&](float m_new) -> bool {
          m_true = fmaxf(m_true, m_new);
          if (!__any_sync(0xffffffffu, m_new > m_use + kRescaleThreshold)) return false;
          const float m_upd = fmaxf(m_use, m_new);
          const float a = (m_upd == -INFINITY) ? 1.0f : ex2(m_use - m_upd);
          m_use = m_upd;
          l *= a;
          alpha *= a;
          rescaled = true;
          return true;
        };
        auto exp_half = [&](const float (&sv)[kBN / 2], uint32_t (&pkh)[32], auto poly_ok) {
          const float m_sub = (m_use == -INFINITY) ? 0.0f : m_use;
          const float2 negm = make_float2(-m_sub, -m_sub);
#pragma unroll
          for (int c = 0; c < kBN / 2; c += 2) {
            const int pair = c >> 1;
            const float2 x = __ffma2_rn(make_float2(sv[c], sv[c + 1]), sl2v, negm);
            float2 pp;
            if (decltype(poly_ok)::value && (pair % kPoly) == kPoly - 1)
              pp = exp2_poly2(x);
            else
              pp = make_float2(ex2(x.x), ex2(x.y));
            // l sums the unrounded fp32 weights
            ls[pair & 1] = __fadd2_rn(ls[pair & 1], pp);
            put_p<DT>(pkh, pair, pp.x, pp.y);
          }
        };
        auto exp_any = [&](const float (&sv)[kBN / 2], uint32_t (&pkh)[32]) {
          // masked entries are -inf: only MUFU's ex2 turns them into exact 0
          if (full)
            exp_half(sv, pkh, std::true_type{});
          else
            exp_half(sv, pkh, std::false_type{});
        };
        // exact pass: the row max first (four chains of 3-input maxima), then
        // the conditional rescale, then P; used for masked blocks, the first
        // block of a row, and whenever the speculative pass is dropped
        auto exact_pass = [&](float (&sv)[kBN]) {
          // exact pass: the row max first (four chains of 3-input maxima)
          float mx[4] = {sv[0], sv[1], sv[2], sv[3]};
#pragma unroll
          for (int c = 4; c < kBN - 4; c += 8)
#pragma unroll
            for (int u = 0; u < 4; ++u) mx[u] = fmax3(mx[u], sv[c + 2 * u], sv[c + 2 * u + 1]);
          const float m_blk = fmax3(fmax3(mx[0], mx[1], sv[kBN - 4]),
                                    fmax3(mx[2], mx[3], sv[kBN - 3]),
                                    fmaxf(sv[kBN - 2], sv[kBN - 1]));
          const float m_new = (m_blk == -INFINITY) ? -INFINITY : m_blk * sl2;
          m_true = fmaxf(m_true, m_new);

          // conditional rescale: only when some row's max grew by > 2^8
          const bool need = m_new > m_use + kRescaleThreshold;
          float alpha = 1.0f;
          const bool warp_rescale = __any_sync(0xffffffffu, need);
          if (warp_rescale) {
            const float m_upd = fmaxf(m_use, m_new);
            alpha = (m_upd == -INFINITY) ? 1.0f : ex2(m_use - m_upd);
            m_use = m_upd;
            l *= alpha;
          }
          const float m_sub = (m_use == -INFINITY) ? 0.0f : m_use;

          // P = 2^(s*scale*log2e - m), packed two per 32-bit TMEM column.
          // P overwrites S columns [0, 64): all of S is already in registers.
          const float2 negm = make_float2(-m_sub, -m_sub);
          float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
          auto exp_block = [&](auto poly_ok) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t pk[32];
#pragma unroll
              for (int c = 0; c < kBN / 2; c += 2) {
                const float2 x =
                    __ffma2_rn(make_float2(sv[half * 64 + c], sv[half * 64 + c + 1]), sl2v, negm);
                const int pair = (half * 64 + c) >> 1;
                float2 pp;
                if (decltype(poly_ok)::value && (pair % kPoly) == kPoly - 1)
                  pp = exp2_poly2(x);
                else
                  pp = make_float2(ex2(x.x), ex2(x.y));
                // l sums the unrounded fp32 weights: lse = m + ln(l) then
                // keeps fp32 accuracy whatever the input type
                ls[(c >> 1) & 1] = __fadd2_rn(ls[(c >> 1) & 1], pp);
                put_p<DT>(pk, c >> 1, pp.x, pp.y);
              }
              store_p_half<DT>(tS, half, pk);
            }
          };
          // masked entries are -inf: only MUFU's ex2 turns them into exact 0
          if (full)
            exp_block(std::true_type{});
          else
            exp_block(std::false_type{});
          l += (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y);

          if (warp_rescale && n > 0) {
            // O_t was completed up to block j-1 (PV_t(j-1) finished before
            // S_t(j) was issued); scale it by alpha row by row.
            scale_o_row<D>(tO, alpha);
          }
        };

        if (kDual && idle_warp) {
          tc_fence_before_sync();
          mbar_arrive(smem_u32(&bars->s_free[0]));
          if (n > 0) {
            const bool got = mbar_wait_warp(smem_u32(&bars->pv_done[t]), (n - 1) & 1, abort_flag);
            ok = ok && got;
          }
        } else if constexpr (kDual) {
          // keys [64t, 64t + 64) of this block: free S (both warpgroups
          // arrive) for the next block's S MMA as soon as it is in
          // registers, then P_t.  Unmasked blocks, once every row of the
          // warp has a reference max, take the exponentials against that
          // reference while the half max is reduced alongside (as the
          // ping-pong's speculative pass); if some row's max grew by more
          // than 2^8 they are redone after the rescale.
          float sv[kBN / 2];
          load64(tS, j * kBN + 64 * t, sv);
          tc_fence_before_sync();
          mbar_arrive(smem_u32(&bars->s_free[0]));
          uint32_t pk[32];
          bool spec_ok = false;
          if (full && __all_sync(0xffffffffu, m_use != -INFINITY)) {
            const float m_half = half_max(sv);
            exp_half(sv, pk, std::true_type{});
            m_true = fmaxf(m_true, m_half);
            spec_ok = !__any_sync(0xffffffffu, m_half > m_use + kRescaleThreshold);
            if (!spec_ok) {
              ls[0] = make_float2(0.f, 0.f);
              ls[1] = make_float2(0.f, 0.f);
              raise(m_half);
              exp_half(sv, pk, std::true_type{});
            }
          } else {
            const float m_half = half_max(sv);
            raise(m_half);
            exp_any(sv, pk);
          }
          l += (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y);
          // P_t and O_t are read / written by PV_t(j-1): wait for it
          if (n > 0) {
            const bool got = mbar_wait_warp(smem_u32(&bars->pv_done[t]), (n - 1) & 1, abort_flag);
            ok = ok && got;
            tc_fence_after_sync();
          }
          if (ok) {
            store_p_half<DT>(tPs, 0, pk);
            if (rescaled && n > 0) scale_o_row<D>(tO, alpha);
          }
        } else if constexpr (G::kSplitP) {
          // row max first, then free S_t for the next block's S MMA, then P
          // (D = 16: S_t is freed right after its load, before the max)
          float s[kBN];
          load_s(s);
          if constexpr (D <= 16) {
            tc_fence_before_sync();
            mbar_arrive(smem_u32(&bars->s_free[t]));
          }
          float mx[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
          for (int c = 4; c < kBN - 4; c += 8)
#pragma unroll
            for (int u = 0; u < 4; ++u) mx[u] = fmax3(mx[u], s[c + 2 * u], s[c + 2 * u + 1]);
          const float m_blk = fmax3(fmax3(mx[0], mx[1], s[kBN - 4]),
                                    fmax3(mx[2], mx[3], s[kBN - 3]),
                                    fmaxf(s[kBN - 2], s[kBN - 1]));
          if constexpr (D > 16) {
            tc_fence_before_sync();
            mbar_arrive(smem_u32(&bars->s_free[t]));
          }
          const float m_new = (m_blk == -INFINITY) ? -INFINITY : m_blk * sl2;
          m_true = fmaxf(m_true, m_new);
          const bool need = m_new > m_use + kRescaleThreshold;
          float alpha = 1.0f;
          const bool warp_rescale = __any_sync(0xffffffffu, need);
          if (warp_rescale) {
            const float m_upd = fmaxf(m_use, m_new);
            alpha = (m_upd == -INFINITY) ? 1.0f : ex2(m_use - m_upd);
            m_use = m_upd;
            l *= alpha;
          }
          const float m_sub = (m_use == -INFINITY) ? 0.0f : m_use;
          const float2 negm = make_float2(-m_sub, -m_sub);
          // P = 2^(s*scale*log2e - m); at D <= 32 the two halves of the row
          // are interleaved (more independent exponentials in flight: the
          // softmax warps are the whole cost there), else in column order
          float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                          make_float2(0.f, 0.f)};
          uint32_t pk[2][32];
          auto exp_pair = [&](int c, float2 &acc) {
            const int pair = c >> 1;
            const float2 x = __ffma2_rn(make_float2(s[c], s[c + 1]), sl2v, negm);
            float2 pp;
            if (full && (pair % kPoly) == kPoly - 1)
              pp = exp2_poly2(x);
            else
              pp = make_float2(ex2(x.x), ex2(x.y));
            acc = __fadd2_rn(acc, pp);
            put_p<DT>(pk[c >> 6], pair & 31, pp.x, pp.y);
          };
          if constexpr (D <= 32) {
#pragma unroll
            for (int c0 = 0; c0 < kBN / 2; c0 += 2) {
              exp_pair(c0, ls[(c0 >> 1) & 1]);
              exp_pair(c0 + kBN / 2, ls[2 + ((c0 >> 1) & 1)]);
            }
          } else {
#pragma unroll
            for (int c = 0; c < kBN; c += 2) exp_pair(c, ls[(c >> 1) & 1]);
          }
          l += ((ls[0].x + ls[0].y) + (ls[1].x + ls[1].y)) + ((ls[2].x + ls[2].y) + (ls[3].x + ls[3].y));
          // P_t and O_t are read / written by PV_t(j-1): wait for it
          if (n > 0) {
            const bool got = mbar_wait_warp(smem_u32(&bars->pv_done[t]), (n - 1) & 1, abort_flag);
            ok = ok && got;
            tc_fence_after_sync();
          }
          if (ok) {
            store_p_half<DT>(tPs, 0, pk[0]);
            store_p_half<DT>(tPs, 1, pk[1]);
            if (warp_rescale && n > 0) scale_o_row<D>(tO, alpha);
          }
        } else {
        // D > 64, two tiles.  Speculative pass (unmasked blocks, once every row has a reference
        // max): P = 2^(s*scale*log2e - m_use) against the current reference
        // while the block max is reduced alongside, so that the exponentials
        // do not wait for the max.  If some row's max grew by more than 2^8
        // the pass is dropped and S, still intact in TMEM (P is stored only
        // after the check), is reloaded for the exact pass.
        if (full && __all_sync(0xffffffffu, m_use != -INFINITY)) {
          float s[kBN];
          load_s(s);
          const float2 negm = make_float2(-m_use, -m_use);
          float2 ls2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
          float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          uint32_t pk[2][32];
#pragma unroll
          for (int c = 0; c < kBN; c += 2) {
            const int pair = c >> 1;
            mx[pair & 3] = fmax3(mx[pair & 3], s[c], s[c + 1]);
            const float2 x = __ffma2_rn(make_float2(s[c], s[c + 1]), sl2v, negm);
            float2 pp;
            if ((pair % kPoly) == kPoly - 1)
              pp = exp2_poly2(x);
            else
              pp = make_float2(ex2(x.x), ex2(x.y));
            ls2[pair & 1] = __fadd2_rn(ls2[pair & 1], pp);
            put_p<DT>(pk[c >> 6], pair & 31, pp.x, pp.y);
          }
          const float m_new = fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]) * sl2;
          m_true = fmaxf(m_true, m_new);
          if (__any_sync(0xffffffffu, m_new > m_use + kRescaleThreshold)) {
            float s2[kBN];
            load_s(s2);
            exact_pass(s2);
          } else {
            store_p_half<DT>(tS, 0, pk[0]);
            store_p_half<DT>(tS, 1, pk[1]);
            l += (ls2[0].x + ls2[0].y) + (ls2[1].x + ls2[1].y);
          }
        } else {
          float s[kBN];
          load_s(s);
          exact_pass(s);
        }
        }   // ping-pong schedule
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(smem_u32(&bars->p_full[t]));
      }

      // ---------------------------------------------- epilogue: O / l, lse
      if (ok && n_blocks > 0) {
        ok = mbar_wait_warp(smem_u32(&bars->pv_done[t]), (n_blocks - 1) & 1, abort_flag);
        if (ok) tc_fence_after_sync();
      }
      // kDual: the two key halves are two slices of the row.  Warpgroup 1
      // hands its (m, l, exact max) to warpgroup 0 through shared memory (Q
      // tile 1's slot, unused with one tile); warpgroup 0 merges them, as
      // the split-KV merge does, and writes the row: O = wa O_0 + wb O_1.
      float wa = 1.0f, wb = 0.0f;
      if constexpr (kDual) {
        float *xch = reinterpret_cast<float *>(smem + G::kOffQ + G::kTileBytes);
        if (t == 1) {
          xch[r] = m_use;
          xch[kBM + r] = l;
          xch[2 * kBM + r] = m_true;
          xch[3 * kBM + r] = ok ? 1.0f : 0.0f;
        }
        tc_fence_before_sync();
        named_barrier_sync(3, 2 * kBM);
        tc_fence_after_sync();
        if (t == 0) {
          const float mb = xch[r], lb = xch[kBM + r], tb = xch[2 * kBM + r];
          ok = ok && xch[3 * kBM + r] != 0.0f;   // uniform: the same rows' warp
          const float m = fmaxf(m_use, mb);
          wa = (m_use == -INFINITY) ? 0.0f : ex2(m_use - m);
          wb = (mb == -INFINITY) ? 0.0f : ex2(mb - m);
          l = wa * l + wb * lb;
          m_use = m;
          m_true = fmaxf(m_true, tb);
        }
      }
      // balanced split pair: the partner slice's weight and O row (receiver)
      constexpr int kUnitsO = D / 4;                  // 16-byte units of an fp32 O row
      float wc = 0.0f;
      const float4 *prow = nullptr;
      // O row chunk (columns [c, c + W)) into registers; kDual: merged
      auto load_o = [&](int c, auto wd, auto &o) {
        constexpr int W = decltype(wd)::value;
        if (n_blocks > 0 && !idle_warp) {
          tmem_ld_cols<W>(tO + c, o);
          if constexpr (kDual) {
            uint32_t ob[W];
            tmem_ld_cols<W>(tO + D + c, ob);
            tmem_wait_ld();
            reg_dep(o);
            reg_dep(ob);
#pragma unroll
            for (int u = 0; u < W; ++u)
              o[u] = __float_as_uint(wa * __uint_as_float(o[u]) + wb * __uint_as_float(ob[u]));
            if (prow != nullptr) {
#pragma unroll
              for (int u = 0; u < W / 4; ++u) {
                const float4 v = prow[(c / 4 + u + r) % kUnitsO];
                o[4 * u] = __float_as_uint(__uint_as_float(o[4 * u]) + wc * v.x);
                o[4 * u + 1] = __float_as_uint(__uint_as_float(o[4 * u + 1]) + wc * v.y);
                o[4 * u + 2] = __float_as_uint(__uint_as_float(o[4 * u + 2]) + wc * v.z);
                o[4 * u + 3] = __float_as_uint(__uint_as_float(o[4 * u + 3]) + wc * v.w);
              }
            }
          } else {
            tmem_wait_ld();
            reg_dep(o);
          }
        } else {
#pragma unroll
          for (int u = 0; u < W; ++u) o[u] = 0u;
        }
      };
      // Balanced split pair (one tile on the two CTAs of a cluster): the
      // sender stages its slice's unnormalised O rows and (m, l, exact max)
      // and copies them into the receiver, one bulk copy per warp of 32
      // rows; the receiver joins them to its own as two key slices and
      // acknowledges, after which the sender may leave.  With a buffer of
      // their own (D <= 64) the rows are staged there and copied at once;
      // otherwise they are staged in the sender's K/V ring and copied into
      // the receiver's once the receiver reports it idle (both halves' last
      // PV complete, which warpgroup 0 knows after the barrier above).  Per
      // warp the buffer holds its 32 O rows, then their (m, l, exact max,
      // ok); the units of a row are stored rotated by the row index, so
      // that a warp's 16-byte accesses spread over the banks.
      if constexpr (kDual) {
        constexpr uint32_t kWarpPartBytes = 32 * (D * 4 + 16);
        constexpr uint32_t kPartnerBytes = 4 * kWarpPartBytes;
        static_assert(kPartnerBytes == G::kPartnerBytes, "partner buffer size");
        static_assert(kPartnerBytes <= G::kSlots * G::kTileBytes,
                      "the partner's rows fit in the K/V ring");
        if (bal_role != 0 && t == 0) {
          uint8_t *part = smem + (G::kPartnerOwn ? G::kOffPartner : G::kOffRing) +
                          (warp & 3) * kWarpPartBytes;   // this warp's rows
          float4 *prow_w = reinterpret_cast<float4 *>(part) + (r & 31) * kUnitsO;
          float4 *pml = reinterpret_cast<float4 *>(part + 32 * D * 4) + (r & 31);
          if (bal_role == 1) {
            // the receiver: with an own buffer it always waits for the
            // sender's rows (bounded), so that no copy reaches it after it
            // has gone; with the ring it first reports the ring idle
            if constexpr (!G::kPartnerOwn) {
              if (r == 0 && ok) {
                mbar_arrive_expect_tx(smem_u32(&bars->partner_full), kPartnerBytes);
                mbar_arrive_cluster(cluster_map(smem_u32(&bars->recv_ready), 1));
              }
            }
            // (once the go-ahead has gone out, or with an own buffer, the
            // sender's copy will come: wait for it, bounded, even after an
            // abort, so that it never lands in a CTA that has gone)
            bool got = false;
            if (ok || G::kPartnerOwn)
              got = mbar_wait_cluster(smem_u32(&bars->partner_full), 0, abort_flag, false);
            got = __all_sync(0xffffffffu, got);
            ok = ok && got;
            if (ok) {
              const float4 ml = *pml;
              ok = __all_sync(0xffffffffu, ml.w != 0.0f);   // the sender's warp is uniform
              const float m = fmaxf(m_use, ml.x);
              const float sa = (m_use == -INFINITY) ? 0.0f : ex2(m_use - m);
              wc = (ml.x == -INFINITY) ? 0.0f : ex2(ml.x - m);
              wa *= sa;
              wb *= sa;
              l = sa * l + wc * ml.y;
              m_use = m;
              m_true = fmaxf(m_true, ml.z);
              prow = prow_w;
            }
          } else {
            if (ok) {
              for_o_chunks<D>([&](int c, auto w) {
                constexpr int W = decltype(w)::value;
                uint32_t o[W];
                load_o(c, w, o);
#pragma unroll
                for (int u = 0; u < W / 4; ++u)
                  prow_w[(c / 4 + u + r) % kUnitsO] =
                      make_float4(__uint_as_float(o[4 * u]), __uint_as_float(o[4 * u + 1]),
                                  __uint_as_float(o[4 * u + 2]), __uint_as_float(o[4 * u + 3]));
              });
            }
            *pml = make_float4(m_use, l, m_true, ok ? 1.0f : 0.0f);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              // always copy (the receiver waits for it) and wait (bounded) for
              // the acknowledgement before leaving: no remote operation may
              // reach this CTA after it has gone
              const bool go =
                  G::kPartnerOwn ||
                  mbar_wait_cluster(smem_u32(&bars->recv_ready), 0, abort_flag, false);
              if (go) {
                bulk_copy_to_cluster(cluster_map(smem_u32(part), 0), smem_u32(part),
                                     kWarpPartBytes,
                                     cluster_map(smem_u32(&bars->partner_full), 0));
                if (r == 0) mbar_wait_cluster(smem_u32(&bars->partner_ack), 0, abort_flag, false);
              }
            }
            __syncwarp();
          }
        }
      }
      if (kDual && t == 1) {
        // warpgroup 1 is done: warpgroup 0 writes the row.  In a balanced
        // receiver whose rows land in its K/V ring, its first thread
        // acknowledges the sender's copy (requested by warpgroup 0 above, so
        // it lands while this CTA is in its epilogue), off warpgroup 0's path.
        if constexpr (!G::kPartnerOwn) {
          if (bal_role == 1 && r == 0 &&
              mbar_wait_cluster(smem_u32(&bars->partner_full), 0, abort_flag, false))
            mbar_arrive_cluster(cluster_map(smem_u32(&bars->partner_ack), 1));
        }
      } else if (bal_role == 2) {
        // the receiver writes the row
      } else if (p.ws_o != nullptr) {
        // split-KV partial: unnormalised O (fp32) and (m, l) of this slice.
        // tcgen05.ld is warp-collective: every lane loads (ok and n_blocks
        // are warp-uniform), only the lanes of real rows store.
        if (ok) {
          const bool mine = r_loc < trows;
          const size_t row = static_cast<size_t>(split) * p.rows_total +
                             static_cast<size_t>(row_head) * p.L_q + i;
          float4 *dst = reinterpret_cast<float4 *>(p.ws_o + row * D);
          for_o_chunks<D>([&](int c, auto w) {
            constexpr int W = decltype(w)::value;
            uint32_t o[W];
            load_o(c, w, o);
            if (mine) {
#pragma unroll
              for (int u = 0; u < W / 4; ++u)
                dst[c / 4 + u] = make_float4(__uint_as_float(o[4 * u]),
                                             __uint_as_float(o[4 * u + 1]),
                                             __uint_as_float(o[4 * u + 2]),
                                             __uint_as_float(o[4 * u + 3]));
            }
          });
          if (mine) p.ws_ml[row] = make_float2(l > 0.0f ? m_use : -INFINITY, l);
        }
      } else {
      const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
      uint8_t *stage = smem + G::kOffQ + t * G::kTileBytes;   // Q_t is free now
      const int sw = ((r * G::kSwBytes) >> 7) & (G::kUnitsPerBoxRow - 1);
      auto put_units = [&](int c0, const uint32_t *w, int nunits) {
        // c0: first column of this chunk; w: packed pairs, 4 words per unit
#pragma unroll
        for (int u = 0; u < nunits; ++u) {
          const int unit = (c0 * 2) / 16 + u;
          const int box = unit / G::kUnitsPerBoxRow;
          const int cc = unit % G::kUnitsPerBoxRow;
          uint4 *dst = reinterpret_cast<uint4 *>(stage + box * G::kBoxBytes + r * G::kSwBytes +
                                                 ((cc ^ sw) << 4));
          *dst = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      };
      if constexpr (kF8) {
        // fp8 inputs: bf16 rows straight to global memory (the 8-bit Q
        // tile is too small to stage them); every lane loads TMEM, the
        // lanes of real rows store
        if (ok) {
          const float sc = inv_l * p.descale_v;
          uint8_t *orow = static_cast<uint8_t *>(p.out_ptr) +
                          (static_cast<size_t>(row_head) * p.L_q + i) * D * 2;
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            uint32_t o[32];
            load_o(c, std::integral_constant<int, 32>{}, o);   // kDual: both halves merged
            if (r_loc < trows) {
#pragma unroll
              for (int u = 0; u < 4; ++u)
                *reinterpret_cast<uint4 *>(orow + (c + 8 * u) * 2) = make_uint4(
                    pack2<1>(__uint_as_float(o[8 * u]) * sc, __uint_as_float(o[8 * u + 1]) * sc),
                    pack2<1>(__uint_as_float(o[8 * u + 2]) * sc, __uint_as_float(o[8 * u + 3]) * sc),
                    pack2<1>(__uint_as_float(o[8 * u + 4]) * sc, __uint_as_float(o[8 * u + 5]) * sc),
                    pack2<1>(__uint_as_float(o[8 * u + 6]) * sc, __uint_as_float(o[8 * u + 7]) * sc));
            }
          }
        }
      } else {
      if (ok) {
        for_o_chunks<D>([&](int c, auto wd) {
          constexpr int W = decltype(wd)::value;
          uint32_t o[W];
          load_o(c, wd, o);
          uint32_t w[W / 2];
#pragma unroll
          for (int u = 0; u < W / 2; ++u)
            w[u] = pack2<kF8 ? 1 : DT>(__uint_as_float(o[2 * u]) * inv_l,
                                       __uint_as_float(o[2 * u + 1]) * inv_l);
          put_units(c, w, W / 8);
        });
      }
      fence_proxy_async_smem();
      named_barrier_sync(1 + t, kBM);
      if (r == 0 && !*abort_flag) {
        for (int bx = 0; bx < G::kNumBox; ++bx)
          tma_store_3d(&p.tm_o, smem_u32(stage + bx * G::kBoxBytes), bx * G::kBoxCols, tq0,
                       bh);
        bulk_commit_group();
        bulk_wait_group_read_all();   // the staging tile has been read
      }
      }   // 16-bit output through TMA
      if (ok && p.smax != nullptr && r_loc < trows) {
        // statistics against the exact max: sum_j 2^(t_j - m_true) = l 2^(m_use - m_true)
        const size_t row = static_cast<size_t>(row_head) * p.L_q + i;
        p.smax[row] = l > 0.0f ? m_true * 0.6931471805599453f : -INFINITY;
        p.ssum[row] = l > 0.0f ? l * ex2(m_use - m_true) : 0.0f;
      }
      if (ok && p.lse != nullptr && r_loc < trows) {
        const float lse = l > 0.0f ? (m_use + __log2f(l)) * 0.6931471805599453f : -INFINITY;
        p.lse[static_cast<size_t>(row_head) * p.L_q + i] = lse;
      }
      }   // normal epilogue
    }
  }

  // ---- teardown
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after_sync();
    mbar_wait_slow(smem_u32(&bars->mma_done), 0, abort_flag, false);
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace fa
