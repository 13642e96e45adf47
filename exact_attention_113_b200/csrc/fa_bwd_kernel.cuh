// fa_bwd_kernel.cuh -- exact attention backward for sm_100a (B200).
//
// The pages keep only the softmax statistics from the forward and recompute
// the attention matrix from Q, K, V when the gradients are taken
// ("FlashAttention算法原理与性能优化实战" §1.2.3; "Flash Attention是怎么做到又快又省
// 显存的？" 总结; the Triton FA2 walkthrough keeps the logsumexp for this).  The
// gradients themselves follow from the chain rule through O = P V,
// P = softmax(S), S = scale Q K^T:
//     dV = P^T dO,   dP = dO V^T,   dS = P o (dP - delta),
//     delta_i = dO_i . O_i  (= sum_j P_ij dP_ij),
//     dQ = scale dS K,   dK = scale dS^T Q.
//
// One CTA owns one block of 128 keys of one (batch, K/V head) and walks the
// query blocks that can see it, for every query head of the GQA group, so
// that dK and dV accumulate in TMEM with no atomics.  Per step (one 128-row
// query block) five tcgen05 MMAs:
//     S^T  = K Q^T      (SS; keys on TMEM lanes, queries along columns)
//     dP^T = V dO^T     (SS)
//     dV  += P^T dO     (TS: P^T from TMEM, dO MN-major from shared memory)
//     dK  += dS^T Q     (TS: dS^T from TMEM)
//     dQ   = dS K       (SS: dS staged in shared memory MN-major, K MN-major)
// dQ of the step is added into an fp32 accumulator in global memory by a
// warpgroup of its own: TMEM -> swizzled fp32 staging in shared memory ->
// TMA bulk reduce-add (the addition happens in L2, a tile at a time); the
// other key blocks add theirs.
//
// Roles: P/dS warpgroups compute P and dS for a share of the query columns
// of every key row (thread = TMEM lane = key): for D <= 64 four of them
// (warpgroups 0, 1, 4 and 5; 32 columns each, 768 threads), so that four
// warps per SM sub-partition share the exponentials and the dS math; for
// D > 64 two (warpgroups 0 and 1; 64 columns each, 512 threads).  Warp 8
// issues the MMAs, warp 9 is the TMA producer; warpgroup 3 drains dQ
// (thread = TMEM lane = query row).
//
// TMEM (512 columns): S^T [0,128); dP^T [128,256) with dS^T (two 16-bit
// values per column) written over the first half of each P/dS warpgroup's
// columns; dV [256, 256+D); dK [256+D, 256+2D).  D > 64: P^T over S^T
// likewise, and dQ [128, 128+D) after dK has read dS^T (tcgen05 MMAs of
// one thread run in order).  D <= 64: dQ [384, 384+D) of its own; D = 16
// also P^T [448, 512), so that S^T of the next step is computed while P of
// this one is.
//
// Every wait is bounded (sm100.cuh); after a timeout each role leaves its
// loop, the producer lets its copies land, and TMEM is freed.
#pragma once

#include "fa_fwd_kernel.cuh"

namespace fa {

struct BwdParams {
  CUtensorMap tm_q;    // [B*H,    L_q, D]
  CUtensorMap tm_k;    // [B*H_kv, L_k, D]
  CUtensorMap tm_v;    // [B*H_kv, L_k, D]
  CUtensorMap tm_do;   // [B*H,    L_q, D]
  CUtensorMap tm_dq;   // dq_acc as [B*H, L_q, D] fp32, box [128 rows, min(32, D) cols]
  const float *lse2;   // [B*H][L_q_pad]: lse * log2(e); +inf where no key is visible / past L_q
  const float *delta;  // [B*H][L_q_pad]: dO_i . O_i; 0 past L_q
  float *dq_acc;       // [B*H][L_q][D] fp32, zero before the launch
  void *dk;            // [B*H_kv][L_k][D]
  void *dv;            // [B*H_kv][L_k][D]
  int H, H_kv, L_q, L_k, L_q_pad, group;
  int n_kblocks;       // ceil(L_k / 128)
  int wl, wr;          // visible iff i - wl <= j <= i + wr; -1 = unbounded
  float scale_log2;    // scale * log2(e), clamped to >= 1e-30
  float scale;
  // optional attention mask (kMask instances), read as the forward reads
  // it: element (b, h, i, j) at mask + b*mask_sb + h*mask_sh + i*mask_sq + j;
  // type 1 bool (nonzero hides), 2 fp16 / 3 fp32 added to the scaled score
  const void *mask;
  int mask_type;
  long long mask_sb, mask_sh, mask_sq;
};

// Launch shape by head dim.  D <= 64 (dQ has TMEM columns of its own): the
// P / dS math sets the step, so four P/dS warpgroups of 32 query columns
// (768 threads, four warps per SM sub-partition); D > 64: the dQ drain ->
// dP chain sets it, and two warpgroups of 64 columns (512 threads) draw less
// power.  setmaxnreg split: P/dS warpgroups, dQ drain warpgroup, MMA/TMA
// warpgroup, adding up to the launch allocation (registers per thread,
// 65536 / threads in steps of 8; the host checks the built count).
template <int D>
struct BwdCfg {
  static constexpr int kPdsGroups = D <= 64 ? 4 : 2;
  static constexpr int kThreads = 256 + 128 * kPdsGroups;
  static constexpr int kPdsCols = kBM / kPdsGroups;       // query columns per warpgroup
  static constexpr uint32_t kLaunchRegs = D <= 64 ? 80 : 128;
  static constexpr uint32_t kRegsPds = D <= 64 ? 80 : 144;
  static constexpr uint32_t kRegsDrain = D <= 64 ? 104 : 168;
  static constexpr uint32_t kRegsIssue = 56;
  // D = 16: P^T goes to TMEM columns [448, 512), free there (S^T, dP^T,
  // dV, dK and dQ take [0, 384 + D)), so S^T of the next step can be
  // computed while P of this one is: once every P/dS thread holds S^T(n).
  // (+9 % at D = 16; at D = 32 and 64 the earlier S MMA cost 1-5 %.)
  static constexpr bool kEarlyS = D <= 16;
  static constexpr uint32_t kPCol = 448;
  static_assert(kPdsGroups * kRegsPds + kRegsDrain + kRegsIssue ==
                    (kThreads / 128) * kLaunchRegs,
                "register split must fit in the launch allocation");
  static_assert(kThreads * kLaunchRegs <= 65536, "launch allocation");
};

template <int D>
struct BwdGeo {
  using G = Geo<D>;
  static constexpr int kTileBytes = G::kTileBytes;        // 128 rows x D, TMA-swizzled
  static constexpr int kDsBoxBytes = 128 * 128;           // [128 keys][64 queries] 16-bit, SW128
  static constexpr int kDsBytes = 2 * kDsBoxBytes;
  // dO is single-buffered at D = 128 (its last reader, dV of the step, runs
  // early) to make room for the dQ staging buffer
  // (D >= 112: K, V, 2 x Q, dS and the dQ staging leave room for one dO)
  static constexpr int kDoStages = D >= 112 ? 1 : 2;
  // dQ staging: up to 32 KB of fp32 boxes of [128 rows][kDqBoxCols] a round
  // (32 columns, 128-byte swizzle; 16 columns, 64-byte swizzle when D is an
  // odd multiple of 16); the last round may hold fewer boxes
  static constexpr int kDqBoxCols = D % 32 == 0 ? 32 : 16;
  static constexpr int kDqBoxBytes = 128 * kDqBoxCols * 4;
  static constexpr int kDqTotalBoxes = D / kDqBoxCols;
  static constexpr int kDqBoxes = (32768 / kDqBoxBytes) < kDqTotalBoxes
                                      ? (32768 / kDqBoxBytes) : kDqTotalBoxes;   // per round
  static constexpr int kDqRounds = (kDqTotalBoxes + kDqBoxes - 1) / kDqBoxes;
  static constexpr int kDqSwBytes = kDqBoxCols * 4;       // 128 (SW128) or 64 (SW64)
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;            // two stages
  static constexpr int kOffDo = 4 * kTileBytes;           // kDoStages stages
  static constexpr int kOffDs = kOffDo + kDoStages * kTileBytes;
  static constexpr int kOffDq = kOffDs + kDsBytes;
  static constexpr int kOffVec = kOffDq + kDqBoxes * kDqBoxBytes;   // lse2[128], delta[128]
  static constexpr int kOffBar = kOffVec + 256 * 4;
  static constexpr int kBarBytes = 256;
  static constexpr int kUsed = kOffBar + kBarBytes;
  // at least ~116 KB: one CTA (one 512-column TMEM allocation) per SM
  static constexpr int kSmemBytes = (kUsed + 1024 > 118 * 1024) ? kUsed + 1024 : 118 * 1024;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(256 + 2 * D <= 512, "TMEM budget");
  // dQ accumulator column: its own columns [384, 384 + D) when they are free
  // (D <= 64), else over dP^T (D = 128, after dK has read dS^T)
  static constexpr uint32_t kDqCol = D <= 64 ? 384u : 128u;
  static constexpr bool kDqOwn = D <= 64;
};

struct BwdBars {
  uint64_t kv_full;
  uint64_t q_full[2];     // Q (and, with two dO stages, dO) of a stage
  uint64_t q_empty[2];
  uint64_t do_full;       // single dO stage: dO of the step
  uint64_t do_empty;      // single dO stage: dV (its last reader) done
  uint64_t s_full;
  uint64_t dp_full;
  uint64_t p_full;
  uint64_t ds_full;
  uint64_t dq_full;
  uint64_t dq_free;
  uint64_t s_free;        // early S^T: every P/dS thread holds S^T of the step
  uint64_t p_free;        // early S^T: dV of the step has read P^T
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

// Query blocks [lo, hi) that can see any key of key block kb.
__device__ __forceinline__ void bwd_query_range(int kb, int L_q, int L_k, int wl, int wr,
                                                int &lo, int &hi) {
  const int k0 = kb * kBN;
  const int k1 = min(L_k - 1, k0 + kBN - 1);
  const int i_lo = wr < 0 ? 0 : max(0, k0 - wr);
  const int i_hi = wl < 0 ? L_q - 1 : min(L_q - 1, k1 + wl);
  if (L_q <= 0 || i_hi < i_lo) {
    lo = hi = 0;
  } else {
    lo = i_lo / kBM;
    hi = i_hi / kBM + 1;
  }
}

// Mask element (b, h, i, j) as a log2-domain bias: -inf where hidden.
__device__ __forceinline__ float bwd_mask_bias2(const BwdParams &p, long long idx) {
  constexpr float kLog2e = 1.4426950408889634f;
  if (p.mask_type == 1)
    return static_cast<const uint8_t *>(p.mask)[idx] ? -INFINITY : 0.0f;
  if (p.mask_type == 2)
    return __half2float(__ushort_as_half(static_cast<const uint16_t *>(p.mask)[idx])) * kLog2e;
  return static_cast<const float *>(p.mask)[idx] * kLog2e;
}

template <int D, int DT, bool kMask>
__global__ void __launch_bounds__(BwdCfg<D>::kThreads, 1)
    fa_bwd_kernel(const __grid_constant__ BwdParams p) {
  using G = Geo<D>;
  using BG = BwdGeo<D>;
  using BC = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  BwdBars *bars = reinterpret_cast<BwdBars *>(smem + BG::kOffBar);
  volatile int *abort_flag = &bars->abort_flag;
  float *s_vec = reinterpret_cast<float *>(smem + BG::kOffVec);   // lse2[128] | delta[128]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;

  // ---- work item: (batch, K/V head, key block)
  const int kb = static_cast<int>(blockIdx.x) % p.n_kblocks;
  const int bh_kv = static_cast<int>(blockIdx.x) / p.n_kblocks;
  const int b = bh_kv / p.H_kv;
  const int hk = bh_kv - b * p.H_kv;
  const int k0 = kb * kBN;
  int qb_lo, qb_hi;
  bwd_query_range(kb, p.L_q, p.L_k, p.wl, p.wr, qb_lo, qb_hi);
  const int nqb = qb_hi - qb_lo;
  const int n_steps = nqb * p.group;          // (query head, query block) pairs
  // step n: query head bh_of(n), first query row q0_of(n)
  auto bh_of = [&](int n) { return b * p.H + hk * p.group + n / max(nqb, 1); };
  auto q0_of = [&](int n) { return (qb_lo + n % max(nqb, 1)) * kBM; };

  // ---- setup
  if (tid == 0) {
    mbar_init(smem_u32(&bars->kv_full), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bars->q_full[s]), 1);
      mbar_init(smem_u32(&bars->q_empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->do_full), 1);
    mbar_init(smem_u32(&bars->do_empty), 1);
    mbar_init(smem_u32(&bars->s_full), 1);
    mbar_init(smem_u32(&bars->dp_full), 1);
    mbar_init(smem_u32(&bars->p_full), 128 * BC::kPdsGroups);
    mbar_init(smem_u32(&bars->ds_full), 128 * BC::kPdsGroups);
    mbar_init(smem_u32(&bars->dq_full), 1);
    mbar_init(smem_u32(&bars->dq_free), 128);
    mbar_init(smem_u32(&bars->s_free), 128 * BC::kPdsGroups);
    mbar_init(smem_u32(&bars->p_free), 1);
    mbar_init(smem_u32(&bars->mma_done), 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == 9 && (tid & 31) == 0) {
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(&p.tm_k);
    prefetch_tensormap(&p.tm_v);
    prefetch_tensormap(&p.tm_do);
    prefetch_tensormap(&p.tm_dq);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t sK = smem_u32(smem + BG::kOffK);
  const uint32_t sV = smem_u32(smem + BG::kOffV);
  const uint32_t sQ = smem_u32(smem + BG::kOffQ);
  const uint32_t sDo = smem_u32(smem + BG::kOffDo);
  const uint32_t sDs = smem_u32(smem + BG::kOffDs);

  if (warp >= 8 && warp < 12) {
  // ===================================================== warpgroup 2
  regs_dec<BC::kRegsIssue>();
  if (warp == 9) {
    // =================================================== TMA producer
    const uint64_t pol_keep = policy_evict_last();
    int issued = 0;       // steps whose Q copy was issued
    int do_issued = 0;    // single dO stage: steps whose dO copy was issued
    bool ok = true;
    if (n_steps > 0) {
      const uint32_t bar = smem_u32(&bars->kv_full);
      if (elect_one()) {
        mbar_arrive_expect_tx(bar, 2 * G::kTileBytes);
#pragma unroll
        for (int bx = 0; bx < G::kNumBox; ++bx) {
          tma_load_3d(sK + bx * G::kBoxBytes, &p.tm_k, bar, bx * G::kBoxCols, k0, bh_kv, pol_keep);
          tma_load_3d(sV + bx * G::kBoxBytes, &p.tm_v, bar, bx * G::kBoxCols, k0, bh_kv, pol_keep);
        }
      }
      __syncwarp();
      for (int n = 0; n < n_steps; ++n) {
        const int st = n & 1;
        if (n >= 2) {
          ok = mbar_wait_warp(smem_u32(&bars->q_empty[st]), ((n >> 1) - 1) & 1, abort_flag);
          if (!ok) break;
        }
        const uint32_t qb = smem_u32(&bars->q_full[st]);
        const int q0 = q0_of(n), bh = bh_of(n);
        if (elect_one()) {
          mbar_arrive_expect_tx(qb, (BG::kDoStages == 2 ? 2 : 1) * G::kTileBytes);
#pragma unroll
          for (int bx = 0; bx < G::kNumBox; ++bx) {
            tma_load_3d(sQ + st * G::kTileBytes + bx * G::kBoxBytes, &p.tm_q, qb,
                        bx * G::kBoxCols, q0, bh, pol_keep);
            if constexpr (BG::kDoStages == 2)
              tma_load_3d(sDo + st * G::kTileBytes + bx * G::kBoxBytes, &p.tm_do, qb,
                          bx * G::kBoxCols, q0, bh, pol_keep);
          }
        }
        __syncwarp();
        if constexpr (BG::kDoStages == 1) {
          if (n >= 1) {
            ok = mbar_wait_warp(smem_u32(&bars->do_empty), (n - 1) & 1, abort_flag);
            if (!ok) {
              issued = n + 1;   // Q of step n is in flight, its dO is not
              break;
            }
          }
          const uint32_t db = smem_u32(&bars->do_full);
          if (elect_one()) {
            mbar_arrive_expect_tx(db, G::kTileBytes);
#pragma unroll
            for (int bx = 0; bx < G::kNumBox; ++bx)
              tma_load_3d(sDo + bx * G::kBoxBytes, &p.tm_do, db, bx * G::kBoxCols, q0, bh,
                          pol_keep);
          }
          __syncwarp();
          do_issued = n + 1;
        }
        issued = n + 1;
      }
      if (!ok) {
        // let the copies already issued land before the CTA exits
        mbar_wait_slow(smem_u32(&bars->kv_full), 0, abort_flag, false);
        for (int n = max(0, issued - 2); n < issued; ++n)
          mbar_wait_slow(smem_u32(&bars->q_full[n & 1]), (n >> 1) & 1, abort_flag, false);
        if constexpr (BG::kDoStages == 1) {
          if (do_issued > 0)   // the latest dO copy (phases complete in order)
            mbar_wait_slow(smem_u32(&bars->do_full), (do_issued - 1) & 1, abort_flag, false);
        }
      }
    }
  } else if (warp == 8) {
    // =================================================== MMA issuer
    constexpr uint32_t kIdescS = make_idesc_f16(kBN, kBM, DT, 0, 0);      // M keys, N queries
    constexpr uint32_t kIdescKV = make_idesc_f16(kBN, D, DT, 0, 1);       // dV, dK (A in TMEM)
    constexpr uint32_t kIdescQ = make_idesc_f16(kBM, D, DT, 1, 1);        // dQ (A MN-major)
    constexpr uint32_t kHi = desc_hi(8 * G::kSwBytes, G::kLayout);
    constexpr uint32_t kHiDs = desc_hi(1024, 2u);                         // SW128
    const uint32_t tS = tmem, tDP = tmem + 128u, tDV = tmem + 256u, tDK = tmem + 256u + D;
    const uint32_t tDQ = tmem + BG::kDqCol;
    if (n_steps > 0) {
      bool ok = mbar_wait_warp(smem_u32(&bars->kv_full), 0, abort_flag);
      // X^T = A B^T over D with A, B K-major 128 x D tiles (A: K or V; B: Q or dO)
      auto issue_kmajor = [&](uint32_t d_tmem, uint32_t a_tile, uint32_t b_tile, uint32_t bar) {
        const uint32_t alo = desc_lo(a_tile, 16), blo = desc_lo(b_tile, 16);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int byte = kk * 32;
            const uint32_t off = ((byte / G::kSwBytes) * G::kBoxBytes + (byte % G::kSwBytes)) >> 4;
            mma_ss(d_tmem, desc_join(alo + off, kHi), desc_join(blo + off, kHi), kIdescS,
                   kk > 0 ? 1u : 0u);
          }
          tc_commit(bar);
        }
        __syncwarp();
      };
      // D_acc += X^T(TMEM, 16-bit, the P/dS warpgroups' packed columns) * B
      // (MN-major tile); 16 queries = 8 packed columns, BC::kPdsCols per warpgroup
      // (wg_stride: TMEM columns between two warpgroups' packed values)
      auto issue_ts = [&](uint32_t d_tmem, uint32_t a_base, uint32_t b_tile, bool first,
                          uint32_t wg_stride) {
        const uint32_t blo = desc_lo(b_tile, G::kBoxBytes);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kBM / 16; ++kk) {
            constexpr int kSteps = BC::kPdsCols / 16;    // K steps per warpgroup
            const uint32_t a = a_base + (kk / kSteps) * wg_stride + (kk % kSteps) * 8u;
            mma_ts(d_tmem, a, desc_join(blo + ((kk * 16 * G::kSwBytes) >> 4), kHi), kIdescKV,
                   (!first || kk > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
      };
      auto commit = [&](uint32_t bar) {
        if (elect_one()) tc_commit(bar);
        __syncwarp();
      };
      // dO of step n: its own stage, or the single stage after do_full(n)
      auto do_tile = [&](int n) -> uint32_t {
        return BG::kDoStages == 2 ? sDo + (n & 1) * G::kTileBytes : sDo;
      };
      auto wait_do = [&](int n) -> bool {
        return BG::kDoStages == 2 || mbar_wait_warp(smem_u32(&bars->do_full), n & 1, abort_flag);
      };
      if (ok) ok = mbar_wait_warp(smem_u32(&bars->q_full[0]), 0, abort_flag);
      if (ok) {
        tc_fence_after_sync();
        issue_kmajor(tS, sK, sQ, smem_u32(&bars->s_full));
        ok = wait_do(0);
        if (ok) {
          tc_fence_after_sync();
          issue_kmajor(tDP, sV, do_tile(0), smem_u32(&bars->dp_full));
        }
      }
      for (int n = 0; n < n_steps && ok; ++n) {
        const int st = n & 1;
        if (BC::kEarlyS && n + 1 < n_steps) {
          // S^T(n+1) as soon as every P/dS thread holds S^T(n)
          const int st1 = (n + 1) & 1;
          ok = mbar_wait_warp(smem_u32(&bars->s_free), n & 1, abort_flag) &&
               mbar_wait_warp(smem_u32(&bars->q_full[st1]), ((n + 1) >> 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after_sync();
          issue_kmajor(tS, sK, sQ + st1 * G::kTileBytes, smem_u32(&bars->s_full));
        }
        ok = mbar_wait_warp(smem_u32(&bars->p_full), n & 1, abort_flag);
        if (!ok) break;
        tc_fence_after_sync();
        if constexpr (BC::kEarlyS) {
          issue_ts(tDV, tmem + BC::kPCol, do_tile(n), n == 0, BC::kPdsCols / 2);
          commit(smem_u32(&bars->p_free));
        } else {
          issue_ts(tDV, tS, do_tile(n), n == 0, BC::kPdsCols);
        }
        if constexpr (BG::kDoStages == 1) commit(smem_u32(&bars->do_empty));
        if (!BC::kEarlyS && n + 1 < n_steps) {
          const int st1 = (n + 1) & 1;
          ok = mbar_wait_warp(smem_u32(&bars->q_full[st1]), ((n + 1) >> 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after_sync();
          issue_kmajor(tS, sK, sQ + st1 * G::kTileBytes, smem_u32(&bars->s_full));
        }
        ok = mbar_wait_warp(smem_u32(&bars->ds_full), n & 1, abort_flag);
        if (!ok) break;
        tc_fence_after_sync();
        issue_ts(tDK, tDP, sQ + st * G::kTileBytes, n == 0, BC::kPdsCols);
        if (BG::kDqOwn && n > 0) {
          // dQ has its own columns: only dQ(n) waits for the drain of dQ(n-1)
          ok = mbar_wait_warp(smem_u32(&bars->dq_free), (n - 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after_sync();
        }
        {
          // dQ = dS K: A = dS [128 q][128 keys] MN-major (two 64-query boxes),
          // B = K [128 keys][D] MN-major
          const uint32_t alo = desc_lo(sDs, BG::kDsBoxBytes);
          const uint32_t blo = desc_lo(sK, G::kBoxBytes);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk)
              mma_ss(tDQ, desc_join(alo + ((kk * 16 * 128) >> 4), kHiDs),
                     desc_join(blo + ((kk * 16 * G::kSwBytes) >> 4), kHi), kIdescQ,
                     kk > 0 ? 1u : 0u);
          }
          __syncwarp();
        }
        commit(smem_u32(&bars->dq_full));
        commit(smem_u32(&bars->q_empty[st]));
        if (n + 1 < n_steps) {
          // dP^T(n+1) reuses dQ's columns when dQ has none of its own
          ok = (BG::kDqOwn || mbar_wait_warp(smem_u32(&bars->dq_free), n & 1, abort_flag)) &&
               wait_do(n + 1);
          if (!ok) break;
          tc_fence_after_sync();
          issue_kmajor(tDP, sV, do_tile(n + 1), smem_u32(&bars->dp_full));
        }
      }
    }
    if (elect_one()) tc_commit(smem_u32(&bars->mma_done));
    __syncwarp();
  }
  } else if (warp < 8 || warp >= 16) {
    // =================================================== P and dS
    if constexpr (BC::kRegsPds > BC::kLaunchRegs) regs_inc<BC::kRegsPds>();
    const int wg = warp >> 2;
    const int pw = wg < 2 ? wg : wg - 2;           // query columns [kPdsCols pw, kPdsCols (pw + 1))
    const int r = tid & 127;                       // key row = TMEM lane
    const int tc = pw * 128 + r;                   // slot in the lse2 / delta buffer if < 256
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + BC::kPdsCols * pw;
    const uint32_t tDP = tmem + lane_base + 128u + BC::kPdsCols * pw;
    const int j = k0 + r;                          // key index of this row
    const float sl2 = p.scale_log2;
    bool ok = true;
    // dS on packed fp32 pairs (every layout); P's exponent argument too
    // where the P/dS math sets the step (four warpgroups; with two the
    // scalar form spills less)
    constexpr bool kPacked = BC::kPdsGroups == 4;
    // lse2 / -delta * scale (the dS form below) of the next step, one value
    // per thread of the first two warpgroups
    auto fetch = [&](int n) -> float {
      const size_t base = static_cast<size_t>(bh_of(n)) * p.L_q_pad + q0_of(n) + (tc & 127);
      if (tc < 128) return p.lse2[base];
      return -p.delta[base] * p.scale;
    };
    float nxt = (n_steps > 0 && tc < 256) ? fetch(0) : 0.0f;
    // Every warp of the four warpgroups passes the two named barriers of
    // every step, also after a timeout (then the step's work is skipped).
    for (int n = 0; n < n_steps; ++n) {
      named_barrier_sync(1, 128 * BC::kPdsGroups);  // the buffer of step n-1 is no longer read
      if (tc < 256) s_vec[tc] = nxt;
      named_barrier_sync(1, 128 * BC::kPdsGroups);
      if (n + 1 < n_steps && tc < 256) nxt = fetch(n + 1);
      if (!ok) continue;
      const int q0 = q0_of(n);
      const int qc = q0 + BC::kPdsCols * pw;        // first query column of this thread
      const bool full = (k0 + kBN - 1 < p.L_k) && (p.wr < 0 || k0 + kBN - 1 <= q0 + p.wr) &&
                        (p.wl < 0 || k0 >= q0 + kBM - 1 - p.wl);
      const float *lse2 = s_vec + BC::kPdsCols * pw;
      const float *dlt = s_vec + 128 + BC::kPdsCols * pw;

      // ---- P^T = 2^(s * scale * log2e - lse2), masked entries 0
      ok = mbar_wait_warp(smem_u32(&bars->s_full), n & 1, abort_flag);
      if (!ok) continue;
      tc_fence_after_sync();
      float pr[BC::kPdsCols];
#pragma unroll
      for (int h = 0; h < BC::kPdsCols / 32; ++h) {   // 32-column chunks
        uint32_t sr[32];
        tmem_ld_x32(tS + 32 * h, sr);
        tmem_wait_ld();
        reg_dep(sr);
        if constexpr (BC::kEarlyS) {
          // S^T(n) is in registers (one chunk): S^T(n+1) may overwrite it
          static_assert(!BC::kEarlyS || BC::kPdsCols == 32, "one S chunk per thread");
          tc_fence_before_sync();
          mbar_arrive(smem_u32(&bars->s_free));
        }
        if constexpr (kMask) {
          // this row's mask entries for the 32 query columns (one key per
          // lane: each load is 32 consecutive elements across the warp)
          const int bh = bh_of(n);
          const long long mrow = static_cast<long long>(bh / p.H) * p.mask_sb +
                                 static_cast<long long>(bh % p.H) * p.mask_sh + j;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int i = qc + 32 * h + c;
            const float bias = (i < p.L_q && j < p.L_k)
                                   ? bwd_mask_bias2(p, mrow + static_cast<long long>(i) * p.mask_sq)
                                   : 0.0f;
            pr[32 * h + c] = ex2(fmaf(__uint_as_float(sr[c]), sl2, bias - lse2[32 * h + c]));
          }
        } else if constexpr (kPacked) {
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float2 x = __ffma2_rn(
                make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])),
                make_float2(sl2, sl2), make_float2(-lse2[32 * h + c], -lse2[32 * h + c + 1]));
            pr[32 * h + c] = ex2(x.x);
            pr[32 * h + c + 1] = ex2(x.y);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            pr[32 * h + c] = ex2(fmaf(__uint_as_float(sr[c]), sl2, -lse2[32 * h + c]));
        }
      }
      if (!full) {
#pragma unroll
        for (int c = 0; c < BC::kPdsCols; ++c) {
          const int i = qc + c;
          const bool vis = (j < p.L_k) && (p.wr < 0 || j <= i + p.wr) && (p.wl < 0 || j >= i - p.wl);
          if (!vis) pr[c] = 0.0f;
        }
      }
      if (BC::kEarlyS && n > 0) {
        // dV(n-1) has read P^T(n-1) from the columns this store reuses
        ok = mbar_wait_warp(smem_u32(&bars->p_free), (n - 1) & 1, abort_flag);
        if (!ok) continue;
      }
      {
        uint32_t pk[BC::kPdsCols / 2];
#pragma unroll
        for (int u = 0; u < BC::kPdsCols / 2; ++u) pk[u] = pack2<DT>(pr[2 * u], pr[2 * u + 1]);
        // early S^T: P^T's own columns; else over S^T columns already read
        tmem_st_cols<BC::kPdsCols / 2>(
            BC::kEarlyS ? tmem + lane_base + BC::kPCol + (BC::kPdsCols / 2) * pw : tS, pk);
        tmem_wait_st();
      }
      tc_fence_before_sync();
      mbar_arrive(smem_u32(&bars->p_full));

      // ---- dS = P o (dP - delta) * scale, to TMEM (for dK) and shared memory (for dQ)
      ok = mbar_wait_warp(smem_u32(&bars->dp_full), n & 1, abort_flag);
      if (!ok) continue;
      tc_fence_after_sync();
      if (n > 0) {
        // the dQ MMA of the previous step has read the dS staging buffer
        ok = mbar_wait_warp(smem_u32(&bars->dq_full), (n - 1) & 1, abort_flag);
        if (!ok) continue;
      }
      // this thread's queries in the box of 64 that holds them: its row of
      // 128 bytes, from 16-byte unit u0 on; chunks of kCh columns
      constexpr int kCh = BC::kPdsCols >= 64 ? 32 : 16;
      const int q_first = BC::kPdsCols * pw;
      uint8_t *ds_row = smem + BG::kOffDs + (q_first >> 6) * BG::kDsBoxBytes + r * 128;
      const int u0 = (q_first & 63) >> 3;
#pragma unroll
      for (int h = 0; h < BC::kPdsCols / kCh; ++h) {
        uint32_t dp[kCh];
        tmem_ld_cols<kCh>(tDP + kCh * h, dp);
        tmem_wait_ld();
        reg_dep(dp);
        uint32_t pk[kCh / 2];
#pragma unroll
        for (int u = 0; u < kCh / 2; ++u) {
          const int c = kCh * h + 2 * u;
          // P * (dP * scale + (-delta * scale))
          const float2 g = __ffma2_rn(
              make_float2(__uint_as_float(dp[2 * u]), __uint_as_float(dp[2 * u + 1])),
              make_float2(p.scale, p.scale), make_float2(dlt[c], dlt[c + 1]));
          const float2 dd = __fmul2_rn(make_float2(pr[c], pr[c + 1]), g);
          pk[u] = pack2<DT>(dd.x, dd.y);
        }
        tmem_st_cols<kCh / 2>(tDP + (kCh / 2) * h, pk);   // over dP^T columns already read
#pragma unroll
        for (int u = 0; u < kCh / 8; ++u) {
          const int unit = u0 + (kCh / 8) * h + u;     // 16-byte unit of the 128-byte row
          *reinterpret_cast<uint4 *>(ds_row + ((unit ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before_sync();
      mbar_arrive(smem_u32(&bars->ds_full));
    }

    // ---- epilogue (row j of this block): P/dS warpgroups 0 (and 2) write
    // dV, 1 (and 3) dK; with four, each the 32-column chunks of one parity
    if (ok && n_steps > 0) {
      ok = mbar_wait_warp(smem_u32(&bars->mma_done), 0, abort_flag);
      if (ok) tc_fence_after_sync();
    }
    if (ok) {
      const int acc = pw & 1;                      // 0: dV, 1: dK
      const uint32_t tAcc = tmem + lane_base + 256u + (acc ? D : 0);
      uint8_t *dst = static_cast<uint8_t *>(acc ? p.dk : p.dv) +
                     (static_cast<size_t>(bh_kv) * p.L_k + j) * D * 2;
      for_o_chunks<D>([&](int c, auto wd) {   // 32-column chunks, 16-column tail
        constexpr int W = decltype(wd)::value;
        if (((c >> 5) % (BC::kPdsGroups / 2)) != (pw >> 1)) return;
        uint32_t o[W];
        if (n_steps > 0) {
          tmem_ld_cols<W>(tAcc + c, o);
          tmem_wait_ld();
          reg_dep(o);
        } else {
#pragma unroll
          for (int u = 0; u < W; ++u) o[u] = 0u;
        }
        if (j < p.L_k) {
#pragma unroll
          for (int u = 0; u < W / 8; ++u)
            *reinterpret_cast<uint4 *>(dst + (c + 8 * u) * 2) = make_uint4(
                pack2<DT>(__uint_as_float(o[8 * u]), __uint_as_float(o[8 * u + 1])),
                pack2<DT>(__uint_as_float(o[8 * u + 2]), __uint_as_float(o[8 * u + 3])),
                pack2<DT>(__uint_as_float(o[8 * u + 4]), __uint_as_float(o[8 * u + 5])),
                pack2<DT>(__uint_as_float(o[8 * u + 6]), __uint_as_float(o[8 * u + 7])));
        }
      });
    }
  } else {
    // =================================================== dQ drain (warps 12-15)
    regs_inc<BC::kRegsDrain>();
    const int r = tid & 127;                       // query row within the block = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tDQ = tmem + lane_base + BG::kDqCol;
    uint8_t *stage = smem + BG::kOffDq;
    const bool leader = tid == 384;                // issues the bulk reductions
    constexpr int kUnits = BG::kDqSwBytes / 16;    // 16-byte units per staged row
    const int sw = ((r * BG::kDqSwBytes) >> 7) & (kUnits - 1);
    bool ok = true;
    // Every drain warp passes the same named barriers, also after a timeout.
    for (int n = 0; n < n_steps; ++n) {
      if (ok) ok = mbar_wait_warp(smem_u32(&bars->dq_full), n & 1, abort_flag);
      if (ok) tc_fence_after_sync();
      const int q0 = q0_of(n), bh = bh_of(n);
      // round by round (loading all of a D = 128 row first measured 6 %
      // slower); the columns are free after the last round's loads
#pragma unroll
      for (int rd = 0; rd < BG::kDqRounds; ++rd) {
        uint32_t v[BG::kDqBoxes][BG::kDqBoxCols];
        // boxes of this round (the last round may have fewer)
        constexpr int kLast = BG::kDqTotalBoxes - (BG::kDqRounds - 1) * BG::kDqBoxes;
        const int nbox = rd == BG::kDqRounds - 1 ? kLast : BG::kDqBoxes;
        if (ok) {
#pragma unroll
          for (int bx = 0; bx < BG::kDqBoxes; ++bx)
            if (bx < nbox)
              tmem_ld_cols<BG::kDqBoxCols>(
                  tDQ + (rd * BG::kDqBoxes + bx) * BG::kDqBoxCols, v[bx]);
          tmem_wait_ld();
#pragma unroll
          for (int bx = 0; bx < BG::kDqBoxes; ++bx) reg_dep(v[bx]);
          if (rd == BG::kDqRounds - 1) {
            tc_fence_before_sync();
            mbar_arrive(smem_u32(&bars->dq_free));
          }
        }
        if (leader) bulk_wait_group_read_all();    // the staging buffer has been read
        named_barrier_sync(2, 128);
        if (ok) {
#pragma unroll
          for (int bx = 0; bx < BG::kDqBoxes; ++bx)
            if (bx < nbox)
#pragma unroll
              for (int u = 0; u < kUnits; ++u)
                *reinterpret_cast<uint4 *>(stage + bx * BG::kDqBoxBytes + r * BG::kDqSwBytes +
                                           ((u ^ sw) << 4)) =
                    make_uint4(v[bx][4 * u], v[bx][4 * u + 1], v[bx][4 * u + 2],
                               v[bx][4 * u + 3]);
        }
        fence_proxy_async_smem();
        named_barrier_sync(2, 128);
        if (leader && ok) {
#pragma unroll
          for (int bx = 0; bx < BG::kDqBoxes; ++bx)
            if (bx < nbox)
              tma_reduce_add_3d(&p.tm_dq, smem_u32(stage + bx * BG::kDqBoxBytes),
                                (rd * BG::kDqBoxes + bx) * BG::kDqBoxCols, q0, bh);
          bulk_commit_group();
        }
      }
    }
    if (leader) bulk_wait_group_all();             // the reductions have landed
  }

  // ---- teardown
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after_sync();
    mbar_wait_slow(smem_u32(&bars->mma_done), 0, abort_flag, false);
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

// delta_i = dO_i . O_i (fp32), lse2_i = lse_i * log2(e) (+inf where lse is
// -inf or i >= L_q), and dQ_acc zeroed: one warp per padded query row.
template <int D, int DT>
__global__ void __launch_bounds__(256) fa_bwd_prep_kernel(const void *out, const void *dout,
                                                          const float *lse, float *lse2,
                                                          float *delta, float *dq_acc, int L_q,
                                                          int L_q_pad, long long rows_pad) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows_pad) return;
  const long long bh = row / L_q_pad;
  const int i = static_cast<int>(row - bh * L_q_pad);
  float dsum = 0.0f;
  if (i < L_q) {
    // 16-byte loads of O and dO (8 elements a lane), 16-byte zero stores of
    // the fp32 dQ accumulator (4 a lane)
    const size_t base = (static_cast<size_t>(bh) * L_q + i) * D;
    for (int u = lane; u < D / 8; u += 32) {
      const uint4 ow = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(out) + base)[u];
      const uint4 gw = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(dout) + base)[u];
      const uint32_t os[4] = {ow.x, ow.y, ow.z, ow.w}, gs[4] = {gw.x, gw.y, gw.z, gw.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float2 o, g;
        if constexpr (DT == 0) {
          o = __half22float2(*reinterpret_cast<const __half2 *>(&os[k]));
          g = __half22float2(*reinterpret_cast<const __half2 *>(&gs[k]));
        } else {
          o = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&os[k]));
          g = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&gs[k]));
        }
        dsum = fmaf(o.x, g.x, fmaf(o.y, g.y, dsum));
      }
    }
    for (int u = lane; u < D / 4; u += 32)
      reinterpret_cast<float4 *>(dq_acc + base)[u] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
  if (lane == 0) {
    delta[row] = dsum;
    float l2 = INFINITY;
    if (i < L_q) {
      const float l = lse[static_cast<size_t>(bh) * L_q + i];
      if (l != -INFINITY) l2 = l * 1.4426950408889634f;
    }
    lse2[row] = l2;
  }
}

// dQ = dQ_acc rounded to the element type (the scale is already in dS).
template <int DT>
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const float *dq_acc, void *dq,
                                                        size_t n) {
  // n is a multiple of 16 (rows of D elements, D a multiple of 16): 16-byte
  // loads, 8-byte stores
  size_t i = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x * 4;
  for (; i < n; i += stride) {
    const float4 v = *reinterpret_cast<const float4 *>(dq_acc + i);
    reinterpret_cast<uint2 *>(dq)[i / 4] = make_uint2(pack2<DT>(v.x, v.y), pack2<DT>(v.z, v.w));
  }
}

}  // namespace fa
