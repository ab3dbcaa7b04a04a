// pba_bwd_sm100.cuh -- backward of pair-biased attention on sm_100a.
//
// Training is distributed too ("Fold-CP: A Context Parallelism Framework for
// Biomolecular Modeling", Figure 3 right, training scaling).  For one (b, h),
// with s_ij = tau q_i.k_j + b_ij over valid keys, lse_i from the forward pass
// and P_ij = exp(s_ij - lse_i) (0 for masked keys):
//     Delta_i = sum_d dO_id O_id                        (pba_bwd_delta_kernel)
//     dP_ij   = dO_i . v_j
//     dS_ij   = P_ij (dP_ij - Delta_i) = dL/db_ij       (dbias, bf16)
//     dq_i    = tau sum_j dS_ij k_j                      (kernel A, fp32)
//     dk_j    = tau sum_i dS_ij q_i,  dv_j = sum_i P_ij dO_i   (kernel B, fp32)
//
// Kernel A walks the key tiles of one 128-row query tile: S = Q K^T and
// dP = dO V^T on the tensor cores (fp32 in Tensor Memory), P and dS on the
// CUDA cores, dS to HBM as dbias and to Tensor Memory as bf16, then
// dQ += dS K (A = dS from Tensor Memory, B = the K tile read MN-major).
// Kernel B walks the query tiles of one 128-row key tile: S^T = K Q^T and
// dP^T = V dO^T, then dV += P^T dO and dK += dS^T Q with P^T and dS^T from
// Tensor Memory and dO, Q read MN-major.  Both recompute P from the saved
// log-sum-exp, so no N^2 intermediate is stored besides dbias.
//
// One CTA per unit, 384 threads: warps 0-7 two compute warpgroups (row =
// thread = Tensor Memory lane; warpgroup g takes columns 64g .. 64g+63 of
// every step), warp 8 the TMA producer of the operand tiles, warp 9 Tensor
// Memory and the MMAs, warp 10 the TMA producer of the bias tiles, warp 11
// idle.  Per step the chain is S, dP -> P, dS -> dQ or dV, dK; the next
// step's S, dP are issued as soon as both warpgroups have read this step's.
// Operand tiles are double-buffered; the bias tiles, streamed from HBM and
// held until the step's compute (and, in A, its dbias store) is done with
// them, run in their own ring of three.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "pba_ptx.cuh"

namespace pba {

constexpr int kBwdTile = 128;
constexpr int kBwdComputeGroups = 2;  // column halves of a step, one warpgroup each
constexpr int kBwdThreads = 128 * (kBwdComputeGroups + 1);
constexpr int kBwdWarpProducer = 4 * kBwdComputeGroups;
constexpr int kBwdWarpMma = kBwdWarpProducer + 1;
constexpr int kBwdWarpBiasProducer = kBwdWarpProducer + 2;
// Per-thread register limits after the warpgroup reallocation: the launch
// gives 168 (384 x 168 = 64512); the producer/MMA warpgroup keeps 56 and the
// compute warpgroups take 224 (128 x 56 + 256 x 224 = 64512).
constexpr int kBwdRegsCompute = 224;
constexpr int kBwdRegsOther = 56;
constexpr int kBwdRegSplitTotal = 128 * kBwdComputeGroups * kBwdRegsCompute + 128 * kBwdRegsOther;

struct BwdParams {
  // A: tm_q/tm_do are the query-side tiles, tm_k/tm_v the key-side tiles;
  // all 4-D (D, n, H, B) bf16 with box {D, 128, 1, 1}.  tm_bias: (Nk, Nq, H, B)
  // bf16, kernel A box {64, 128} 128-byte swizzle, kernel B box {128, 128}
  // no swizzle.
  CUtensorMap tm_q, tm_k, tm_v, tm_do, tm_bias;
  // A: dbias (Nk, Nq, H, B) bf16, box {64, 32} 128-byte swizzle: one warp's
  // 32 rows of a 64-key half of a step, stored from the step's bias slot
  CUtensorMap tm_dbias;
  int32_t B, H, Nq, Nk;
  int32_t n_tiles;      // A: ceil(Nq/128), B: ceil(Nk/128) per (b, h)
  int32_t bias_h_bcast, bias_b_bcast;  // bias head / batch stride 0 (map extent 1)
  float tau;
  const uint8_t *mask;  // [B][Nk] or null
  int64_t mask_sb;
  const float *lse, *delta;  // [B][H][Nq]
  int64_t row_sb, row_sh;    // strides of lse / delta (elements); row stride 1
  uint16_t *dbias;           // [B][H][Nq][Nk] bf16 (contiguous rows of Nk)
  int64_t db_sb, db_sh, db_sn;
  float *dq, *dk, *dv;       // fp32 [B][H][n][D] contiguous
  int *err;
  uint64_t timeout_ns;
};

template <int D>
struct BwdLayout {
  static_assert(D == 32 || D == 64, "head dimension");
  static constexpr int kRowBytes = D * 2;
  static constexpr int kSwizzleMode = (D == 64) ? 2 : 4;
  static constexpr int kAtomBytes = 8 * kRowBytes;
  static constexpr int kTileBytes = kBwdTile * kRowBytes;  // one [128][D] bf16 tile
  static constexpr int kBiasBytes = kBwdTile * kBwdTile * 2;
  static constexpr int kStages = 2;      // operand tiles (A: K, V; B: Q, dO)
  // bias tiles: a third stage gives each HBM load a step more of lead
  // (ring8k shapes: 2.20 -> 2.02 ms per backward call)
  static constexpr int kBiasStages = 3;
  // fixed operands of the unit (A: Q, dO; B: K, V), then per-step operands
  // (A: K, V; B: Q, dO), double-buffered, and the bias tiles in a ring of
  // three
  static constexpr int kOffFix0 = 0;
  static constexpr int kOffFix1 = kOffFix0 + kTileBytes;
  static constexpr int kOffStep0 = kOffFix1 + kTileBytes;                   // [stage]
  static constexpr int kOffStep1 = kOffStep0 + kStages * kTileBytes;        // [stage]
  static constexpr int kOffBias = kOffStep1 + kStages * kTileBytes;         // [bias stage]
  // per-step column data, one copy per compute warp (so that a warp needs no
  // barrier with the others of its warpgroup), double-buffered by step
  // parity: A: 32 keep words; B: -lse log2(e) and -Delta of 64 query columns
  static constexpr int kRowvWarpFloats = kBwdTile;
  static constexpr int kOffRowv = kOffBias + kBiasStages * kBiasBytes;
  static constexpr int kOffBar = kOffRowv + 2 * (4 * kBwdComputeGroups) * kRowvWarpFloats * 4;
  static constexpr int kBarFixFull = 0;
  static constexpr int kBarStepFull = 1;                       // [stage]
  static constexpr int kBarStepEmpty = kBarStepFull + kStages;  // [stage]
  static constexpr int kBarBiasFull = kBarStepEmpty + kStages;       // [bias stage]
  static constexpr int kBarBiasEmpty = kBarBiasFull + kBiasStages;   // [bias stage]
  static constexpr int kBarSFull = kBarBiasEmpty + kBiasStages;
  static constexpr int kBarSFree = kBarSFull + 1;
  static constexpr int kBarGFull = kBarSFree + 1;  // P / dS written to Tensor Memory
  static constexpr int kBarGDone = kBarGFull + 1;  // the accumulating MMAs of a step are done
  static constexpr int kBarDrain = kBarGDone + 1;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemSlot + 4;
  static constexpr int kBytes = kOffAbort + 4;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  // Tensor Memory columns
  static constexpr uint32_t kColS = 0, kColDP = 128, kColG0 = 256, kColG1 = 320, kColAcc0 = 384,
                            kColAcc1 = 384 + D;
  static_assert(kColAcc1 + D <= 512, "Tensor Memory budget");
};

// kB = false: kernel A (dq, dbias); kB = true: kernel B (dk, dv).
template <int D, bool kB>
__global__ void __launch_bounds__(kBwdThreads, 1) pba_bwd_sm100_kernel(const __grid_constant__ BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffTmemSlot);
  int *abort_flag = reinterpret_cast<int *>(smem + L::kOffAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // unit: (b, h, tile of 128 rows); steps: the tiles of the other side
  const int unit = blockIdx.x;
  const int tile = unit % p.n_tiles;
  const int bh = unit / p.n_tiles;
  const int h = bh % p.H, b = bh / p.H;
  const int row0 = tile * kBwdTile;
  const int n_other = kB ? p.Nq : p.Nk;
  const int nsteps = (n_other + kBwdTile - 1) / kBwdTile;

  if (threadIdx.x == 0) {
    mbar_init(&bars[L::kBarFixFull], 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&bars[L::kBarStepFull + s], 1);
      mbar_init(&bars[L::kBarStepEmpty + s], 1);  // the MMA commit after the step's last MMAs
    }
    for (int s = 0; s < L::kBiasStages; ++s) {
      mbar_init(&bars[L::kBarBiasFull + s], 1);
      // each compute warp (A: once its dbias store has read the slot)
      mbar_init(&bars[L::kBarBiasEmpty + s], 4 * kBwdComputeGroups);
    }
    mbar_init(&bars[L::kBarSFull], 1);
    mbar_init(&bars[L::kBarSFree], kBwdComputeGroups * kBwdTile);
    mbar_init(&bars[L::kBarGFull], kBwdComputeGroups * kBwdTile);
    mbar_init(&bars[L::kBarGDone], 1);
    mbar_init(&bars[L::kBarDrain], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kBwdWarpMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, p.err, p.timeout_ns};
  WaitCtl wc_drain = wc;
  int drain_abort = 0;
  wc_drain.abort_flag = &drain_abort;

  if (warp >= kBwdWarpProducer) {
    setmaxnreg_dec<kBwdRegsOther>();
    if (warp == kBwdWarpProducer) {
      // ================================================================ TMA producer
      if (lane == 0) {
        const uint64_t pol = l2_policy_evict_last();
        // fixed tiles of the unit: A: Q, dO rows; B: K, V rows
        mbar_arrive_expect_tx(&bars[L::kBarFixFull], 2 * L::kTileBytes);
        tma_load_4d(smem + L::kOffFix0, kB ? &p.tm_k : &p.tm_q, &bars[L::kBarFixFull], 0, row0, h, b, pol);
        tma_load_4d(smem + L::kOffFix1, kB ? &p.tm_v : &p.tm_do, &bars[L::kBarFixFull], 0, row0, h, b, pol);
        bool ok = true;
        int it = 0;
        for (; it < nsteps && ok; ++it) {
          const int s = it % L::kStages;
          if (it >= L::kStages) ok = mbar_wait(&bars[L::kBarStepEmpty + s], ((it / L::kStages) - 1) & 1, wc);
          if (!ok) break;
          const int o0 = it * kBwdTile;
          uint64_t *full = &bars[L::kBarStepFull + s];
          mbar_arrive_expect_tx(full, 2 * L::kTileBytes);
          tma_load_4d(smem + L::kOffStep0 + s * L::kTileBytes, kB ? &p.tm_q : &p.tm_k, full, 0, o0, h, b, pol);
          tma_load_4d(smem + L::kOffStep1 + s * L::kTileBytes, kB ? &p.tm_do : &p.tm_v, full, 0, o0, h, b, pol);
        }
        mbar_wait(&bars[L::kBarFixFull], 0, wc_drain);
        if (!ok)
          for (int s = 0; s < L::kStages; ++s) {
            const int a = (it - s + L::kStages - 1) / L::kStages;
            if (a > 0) mbar_wait(&bars[L::kBarStepFull + s], (a - 1) & 1, wc_drain);
          }
      }
    } else if (warp == kBwdWarpBiasProducer) {
      // ================================================================ bias tiles
      if (lane == 0) {
        const uint64_t pol = l2_policy_evict_last();
        const int hb = p.bias_h_bcast ? 0 : h, bb = p.bias_b_bcast ? 0 : b;
        bool ok = true;
        int it = 0;
        for (; it < nsteps && ok; ++it) {
          const int s = it % L::kBiasStages;
          if (it >= L::kBiasStages)
            ok = mbar_wait(&bars[L::kBarBiasEmpty + s], ((it / L::kBiasStages) - 1) & 1, wc);
          if (!ok) break;
          const int o0 = it * kBwdTile;
          uint64_t *full = &bars[L::kBarBiasFull + s];
          uint8_t *bdst = smem + L::kOffBias + s * L::kBiasBytes;
          mbar_arrive_expect_tx(full, L::kBiasBytes);
          if (kB) {
            // [128 queries][128 keys], no swizzle: the thread of key j reads column j
            tma_load_4d(bdst, &p.tm_bias, full, row0, o0, hb, bb, pol);
          } else {
            // [128 queries][128 keys] as two 64-key boxes, 128-byte swizzle
            tma_load_4d(bdst, &p.tm_bias, full, o0, row0, hb, bb, pol);
            tma_load_4d(bdst + L::kBiasBytes / 2, &p.tm_bias, full, o0 + 64, row0, hb, bb, pol);
          }
        }
        if (!ok)
          for (int s = 0; s < L::kBiasStages; ++s) {
            const int a = (it - s + L::kBiasStages - 1) / L::kBiasStages;
            if (a > 0) mbar_wait(&bars[L::kBarBiasFull + s], (a - 1) & 1, wc_drain);
          }
      }
    } else if (warp == kBwdWarpMma) {
      // ================================================================ MMA issuer
      if (lane == 0) {
        const uint32_t idesc_s = idesc_bf16_f32(kBwdTile, kBwdTile, false);  // both operands K-major
        const uint32_t idesc_g = idesc_bf16_f32(kBwdTile, D, true);          // B MN-major
        constexpr uint32_t kHi = smem_desc_hi(L::kAtomBytes, L::kSwizzleMode);
        const uint32_t sF0 = smem_u32(smem + L::kOffFix0), sF1 = smem_u32(smem + L::kOffFix1);
        // S, dP of step `it` (A: S = Q K^T, dP = dO V^T; B: S^T = K Q^T,
        // dP^T = V dO^T) once its tiles have landed and the compute warpgroup has
        // read the previous step's S and dP
        auto issue_s = [&](int it) -> bool {
          const int s = it % L::kStages;
          if (!mbar_wait(&bars[L::kBarStepFull + s], (it / L::kStages) & 1, wc)) return false;
          if (it > 0 && !mbar_wait(&bars[L::kBarSFree], (it - 1) & 1, wc)) return false;
          tc_fence_after_sync();
          const uint32_t sS0 = smem_u32(smem + L::kOffStep0 + s * L::kTileBytes);
          const uint32_t sS1 = smem_u32(smem + L::kOffStep1 + s * L::kTileBytes);
          const uint32_t a0 = smem_desc_lo(sF0, 16), b0 = smem_desc_lo(sS0, 16);
          const uint32_t a1 = smem_desc_lo(sF1, 16), b1 = smem_desc_lo(sS1, 16);
  #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(tmem + L::kColS, desc_join(a0 + kk * 2, kHi), desc_join(b0 + kk * 2, kHi), idesc_s, kk > 0);
  #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(tmem + L::kColDP, desc_join(a1 + kk * 2, kHi), desc_join(b1 + kk * 2, kHi), idesc_s, kk > 0);
          tc_commit(&bars[L::kBarSFull]);
          return true;
        };
        // Software-pipelined: S, dP of step it+1 go out as soon as step it's
        // S, dP have been read, before the accumulating products of step it.
        bool ok = mbar_wait(&bars[L::kBarFixFull], 0, wc);
        if (ok) ok = issue_s(0);
        for (int it = 0; it < nsteps && ok; ++it) {
          const int s = it % L::kStages;
          if (it + 1 < nsteps && !(ok = issue_s(it + 1))) break;
          // the accumulating products once P / dS are in Tensor Memory
          ok = mbar_wait(&bars[L::kBarGFull], it & 1, wc);
          if (!ok) break;
          tc_fence_after_sync();
          const uint32_t sS0 = smem_u32(smem + L::kOffStep0 + s * L::kTileBytes);
          const uint32_t sS1 = smem_u32(smem + L::kOffStep1 + s * L::kTileBytes);
          const uint32_t acc = (it > 0) ? 1u : 0u;
          if (!kB) {
            // dQ += dS K: B = the K tile, keys are the reduction (MN-major read)
            const uint32_t kb = smem_desc_lo(sS0, L::kTileBytes);
  #pragma unroll
            for (int kk = 0; kk < kBwdTile / 16; ++kk)
              mma_bf16_ts(tmem + L::kColAcc0, tmem + L::kColG0 + kk * 8,
                          desc_join(kb + kk * (16 * L::kRowBytes / 16), kHi), idesc_g, (acc || kk > 0) ? 1u : 0u);
          } else {
            // dV += P^T dO and dK += dS^T Q: queries are the reduction
            const uint32_t qb = smem_desc_lo(sS0, L::kTileBytes), ob = smem_desc_lo(sS1, L::kTileBytes);
  #pragma unroll
            for (int kk = 0; kk < kBwdTile / 16; ++kk)
              mma_bf16_ts(tmem + L::kColAcc1, tmem + L::kColG0 + kk * 8,
                          desc_join(ob + kk * (16 * L::kRowBytes / 16), kHi), idesc_g, (acc || kk > 0) ? 1u : 0u);
  #pragma unroll
            for (int kk = 0; kk < kBwdTile / 16; ++kk)
              mma_bf16_ts(tmem + L::kColAcc0, tmem + L::kColG1 + kk * 8,
                          desc_join(qb + kk * (16 * L::kRowBytes / 16), kHi), idesc_g, (acc || kk > 0) ? 1u : 0u);
          }
          tc_commit(&bars[L::kBarGDone]);
          tc_commit(&bars[L::kBarStepEmpty + s]);
        }
        tc_commit(&bars[L::kBarDrain]);
        mbar_wait(&bars[L::kBarDrain], 0, wc_drain);
      }
    }
  } else {
    // ================================================================ compute warpgroups
    setmaxnreg_inc<kBwdRegsCompute>();
    const int g = warp >> 2;           // column half of each step
    const int t = threadIdx.x & 127;   // row of the unit's tile = Tensor Memory lane
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const int r = row0 + t;     // A: query row; B: key row
    const float l2e = 1.4426950408889634f;
    const float c_s = p.tau * l2e;
    const uint8_t *mrow = p.mask ? p.mask + int64_t(b) * p.mask_sb : nullptr;
    // A: this row's lse and Delta; B: this key's mask flag
    float lse2 = 0.f, delta = 0.f;
    bool key_ok = true;
    if (!kB) {
      if (r < p.Nq) {
        const int64_t at = int64_t(b) * p.row_sb + int64_t(h) * p.row_sh + r;
        // a row with no valid key (lse = -inf) has -inf exponents for every
        // key already; a finite stand-in keeps -lse from forming inf - inf
        const float lse = p.lse[at];
        lse2 = (lse == -INFINITY) ? 0.f : lse * l2e;
        delta = p.delta[at];
      }
    } else {
      key_ok = r < p.Nk && (mrow == nullptr || mrow[r] != 0);
    }
    // Column data of a step, loaded from global memory one step ahead so
    // that the loads' latency overlaps a step of work; every warp loads the
    // data of its warpgroup's columns for itself.  A: the mask bytes of key
    // pair `lane`; B: lse and Delta of query columns `lane` and `lane + 32`.
    uint32_t nm0 = 1u, nm1 = 1u;
    float nlse[2] = {0.f, 0.f}, ndelta[2] = {0.f, 0.f};
    auto load_cols = [&](int step) {
      const int o = step * kBwdTile;
      if (!kB) {
        if (mrow != nullptr) {
          const int key = o + 2 * (g * (kBwdTile / 4) + lane);
          nm0 = key < p.Nk ? uint32_t(mrow[key]) : 0u;
          nm1 = key + 1 < p.Nk ? uint32_t(mrow[key + 1]) : 0u;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int qi = o + g * (kBwdTile / 2) + lane + 32 * e;
          if (qi < p.Nq) {
            const int64_t at = int64_t(b) * p.row_sb + int64_t(h) * p.row_sh + qi;
            nlse[e] = p.lse[at];
            ndelta[e] = p.delta[at];
          }
        }
      }
    };
    if (nsteps > 0) load_cols(0);
    bool ok = true;
    uint32_t bias_off = 0, bias_ph = 0;  // the step's bias slot (bytes) and its phase
    for (int it = 0; it < nsteps && ok; ++it) {
      const int o0 = it * kBwdTile;
      const uint32_t cm0 = nm0, cm1 = nm1;
      const float clse[2] = {nlse[0], nlse[1]}, cdelta[2] = {ndelta[0], ndelta[1]};
      if (it + 1 < nsteps) load_cols(it + 1);
      // S, dP and the step's bias tile.  The waits only set ok; the warp
      // leaves together at the vote below.
      const int bs = bias_off / L::kBiasBytes;
      ok = mbar_wait<false>(&bars[L::kBarSFull], it & 1, wc);
      if (ok) ok = mbar_wait<false>(&bars[L::kBarBiasFull + bs], bias_ph, wc);
      const uint8_t *bt = smem + L::kOffBias + bias_off;
      // Per-step column data in this warp's own shared-memory copy
      // (double-buffered by step parity), written and read by the warp alone.
      // A: one keep word per key pair of the warpgroup's 64 columns (0xFFFF
      // per kept half: masked keys and keys past Nk turn into bf16 -inf in
      // the bias).  B: -lse*log2(e) at [0, 64) and -Delta at [64, 128) for
      // the warpgroup's query columns (columns past Nq get -lse = -inf, so
      // P = 0 there).
      float *rv = reinterpret_cast<float *>(smem + L::kOffRowv) +
                  ((it & 1) * (4 * kBwdComputeGroups) + warp) * L::kRowvWarpFloats;
      if (!kB) {
        const int key = o0 + 2 * (g * (kBwdTile / 4) + lane);  // key pair `lane` of the warpgroup
        const uint32_t keep = ((key < p.Nk && cm0 != 0u) ? 0x0000FFFFu : 0u) |
                              ((key + 1 < p.Nk && cm1 != 0u) ? 0xFFFF0000u : 0u);
        reinterpret_cast<uint32_t *>(rv)[lane] = keep;
      } else {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int col = lane + 32 * e;  // query column of the warpgroup's half
          const int qi = o0 + g * (kBwdTile / 2) + col;
          rv[col] = qi >= p.Nq ? -INFINITY : (clse[e] == -INFINITY ? 0.f : -clse[e] * l2e);  // see the A side
          rv[kBwdTile / 2 + col] = qi < p.Nq ? -cdelta[e] : 0.f;
        }
      }
      __syncwarp();
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after_sync();
      const float2 cs2 = make_float2(c_s, c_s), l2e2 = make_float2(l2e, l2e);
      // A: this row's -lse and -Delta; B: a masked key row gets -inf exponents
      const float2 rowl2 = make_float2(-lse2, -lse2), rowd2 = make_float2(-delta, -delta);
      const float kill = key_ok ? 0.f : -INFINITY;
      const float2 kill2 = make_float2(kill, kill);
      // this warpgroup's 64 columns: S, dP -> P, dS, two columns per packed op
      {
        const int hf = g;
        uint32_t sv[64], dpv[64];
        tmem_ld32(tmem + lane_base + L::kColS + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(tmem + lane_base + L::kColS + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_ld32(tmem + lane_base + L::kColDP + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(&dpv[0]));
        tmem_ld32(tmem + lane_base + L::kColDP + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&dpv[32]));
        tmem_wait_ld();
        reg_fence(sv);
        reg_fence(dpv);
        // S and dP are in registers: the next step's S, dP may overwrite them
        // once both warpgroups have arrived
        tc_fence_before_sync();
        mbar_arrive(&bars[L::kBarSFree]);
        // two quarters of 32 columns, each stored to Tensor Memory (and, in
        // A, to dbias) before the next is formed
#pragma unroll
        for (int qt = 0; qt < 2; ++qt) {
          uint32_t pk[16], dk[16];
#pragma unroll
          for (int c8 = 4 * qt; c8 < 4 * qt + 4; ++c8) {
            const int c = hf * 64 + c8 * 8;  // first of eight columns
            float2 b2[4], nl2[4], nd2[4];
            if (!kB) {
              // 128-byte swizzled [query][key] tile: keys c .. c+7 of row t,
              // masked halves become bf16 -inf: (w & keep) | (~keep & -inf)
              const int box = c >> 6, chunk = (c & 63) >> 3;
              const uint4 w4 = *reinterpret_cast<const uint4 *>(bt + box * (L::kBiasBytes / 2) + t * 128 +
                                                                ((chunk ^ (t & 7)) << 4));
              const uint4 k4 = reinterpret_cast<const uint4 *>(rv)[c8];
              const uint32_t ww[4] = {w4.x, w4.y, w4.z, w4.w}, kw[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const uint32_t w = (ww[e] & kw[e]) | (~kw[e] & 0xFF80FF80u);
                b2[e] = make_float2(bf16lo_to_f32(w), bf16hi_to_f32(w));
                nl2[e] = rowl2;
                nd2[e] = rowd2;
              }
            } else {
              // plain [query][key] tile: queries c .. c+7 of key column t
              const int cl = c8 * 8;  // the columns' place in the warp's copy
              const float4 la = *reinterpret_cast<const float4 *>(rv + cl);
              const float4 lb = *reinterpret_cast<const float4 *>(rv + cl + 4);
              const float4 da = *reinterpret_cast<const float4 *>(rv + kBwdTile / 2 + cl);
              const float4 db = *reinterpret_cast<const float4 *>(rv + kBwdTile / 2 + cl + 4);
              const float2 lv[4] = {make_float2(la.x, la.y), make_float2(la.z, la.w), make_float2(lb.x, lb.y),
                                    make_float2(lb.z, lb.w)};
              const float2 dv[4] = {make_float2(da.x, da.y), make_float2(da.z, da.w), make_float2(db.x, db.y),
                                    make_float2(db.z, db.w)};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const uint32_t b0 = *reinterpret_cast<const uint16_t *>(bt + (c + 2 * e) * 256 + t * 2);
                const uint32_t b1 = *reinterpret_cast<const uint16_t *>(bt + (c + 2 * e + 1) * 256 + t * 2);
                b2[e] = make_float2(__uint_as_float(b0 << 16), __uint_as_float(b1 << 16));
                nl2[e] = fadd2(lv[e], kill2);
                nd2[e] = dv[e];
              }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = c8 * 4 + e;  // column pair
              // log2 of P: (tau s + b - lse) log2(e); -inf for masked keys and -inf bias
              const float2 a = ffma2(make_float2(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1])), cs2,
                                     ffma2(b2[e], l2e2, nl2[e]));
              const float2 pe = make_float2(ex2_approx(a.x), ex2_approx(a.y));
              const float2 dp = make_float2(__uint_as_float(dpv[2 * j]), __uint_as_float(dpv[2 * j + 1]));
              const float2 ds = fmul2(pe, fadd2(dp, nd2[e]));
              pk[j - 16 * qt] = pack_bf16x2(pe.x, pe.y);
              dk[j - 16 * qt] = pack_bf16x2(ds.x, ds.y);
            }
          }
          if (!kB) {
            // dbias: this row's dS over the quarter's 32 keys, written in
            // place of the bias values it came from (same swizzled 16-byte
            // chunks of the step's bias slot, read by this thread alone); the
            // warp stores its rows with one tensor store at the end of the step
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int c = hf * 64 + qt * 32 + q * 8;
              const int box = c >> 6, chunk = (c & 63) >> 3;
              *reinterpret_cast<uint4 *>(const_cast<uint8_t *>(bt) + box * (L::kBiasBytes / 2) + t * 128 +
                                         ((chunk ^ (t & 7)) << 4)) =
                  make_uint4(dk[4 * q], dk[4 * q + 1], dk[4 * q + 2], dk[4 * q + 3]);
            }
          }
          if (qt == 0 && it > 0) {
            // the previous step's accumulating MMAs read G0/G1, which the
            // stores below overwrite: wait for them only now, so that they
            // overlap this quarter's arithmetic
            ok = __all_sync(0xffffffffu, mbar_wait<false>(&bars[L::kBarGDone], (it - 1) & 1, wc));
            if (!ok) break;
            tc_fence_after_sync();
          }
          if (!kB) {
            tmem_st16(tmem + lane_base + L::kColG0 + hf * 32 + qt * 16, dk);
          } else {
            tmem_st16(tmem + lane_base + L::kColG0 + hf * 32 + qt * 16, pk);  // P^T
            tmem_st16(tmem + lane_base + L::kColG1 + hf * 32 + qt * 16, dk);  // dS^T
          }
        }
      }
      if (!ok) break;
      tmem_wait_st();
      tc_fence_before_sync();
      mbar_arrive(&bars[L::kBarGFull]);
      if (!kB) {
        // the warp's 32 rows of dbias for its warpgroup's 64 keys: one tensor
        // store from the slot (rows past Nq and keys past Nk are clipped);
        // the slot is released once the store has read it
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int w4 = warp & 3;
          tma_store_4d(&p.tm_dbias, bt + g * (L::kBiasBytes / 2) + w4 * 32 * 128, o0 + g * 64, row0 + 32 * w4, h,
                       b);
          bulk_commit_group();
          bulk_wait_group_read<0>();
          mbar_arrive(&bars[L::kBarBiasEmpty + bias_off / L::kBiasBytes]);
        }
      } else {
        // this warp's reads of the bias slot are done
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[L::kBarBiasEmpty + bias_off / L::kBiasBytes]);
      }
      bias_off += L::kBiasBytes;
      if (bias_off == uint32_t(L::kBiasStages * L::kBiasBytes)) {
        bias_off = 0;
        bias_ph ^= 1u;
      }
    }
    // -------------------------------------------------------------- epilogue
    if (ok) ok = mbar_wait<false>(&bars[L::kBarGDone], (nsteps - 1) & 1, wc);
    // the loads below are warp-collective: the warp leaves the wait as one
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after_sync();
      const int nrows = kB ? p.Nk : p.Nq;
      {
        // A: dQ (acc0, scaled by tau), columns 32g .. 32g+31 (D = 32: the
        // first warpgroup alone).  B: warpgroup 0 dK (acc0, scaled by tau),
        // warpgroup 1 dV (acc1), all D columns.
        const int a = kB ? g : 0;
        const uint32_t col = (a == 0) ? L::kColAcc0 : L::kColAcc1;
        const float scale = (a == 0) ? p.tau : 1.f;
        float *dst = !kB ? p.dq : (a == 0 ? p.dk : p.dv);
        const int c_begin = kB ? 0 : 32 * g, c_step = kB ? 32 : D;
#pragma unroll 1
        for (int c = c_begin; c < D; c += c_step) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + col + c, v);
          tmem_wait_ld();
          reg_fence(v);
          if (r < nrows) {
            float4 *o = reinterpret_cast<float4 *>(dst + ((int64_t(b) * p.H + h) * nrows + r) * D + c);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              o[q] = make_float4(__uint_as_float(v[4 * q]) * scale, __uint_as_float(v[4 * q + 1]) * scale,
                                 __uint_as_float(v[4 * q + 2]) * scale, __uint_as_float(v[4 * q + 3]) * scale);
          }
        }
      }
    }
  }

  // the warps' dbias tensor stores are complete before the CTA ends
  if (!kB && warp < kBwdWarpProducer && lane == 0) bulk_wait_group_all();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == kBwdWarpMma) tmem_dealloc(tmem, 512);
}

// Delta_i = sum_d dO_id O_id (bf16 inputs, fp32 sum).  D / 8 lanes per row
// (D = 32 or 64), each with one 16-byte load of dO and of O (8 features); the
// lanes of a row add their sums by shuffles.  dO and O are contiguous
// [rows][D] bf16 rows starting on 16-byte boundaries.
__global__ void pba_bwd_delta_kernel(const uint16_t *dout, const uint16_t *out, float *delta, int64_t rows, int D) {
  const int lpr = D >> 3;  // lanes per row, a divisor of 32
  const int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t row = t / lpr;
  const int c = int(t - row * lpr);
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = reinterpret_cast<const uint4 *>(dout + row * D)[c];
    const uint4 b = reinterpret_cast<const uint4 *>(out + row * D)[c];
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      acc += __uint_as_float(aw[e] << 16) * __uint_as_float(bw[e] << 16) +
             __uint_as_float(aw[e] & 0xFFFF0000u) * __uint_as_float(bw[e] & 0xFFFF0000u);
  }
  // every lane of the warp takes part; rows past the end add zeros
  for (int o = lpr >> 1; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (row < rows && c == 0) delta[row] = acc;
}

}  // namespace pba
