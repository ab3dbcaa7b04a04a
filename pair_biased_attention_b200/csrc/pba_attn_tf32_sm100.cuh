// pba_attn_tf32_sm100.cuh -- pair-biased attention for fp32 inputs on the
// sm_100a tensor cores (tcgen05.mma kind::tf32).
//
// The same computation as pba_attn_sm100.cuh ("Fold-CP: A Context Parallelism
// Framework for Biomolecular Modeling", Table 1 "Attn Pair Bias" and the
// key-block step of Figure 2(c)): per (b, h) and query row i,
//     O_i = sum_j softmax_j( tau q_i.k_j + b_ij ) v_j,
// accumulated online over 64-key tiles, with either the forward epilogue
// (fp32 O and the natural log-sum-exp) or the partial one (fp32 O_p, m_p, l_p
// for the tiled-softmax merge).
//
// fp32 accuracy from tf32 products.  A tf32 operand keeps 10 of fp32's 23
// mantissa bits, so one tf32 product of x and y is off by about 2^-11 |x y|.
// Every operand x is therefore split into x_hi = tf32(x) and
// x_lo = tf32(x - x_hi) (both rounded to nearest, x - x_hi exact in fp32), and
// each product takes three instructions,
//     x y ~= x_lo y_hi + x_hi y_lo + x_hi y_hi,
// which leaves out x_lo y_lo and the rounding of the low parts: about
// 3 * 2^-22 |x y| per product (the split of "Recovering single precision
// accuracy from Tensor Cores while surpassing the FP32 theoretical peak
// performance", Ootomo and Yokota, 2022).  The sums are the tensor core's
// fp32 accumulation.  This applies to S = Q K^T (Q's high part and K's two
// parts in shared memory, Q's low part in Tensor Memory) and to O += P V (P
// split by the softmax threads into Tensor Memory, V split and transposed in
// shared memory).
//
// Operand layouts: every operand is K-major (the contraction dimension
// contiguous).  Q's two parts and P's two parts are the A operands, read from
// Tensor Memory; K's parts and V^T's parts are the B operands, in shared
// memory with the 128-byte swizzle (rows of D or 64 fp32 as 128-byte chunks of
// 32).  V arrives key-major and is written transposed (one row per feature,
// keys contiguous) by its split warps.
//
// One CTA per (b, h, 128 query rows), sixteen warps:
//   warps 0-3    softmax (thread t owns query row t)
//   warps 4-7    K split: Q once (row by row, both parts into Tensor Memory),
//                then per key tile K (high part in place, low part beside it)
//   warps 8-11   V split: per key tile V^T's high and low parts
//   warp 12      TMA producer of Q, K and V
//   warp 13      allocates Tensor Memory and issues every tcgen05.mma
//   warp 14      TMA producer of the bias tiles
//   warp 15      no role (completes the fourth warpgroup)
// Tensor Memory (512 columns x 128 lanes of fp32):
//   [0,64) S0  [64,128) S1  [128,192) P_hi  [192,256) P_lo  [256,256+D) O
//   [256+D,256+2D) Q_hi  [256+2D,256+3D) Q_lo
// Issue order of the MMA warp: S(0), S(1), PV(0), S(2), PV(1), ...  The K and
// V splits run on their own warps, ahead of the MMAs by their ring depths, so
// the tensor pipe, not a chain of loads and splits, sets the pace: a tile is
// S(j+1) and PV(j) back to back, while the softmax works on tile j+1.
#pragma once

#include <cuda.h>

#include "pba_ptx.cuh"

namespace pba {

constexpr int kTfBM = 128;  // query rows per CTA (one TMEM lane each)
constexpr int kTfBN = 64;   // keys per tile
constexpr int kTfThreads = 512;
constexpr int kTfWarpKSplit0 = 4;
constexpr int kTfWarpVSplit0 = 8;
constexpr int kTfWarpProducer = 12;
constexpr int kTfWarpMma = 13;
constexpr int kTfWarpBias = 14;
constexpr uint32_t kTfTmemCols = 512;
constexpr uint32_t kTfColS = 0, kTfColPhi = 128, kTfColPlo = 192, kTfColO = 256;
// Per-thread register limits after the warpgroup reallocation (launch: 128).
constexpr int kTfRegsSoftmax = 248;
constexpr int kTfRegsOther = 88;
constexpr int kTfRegSplitTotal = 128 * kTfRegsSoftmax + 384 * kTfRegsOther;

struct Tf32Params {
  CUtensorMap tm_q, tm_k, tm_v, tm_bias;
  int32_t B, H, Nq, Nk;
  int32_t n_qblocks;     // ceil(Nq / 128)
  int32_t bias_h_bcast;  // bias head stride 0
  int32_t bias_b_bcast;  // bias batch stride 0
  int32_t mask_vec16;    // mask rows readable as aligned 16-byte words
  float tau;
  const uint8_t *mask;  // [B][Nk] (row stride mask_sb) or null
  int64_t mask_sb;
  float *out;  // fp32 O (forward) or O_p (partial)
  int64_t out_sb, out_sh, out_sn;
  float *lse;  // forward: log-sum-exp (nullable); partial: m_p
  int64_t lse_sb, lse_sh, lse_sn;
  float *l_part;  // partial: l_p (strides of lse)
  int *err;
  uint64_t timeout_ns;
};

template <int D>
struct Tf32Layout {
  static_assert(D == 32 || D == 64, "head dimension");
  static constexpr int kChunks = D / 32;                // 128-byte K chunks per Q/K row
  static constexpr int kQChunkBytes = kTfBM * 128;      // 128 rows x 32 fp32
  static constexpr int kQBytes = kChunks * kQChunkBytes;
  static constexpr int kKChunkBytes = kTfBN * 128;      // 64 rows x 32 fp32
  static constexpr int kKBytes = kChunks * kKChunkBytes;  // one K tile (or raw V tile)
  static constexpr int kVtChunkBytes = D * 128;         // D feature rows x 32 keys
  static constexpr int kVtBytes = 2 * kVtChunkBytes;    // 64 keys
  static constexpr int kBiasBoxBytes = kTfBM * 128;     // 128 rows x 32 keys
  static constexpr int kBiasBytes = 2 * kBiasBoxBytes;  // 64 keys
  static constexpr int kKStages = (D == 32) ? 3 : 2;
  static constexpr int kVRawStages = (D == 32) ? 3 : 2;
  static constexpr int kVtStages = (D == 32) ? 3 : 2;
  static constexpr int kBiasStages = 2;
  static constexpr uint32_t kColQhi = kTfColO + D;
  static constexpr uint32_t kColQlo = kTfColO + 2 * D;
  static constexpr int kOffKhi = 0;
  static constexpr int kOffKlo = kOffKhi + kKStages * kKBytes;
  static constexpr int kOffVraw = kOffKlo + kKStages * kKBytes;
  static constexpr int kOffVthi = kOffVraw + kVRawStages * kKBytes;
  static constexpr int kOffVtlo = kOffVthi + kVtStages * kVtBytes;
  static constexpr int kOffBias = kOffVtlo + kVtStages * kVtBytes;
  static constexpr int kOffBar = kOffBias + kBiasStages * kBiasBytes;
  // Q lands in the V^T high-part ring, which its split empties before the
  // V split writes the first V^T tile there
  static constexpr int kOffQraw = kOffVthi;
  static_assert(kVtStages * kVtBytes >= kQBytes, "Q staging");
  // barriers
  static constexpr int kBarQFull = 0;
  static constexpr int kBarQReady = 1;
  static constexpr int kBarKFull = 2;
  static constexpr int kBarKReady = kBarKFull + kKStages;
  static constexpr int kBarKEmpty = kBarKReady + kKStages;
  static constexpr int kBarVFull = kBarKEmpty + kKStages;
  static constexpr int kBarVRawEmpty = kBarVFull + kVRawStages;
  static constexpr int kBarVtReady = kBarVRawEmpty + kVRawStages;
  static constexpr int kBarVtEmpty = kBarVtReady + kVtStages;
  static constexpr int kBarBiasFull = kBarVtEmpty + kVtStages;
  static constexpr int kBarBiasEmpty = kBarBiasFull + kBiasStages;
  static constexpr int kBarSFull = kBarBiasEmpty + kBiasStages;  // [2]
  static constexpr int kBarSFree = kBarSFull + 2;                // [2]
  static constexpr int kBarPFull = kBarSFree + 2;
  static constexpr int kBarPDone = kBarPFull + 1;  // a P V has completed
  static constexpr int kBarDrain = kBarPDone + 1;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemSlot + 4;
  static constexpr int kBytes = kOffAbort + 4;
  static constexpr int kSmemAlloc = kBytes + 1024;  // room to align the base to 1024
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(kOffKlo % 1024 == 0 && kOffVraw % 1024 == 0 && kOffVthi % 1024 == 0 && kOffVtlo % 1024 == 0 &&
                    kOffBias % 1024 == 0,
                "swizzle atoms");
};

// Splits four fp32 values into their tf32 high parts and tf32 low parts.
__device__ __forceinline__ void tf32_split4(const uint4 v, uint4 &hi, uint4 &lo) {
  hi.x = to_tf32(__uint_as_float(v.x));
  hi.y = to_tf32(__uint_as_float(v.y));
  hi.z = to_tf32(__uint_as_float(v.z));
  hi.w = to_tf32(__uint_as_float(v.w));
  lo.x = to_tf32(__uint_as_float(v.x) - __uint_as_float(hi.x));
  lo.y = to_tf32(__uint_as_float(v.y) - __uint_as_float(hi.y));
  lo.z = to_tf32(__uint_as_float(v.z) - __uint_as_float(hi.z));
  lo.w = to_tf32(__uint_as_float(v.w) - __uint_as_float(hi.w));
}

// Splits kBytes of fp32 at `hi` in place and writes the low parts at the
// same offsets from `lo` (the split is element-wise, so any swizzle carries
// over).  Thread st of 128 takes 16-byte words st, st + 128, ...; all loads
// are issued before the first store.
template <int kBytes>
__device__ __forceinline__ void tf32_split_tile(uint8_t *hi, uint8_t *lo, int st) {
  constexpr int kWords = kBytes / (128 * 16);
  static_assert(kBytes % (128 * 16) == 0, "whole words per thread");
  uint4 v[kWords];
#pragma unroll
  for (int i = 0; i < kWords; ++i) v[i] = *reinterpret_cast<const uint4 *>(hi + (i * 128 + st) * 16);
#pragma unroll
  for (int i = 0; i < kWords; ++i) {
    uint4 h, l;
    tf32_split4(v[i], h, l);
    *reinterpret_cast<uint4 *>(hi + (i * 128 + st) * 16) = h;
    *reinterpret_cast<uint4 *>(lo + (i * 128 + st) * 16) = l;
  }
}

// Splits the raw V tile (kChunks boxes of [64 keys][32 fp32], 128-byte
// swizzle) into V^T high and low parts: two key chunks (keys 0-31, 32-63),
// each [D feature rows][32 keys] with the 128-byte swizzle, the K-major B
// operand of O += P V.  Thread st takes key st & 63 and half st >> 6 of the
// features; a warp reads eight consecutive keys' words per phase (distinct
// swizzled banks) and writes one feature row's 32 keys (32 distinct banks).
template <int D>
__device__ __forceinline__ void tf32_split_vt(const uint8_t *vraw, uint8_t *vthi, uint8_t *vtlo, int st) {
  using L = Tf32Layout<D>;
  const int key = st & 63, half = st >> 6;
  const int kk = key & 31;
  uint8_t *dhi = vthi + (key >> 5) * L::kVtChunkBytes;
  uint8_t *dlo = vtlo + (key >> 5) * L::kVtChunkBytes;
#pragma unroll
  for (int w = 0; w < D / 8; ++w) {
    const int dq = half * (D / 8) + w;  // 16-byte word along the features: features 4 dq .. 4 dq + 3
    const int chunk = dq >> 3, g = dq & 7;
    const uint4 v =
        *reinterpret_cast<const uint4 *>(vraw + chunk * L::kKChunkBytes + key * 128 + ((g ^ (key & 7)) << 4));
    uint4 hi, lo;
    tf32_split4(v, hi, lo);
    const uint32_t hv[4] = {hi.x, hi.y, hi.z, hi.w}, lv[4] = {lo.x, lo.y, lo.z, lo.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int d = dq * 4 + e;
      const int off = d * 128 + (((kk >> 2) ^ (d & 7)) << 4) + (kk & 3) * 4;
      *reinterpret_cast<uint32_t *>(dhi + off) = hv[e];
      *reinterpret_cast<uint32_t *>(dlo + off) = lv[e];
    }
  }
}

// A wait of a full warp before warp-collective Tensor Memory accesses: every
// lane waits on the same phase, and the vote makes the warp leave as one even
// if the lanes' time limits ran out at different moments.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, const WaitCtl &w) {
  return __all_sync(0xffffffffu, mbar_wait<false>(bar, parity, w));
}

constexpr float kTfLog2e = 1.4426950408889634f;
// The running maximum is replaced only when a tile's maximum exceeds it by
// more than 8 / ln 2 (P and l share the stale maximum, so the result is the
// same; probabilities stay below 2^8 and most tiles skip the rescale of O).
constexpr float kTfRescaleThreshold = 8.0f / kTfLog2e;

template <int D, bool kPartial, bool kMasked>
__global__ void __launch_bounds__(kTfThreads, 1) pba_attn_tf32_sm100_kernel(const __grid_constant__ Tf32Params p) {
  using L = Tf32Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffTmemSlot);
  int *abort_flag = reinterpret_cast<int *>(smem + L::kOffAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nt = (p.Nk + kTfBN - 1) / kTfBN;  // key tiles
  const int qblk = int(blockIdx.x % uint32_t(p.n_qblocks));
  const int bh = int(blockIdx.x / uint32_t(p.n_qblocks));
  const int b = bh / p.H, h = bh % p.H, q0 = qblk * kTfBM;

  if (threadIdx.x == 0) {
    mbar_init(&bars[L::kBarQFull], 1);
    mbar_init(&bars[L::kBarQReady], 128);
    for (int s = 0; s < L::kKStages; ++s) {
      mbar_init(&bars[L::kBarKFull + s], 1);
      mbar_init(&bars[L::kBarKReady + s], 128);
      mbar_init(&bars[L::kBarKEmpty + s], 1);
    }
    for (int s = 0; s < L::kVRawStages; ++s) {
      mbar_init(&bars[L::kBarVFull + s], 1);
      mbar_init(&bars[L::kBarVRawEmpty + s], 128);
    }
    for (int s = 0; s < L::kVtStages; ++s) {
      mbar_init(&bars[L::kBarVtReady + s], 128);
      mbar_init(&bars[L::kBarVtEmpty + s], 1);
    }
    for (int s = 0; s < L::kBiasStages; ++s) {
      mbar_init(&bars[L::kBarBiasFull + s], 1);
      mbar_init(&bars[L::kBarBiasEmpty + s], kTfBM);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[L::kBarSFull + i], 1);
      mbar_init(&bars[L::kBarSFree + i], kTfBM);
    }
    mbar_init(&bars[L::kBarPFull], kTfBM);
    mbar_init(&bars[L::kBarPDone], 1);
    mbar_init(&bars[L::kBarDrain], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kTfWarpMma) {
    tmem_alloc(tmem_slot, kTfTmemCols);
    tmem_relinquish();
  }
  if (warp == kTfWarpProducer && lane == 0) {
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
  }
  if (warp == kTfWarpBias && lane == 0) tma_prefetch_desc(&p.tm_bias);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, p.err, p.timeout_ns};
  WaitCtl wc_drain = wc;  // clean-up waits: ignore the abort word, keep the time limit
  int drain_abort = 0;
  wc_drain.abort_flag = &drain_abort;

  // Registers: the launch gives 128 per thread (512 x 128 = 65536); the
  // split, producer and MMA warpgroups give part of theirs to the softmax
  // warpgroup (128 x 248 + 384 x 88 = 65536).  Each warpgroup changes its
  // limit once, at the top of its own branch.
  if (warp >= kTfWarpProducer) {
    setmaxnreg_dec<kTfRegsOther>();
    if (warp == kTfWarpProducer) {
      // ================================================================ Q/K/V TMA producer
      if (lane == 0) {
        const uint64_t pol_stream = l2_policy_evict_first();
        const uint64_t pol_keep = l2_policy_evict_last();
        bool ok = true;
        int nk = 0, nv = 0;  // K and V tiles issued
        mbar_arrive_expect_tx(&bars[L::kBarQFull], L::kQBytes);
  #pragma unroll
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_4d(smem + L::kOffQraw + c * L::kQChunkBytes, &p.tm_q, &bars[L::kBarQFull], c * 32, q0, h, b,
                      pol_stream);
        for (int j = 0; j < nt && ok; ++j) {
          const int sk = j % L::kKStages;
          if (j >= L::kKStages && !(ok = mbar_wait(&bars[L::kBarKEmpty + sk], ((j / L::kKStages) - 1) & 1, wc)))
            break;
          mbar_arrive_expect_tx(&bars[L::kBarKFull + sk], L::kKBytes);
  #pragma unroll
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_4d(smem + L::kOffKhi + sk * L::kKBytes + c * L::kKChunkBytes, &p.tm_k, &bars[L::kBarKFull + sk],
                        c * 32, j * kTfBN, h, b, pol_keep);
          ++nk;
          const int sv = j % L::kVRawStages;
          if (j >= L::kVRawStages &&
              !(ok = mbar_wait(&bars[L::kBarVRawEmpty + sv], ((j / L::kVRawStages) - 1) & 1, wc)))
            break;
          mbar_arrive_expect_tx(&bars[L::kBarVFull + sv], L::kKBytes);
  #pragma unroll
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_4d(smem + L::kOffVraw + sv * L::kKBytes + c * L::kKChunkBytes, &p.tm_v, &bars[L::kBarVFull + sv],
                        c * 32, j * kTfBN, h, b, pol_keep);
          ++nv;
        }
        if (!ok) {
          // Let every copy already issued land before the CTA exits: slot s of a
          // ring of S slots was armed (n - s + S - 1) / S times after n issues.
          mbar_wait(&bars[L::kBarQFull], 0, wc_drain);
          for (int s = 0; s < L::kKStages; ++s) {
            const int a = (nk - s + L::kKStages - 1) / L::kKStages;
            if (a > 0) mbar_wait(&bars[L::kBarKFull + s], (a - 1) & 1, wc_drain);
          }
          for (int s = 0; s < L::kVRawStages; ++s) {
            const int a = (nv - s + L::kVRawStages - 1) / L::kVRawStages;
            if (a > 0) mbar_wait(&bars[L::kBarVFull + s], (a - 1) & 1, wc_drain);
          }
        }
      }
    } else if (warp == kTfWarpBias) {
      // ================================================================ bias TMA producer
      if (lane == 0) {
        const uint64_t pol_stream = l2_policy_evict_first();
        const int hb = p.bias_h_bcast ? 0 : h;
        const int bb = p.bias_b_bcast ? 0 : b;
        bool ok = true;
        int nb = 0;
        for (int j = 0; j < nt && ok; ++j) {
          const int s = j % L::kBiasStages;
          if (j >= L::kBiasStages &&
              !(ok = mbar_wait(&bars[L::kBarBiasEmpty + s], ((j / L::kBiasStages) - 1) & 1, wc)))
            break;
          mbar_arrive_expect_tx(&bars[L::kBarBiasFull + s], L::kBiasBytes);
          // [128 queries][64 keys] as two 32-key boxes, 128-byte swizzle
  #pragma unroll
          for (int c = 0; c < 2; ++c)
            tma_load_4d(smem + L::kOffBias + s * L::kBiasBytes + c * L::kBiasBoxBytes, &p.tm_bias,
                        &bars[L::kBarBiasFull + s], j * kTfBN + c * 32, q0, hb, bb, pol_stream);
          ++nb;
        }
        if (!ok)
          for (int s = 0; s < L::kBiasStages; ++s) {
            const int a = (nb - s + L::kBiasStages - 1) / L::kBiasStages;
            if (a > 0) mbar_wait(&bars[L::kBarBiasFull + s], (a - 1) & 1, wc_drain);
          }
      }
    } else if (warp == kTfWarpMma) {
      // ================================================================ MMA issuer
      if (lane == 0) {
        const uint32_t idesc_s = idesc_tf32_f32(kTfBM, kTfBN);
        const uint32_t idesc_o = idesc_tf32_f32(kTfBM, D);
        constexpr uint32_t kDescHi = smem_desc_hi(1024, 2);  // 8-row atoms of 128 bytes, 128-byte swizzle
        // S(buf) = Q K^T over D / 8 steps of 8 features, three products per step
        // (Q_lo x K_hi, Q_hi x K_lo, Q_hi x K_hi): Q from Tensor Memory (8
        // columns per step), K from shared memory (32 bytes further along a
        // 128-byte swizzle row per step, or the next 32-feature chunk).
        auto issue_s = [&](int buf, int sk) {
          const uint32_t d_tmem = tmem + kTfColS + buf * kTfBN;
          const uint32_t khi = smem_desc_lo(smem_u32(smem + L::kOffKhi + sk * L::kKBytes), 16);
          const uint32_t klo = smem_desc_lo(smem_u32(smem + L::kOffKlo + sk * L::kKBytes), 16);
  #pragma unroll
          for (int pass = 0; pass < 3; ++pass) {
            const uint32_t a = tmem + (pass == 0 ? L::kColQlo : L::kColQhi);
            const uint32_t bk = pass == 1 ? klo : khi;
  #pragma unroll
            for (int k = 0; k < D / 8; ++k) {
              const uint32_t ka = uint32_t((k >> 2) * L::kKChunkBytes + (k & 3) * 32) >> 4;
              mma_tf32_ts(d_tmem, a + k * 8, desc_at(bk, ka, kDescHi), idesc_s, (pass > 0 || k > 0) ? 1u : 0u);
            }
          }
          tc_commit(&bars[L::kBarSFull + buf]);
        };
        // O += P V over 8 steps of 8 keys: P from Tensor Memory (8 columns per
        // step), V^T from shared memory (32 bytes per step inside a key chunk).
        auto issue_pv = [&](int sv, bool first) {
          const uint32_t d_tmem = tmem + kTfColO;
          const uint32_t vhi = smem_desc_lo(smem_u32(smem + L::kOffVthi + sv * L::kVtBytes), 16);
          const uint32_t vlo = smem_desc_lo(smem_u32(smem + L::kOffVtlo + sv * L::kVtBytes), 16);
  #pragma unroll
          for (int pass = 0; pass < 3; ++pass) {
            const uint32_t a = tmem + (pass == 0 ? kTfColPlo : kTfColPhi);
            const uint32_t bv = pass == 1 ? vlo : vhi;
  #pragma unroll
            for (int k = 0; k < kTfBN / 8; ++k) {
              const uint32_t va = uint32_t((k >> 2) * L::kVtChunkBytes + (k & 3) * 32) >> 4;
              mma_tf32_ts(d_tmem, a + k * 8, desc_at(bv, va, kDescHi), idesc_o,
                          (!first || pass > 0 || k > 0) ? 1u : 0u);
            }
          }
          tc_commit(&bars[L::kBarPDone]);
        };
        bool ok = mbar_wait(&bars[L::kBarQReady], 0, wc);
        if (ok) ok = mbar_wait(&bars[L::kBarKReady], 0, wc);
        if (ok) {
          tc_fence_after_sync();
          issue_s(0, 0);
          tc_commit(&bars[L::kBarKEmpty]);
        }
        for (int j = 0; j < nt && ok; ++j) {
          if (j + 1 < nt) {
            // S(j+1) into the other buffer: its K tile split, and S(j-1) read by the softmax
            const int jn = j + 1, sk = jn % L::kKStages, buf = jn & 1;
            ok = mbar_wait(&bars[L::kBarKReady + sk], (jn / L::kKStages) & 1, wc);
            if (ok && jn >= 2) ok = mbar_wait(&bars[L::kBarSFree + buf], ((jn >> 1) - 1) & 1, wc);
            if (!ok) break;
            tc_fence_after_sync();
            issue_s(buf, sk);
            tc_commit(&bars[L::kBarKEmpty + sk]);
          }
          // P V(j): V^T(j) split, P(j) written
          const int sv = j % L::kVtStages;
          ok = mbar_wait(&bars[L::kBarVtReady + sv], (j / L::kVtStages) & 1, wc);
          if (ok) ok = mbar_wait(&bars[L::kBarPFull], j & 1, wc);
          if (!ok) break;
          tc_fence_after_sync();
          issue_pv(sv, j == 0);
          tc_commit(&bars[L::kBarVtEmpty + sv]);
        }
        // Every MMA issued above completes before Tensor Memory is released.
        tc_commit(&bars[L::kBarDrain]);
        mbar_wait(&bars[L::kBarDrain], 0, wc_drain);
      }
    }
    // warp 15 has no role
  } else if (warp < kTfWarpVSplit0 && warp >= kTfWarpKSplit0) {
    // ================================================================ K split warps
    setmaxnreg_dec<kTfRegsOther>();
    const int st = threadIdx.x - kTfWarpKSplit0 * 32;
    // Q: thread st takes query row st, both parts into this warp's lanes of
    // Tensor Memory
    bool ok = warp_wait(&bars[L::kBarQFull], 0, wc);
    if (ok) {
      const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
      const uint8_t *qrow = smem + L::kOffQraw + st * 128;
#pragma unroll
      for (int c = 0; c < L::kChunks; ++c) {
        uint32_t hi[32], lo[32];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const uint4 v = *reinterpret_cast<const uint4 *>(qrow + c * L::kQChunkBytes + ((g ^ (st & 7)) << 4));
          uint4 h4, l4;
          tf32_split4(v, h4, l4);
          hi[4 * g] = h4.x, hi[4 * g + 1] = h4.y, hi[4 * g + 2] = h4.z, hi[4 * g + 3] = h4.w;
          lo[4 * g] = l4.x, lo[4 * g + 1] = l4.y, lo[4 * g + 2] = l4.z, lo[4 * g + 3] = l4.w;
        }
        tmem_st32(tmem + lane_base + L::kColQhi + c * 32, hi);
        tmem_st32(tmem + lane_base + L::kColQlo + c * 32, lo);
      }
      tmem_wait_st();
      tc_fence_before_sync();
      mbar_arrive(&bars[L::kBarQReady]);
    }
    for (int j = 0; j < nt && ok; ++j) {
      const int sk = j % L::kKStages;
      if (!(ok = mbar_wait(&bars[L::kBarKFull + sk], (j / L::kKStages) & 1, wc))) break;
      tf32_split_tile<L::kKBytes>(smem + L::kOffKhi + sk * L::kKBytes, smem + L::kOffKlo + sk * L::kKBytes, st);
      fence_proxy_async_smem();
      mbar_arrive(&bars[L::kBarKReady + sk]);
    }
  } else if (warp >= kTfWarpVSplit0) {
    // ================================================================ V split warps
    setmaxnreg_dec<kTfRegsOther>();
    const int st = threadIdx.x - kTfWarpVSplit0 * 32;
    // the first V^T tiles overwrite the Q staging area: its split must be done
    bool ok = mbar_wait(&bars[L::kBarQReady], 0, wc);
    for (int j = 0; j < nt && ok; ++j) {
      const int sv = j % L::kVRawStages, stv = j % L::kVtStages;
      if (!(ok = mbar_wait(&bars[L::kBarVFull + sv], (j / L::kVRawStages) & 1, wc))) break;
      if (j >= L::kVtStages && !(ok = mbar_wait(&bars[L::kBarVtEmpty + stv], ((j / L::kVtStages) - 1) & 1, wc)))
        break;
      tf32_split_vt<D>(smem + L::kOffVraw + sv * L::kKBytes, smem + L::kOffVthi + stv * L::kVtBytes,
                       smem + L::kOffVtlo + stv * L::kVtBytes, st);
      fence_proxy_async_smem();
      mbar_arrive(&bars[L::kBarVtReady + stv]);
      // the raw slot's loads fed the stores above, so they have returned
      mbar_arrive(&bars[L::kBarVRawEmpty + sv]);
    }
  } else {
    // ================================================================ softmax warps
    setmaxnreg_inc<kTfRegsSoftmax>();
    const int t = threadIdx.x;  // query row inside the tile
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t tS = tmem + lane_base + kTfColS;
    const uint32_t tPhi = tmem + lane_base + kTfColPhi;
    const uint32_t tPlo = tmem + lane_base + kTfColPlo;
    const uint32_t tO = tmem + lane_base + kTfColO;
    const float tau = p.tau;
    const uint8_t *mrow = p.mask ? p.mask + int64_t(b) * p.mask_sb : nullptr;
    // bit c: key j * 64 + c exists and is not masked
    auto tile_keep = [&](int j) -> uint64_t {
      const int k0 = j * kTfBN;
      uint64_t kp = 0;
      if (mrow != nullptr && p.mask_vec16 && k0 + kTfBN <= p.Nk) {
        const uint4 *mp = reinterpret_cast<const uint4 *>(mrow + k0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 w = __ldg(mp + q);
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 16; ++e)
            kp |= uint64_t(((ws[e >> 2] >> (8 * (e & 3))) & 0xFFu) != 0) << (16 * q + e);
        }
      } else {
        for (int c = 0; c < kTfBN; ++c) {
          const int key = k0 + c;
          if (key < p.Nk && (mrow == nullptr || __ldg(mrow + key) != 0)) kp |= uint64_t(1) << c;
        }
      }
      return kp;
    };
    float m_cur = -INFINITY;   // maximum used for P and l
    float m_true = -INFINITY;  // true running maximum
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < nt && ok; ++j) {
      const int bs = j % L::kBiasStages, buf = j & 1;
      const uint64_t keep = kMasked ? tile_keep(j) : ~uint64_t(0);
      // x = bias first (the tile lands long before the score tile)
      if (!(ok = warp_wait(&bars[L::kBarBiasFull + bs], (j / L::kBiasStages) & 1, wc))) break;
      float x[kTfBN];
      {
        const uint8_t *row = smem + L::kOffBias + bs * L::kBiasBytes + t * 128;
#pragma unroll
        for (int g = 0; g < kTfBN / 4; ++g) {
          const uint4 v =
              *reinterpret_cast<const uint4 *>(row + (g >> 3) * L::kBiasBoxBytes + (((g & 7) ^ (t & 7)) << 4));
          x[4 * g] = __uint_as_float(v.x);
          x[4 * g + 1] = __uint_as_float(v.y);
          x[4 * g + 2] = __uint_as_float(v.z);
          x[4 * g + 3] = __uint_as_float(v.w);
        }
      }
      if (!(ok = warp_wait(&bars[L::kBarSFull + buf], (j >> 1) & 1, wc))) break;
      tc_fence_after_sync();
      uint32_t s[kTfBN];
      tmem_ld32(tS + buf * kTfBN, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld32(tS + buf * kTfBN + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_wait_ld();
      reg_fence(s);
      tc_fence_before_sync();
      mbar_arrive(&bars[L::kBarSFree + buf]);
#pragma unroll
      for (int c = 0; c < kTfBN; ++c) {
        x[c] = fmaf(tau, __uint_as_float(s[c]), x[c]);
        if (kMasked && !((keep >> c) & 1u)) x[c] = -INFINITY;
      }
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = x[i];
#pragma unroll
      for (int c = 8; c < kTfBN; ++c) m8[c & 7] = fmaxf(m8[c & 7], x[c]);
      const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      // Released under a condition on mx, which depends on every bias value
      // of the tile, so the arrive waits for all of the slot's loads and the
      // next TMA write into the slot cannot overtake one of them.  (No
      // maximum is this NaN pattern.)
      if (__float_as_uint(mx) != 0x7FC0DEADu) mbar_arrive(&bars[L::kBarBiasEmpty + bs]);
      m_true = fmaxf(m_true, mx);
      const bool need = mx > m_cur + kTfRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = (m_cur == -INFINITY) ? 0.f : ex2_approx((m_cur - mx) * kTfLog2e);
        l *= alpha;
        m_cur = mx;
      }
      const float neg_m = (m_cur == -INFINITY) ? 0.f : -m_cur * kTfLog2e;
#pragma unroll
      for (int c = 0; c < kTfBN; ++c) x[c] = ex2_approx(fmaf(x[c], kTfLog2e, neg_m));
      // pairwise sum of the 64 probabilities
      float ps[kTfBN / 2];
#pragma unroll
      for (int c = 0; c < kTfBN / 2; ++c) ps[c] = x[c] + x[c + kTfBN / 2];
#pragma unroll
      for (int w = kTfBN / 4; w >= 1; w >>= 1)
#pragma unroll
        for (int c = 0; c < w; ++c) ps[c] += ps[c + w];
      l += ps[0];

      // P(j) overwrites the P that P V(j-1) read, and a rescale of O needs
      // P V(j-1) done as well
      if (j >= 1) {
        if (!(ok = warp_wait(&bars[L::kBarPDone], (j - 1) & 1, wc))) break;
        tc_fence_after_sync();
        if (__any_sync(0xffffffffu, need)) {
          // rescale this warp's rows of O (lanes without a new maximum use 1)
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            uint32_t o[32];
            tmem_ld32(tO + c, o);
            tmem_wait_ld();
            reg_fence(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tO + c, o);
          }
        }
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t hi[32], lo[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float v = x[half * 32 + e];
          hi[e] = to_tf32(v);
          lo[e] = to_tf32(v - __uint_as_float(hi[e]));
        }
        tmem_st32(tPhi + half * 32, hi);
        tmem_st32(tPlo + half * 32, lo);
      }
      tmem_wait_st();
      tc_fence_before_sync();
      mbar_arrive(&bars[L::kBarPFull]);
    }

    // ---------------------------------------------------------------- epilogue
    if (ok) ok = warp_wait(&bars[L::kBarPDone], (nt - 1) & 1, wc);  // the last P V
    if (ok) {
      tc_fence_after_sync();
      float o[D];
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t r[32];
        tmem_ld32(tO + c, r);
        tmem_wait_ld();
        reg_fence(r);
#pragma unroll
        for (int e = 0; e < 32; ++e) o[c + e] = __uint_as_float(r[e]);
      }
      const int row = q0 + t;
      if (row < p.Nq) {
        float4 *op = reinterpret_cast<float4 *>(p.out + b * p.out_sb + h * p.out_sh + int64_t(row) * p.out_sn);
        if (l > 0.f) {
#pragma unroll
          for (int c = 0; c < D / 4; ++c)
            op[c] = make_float4(o[4 * c] / l, o[4 * c + 1] / l, o[4 * c + 2] / l, o[4 * c + 3] / l);
        } else {
#pragma unroll
          for (int c = 0; c < D / 4; ++c) op[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        const int64_t li = b * p.lse_sb + h * p.lse_sh + int64_t(row) * p.lse_sn;
        if (!kPartial) {
          if (p.lse != nullptr) p.lse[li] = (l > 0.f) ? m_cur + logf(l) : -INFINITY;
        } else {
          p.lse[li] = (l > 0.f) ? m_true : -INFINITY;
          p.l_part[li] = (l > 0.f) ? l * ex2_approx((m_cur - m_true) * kTfLog2e) : 0.f;
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == kTfWarpMma) tmem_dealloc(tmem, kTfTmemCols);
}

}  // namespace pba
