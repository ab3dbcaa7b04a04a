// pba_oproj_sm100.cuh -- output projection of triangle attention (sm_100a).
//
// Triangle attention draws its inputs from the pair representation and
// writes its result back to it ("Fold-CP: A Context Parallelism Framework for
// Biomolecular Modeling", Figure 2(a)); the per-head outputs [N*N][H*D] are
// projected back to the pair channels:
//     out[r][0:c] = o[r][0:128] W_o          (o [N*N][H*D = 128], W_o [128][c])
// as fp32 sums of bf16 products, rounded once to bf16.
//
// Persistent, one CTA per SM, 192 threads:
//   warps 0-3  epilogue: thread t owns pair row t of the tile (TMEM lane t);
//              32-column chunks of the accumulator -> bf16 -> swizzled
//              staging buffer -> one tensor store per chunk
//   warp 4     TMA producer: W_o once (resident), then one [128 rows][128]
//              o tile per stage of a kOprojStages ring
//   warp 5     allocates Tensor Memory and issues the MMAs
// Per tile: 8 MMAs of M128 N(c) K16, A = the o tile (K-major, 128-byte
// swizzle, two 64-column boxes), B = c/64 slabs of W_o (MN-major, 128-byte
// swizzle, slabs LBO apart), into one of two c-column accumulators in Tensor
// Memory so that the epilogue of one tile overlaps the MMAs of the next.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "pba_ptx.cuh"

namespace pba {

constexpr int kOprojRows = 128;    // pair rows per tile
constexpr int kOprojK = 128;       // H*D
constexpr int kOprojThreads = 192;
constexpr int kOprojStages = 4;

struct OprojParams {
  CUtensorMap tm_o;    // o [rows][128] bf16, box {64, 128}, 128-byte swizzle
  CUtensorMap tm_w;    // W_o [128][c] bf16, box {64, 128}, 128-byte swizzle
  CUtensorMap tm_out;  // out [rows][c] bf16, box {32, 32}, 64-byte swizzle (stores, one warp's rows each)
  int64_t rows;        // N*N
  int32_t n_tiles;     // ceil(rows / 128)
  int *err;
  uint64_t timeout_ns;
};

template <int kC>
struct OprojLayout {
  static_assert(kC == 64 || kC == 128, "pair channels");
  static constexpr int kSlabs = kC / 64;
  static constexpr int kSlabBytes = kOprojK * 128;          // 128 K rows of 64 bf16 columns
  static constexpr int kTileBytes = kOprojRows * kOprojK * 2;  // one o tile, two 64-column boxes
  static constexpr int kStageBufs = 3;                      // output staging: [128 rows][32 cols]
  static constexpr int kStageBytes = kOprojRows * 64;
  static constexpr int kOffW = 0;
  static constexpr int kOffO = kOffW + kSlabs * kSlabBytes;
  static constexpr int kOffStage = kOffO + kOprojStages * kTileBytes;
  static constexpr int kOffBar = kOffStage + kStageBufs * kStageBytes;
  static constexpr int kBarW = 0;
  static constexpr int kBarOFull = 1;
  static constexpr int kBarOEmpty = kBarOFull + kOprojStages;
  static constexpr int kBarAccFull = kBarOEmpty + kOprojStages;  // [accumulator]
  static constexpr int kBarAccEmpty = kBarAccFull + 2;           // [accumulator]
  static constexpr int kBarDrain = kBarAccEmpty + 2;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemSlot + 4;
  static constexpr int kBytes = kOffAbort + 4;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static constexpr uint32_t kTmemCols = 256;  // two accumulators of up to 128 columns
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(kOffO % 1024 == 0 && kOffStage % 1024 == 0, "swizzle alignment");
};

template <int kC>
__global__ void __launch_bounds__(kOprojThreads, 1) pba_oproj_sm100_kernel(const __grid_constant__ OprojParams p) {
  using L = OprojLayout<kC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffTmemSlot);
  int *abort_flag = reinterpret_cast<int *>(smem + L::kOffAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars[L::kBarW], 1);
    for (int s = 0; s < kOprojStages; ++s) {
      mbar_init(&bars[L::kBarOFull + s], 1);
      mbar_init(&bars[L::kBarOEmpty + s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[L::kBarAccFull + b], 1);
      mbar_init(&bars[L::kBarAccEmpty + b], kOprojRows);
    }
    mbar_init(&bars[L::kBarDrain], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&p.tm_o);
    tma_prefetch_desc(&p.tm_w);
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&p.tm_out);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, p.err, p.timeout_ns};
  WaitCtl wc_drain = wc;  // clean-up waits: ignore the abort word, keep the time limit
  int drain_abort = 0;
  wc_drain.abort_flag = &drain_abort;

  if (warp == 4) {
    // ================================================================ TMA producer
    if (lane == 0) {
      const uint64_t pol_stream = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_last();
      mbar_arrive_expect_tx(&bars[L::kBarW], L::kSlabs * L::kSlabBytes);
      for (int s = 0; s < L::kSlabs; ++s)
        tma_load_4d(smem + L::kOffW + s * L::kSlabBytes, &p.tm_w, &bars[L::kBarW], s * 64, 0, 0, 0, pol_keep);
      bool ok = true;
      int it = 0;  // tiles issued
      for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x, ++it) {
        const int s = it % kOprojStages;
        if (it >= kOprojStages) ok = mbar_wait(&bars[L::kBarOEmpty + s], ((it / kOprojStages) - 1) & 1, wc);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars[L::kBarOFull + s], L::kTileBytes);
        for (int bx = 0; bx < kOprojK / 64; ++bx)
          tma_load_4d(smem + L::kOffO + s * L::kTileBytes + bx * (kOprojRows * 128), &p.tm_o, &bars[L::kBarOFull + s],
                      bx * 64, tile * kOprojRows, 0, 0, pol_stream);
      }
      // Let every copy already issued land before the CTA exits.
      mbar_wait(&bars[L::kBarW], 0, wc_drain);
      if (!ok)
        for (int s = 0; s < kOprojStages; ++s) {
          const int a = (it - s + kOprojStages - 1) / kOprojStages;
          if (a > 0) mbar_wait(&bars[L::kBarOFull + s], (a - 1) & 1, wc_drain);
        }
    }
  } else if (warp == 5) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kOprojRows, kC, true);  // B (W_o) is MN-major
      const uint32_t sW = smem_u32(smem + L::kOffW);
      const uint32_t sO = smem_u32(smem + L::kOffO);
      constexpr uint32_t kHi = smem_desc_hi(1024, 2);  // 8-row atoms of 128 bytes, 128-byte swizzle
      bool ok = mbar_wait(&bars[L::kBarW], 0, wc);
      int it = 0;
      for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x, ++it) {
        const int s = it % kOprojStages;
        const int b = it & 1;  // accumulator
        ok = mbar_wait(&bars[L::kBarOFull + s], (it / kOprojStages) & 1, wc);
        // the accumulator was last read by the epilogue of tile it - 2
        if (ok && it >= 2) ok = mbar_wait(&bars[L::kBarAccEmpty + b], ((it >> 1) - 1) & 1, wc);
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t obase = sO + s * L::kTileBytes;
        const uint32_t wlo = smem_desc_lo(sW, L::kSlabBytes);
#pragma unroll
        for (int kk = 0; kk < kOprojK / 16; ++kk) {
          // A: columns 16 kk .. 16 kk + 15 of the o tile (box kk/4, 32 bytes per K step inside a swizzle row)
          const uint32_t alo = smem_desc_lo(obase + (kk >> 2) * (kOprojRows * 128) + (kk & 3) * 32, 16);
          // B: rows 16 kk .. 16 kk + 15 of the W_o slabs (2 KB per K step)
          mma_bf16_ss(tmem + b * kC, desc_join(alo, kHi), desc_join(wlo + kk * 128, kHi), idesc, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars[L::kBarAccFull + b]);
        tc_commit(&bars[L::kBarOEmpty + s]);
      }
      tc_commit(&bars[L::kBarDrain]);
      mbar_wait(&bars[L::kBarDrain], 0, wc_drain);
    }
  } else {
    // ================================================================ epilogue warpgroup
    const int t = threadIdx.x;  // pair row inside the tile, TMEM lane
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    bool ok = true;
    int it = 0;
    int sc = 0;  // output chunks staged
    for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x, ++it) {
      const int b = it & 1;
      // the warp leaves the wait as one (the loads below are warp-collective)
      ok = __all_sync(0xffffffffu, mbar_wait<false>(&bars[L::kBarAccFull + b], (it >> 1) & 1, wc));
      if (!ok) break;
      tc_fence_after_sync();
#pragma unroll 1
      for (int ch = 0; ch < kC / 32; ++ch) {
        uint32_t a[32];
        tmem_ld32(tmem + lane_base + b * kC + 32 * ch, a);
        tmem_wait_ld();
        reg_fence(a);
        if (ch + 1 == kC / 32) {
          tc_fence_before_sync();
          mbar_arrive(&bars[L::kBarAccEmpty + b]);  // this accumulator is free
        }
        uint8_t *buf = smem + L::kOffStage + (sc % L::kStageBufs) * L::kStageBytes;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 v = make_uint4(pack_bf16x2(__uint_as_float(a[8 * j]), __uint_as_float(a[8 * j + 1])),
                                     pack_bf16x2(__uint_as_float(a[8 * j + 2]), __uint_as_float(a[8 * j + 3])),
                                     pack_bf16x2(__uint_as_float(a[8 * j + 4]), __uint_as_float(a[8 * j + 5])),
                                     pack_bf16x2(__uint_as_float(a[8 * j + 6]), __uint_as_float(a[8 * j + 7])));
          // 64-byte swizzle: the 16-byte chunk index XOR bits 7-8 of the row address
          *reinterpret_cast<uint4 *>(buf + t * 64 + ((j ^ ((t >> 1) & 3)) << 4)) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // this warp's 32 rows (the 2 KB at 2 KB warp of the buffer)
          tma_store_4d(&p.tm_out, buf + warp * 2048, ch * 32, tile * kOprojRows + warp * 32, 0, 0);
          bulk_commit_group();
          // the buffer the chunk after next writes is free once this chunk's
          // predecessor has been read out
          bulk_wait_group_read<1>();
        }
        __syncwarp();
        ++sc;
      }
    }
    if (lane == 0) bulk_wait_group_all();  // this warp's staging buffers are read and its rows written
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 5) tmem_dealloc(tmem, L::kTmemCols);
}

}  // namespace pba
