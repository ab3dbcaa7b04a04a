// pba_proj_sm100.cuh -- triangle projections on the tensor cores (sm_100a).
//
// For the pair tensor z [N*N][c] (pair row r = i*N + j) this computes, as in
// "Fold-CP: A Context Parallelism Framework for Biomolecular Modeling"
// (Figure 2(a): triangle attention takes its queries, keys, values, gate and
// per-head bias from the pair representation),
//     q|k|v|g [r][0:128] = z[r] W_{q|k|v|g}     (W [c][512], H*D = 128 columns each)
//     bias[h][r]         = z[r] W_b[:, h]       (W_b [c][H], bias laid out [H][N][N])
// in one pass over z: the products are fp32 sums of bf16 products, rounded
// once to bf16 on output.
//
// Persistent, one CTA per SM, 192 threads:
//   warps 0-3  epilogue: thread t owns pair row t of the tile (TMEM lane t);
//              reads the fp32 accumulators, writes bf16 rows of q, k, v, g
//              and the row's H bias values
//   warp 4     TMA producer: W once (resident, 128 KB at c = 128), then one
//              128-row z tile per stage of a 2-stage ring
//   warp 5     allocates Tensor Memory and issues every tcgen05.mma
// Tensor Memory: two 256-column fp32 halves, [0,256) = q|k and [256,512) =
// v|g of a tile, so that the epilogue of one half overlaps the MMAs of the
// other.  Each half is c/16 MMAs of M128 N256 K16: A = the z tile (K-major,
// 128-byte swizzle), B = four 64-column slabs of W (MN-major, 128-byte
// swizzle, slabs LBO apart).  The bias columns are c/16 more MMAs of
// M128 N16 K16 against W_b^T (K-major, H rows padded to 16), issued after
// the v|g half into the first 16 columns of the q|k half once the epilogue
// has read them; the epilogue reads the bias after the rest of q|k and only
// then frees that half for the next tile.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "pba_ptx.cuh"

namespace pba {

constexpr int kProjRows = 128;     // pair rows per tile
constexpr int kProjCols = 512;     // q|k|v|g columns (H*D = 128 each)
constexpr int kProjThreads = 192;  // 6 warps
constexpr int kProjZStages = 2;
constexpr int kProjMaxC = 128;

struct ProjParams {
  CUtensorMap tm_z;  // z [rows][c] bf16, box {64, 128}
  CUtensorMap tm_w;  // W [c][512] bf16, box {64, c}
  CUtensorMap tm_out[4];  // q, k, v, g [rows][128] bf16, box {32, 32}, 64-byte swizzle (stores)
  int64_t rows;      // N*N
  int32_t c;         // 64 or 128
  int32_t n_tiles;   // ceil(rows / 128)
  const uint16_t *wb;  // W_b [c][H] bf16
  uint16_t *out[4];    // q, k, v, g: [rows][128] bf16
  uint16_t *bias;      // [H][rows] bf16
  int *err;
  uint64_t timeout_ns;
};

struct ProjLayout {
  static constexpr int kSlabs = kProjCols / 64;                 // 64-column slabs of W
  static constexpr int kSlabMax = kProjMaxC * 128;              // bytes of one slab at c = 128
  static constexpr int kOffW = 0;
  static constexpr int kZStageMax = kProjRows * kProjMaxC * 2;  // one z tile at c = 128
  static constexpr int kOffZ = kOffW + kSlabs * kSlabMax;
  // W_b^T as the bias MMA's B operand: [16 rows (h, zero past H)][c] bf16,
  // K-major, 128-byte swizzle, one 2 KB block per 64 columns of c
  static constexpr int kOffWb = kOffZ + kProjZStages * kZStageMax;
  static constexpr int kWbChunkBytes = 16 * 128;
  static constexpr int kWbMax = (kProjMaxC / 64) * kWbChunkBytes;
  // output staging: 32-column chunks of a tile ([128 rows][64 bytes], 64-byte
  // swizzle; warp w's rows are the 2 KB at 2 KB w, stored by the warp on its
  // own), three buffers
  static constexpr int kStageBufs = 3;
  static constexpr int kStageBytes = kProjRows * 64;
  static constexpr int kOffStage = kOffWb + kWbMax;
  static constexpr int kOffBar = kOffStage + kStageBufs * kStageBytes;
  static constexpr int kBarW = 0;
  static constexpr int kBarZFull = 1;
  static constexpr int kBarZEmpty = kBarZFull + kProjZStages;
  static constexpr int kBarAccFull = kBarZEmpty + kProjZStages;
  static constexpr int kBarAccEmpty = kBarAccFull + 2;
  static constexpr int kBarBiasSlot = kBarAccEmpty + 2;  // the epilogue has read columns [0, 64) of q|k
  static constexpr int kBarBiasFull = kBarBiasSlot + 1;  // the bias MMAs are done
  static constexpr int kBarDrain = kBarBiasFull + 1;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemSlot + 4;
  static constexpr int kBytes = kOffAbort + 4;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
};

template <int kH>
__global__ void __launch_bounds__(kProjThreads, 1) pba_proj_sm100_kernel(const __grid_constant__ ProjParams p) {
  using L = ProjLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffTmemSlot);
  int *abort_flag = reinterpret_cast<int *>(smem + L::kOffAbort);
  uint8_t *wb_s = smem + L::kOffWb;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c = p.c;
  const int slab_bytes = c * 128;               // one 64-column slab of W: c rows of 128 bytes
  const int zstage_bytes = kProjRows * c * 2;  // c/64 boxes of [128 rows][64 c]

  if (threadIdx.x == 0) {
    mbar_init(&bars[L::kBarW], 1);
    for (int s = 0; s < kProjZStages; ++s) {
      mbar_init(&bars[L::kBarZFull + s], 1);
      mbar_init(&bars[L::kBarZEmpty + s], 1);  // the MMA commit after the tile's last MMAs
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bars[L::kBarAccFull + h], 1);
      mbar_init(&bars[L::kBarAccEmpty + h], kProjRows);
    }
    mbar_init(&bars[L::kBarBiasSlot], kProjRows);
    mbar_init(&bars[L::kBarBiasFull], 1);
    mbar_init(&bars[L::kBarDrain], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // W_b^T into its swizzled K-major tile: element (h, k) in block k / 64, row
  // h, 16-byte granule ((k % 64) / 8) ^ (h % 8); rows h >= H are zero
  for (int i = threadIdx.x; i < 16 * c; i += kProjThreads) {
    const int hh = i / c, k = i % c;
    const uint16_t v = hh < kH ? p.wb[k * kH + hh] : uint16_t(0);
    *reinterpret_cast<uint16_t *>(wb_s + (k >> 6) * L::kWbChunkBytes + hh * 128 + ((((k & 63) >> 3) ^ (hh & 7)) << 4) +
                                  (k & 7) * 2) = v;
  }
  fence_proxy_async_smem();
  if (warp == 5) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&p.tm_z);
    tma_prefetch_desc(&p.tm_w);
  }
  if (warp == 0 && lane == 0)
    for (int m = 0; m < 4; ++m) tma_prefetch_desc(&p.tm_out[m]);
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
      mbar_arrive_expect_tx(&bars[L::kBarW], L::kSlabs * slab_bytes);
      for (int s = 0; s < L::kSlabs; ++s)
        tma_load_4d(smem + L::kOffW + s * slab_bytes, &p.tm_w, &bars[L::kBarW], s * 64, 0, 0, 0, pol_keep);
      bool ok = true;
      int it = 0;  // tiles issued
      for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x, ++it) {
        const int s = it % kProjZStages;
        if (it >= kProjZStages) ok = mbar_wait(&bars[L::kBarZEmpty + s], ((it / kProjZStages) - 1) & 1, wc);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars[L::kBarZFull + s], zstage_bytes);
        for (int bx = 0; bx < c / 64; ++bx)
          tma_load_4d(smem + L::kOffZ + s * L::kZStageMax + bx * (kProjRows * 128), &p.tm_z, &bars[L::kBarZFull + s],
                      bx * 64, tile * kProjRows, 0, 0, pol_stream);
      }
      // Let every copy already issued land before the CTA exits.
      mbar_wait(&bars[L::kBarW], 0, wc_drain);
      if (!ok)
        for (int s = 0; s < kProjZStages; ++s) {
          const int a = (it - s + kProjZStages - 1) / kProjZStages;
          if (a > 0) mbar_wait(&bars[L::kBarZFull + s], (a - 1) & 1, wc_drain);
        }
    }
  } else if (warp == 5) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kProjRows, 256, true);  // B (W) is MN-major
      const uint32_t sW = smem_u32(smem + L::kOffW);
      const uint32_t sZ = smem_u32(smem + L::kOffZ);
      constexpr uint32_t kHi = smem_desc_hi(1024, 2);  // 8-row atoms of 128 bytes, 128-byte swizzle
      bool ok = mbar_wait(&bars[L::kBarW], 0, wc);
      int it = 0;
      for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x, ++it) {
        const int s = it % kProjZStages;
        ok = mbar_wait(&bars[L::kBarZFull + s], (it / kProjZStages) & 1, wc);
        for (int hf = 0; hf < 2 && ok; ++hf) {
          if (it > 0) ok = mbar_wait(&bars[L::kBarAccEmpty + hf], (it - 1) & 1, wc);
          if (!ok) break;
          tc_fence_after_sync();
          const uint32_t zbase = sZ + s * L::kZStageMax;
          const uint32_t wlo = smem_desc_lo(sW + 4 * hf * slab_bytes, slab_bytes);
#pragma unroll 4
          for (int kk = 0; kk < c / 16; ++kk) {
            // A: c-chunk kk of the z tile (box kk/4, 32 bytes per K step inside a swizzle row)
            const uint32_t alo = smem_desc_lo(zbase + (kk >> 2) * (kProjRows * 128) + (kk & 3) * 32, 16);
            // B: rows 16 kk .. 16 kk + 15 of four W slabs (2 KB per K step)
            mma_bf16_ss(tmem + 256 * hf, desc_join(alo, kHi), desc_join(wlo + kk * 128, kHi), idesc,
                        kk > 0 ? 1u : 0u);
          }
          tc_commit(&bars[L::kBarAccFull + hf]);
        }
        // the bias columns, into the first 16 columns of q|k once the
        // epilogue has read them: A = the z tile, B = W_b^T (K-major)
        if (ok) ok = mbar_wait(&bars[L::kBarBiasSlot], it & 1, wc);
        if (ok) {
          tc_fence_after_sync();
          const uint32_t zbase = sZ + s * L::kZStageMax;
          const uint32_t sWb = smem_u32(smem + L::kOffWb);
          const uint32_t idesc_b = idesc_bf16_f32(kProjRows, 16, false);
#pragma unroll 4
          for (int kk = 0; kk < c / 16; ++kk) {
            const uint32_t alo = smem_desc_lo(zbase + (kk >> 2) * (kProjRows * 128) + (kk & 3) * 32, 16);
            const uint32_t blo = smem_desc_lo(sWb + (kk >> 2) * L::kWbChunkBytes + (kk & 3) * 32, 16);
            mma_bf16_ss(tmem, desc_join(alo, kHi), desc_join(blo, kHi), idesc_b, kk > 0 ? 1u : 0u);
          }
          tc_commit(&bars[L::kBarBiasFull]);
          tc_commit(&bars[L::kBarZEmpty + s]);
        }
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
      const int64_t r = int64_t(tile) * kProjRows + t;
      const bool live = r < p.rows;
      // q|k from half 0, v|g from half 1, as 32-column chunks: Tensor Memory ->
      // registers -> bf16 -> swizzled staging buffer -> one tensor store per
      // chunk (issued by thread 0 after a barrier of the four warps).
      for (int hf = 0; hf < 2 && ok; ++hf) {
        ok = __all_sync(0xffffffffu, mbar_wait<false>(&bars[L::kBarAccFull + hf], it & 1, wc));
        if (!ok) break;
        tc_fence_after_sync();
#pragma unroll 1
        for (int cc = 0; cc < 8; cc += 2) {
          uint32_t a[2][32];
          tmem_ld32(tmem + lane_base + 256 * hf + 32 * cc, a[0]);
          tmem_ld32(tmem + lane_base + 256 * hf + 32 * (cc + 1), a[1]);
          tmem_wait_ld();
          reg_fence(a[0]);
          reg_fence(a[1]);
          if (hf == 0 && cc == 0) {
            tc_fence_before_sync();
            mbar_arrive(&bars[L::kBarBiasSlot]);  // columns [0, 64) read: the bias MMAs may write there
          }
          if (hf == 1 && cc == 6) {
            tc_fence_before_sync();
            mbar_arrive(&bars[L::kBarAccEmpty + 1]);  // this half of Tensor Memory is free
          }
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int chunk = hf * 8 + cc + u;  // 0..15 over q|k|v|g
            uint8_t *buf = smem + L::kOffStage + (sc % L::kStageBufs) * L::kStageBytes;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint4 v = make_uint4(pack_bf16x2(__uint_as_float(a[u][8 * j]), __uint_as_float(a[u][8 * j + 1])),
                                         pack_bf16x2(__uint_as_float(a[u][8 * j + 2]), __uint_as_float(a[u][8 * j + 3])),
                                         pack_bf16x2(__uint_as_float(a[u][8 * j + 4]), __uint_as_float(a[u][8 * j + 5])),
                                         pack_bf16x2(__uint_as_float(a[u][8 * j + 6]), __uint_as_float(a[u][8 * j + 7])));
              *reinterpret_cast<uint4 *>(buf + t * 64 + ((j ^ ((t >> 1) & 3)) << 4)) = v;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              const int m = chunk >> 2;  // 0 q, 1 k, 2 v, 3 g
              const CUtensorMap *map = m == 0 ? &p.tm_out[0] : m == 1 ? &p.tm_out[1] : m == 2 ? &p.tm_out[2] : &p.tm_out[3];
              tma_store_4d(map, buf + warp * 2048, (chunk & 3) * 32, tile * kProjRows + warp * 32, 0, 0);
              bulk_commit_group();
              // the buffer the next chunk but one writes is free once this
              // chunk's predecessor has been read out
              bulk_wait_group_read<1>();
            }
            __syncwarp();
            ++sc;
          }
        }
        if (hf == 0) {
          // the row's bias values, then q|k's columns are free for the next tile
          ok = __all_sync(0xffffffffu, mbar_wait<false>(&bars[L::kBarBiasFull], it & 1, wc));
          if (!ok) break;
          tc_fence_after_sync();
          uint32_t bv[16];
          tmem_ld16(tmem + lane_base, bv);
          tmem_wait_ld();
          reg_fence(bv);
          tc_fence_before_sync();
          mbar_arrive(&bars[L::kBarAccEmpty + 0]);
          if (live)
#pragma unroll
            for (int h = 0; h < kH; ++h)
              p.bias[int64_t(h) * p.rows + r] = uint16_t(pack_bf16x2(__uint_as_float(bv[h]), 0.f) & 0xFFFFu);
        }
      }
    }
    if (lane == 0) bulk_wait_group_all();  // this warp's staging buffers are read and its rows written
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 5) tmem_dealloc(tmem, 512);
}

}  // namespace pba
