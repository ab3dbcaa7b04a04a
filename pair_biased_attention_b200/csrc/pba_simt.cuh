// pba_simt.cuh -- the CUDA-core kernels of the library:
//   * pba_attn_f32_kernel: pair-biased attention in fp32 for fp32 inputs
//     whose rows the tile loads cannot address (one warp per query row,
//     expf, fp32 accumulation); aligned fp32 inputs run on the tensor cores
//     (pba_attn_tf32_sm100.cuh).
//   * softmax_merge_kernel: the tiled-softmax merge of key-block partials
//     ("Fold-CP: A Context Parallelism Framework for Biomolecular Modeling",
//     Figure 2 (a) and (c)), a bandwidth-bound pass with 16-byte vector loads.
//   * pba_empty_keys_kernel: outputs for a call with no keys.
//   * pba_wait_selftest_kernel: exercises the bounded wait.
#pragma once

#include <cstdint>

#include "pba_ptx.cuh"

namespace pba {

struct SimtParams {
  int32_t B, H, Nq, Nk;
  float tau;
  const float *q, *k, *v, *bias;
  int64_t q_sb, q_sh, q_sn, k_sb, k_sh, k_sn, v_sb, v_sh, v_sn, bias_sb, bias_sh, bias_sn;
  const uint8_t *mask;
  int64_t mask_sb;
  float *out;  // forward O or partial O_p
  int64_t out_sb, out_sh, out_sn;
  float *lse;  // forward lse or partial m_p (nullable in forward)
  int64_t lse_sb, lse_sh, lse_sn;
  float *l_part;  // partial only
};

// One warp per (b, h, query row).  Keys are visited 32 at a time (lane = key
// inside the chunk); the running maximum m, sum l and output O (D/32 values
// per lane) follow the online softmax.
template <int D, bool kPartial>
__global__ void __launch_bounds__(128) pba_attn_f32_kernel(const SimtParams p) {
  constexpr int DPL = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t row = int64_t(blockIdx.x) * 4 + (threadIdx.x >> 5);
  const int64_t rows = int64_t(p.B) * p.H * p.Nq;
  if (row >= rows) return;
  const int i = int(row % p.Nq);
  const int64_t bh = row / p.Nq;
  const int h = int(bh % p.H);
  const int b = int(bh / p.H);

  float qv[D];
  const float *qp = p.q + b * p.q_sb + h * p.q_sh + int64_t(i) * p.q_sn;
#pragma unroll
  for (int d = 0; d < D; ++d) qv[d] = qp[d];
  const float *kb = p.k + b * p.k_sb + h * p.k_sh;
  const float *vb = p.v + b * p.v_sb + h * p.v_sh;
  const float *brow = p.bias + b * p.bias_sb + h * p.bias_sh + int64_t(i) * p.bias_sn;
  const uint8_t *mrow = p.mask ? p.mask + b * p.mask_sb : nullptr;

  float m = -INFINITY, l = 0.f;
  float o[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) o[e] = 0.f;

  for (int c0 = 0; c0 < p.Nk; c0 += 32) {
    const int key = c0 + lane;
    float s = -INFINITY;
    if (key < p.Nk && (mrow == nullptr || mrow[key] != 0)) {
      const float bij = brow[key];
      if (bij != -INFINITY) {
        const float *kr = kb + int64_t(key) * p.k_sn;
        float dot = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) dot = fmaf(qv[d], kr[d], dot);
        s = fmaf(p.tau, dot, bij);
      }
    }
    float cmax = s;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, off));
    if (cmax == -INFINITY) continue;
    const float m_new = fmaxf(m, cmax);
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
    const float pv = (s == -INFINITY) ? 0.f : expf(s - m_new);
    float psum = pv;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
    l = l * alpha + psum;
#pragma unroll
    for (int e = 0; e < DPL; ++e) o[e] *= alpha;
    const int nkeys = min(32, p.Nk - c0);
    for (int jj = 0; jj < nkeys; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, pv, jj);
      if (pj == 0.f) continue;
      const float *vr = vb + int64_t(c0 + jj) * p.v_sn;
#pragma unroll
      for (int e = 0; e < DPL; ++e) o[e] = fmaf(pj, vr[lane + 32 * e], o[e]);
    }
    m = m_new;
  }

  const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
  float *op = p.out + b * p.out_sb + h * p.out_sh + int64_t(i) * p.out_sn;
#pragma unroll
  for (int e = 0; e < DPL; ++e) op[lane + 32 * e] = o[e] * inv_l;
  if (lane == 0) {
    const int64_t li = b * p.lse_sb + h * p.lse_sh + int64_t(i) * p.lse_sn;
    if (kPartial) {
      p.lse[li] = (l > 0.f) ? m : -INFINITY;
      p.l_part[li] = l;
    } else if (p.lse != nullptr) {
      p.lse[li] = (l > 0.f) ? m + logf(l) : -INFINITY;
    }
  }
}

// Tiled-softmax merge.  Each thread owns 4 consecutive elements of one row
// (D/4 threads per row); the per-row maxima and weights are recomputed by each
// of those threads from the m_p, l_p values (cached loads).  kUnrollP > 0
// handles P <= kUnrollP with every partial's loads issued before any of the
// arithmetic (P independent 16-byte loads in flight per thread, which the
// bandwidth-bound pass needs); kUnrollP = 0 is the loop for any P.  Four
// resident blocks per SM (at most 64 registers): the pass is latency-bound
// on its loads, and 32 warps per SM keep more of them in flight than the 24
// that 77 registers allowed (ring8k merge 65.5 -> 56.4 us).
template <bool kOutBf16, int kUnrollP>
__global__ void __launch_bounds__(256, 4) softmax_merge_kernel(int P, int64_t rows, int D, const float *o_parts,
                                                            const float *m_parts, const float *l_parts, void *out,
                                                            float *lse) {
  const int tpr = D >> 2;
  const int64_t total = rows * tpr;
  for (int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = idx / tpr;
    const int c = int(idx - r * tpr);
    float M = -INFINITY;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float Lsum = 0.f;
    if (kUnrollP > 0) {
      float lp[kUnrollP > 0 ? kUnrollP : 1], mp[kUnrollP > 0 ? kUnrollP : 1];
      float4 ov[kUnrollP > 0 ? kUnrollP : 1];
#pragma unroll
      for (int pp = 0; pp < kUnrollP; ++pp) {
        if (pp < P) {
          lp[pp] = __ldg(l_parts + int64_t(pp) * rows + r);
          mp[pp] = __ldg(m_parts + int64_t(pp) * rows + r);
          ov[pp] = __ldcs(reinterpret_cast<const float4 *>(o_parts + (int64_t(pp) * rows + r) * D) + c);
        } else {
          lp[pp] = 0.f;
          mp[pp] = -INFINITY;
          ov[pp] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int pp = 0; pp < kUnrollP; ++pp)
        if (lp[pp] > 0.f && mp[pp] > M) M = mp[pp];
      if (M != -INFINITY) {
#pragma unroll
        for (int pp = 0; pp < kUnrollP; ++pp) {
          if (!(lp[pp] > 0.f)) continue;  // an empty block adds nothing, whatever its O holds
          const float wgt = lp[pp] * expf(mp[pp] - M);
          Lsum += wgt;
          acc.x = fmaf(wgt, ov[pp].x, acc.x);
          acc.y = fmaf(wgt, ov[pp].y, acc.y);
          acc.z = fmaf(wgt, ov[pp].z, acc.z);
          acc.w = fmaf(wgt, ov[pp].w, acc.w);
        }
      }
    } else {
      for (int pp = 0; pp < P; ++pp) {
        const float lp = __ldg(l_parts + int64_t(pp) * rows + r);
        const float mp = __ldg(m_parts + int64_t(pp) * rows + r);
        if (lp > 0.f && mp > M) M = mp;
      }
      if (M != -INFINITY) {
        for (int pp = 0; pp < P; ++pp) {
          const float lp = __ldg(l_parts + int64_t(pp) * rows + r);
          if (!(lp > 0.f)) continue;
          const float wgt = lp * expf(__ldg(m_parts + int64_t(pp) * rows + r) - M);
          const float4 ov = __ldcs(reinterpret_cast<const float4 *>(o_parts + (int64_t(pp) * rows + r) * D) + c);
          Lsum += wgt;
          acc.x = fmaf(wgt, ov.x, acc.x);
          acc.y = fmaf(wgt, ov.y, acc.y);
          acc.z = fmaf(wgt, ov.z, acc.z);
          acc.w = fmaf(wgt, ov.w, acc.w);
        }
      }
    }
    const float inv = (Lsum > 0.f) ? 1.f / Lsum : 0.f;
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
    if (kOutBf16) {
      uint2 pk = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
      reinterpret_cast<uint2 *>(static_cast<uint16_t *>(out) + r * D)[c] = pk;
    } else {
      reinterpret_cast<float4 *>(static_cast<float *>(out) + r * D)[c] = acc;
    }
    if (c == 0 && lse != nullptr) lse[r] = (Lsum > 0.f) ? M + logf(Lsum) : -INFINITY;
  }
}

// Outputs of a call with no keys: every row is empty.
struct EmptyParams {
  int32_t B, H, Nq, D;
  int32_t out_bf16;  // forward out dtype
  int32_t partial;
  void *out;
  int64_t out_sb, out_sh, out_sn;
  float *lse;  // forward lse or partial m_p
  int64_t lse_sb, lse_sh, lse_sn;
  float *l_part;
};

__global__ void pba_empty_keys_kernel(const EmptyParams p) {
  const int64_t rows = int64_t(p.B) * p.H * p.Nq;
  for (int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < rows * p.D;
       idx += int64_t(gridDim.x) * blockDim.x) {
    const int64_t row = idx / p.D;
    const int d = int(idx - row * p.D);
    const int i = int(row % p.Nq);
    const int64_t bh = row / p.Nq;
    const int h = int(bh % p.H), b = int(bh / p.H);
    const int64_t o = b * p.out_sb + h * p.out_sh + int64_t(i) * p.out_sn + d;
    if (p.out_bf16)
      static_cast<uint16_t *>(p.out)[o] = 0;
    else
      static_cast<float *>(p.out)[o] = 0.f;
    if (d == 0) {
      const int64_t li = b * p.lse_sb + h * p.lse_sh + int64_t(i) * p.lse_sn;
      if (p.lse) p.lse[li] = -INFINITY;
      if (p.partial) p.l_part[li] = 0.f;
    }
  }
}

// Applies the attention kernel's software exp2 (exp2_poly2) to n values.
__global__ void pba_exp2_selftest_kernel(const float *in, float *out, int64_t n) {
  for (int64_t i = 2 * (int64_t(blockIdx.x) * blockDim.x + threadIdx.x); i < n;
       i += 2 * int64_t(gridDim.x) * blockDim.x) {
    const float2 r = exp2_poly2(make_float2(in[i], i + 1 < n ? in[i + 1] : 0.f));
    out[i] = r.x;
    if (i + 1 < n) out[i + 1] = r.y;
  }
}

// Waits on a barrier that no thread ever completes; the bounded wait must give
// up after timeout_ns and record kErrTimeout.
__global__ void pba_wait_selftest_kernel(int *err, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const WaitCtl wc{&abort_flag, err, timeout_ns};
  mbar_wait(&bar, 0, wc);
  __syncthreads();
}

}  // namespace pba
