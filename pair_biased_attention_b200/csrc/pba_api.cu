// pba_api.cu -- the C ABI declared in include/pba.h: argument checks, Tensor
// Memory Accelerator descriptors and kernel launches.  Every step of the
// computation runs in the kernels of pba_attn_sm100.cuh and pba_simt.cuh.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "pba.h"
#include "pba_attn_sm100.cuh"
#include "pba_attn_tf32_sm100.cuh"
#include "pba_proj_sm100.cuh"
#include "pba_oproj_sm100.cuh"
#include "pba_pwa_sm100.cuh"
#include "pba_bwd_sm100.cuh"
#include "pba_simt.cuh"

// Device error word: written by kernels whose bounded waits ran out, read and
// cleared by pba_last_device_error().
__device__ int g_pba_err = 0;

// pba_last_device_error takes the word with one atomic exchange on the device
// (so an error recorded between a read and a separate clear is never lost)
// into one of these slots; concurrent callers use different slots.
constexpr int kErrTakeSlots = 64;
__device__ int g_pba_err_taken[kErrTakeSlots];
__global__ void pba_take_error_kernel(int slot) { g_pba_err_taken[slot] = atomicExch(&g_pba_err, 0); }

namespace {

constexpr uint64_t kDefaultTimeoutNs = 1000000000ull;
std::atomic<uint64_t> g_timeout_ns{kDefaultTimeoutNs};

using EncodeTiledFn = PFN_cuTensorMapEncodeTiled_v12000;

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

pba_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PBA_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return PBA_ERR_CUDA;
  if (major != 10 || minor != 0) return PBA_ERR_UNSUPPORTED;  // built for sm_100a only
  return PBA_OK;
}

int *device_error_word() {
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_pba_err) != cudaSuccess) return nullptr;
  return static_cast<int *>(p);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// One-time per-device kernel set-up (the dynamic shared memory limit is a
// per-device attribute of a kernel): `setup` runs once for each device it is
// called on, with that device current, and its result is kept per device.
constexpr int kMaxDevices = 64;
struct PerDeviceOnce {
  std::once_flag flag[kMaxDevices];
  cudaError_t err[kMaxDevices] = {};
};
template <typename F>
cudaError_t once_per_device(PerDeviceOnce &o, F &&setup) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(o.flag[dev], [&] { o.err[dev] = setup(); });
  return o.err[dev];
}

constexpr int64_t kMaxI32 = 2147483647;

// 4-D tiled tensor map of bf16 (or, with f32, fp32) elements.  dims/strides
// innermost first; strides in bytes for dims 1..3.  A dim of extent 1 gets a
// harmless positive stride (its coordinate is always 0).
bool make_map(CUtensorMap *map, const void *base, const uint64_t dims[4], const int64_t strides_bytes[3],
              const uint32_t box[4], CUtensorMapSwizzle swizzle, bool f32 = false) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t gdim[4] = {dims[0], dims[1], dims[2], dims[3]};
  cuuint64_t gstride[3];
  int64_t prev_extent = int64_t(dims[0]) * (f32 ? 4 : 2);
  for (int i = 0; i < 3; ++i) {
    int64_t s = strides_bytes[i];
    if (dims[i + 1] == 1 || s <= 0) s = (prev_extent + 15) / 16 * 16;
    gstride[i] = cuuint64_t(s);
    prev_extent = s * int64_t(dims[i + 1]);
  }
  cuuint32_t bdim[4] = {box[0], box[1], box[2], box[3]};
  cuuint32_t estride[4] = {1, 1, 1, 1};
  CUresult r = enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), gdim, gstride, bdim, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool stride_ok_bf16(int64_t s, int64_t extent) { return extent <= 1 || (s > 0 && s % 8 == 0); }
bool stride_ok_f32(int64_t s, int64_t extent) { return extent <= 1 || (s > 0 && s % 4 == 0); }

// ------------------------------------------------------------ tensor-core path
struct TcProblem {
  int B, H, Nq, Nk, D;
  float tau;
  const void *q, *k, *v, *bias;
  int64_t q_s[3], k_s[3], v_s[3];  // (b, h, n) elements
  // bias: either [query][key] rows (bias_t = false) or [key][query] rows (true)
  bool bias_t;
  int64_t bias_s[3];  // (b, h, row) elements
  bool bias_b_bcast, bias_h_bcast;
  const uint8_t *mask;
  int64_t mask_sb, mask_sk;
  int epi;  // pba::kEpiForward / kEpiPartial
  void *out;
  int64_t out_s[3];
  float *lse;
  int64_t lse_s[3];
  float *l_part;
  const void *gate;
  int64_t gate_s[3];
};

template <int D, bool kBiasT, int kEpi, bool kGate, bool kMasked>
cudaError_t launch_tc(const pba::AttnParams &p, int grid, cudaStream_t stream) {
  using L = pba::AttnLayout<D>;
  auto kern = pba::pba_attn_sm100_kernel<D, kBiasT, kEpi, kGate, kMasked>;
  static PerDeviceOnce once;
  const cudaError_t attr_err = once_per_device(once, [&] {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemAlloc);
    // The kernel moves registers between its warpgroups with setmaxnreg; the
    // split must fit in what the block is launched with, or the increase
    // would wait forever.  Refuse to launch a build where it would not.
    cudaFuncAttributes fa;
    if (e == cudaSuccess && cudaFuncGetAttributes(&fa, kern) == cudaSuccess &&
        fa.numRegs * pba::kAttnThreads < pba::kRegSplitTotal)
      e = cudaErrorInvalidConfiguration;
    return e;
  });
  if (attr_err != cudaSuccess) return attr_err;
  kern<<<grid, pba::kAttnThreads, L::kSmemAlloc, stream>>>(p);
  return cudaGetLastError();
}

// Instantiations: untransposed bias tiles with and without key masking
// (masked keys and a ragged key tail are applied as mask words), transposed
// bias tiles (triangle attention, ending node; masking by the mask warp).
template <int D>
cudaError_t dispatch_tc(const pba::AttnParams &p, int grid, bool bias_t, int epi, bool gate, cudaStream_t st) {
  const bool m = p.needs_mask != 0;
  if (epi == pba::kEpiPartial)
    return m ? launch_tc<D, false, pba::kEpiPartial, false, true>(p, grid, st)
             : launch_tc<D, false, pba::kEpiPartial, false, false>(p, grid, st);
  if (bias_t)
    return gate ? launch_tc<D, true, pba::kEpiForward, true, false>(p, grid, st)
                : launch_tc<D, true, pba::kEpiForward, false, false>(p, grid, st);
  if (gate)
    return m ? launch_tc<D, false, pba::kEpiForward, true, true>(p, grid, st)
             : launch_tc<D, false, pba::kEpiForward, true, false>(p, grid, st);
  return m ? launch_tc<D, false, pba::kEpiForward, false, true>(p, grid, st)
           : launch_tc<D, false, pba::kEpiForward, false, false>(p, grid, st);
}

pba_status run_tc(const TcProblem &t, cudaStream_t stream) {
  pba::AttnParams p;
  std::memset(&p, 0, sizeof(p));
  const uint32_t qbox[4] = {uint32_t(t.D), uint32_t(pba::kBM), 1, 1};
  const uint32_t kbox[4] = {uint32_t(t.D), uint32_t(pba::kBN), 1, 1};
  const CUtensorMapSwizzle swz = (t.D == 64) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  {
    const uint64_t dims[4] = {uint64_t(t.D), uint64_t(t.Nq), uint64_t(t.H), uint64_t(t.B)};
    const int64_t st[3] = {t.q_s[2] * 2, t.q_s[1] * 2, t.q_s[0] * 2};
    if (!make_map(&p.tm_q, t.q, dims, st, qbox, swz)) return PBA_ERR_INVALID_ARG;
  }
  {
    const uint64_t dims[4] = {uint64_t(t.D), uint64_t(t.Nk), uint64_t(t.H), uint64_t(t.B)};
    const int64_t sk[3] = {t.k_s[2] * 2, t.k_s[1] * 2, t.k_s[0] * 2};
    const int64_t sv[3] = {t.v_s[2] * 2, t.v_s[1] * 2, t.v_s[0] * 2};
    if (!make_map(&p.tm_k, t.k, dims, sk, kbox, swz)) return PBA_ERR_INVALID_ARG;
    if (!make_map(&p.tm_v, t.v, dims, sv, kbox, swz)) return PBA_ERR_INVALID_ARG;
  }
  {
    const uint64_t hb = t.bias_h_bcast ? 1 : uint64_t(t.H), bb = t.bias_b_bcast ? 1 : uint64_t(t.B);
    const int64_t st[3] = {t.bias_s[2] * 2, t.bias_s[1] * 2, t.bias_s[0] * 2};
    if (t.bias_t) {
      const uint64_t dims[4] = {uint64_t(t.Nq), uint64_t(t.Nk), hb, bb};
      const uint32_t box[4] = {uint32_t(pba::kBM), uint32_t(pba::kBN), 1, 1};
      if (!make_map(&p.tm_bias, t.bias, dims, st, box, CU_TENSOR_MAP_SWIZZLE_NONE)) return PBA_ERR_INVALID_ARG;
    } else {
      const uint64_t dims[4] = {uint64_t(t.Nk), uint64_t(t.Nq), hb, bb};
      const uint32_t box[4] = {64, uint32_t(pba::kBM), 1, 1};
      if (!make_map(&p.tm_bias, t.bias, dims, st, box, CU_TENSOR_MAP_SWIZZLE_128B)) return PBA_ERR_INVALID_ARG;
    }
  }
  if (t.D == 32 && t.epi == pba::kEpiForward) {
    // the bf16 output rows, stored by warps of 32 rows from the staging buffer
    const uint64_t dims[4] = {uint64_t(t.D), uint64_t(t.Nq), uint64_t(t.H), uint64_t(t.B)};
    const int64_t st[3] = {t.out_s[2] * 2, t.out_s[1] * 2, t.out_s[0] * 2};
    const uint32_t box[4] = {32, 32, 1, 1};
    if (!make_map(&p.tm_out, t.out, dims, st, box, CU_TENSOR_MAP_SWIZZLE_64B)) return PBA_ERR_INVALID_ARG;
  }
  p.B = t.B;
  p.H = t.H;
  p.Nq = t.Nq;
  p.Nk = t.Nk;
  p.n_qblocks = (t.Nq + pba::kQTiles * pba::kBM - 1) / (pba::kQTiles * pba::kBM);
  const int64_t n_units = int64_t(t.B) * t.H * p.n_qblocks;
  if (n_units > kMaxI32) return PBA_ERR_INVALID_ARG;
  p.n_units = int(n_units);
  p.bias_h_bcast = t.bias_h_bcast;
  p.bias_b_bcast = t.bias_b_bcast;
  p.needs_mask = (t.mask != nullptr) || (t.Nk % pba::kBN != 0);
  p.mask_vec4 = t.mask != nullptr && t.mask_sk == 1 && (reinterpret_cast<uintptr_t>(t.mask) & 3u) == 0 &&
                t.mask_sb % 4 == 0;
  p.tau = t.tau;
  p.mask = t.mask;
  p.mask_sb = t.mask_sb;
  p.mask_sk = t.mask_sk;
  p.out = t.out;
  p.out_sb = t.out_s[0];
  p.out_sh = t.out_s[1];
  p.out_sn = t.out_s[2];
  p.lse = t.lse;
  p.lse_sb = t.lse_s[0];
  p.lse_sh = t.lse_s[1];
  p.lse_sn = t.lse_s[2];
  p.l_part = t.l_part;
  p.gate = static_cast<const uint16_t *>(t.gate);
  p.gate_sb = t.gate_s[0];
  p.gate_sh = t.gate_s[1];
  p.gate_sn = t.gate_s[2];
  p.err = device_error_word();
  if (p.err == nullptr) return PBA_ERR_CUDA;
  p.timeout_ns = g_timeout_ns.load();
  // persistent: one CTA per SM (each needs most of the SM's shared memory)
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return PBA_ERR_CUDA;
#ifndef PBA_PERSISTENT_GRID
#define PBA_PERSISTENT_GRID 1
#endif
  const int64_t grid = (PBA_PERSISTENT_GRID && n_units > sms) ? sms : n_units;
  cudaError_t e = (t.D == 64) ? dispatch_tc<64>(p, int(grid), t.bias_t, t.epi, t.gate != nullptr, stream)
                              : dispatch_tc<32>(p, int(grid), t.bias_t, t.epi, t.gate != nullptr, stream);
  return e == cudaSuccess ? PBA_OK : PBA_ERR_CUDA;
}

// ------------------------------------------------------------ fp32 on the tensor cores
template <int D, bool kPartial, bool kMasked>
cudaError_t launch_tf32(const pba::Tf32Params &p, int64_t grid, cudaStream_t stream) {
  using L = pba::Tf32Layout<D>;
  auto kern = pba::pba_attn_tf32_sm100_kernel<D, kPartial, kMasked>;
  static PerDeviceOnce once;
  const cudaError_t attr_err = once_per_device(once, [&] {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemAlloc);
    // the warpgroup register split must fit in what the block is launched with
    cudaFuncAttributes fa;
    if (e == cudaSuccess && cudaFuncGetAttributes(&fa, kern) == cudaSuccess &&
        fa.numRegs * pba::kTfThreads < pba::kTfRegSplitTotal)
      e = cudaErrorInvalidConfiguration;
    return e;
  });
  if (attr_err != cudaSuccess) return attr_err;
  kern<<<unsigned(grid), pba::kTfThreads, L::kSmemAlloc, stream>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t dispatch_tf32(const pba::Tf32Params &p, int64_t grid, bool partial, bool masked, cudaStream_t st) {
  if (partial) return masked ? launch_tf32<D, true, true>(p, grid, st) : launch_tf32<D, true, false>(p, grid, st);
  return masked ? launch_tf32<D, false, true>(p, grid, st) : launch_tf32<D, false, false>(p, grid, st);
}

// fp32 inputs whose tiles the Tensor Memory Accelerator can load (16-byte
// aligned bases and row strides) run on the tensor cores; the caller routes
// the others to the CUDA-core kernel.
bool tf32_layout_ok(const pba_attn_desc *d, const void *q, const void *k, const void *v, const void *bias,
                    const void *out) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(bias) || !aligned16(out)) return false;
  const int64_t *qs = d->q_stride, *ks = d->k_stride, *vs = d->v_stride, *bs = d->bias_stride, *os = d->out_stride;
  if (!stride_ok_f32(qs[0], d->B) || !stride_ok_f32(qs[1], d->H) || !stride_ok_f32(qs[2], d->Nq) ||
      !stride_ok_f32(ks[0], d->B) || !stride_ok_f32(ks[1], d->H) || !stride_ok_f32(ks[2], d->Nk) ||
      !stride_ok_f32(vs[0], d->B) || !stride_ok_f32(vs[1], d->H) || !stride_ok_f32(vs[2], d->Nk) ||
      !stride_ok_f32(bs[2], d->Nq))
    return false;
  if ((bs[0] != 0 && !stride_ok_f32(bs[0], d->B)) || (bs[1] != 0 && !stride_ok_f32(bs[1], d->H))) return false;
  for (int i = 0; i < 3; ++i)
    if (os[i] % 4 != 0) return false;  // 16-byte stores of whole output rows
  return true;
}

pba_status run_tf32(const pba_attn_desc *d, float tau, const void *q, const void *k, const void *v, const void *bias,
                    const uint8_t *mask, bool partial, void *out, float *lse, float *l_part, cudaStream_t stream) {
  pba::Tf32Params p;
  std::memset(&p, 0, sizeof(p));
  const int64_t B = d->B, H = d->H, Nq = d->Nq, Nk = d->Nk, D = d->D;
  const int64_t *qs = d->q_stride, *ks = d->k_stride, *vs = d->v_stride, *bs = d->bias_stride;
  {
    // Q, K, V [B][H][n][D] as (D, n, H, B): 32-feature boxes of 128 query / 64 key rows
    const uint64_t dq[4] = {uint64_t(D), uint64_t(Nq), uint64_t(H), uint64_t(B)};
    const uint64_t dk[4] = {uint64_t(D), uint64_t(Nk), uint64_t(H), uint64_t(B)};
    const int64_t sq[3] = {qs[2] * 4, qs[1] * 4, qs[0] * 4};
    const int64_t sk[3] = {ks[2] * 4, ks[1] * 4, ks[0] * 4};
    const int64_t sv[3] = {vs[2] * 4, vs[1] * 4, vs[0] * 4};
    const uint32_t qbox[4] = {32, uint32_t(pba::kTfBM), 1, 1};
    const uint32_t kbox[4] = {32, uint32_t(pba::kTfBN), 1, 1};
    if (!make_map(&p.tm_q, q, dq, sq, qbox, CU_TENSOR_MAP_SWIZZLE_128B, true) ||
        !make_map(&p.tm_k, k, dk, sk, kbox, CU_TENSOR_MAP_SWIZZLE_128B, true) ||
        !make_map(&p.tm_v, v, dk, sv, kbox, CU_TENSOR_MAP_SWIZZLE_128B, true))
      return PBA_ERR_INVALID_ARG;
  }
  {
    // bias [B|1][H|1][Nq][Nk] as (keys, rows, H, B): 32-key boxes of 128 rows
    const uint64_t hb = bs[1] == 0 ? 1 : uint64_t(H), bb = bs[0] == 0 ? 1 : uint64_t(B);
    const uint64_t dims[4] = {uint64_t(Nk), uint64_t(Nq), hb, bb};
    const int64_t st[3] = {bs[2] * 4, bs[1] * 4, bs[0] * 4};
    const uint32_t box[4] = {32, uint32_t(pba::kTfBM), 1, 1};
    if (!make_map(&p.tm_bias, bias, dims, st, box, CU_TENSOR_MAP_SWIZZLE_128B, true)) return PBA_ERR_INVALID_ARG;
  }
  p.B = int(B);
  p.H = int(H);
  p.Nq = int(Nq);
  p.Nk = int(Nk);
  p.n_qblocks = int((Nq + pba::kTfBM - 1) / pba::kTfBM);
  const int64_t grid = B * H * p.n_qblocks;
  if (grid > kMaxI32) return PBA_ERR_INVALID_ARG;
  p.bias_h_bcast = bs[1] == 0;
  p.bias_b_bcast = bs[0] == 0;
  p.mask = mask;
  p.mask_sb = d->mask_stride_b;
  p.mask_vec16 = mask != nullptr && aligned16(mask) && (B == 1 || d->mask_stride_b % 16 == 0);
  p.tau = tau;
  p.out = static_cast<float *>(out);
  p.out_sb = d->out_stride[0];
  p.out_sh = d->out_stride[1];
  p.out_sn = d->out_stride[2];
  p.lse = lse;
  p.lse_sb = d->lse_stride[0];
  p.lse_sh = d->lse_stride[1];
  p.lse_sn = d->lse_stride[2];
  p.l_part = l_part;
  p.err = device_error_word();
  if (p.err == nullptr) return PBA_ERR_CUDA;
  p.timeout_ns = g_timeout_ns.load();
  const bool masked = mask != nullptr || Nk % pba::kTfBN != 0;
  const cudaError_t e = (D == 64) ? dispatch_tf32<64>(p, grid, partial, masked, stream)
                                  : dispatch_tf32<32>(p, grid, partial, masked, stream);
  return e == cudaSuccess ? PBA_OK : PBA_ERR_CUDA;
}

// ------------------------------------------------------------ shared checks
pba_status check_desc(const pba_attn_desc *d) {
  if (d == nullptr) return PBA_ERR_INVALID_ARG;
  if (d->B < 1 || d->H < 1 || d->Nq < 0 || d->Nk < 0) return PBA_ERR_INVALID_ARG;
  if (d->B > kMaxI32 || d->H > kMaxI32 || d->Nq > kMaxI32 || d->Nk > kMaxI32) return PBA_ERR_INVALID_ARG;
  if (d->dtype != PBA_BF16 && d->dtype != PBA_F32) return PBA_ERR_UNSUPPORTED;
  if (d->D != 32 && d->D != 64) return PBA_ERR_UNSUPPORTED;
  if (!(d->softmax_scale >= 0.f) || std::isinf(d->softmax_scale)) return PBA_ERR_INVALID_ARG;
  return PBA_OK;
}

float tau_of(float scale, int64_t D) { return scale > 0.f ? scale : float(1.0 / std::sqrt(double(D))); }

pba_status launch_empty(const pba_attn_desc *d, bool partial, void *out, float *lse, float *l_part,
                        cudaStream_t stream) {
  pba::EmptyParams e;
  e.B = int(d->B);
  e.H = int(d->H);
  e.Nq = int(d->Nq);
  e.D = int(d->D);
  e.out_bf16 = (!partial && d->dtype == PBA_BF16) ? 1 : 0;
  e.partial = partial ? 1 : 0;
  e.out = out;
  e.out_sb = d->out_stride[0];
  e.out_sh = d->out_stride[1];
  e.out_sn = d->out_stride[2];
  e.lse = lse;
  e.lse_sb = d->lse_stride[0];
  e.lse_sh = d->lse_stride[1];
  e.lse_sn = d->lse_stride[2];
  e.l_part = l_part;
  pba::pba_empty_keys_kernel<<<296, 256, 0, stream>>>(e);
  return cudaGetLastError() == cudaSuccess ? PBA_OK : PBA_ERR_CUDA;
}

pba_status attn_common(const pba_attn_desc *d, const void *q, const void *k, const void *v, const void *bias,
                       const uint8_t *mask, bool partial, void *out, float *lse, float *l_part, void *stream_ptr) {
  pba_status s = check_desc(d);
  if (s != PBA_OK) return s;
  // a pointer may be NULL only when the tensor it stands for has no element
  const bool has_q = d->Nq > 0, has_k = d->Nk > 0;
  if ((has_q && (q == nullptr || out == nullptr)) || (has_k && (k == nullptr || v == nullptr)) ||
      (has_q && has_k && bias == nullptr))
    return PBA_ERR_INVALID_ARG;
  if (has_q && partial && (lse == nullptr || l_part == nullptr)) return PBA_ERR_INVALID_ARG;
  s = check_device();
  if (s != PBA_OK) return s;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  if (d->Nq == 0) return PBA_OK;
  if (d->Nk == 0) return launch_empty(d, partial, out, lse, l_part, stream);
  const float tau = tau_of(d->softmax_scale, d->D);

  if (d->dtype == PBA_F32 && tf32_layout_ok(d, q, k, v, bias, out))
    return run_tf32(d, tau, q, k, v, bias, mask, partial, out, lse, l_part, stream);
  if (d->dtype == PBA_F32) {
    // rows the tile loads cannot address: one warp per query row on the CUDA cores
    pba::SimtParams p;
    p.B = int(d->B);
    p.H = int(d->H);
    p.Nq = int(d->Nq);
    p.Nk = int(d->Nk);
    p.tau = tau;
    p.q = static_cast<const float *>(q);
    p.k = static_cast<const float *>(k);
    p.v = static_cast<const float *>(v);
    p.bias = static_cast<const float *>(bias);
    p.q_sb = d->q_stride[0], p.q_sh = d->q_stride[1], p.q_sn = d->q_stride[2];
    p.k_sb = d->k_stride[0], p.k_sh = d->k_stride[1], p.k_sn = d->k_stride[2];
    p.v_sb = d->v_stride[0], p.v_sh = d->v_stride[1], p.v_sn = d->v_stride[2];
    p.bias_sb = d->bias_stride[0], p.bias_sh = d->bias_stride[1], p.bias_sn = d->bias_stride[2];
    p.mask = mask;
    p.mask_sb = d->mask_stride_b;
    p.out = static_cast<float *>(out);
    p.out_sb = d->out_stride[0], p.out_sh = d->out_stride[1], p.out_sn = d->out_stride[2];
    p.lse = lse;
    p.lse_sb = d->lse_stride[0], p.lse_sh = d->lse_stride[1], p.lse_sn = d->lse_stride[2];
    p.l_part = l_part;
    const int64_t rows = d->B * d->H * d->Nq;
    const int64_t grid = (rows + 3) / 4;
    if (grid > kMaxI32) return PBA_ERR_INVALID_ARG;
    if (d->D == 64) {
      if (partial)
        pba::pba_attn_f32_kernel<64, true><<<int(grid), 128, 0, stream>>>(p);
      else
        pba::pba_attn_f32_kernel<64, false><<<int(grid), 128, 0, stream>>>(p);
    } else {
      if (partial)
        pba::pba_attn_f32_kernel<32, true><<<int(grid), 128, 0, stream>>>(p);
      else
        pba::pba_attn_f32_kernel<32, false><<<int(grid), 128, 0, stream>>>(p);
    }
    return cudaGetLastError() == cudaSuccess ? PBA_OK : PBA_ERR_CUDA;
  }

  // bf16 on the tensor cores: tile loads need 16-byte aligned bases and strides
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(bias) || !aligned16(out))
    return PBA_ERR_INVALID_ARG;
  const int64_t *qs = d->q_stride, *ks = d->k_stride, *vs = d->v_stride, *bs = d->bias_stride;
  if (!stride_ok_bf16(qs[0], d->B) || !stride_ok_bf16(qs[1], d->H) || !stride_ok_bf16(qs[2], d->Nq) ||
      !stride_ok_bf16(ks[0], d->B) || !stride_ok_bf16(ks[1], d->H) || !stride_ok_bf16(ks[2], d->Nk) ||
      !stride_ok_bf16(vs[0], d->B) || !stride_ok_bf16(vs[1], d->H) || !stride_ok_bf16(vs[2], d->Nk) ||
      !stride_ok_bf16(bs[2], d->Nq))
    return PBA_ERR_INVALID_ARG;
  if ((bs[0] != 0 && !stride_ok_bf16(bs[0], d->B)) || (bs[1] != 0 && !stride_ok_bf16(bs[1], d->H)))
    return PBA_ERR_INVALID_ARG;
  // outputs: 16-byte vector stores of whole rows
  const int64_t out_mult = partial ? 4 : 8;
  for (int i = 0; i < 3; ++i)
    if (d->out_stride[i] % out_mult != 0) return PBA_ERR_INVALID_ARG;
  TcProblem t;
  std::memset(&t, 0, sizeof(t));
  t.B = int(d->B);
  t.H = int(d->H);
  t.Nq = int(d->Nq);
  t.Nk = int(d->Nk);
  t.D = int(d->D);
  t.tau = tau;
  t.q = q;
  t.k = k;
  t.v = v;
  t.bias = bias;
  for (int i = 0; i < 3; ++i) {
    t.q_s[i] = qs[i];
    t.k_s[i] = ks[i];
    t.v_s[i] = vs[i];
    t.bias_s[i] = bs[i];
    t.out_s[i] = d->out_stride[i];
    t.lse_s[i] = d->lse_stride[i];
  }
  t.bias_t = false;
  t.bias_b_bcast = bs[0] == 0;
  t.bias_h_bcast = bs[1] == 0;
  t.mask = mask;
  t.mask_sb = d->mask_stride_b;
  t.mask_sk = 1;
  t.epi = partial ? pba::kEpiPartial : pba::kEpiForward;
  t.out = out;
  t.lse = lse;
  t.l_part = l_part;
  t.gate = nullptr;
  return run_tc(t, stream);
}

// ------------------------------------------------------------ triangle projections
template <int kH>
cudaError_t launch_proj(const pba::ProjParams &p, int grid, cudaStream_t stream) {
  auto kern = pba::pba_proj_sm100_kernel<kH>;
  static PerDeviceOnce once;
  const cudaError_t attr_err = once_per_device(
      once, [&] { return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pba::ProjLayout::kSmemAlloc); });
  if (attr_err != cudaSuccess) return attr_err;
  kern<<<grid, pba::kProjThreads, pba::ProjLayout::kSmemAlloc, stream>>>(p);
  return cudaGetLastError();
}

template <int kC>
cudaError_t launch_oproj(const pba::OprojParams &p, int grid, cudaStream_t stream) {
  using L = pba::OprojLayout<kC>;
  auto kern = pba::pba_oproj_sm100_kernel<kC>;
  static PerDeviceOnce once;
  const cudaError_t attr_err = once_per_device(
      once, [&] { return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemAlloc); });
  if (attr_err != cudaSuccess) return attr_err;
  kern<<<grid, pba::kOprojThreads, L::kSmemAlloc, stream>>>(p);
  return cudaGetLastError();
}

// ------------------------------------------------------------ pair weighted averaging
template <int D, bool kGate, bool kMasked>
cudaError_t launch_pwa(const pba::PwaParams &p, int grid, cudaStream_t stream) {
  using L = pba::PwaLayout<D>;
  auto kern = pba::pba_pwa_sm100_kernel<D, kGate, kMasked>;
  static PerDeviceOnce once;
  const cudaError_t attr_err = once_per_device(
      once, [&] { return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemAlloc); });
  if (attr_err != cudaSuccess) return attr_err;
  kern<<<grid, pba::kPwaThreads, L::kSmemAlloc, stream>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t dispatch_pwa(const pba::PwaParams &p, int grid, bool gate, cudaStream_t st) {
  const bool m = p.masked != 0;
  if (gate) return m ? launch_pwa<D, true, true>(p, grid, st) : launch_pwa<D, true, false>(p, grid, st);
  return m ? launch_pwa<D, false, true>(p, grid, st) : launch_pwa<D, false, false>(p, grid, st);
}

// ------------------------------------------------------------ backward
template <int D, bool kB>
cudaError_t launch_bwd(const pba::BwdParams &p, int grid, cudaStream_t stream) {
  using L = pba::BwdLayout<D>;
  auto kern = pba::pba_bwd_sm100_kernel<D, kB>;
  static PerDeviceOnce once;
  const cudaError_t attr_err = once_per_device(once, [&] {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemAlloc);
    // the register split must fit in what the block is launched with (see launch_tc)
    cudaFuncAttributes fa;
    if (e == cudaSuccess && cudaFuncGetAttributes(&fa, kern) == cudaSuccess &&
        fa.numRegs * pba::kBwdThreads < pba::kBwdRegSplitTotal)
      e = cudaErrorInvalidConfiguration;
    return e;
  });
  if (attr_err != cudaSuccess) return attr_err;
  kern<<<grid, pba::kBwdThreads, L::kSmemAlloc, stream>>>(p);
  return cudaGetLastError();
}

// Dense [B][H][N][D]; the stride of an extent-1 dimension does not matter.
bool contiguous_bhnd(const int64_t s[3], int64_t B, int64_t H, int64_t N, int64_t D) {
  return (N <= 1 || s[2] == D) && (H <= 1 || s[1] == N * D) && (B <= 1 || s[0] == H * N * D);
}

}  // namespace

extern "C" {

pba_status pba_forward(const pba_attn_desc *desc, const void *q, const void *k, const void *v, const void *bias,
                       const uint8_t *key_mask, void *out, float *lse, void *stream) {
  return attn_common(desc, q, k, v, bias, key_mask, false, out, lse, nullptr, stream);
}

pba_status pba_partial(const pba_attn_desc *desc, const void *q, const void *k, const void *v, const void *bias,
                       const uint8_t *key_mask, float *o_part, float *m_part, float *l_part, void *stream) {
  return attn_common(desc, q, k, v, bias, key_mask, true, o_part, m_part, l_part, stream);
}

pba_status softmax_merge(int32_t P, int64_t rows, int64_t D, const float *o_parts, const float *m_parts,
                         const float *l_parts, int32_t out_dtype, void *out, float *lse, void *stream_ptr) {
  if (P < 1 || rows < 0 || D < 4 || D > 256 || D % 4 != 0) return PBA_ERR_INVALID_ARG;
  if (out_dtype != PBA_BF16 && out_dtype != PBA_F32) return PBA_ERR_UNSUPPORTED;
  if (o_parts == nullptr || m_parts == nullptr || l_parts == nullptr || out == nullptr) return PBA_ERR_INVALID_ARG;
  if (!aligned16(o_parts) || (reinterpret_cast<uintptr_t>(out) & (out_dtype == PBA_BF16 ? 7u : 15u)) != 0)
    return PBA_ERR_INVALID_ARG;
  pba_status s = check_device();
  if (s != PBA_OK) return s;
  if (rows == 0) return PBA_OK;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  const int64_t total = rows * (D / 4);
  int64_t grid = (total + 255) / 256;
  // One thread per 4-element chunk: blocks that finish make room for new
  // ones, whose loads overlap the others' arithmetic (ring8k merge 57.3 ->
  // 53.2 us against a grid of 8 blocks per SM looping over the rows).  The
  // kernel's grid-stride loop covers sizes beyond the cap.
  const int64_t cap = int64_t(1) << 30;
  if (grid > cap) grid = cap;
  const bool bf = out_dtype == PBA_BF16;
  // P up to 8 (the ring steps of one node) unrolled with all loads up front; larger P loops
  if (P <= 4)
    (bf ? pba::softmax_merge_kernel<true, 4> : pba::softmax_merge_kernel<false, 4>)<<<int(grid), 256, 0, stream>>>(
        P, rows, int(D), o_parts, m_parts, l_parts, out, lse);
  else if (P <= 8)
    (bf ? pba::softmax_merge_kernel<true, 8> : pba::softmax_merge_kernel<false, 8>)<<<int(grid), 256, 0, stream>>>(
        P, rows, int(D), o_parts, m_parts, l_parts, out, lse);
  else
    (bf ? pba::softmax_merge_kernel<true, 0> : pba::softmax_merge_kernel<false, 0>)<<<int(grid), 256, 0, stream>>>(
        P, rows, int(D), o_parts, m_parts, l_parts, out, lse);
  return cudaGetLastError() == cudaSuccess ? PBA_OK : PBA_ERR_CUDA;
}

pba_status tri_attn_forward(int64_t N, int64_t H, int64_t D, int32_t orient, float softmax_scale, const void *q,
                            const void *k, const void *v, const void *bias, const void *gate,
                            const uint8_t *pair_mask, void *out, float *lse, void *stream_ptr) {
  if (N < 0 || H < 1 || N > 65535 || H > 4096) return PBA_ERR_INVALID_ARG;
  if (D != 32 && D != 64) return PBA_ERR_UNSUPPORTED;
  if (orient != PBA_TRI_STARTING && orient != PBA_TRI_ENDING) return PBA_ERR_INVALID_ARG;
  if (!(softmax_scale >= 0.f) || std::isinf(softmax_scale)) return PBA_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr || v == nullptr || bias == nullptr || out == nullptr) return PBA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(bias) || !aligned16(out) ||
      (gate != nullptr && !aligned16(gate)))
    return PBA_ERR_INVALID_ARG;
  if (N % 8 != 0 || (H * D) % 8 != 0) return PBA_ERR_INVALID_ARG;
  pba_status s = check_device();
  if (s != PBA_OK) return s;
  if (N == 0) return PBA_OK;
  const bool ending = orient == PBA_TRI_ENDING;
  const int64_t HD = H * D, NHD = N * H * D;
  TcProblem t;
  std::memset(&t, 0, sizeof(t));
  t.B = int(N);  // one problem per pair-tensor line
  t.H = int(H);
  t.Nq = int(N);
  t.Nk = int(N);
  t.D = int(D);
  t.tau = tau_of(softmax_scale, D);
  t.q = q;
  t.k = k;
  t.v = v;
  t.bias = bias;
  // (line, head, position): starting node line = row i, position = column j;
  // ending node line = column j, position = row i (outer strides swapped).
  const int64_t s_line = ending ? HD : NHD, s_pos = ending ? NHD : HD;
  const int64_t qkv_s[3] = {s_line, D, s_pos};
  for (int i = 0; i < 3; ++i) {
    t.q_s[i] = qkv_s[i];
    t.k_s[i] = qkv_s[i];
    t.v_s[i] = qkv_s[i];
    t.out_s[i] = qkv_s[i];
    t.gate_s[i] = qkv_s[i];
  }
  // bias [H][N][N]: starting node reads rows b[h][j][:] (query j, keys k);
  // ending node reads b[h][k][i] as a [key][query] tile.
  t.bias_t = ending;
  t.bias_s[0] = 0;
  t.bias_s[1] = N * N;
  t.bias_s[2] = N;
  t.bias_b_bcast = true;
  t.bias_h_bcast = false;
  t.mask = pair_mask;
  t.mask_sb = ending ? 1 : N;
  t.mask_sk = ending ? N : 1;
  t.epi = pba::kEpiForward;
  t.out = out;
  t.lse = lse;
  t.lse_s[0] = ending ? H : N * H;
  t.lse_s[1] = 1;
  t.lse_s[2] = ending ? N * H : H;
  t.gate = gate;
  return run_tc(t, static_cast<cudaStream_t>(stream_ptr));
}

pba_status tri_proj_forward(int64_t N, int64_t c, int64_t H, int64_t D, const void *z, const void *w_qkvg,
                            const void *w_b, void *q, void *k, void *v, void *g, void *bias, void *stream_ptr) {
  if (N < 0 || N > 32768 || H < 1 || D < 1) return PBA_ERR_INVALID_ARG;
  if ((c != 64 && c != 128) || H * D != 128 || (H != 1 && H != 2 && H != 4 && H != 8)) return PBA_ERR_UNSUPPORTED;
  if (N == 0) return PBA_OK;  // nothing to read or write; zero-extent buffers may be NULL
  if (z == nullptr || w_qkvg == nullptr || w_b == nullptr || q == nullptr || k == nullptr || v == nullptr ||
      g == nullptr || bias == nullptr)
    return PBA_ERR_INVALID_ARG;
  if (!aligned16(z) || !aligned16(w_qkvg) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) ||
      (reinterpret_cast<uintptr_t>(w_b) & 1u) || (reinterpret_cast<uintptr_t>(bias) & 1u))
    return PBA_ERR_INVALID_ARG;
  pba_status s = check_device();
  if (s != PBA_OK) return s;
  const int64_t rows = N * N;
  pba::ProjParams p;
  std::memset(&p, 0, sizeof(p));
  {
    const uint64_t dims[4] = {uint64_t(c), uint64_t(rows), 1, 1};
    const int64_t st[3] = {c * 2, 0, 0};
    const uint32_t box[4] = {64, uint32_t(pba::kProjRows), 1, 1};
    if (!make_map(&p.tm_z, z, dims, st, box, CU_TENSOR_MAP_SWIZZLE_128B)) return PBA_ERR_INVALID_ARG;
  }
  {
    const uint64_t dims[4] = {uint64_t(pba::kProjCols), uint64_t(c), 1, 1};
    const int64_t st[3] = {int64_t(pba::kProjCols) * 2, 0, 0};
    const uint32_t box[4] = {64, uint32_t(c), 1, 1};
    if (!make_map(&p.tm_w, w_qkvg, dims, st, box, CU_TENSOR_MAP_SWIZZLE_128B)) return PBA_ERR_INVALID_ARG;
  }
  for (int m = 0; m < 4; ++m) {
    void *const dst[4] = {q, k, v, g};
    const uint64_t dims[4] = {uint64_t(pba::kProjCols / 4), uint64_t(rows), 1, 1};
    const int64_t st[3] = {int64_t(pba::kProjCols / 4) * 2, 0, 0};
    // one warp's 32 rows of a 32-column chunk per tensor store
    const uint32_t box[4] = {32, 32, 1, 1};
    if (!make_map(&p.tm_out[m], dst[m], dims, st, box, CU_TENSOR_MAP_SWIZZLE_64B)) return PBA_ERR_INVALID_ARG;
  }
  p.rows = rows;
  p.c = int(c);
  p.n_tiles = int((rows + pba::kProjRows - 1) / pba::kProjRows);
  p.wb = static_cast<const uint16_t *>(w_b);
  p.out[0] = static_cast<uint16_t *>(q);
  p.out[1] = static_cast<uint16_t *>(k);
  p.out[2] = static_cast<uint16_t *>(v);
  p.out[3] = static_cast<uint16_t *>(g);
  p.bias = static_cast<uint16_t *>(bias);
  p.err = device_error_word();
  if (p.err == nullptr) return PBA_ERR_CUDA;
  p.timeout_ns = g_timeout_ns.load();
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return PBA_ERR_CUDA;
  const int grid = std::min(p.n_tiles, sms);
  cudaStream_t st = static_cast<cudaStream_t>(stream_ptr);
  cudaError_t e = H == 1   ? launch_proj<1>(p, grid, st)
                  : H == 2 ? launch_proj<2>(p, grid, st)
                  : H == 4 ? launch_proj<4>(p, grid, st)
                           : launch_proj<8>(p, grid, st);
  return e == cudaSuccess ? PBA_OK : PBA_ERR_CUDA;
}

pba_status tri_out_proj_forward(int64_t N, int64_t c, int64_t H, int64_t D, const void *o, const void *w_o,
                                void *out, void *stream_ptr) {
  if (N < 0 || N > 32768 || H < 1 || D < 1) return PBA_ERR_INVALID_ARG;
  if ((c != 64 && c != 128) || H * D != pba::kOprojK) return PBA_ERR_UNSUPPORTED;
  if (N == 0) return PBA_OK;  // nothing to read or write; zero-extent buffers may be NULL
  if (o == nullptr || w_o == nullptr || out == nullptr) return PBA_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(w_o) || !aligned16(out)) return PBA_ERR_INVALID_ARG;
  pba_status s = check_device();
  if (s != PBA_OK) return s;
  const int64_t rows = N * N;
  pba::OprojParams p;
  std::memset(&p, 0, sizeof(p));
  {
    const uint64_t dims[4] = {uint64_t(pba::kOprojK), uint64_t(rows), 1, 1};
    const int64_t st[3] = {int64_t(pba::kOprojK) * 2, 0, 0};
    const uint32_t box[4] = {64, uint32_t(pba::kOprojRows), 1, 1};
    if (!make_map(&p.tm_o, o, dims, st, box, CU_TENSOR_MAP_SWIZZLE_128B)) return PBA_ERR_INVALID_ARG;
  }
  {
    // W_o [128][c]: 64-column slabs of all 128 rows
    const uint64_t dims[4] = {uint64_t(c), uint64_t(pba::kOprojK), 1, 1};
    const int64_t st[3] = {c * 2, 0, 0};
    const uint32_t box[4] = {64, uint32_t(pba::kOprojK), 1, 1};
    if (!make_map(&p.tm_w, w_o, dims, st, box, CU_TENSOR_MAP_SWIZZLE_128B)) return PBA_ERR_INVALID_ARG;
  }
  {
    const uint64_t dims[4] = {uint64_t(c), uint64_t(rows), 1, 1};
    const int64_t st[3] = {c * 2, 0, 0};
    // one warp's 32 rows of a 32-column chunk per tensor store
    const uint32_t box[4] = {32, 32, 1, 1};
    if (!make_map(&p.tm_out, out, dims, st, box, CU_TENSOR_MAP_SWIZZLE_64B)) return PBA_ERR_INVALID_ARG;
  }
  p.rows = rows;
  p.n_tiles = int((rows + pba::kOprojRows - 1) / pba::kOprojRows);
  p.err = device_error_word();
  if (p.err == nullptr) return PBA_ERR_CUDA;
  p.timeout_ns = g_timeout_ns.load();
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return PBA_ERR_CUDA;
  const int grid = std::min(p.n_tiles, sms);
  cudaStream_t st = static_cast<cudaStream_t>(stream_ptr);
  const cudaError_t e = c == 64 ? launch_oproj<64>(p, grid, st) : launch_oproj<128>(p, grid, st);
  return e == cudaSuccess ? PBA_OK : PBA_ERR_CUDA;
}

pba_status pwa_forward(int64_t S, int64_t N, int64_t H, int64_t D, const void *v, const void *bias,
                       const uint8_t *key_mask, const void *gate, void *out, float *lse, void *stream_ptr) {
  if (S < 0 || N < 0 || H < 1 || S > 65535 || N > 65535 || H > 4096) return PBA_ERR_INVALID_ARG;
  if (D != 32 && D != 64) return PBA_ERR_UNSUPPORTED;
  if (N % 8 != 0) return PBA_ERR_INVALID_ARG;  // bias rows are tile rows: 16-byte strides
  if (S == 0 || N == 0) return PBA_OK;        // nothing to write; zero-extent buffers may be NULL
  if (v == nullptr || bias == nullptr || out == nullptr || lse == nullptr) return PBA_ERR_INVALID_ARG;
  if (!aligned16(v) || !aligned16(bias) || !aligned16(out) || (gate != nullptr && !aligned16(gate)) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
    return PBA_ERR_INVALID_ARG;
  pba_status s = check_device();
  if (s != PBA_OK) return s;
  const int slabs = pba::kPwaDF / int(D);
  pba::PwaParams p;
  std::memset(&p, 0, sizeof(p));
  {
    // v [S][N][H][D] as (D, N, H, S)
    const uint64_t dims[4] = {uint64_t(D), uint64_t(N), uint64_t(H), uint64_t(S)};
    const int64_t st[3] = {H * D * 2, D * 2, N * H * D * 2};
    const uint32_t box[4] = {uint32_t(D), uint32_t(pba::kPwaBN), 1, uint32_t(slabs)};
    if (!make_map(&p.tm_v, v, dims, st, box, D == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
      return PBA_ERR_INVALID_ARG;
  }
  {
    // bias [H][N][N] as (keys, rows, H, 1): two 64-key boxes per tile
    const uint64_t dims[4] = {uint64_t(N), uint64_t(N), uint64_t(H), 1};
    const int64_t st[3] = {N * 2, N * N * 2, 0};
    const uint32_t box[4] = {64, uint32_t(pba::kPwaBM), 1, 1};
    if (!make_map(&p.tm_bias, bias, dims, st, box, CU_TENSOR_MAP_SWIZZLE_128B)) return PBA_ERR_INVALID_ARG;
  }
  p.S = int(S);
  p.N = int(N);
  p.H = int(H);
  p.n_qblocks = int((N + pba::kPwaBM - 1) / pba::kPwaBM);
  p.n_ftiles = int((S + slabs - 1) / slabs);
  const int64_t n_units = int64_t(H) * p.n_qblocks * p.n_ftiles;
  if (n_units > kMaxI32) return PBA_ERR_INVALID_ARG;
  p.n_units = int(n_units);
  p.masked = (key_mask != nullptr) || (N % pba::kPwaBN != 0);
  p.mask_vec4 = key_mask != nullptr && (reinterpret_cast<uintptr_t>(key_mask) & 3u) == 0;
  p.mask = key_mask;
  p.out = static_cast<uint16_t *>(out);
  p.gate = static_cast<const uint16_t *>(gate);
  p.lse = lse;
  p.err = device_error_word();
  if (p.err == nullptr) return PBA_ERR_CUDA;
  p.timeout_ns = g_timeout_ns.load();
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return PBA_ERR_CUDA;
  const int grid = int(std::min<int64_t>(n_units, sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream_ptr);
  // first pass: the log-sum-exp of every weight row (one warp per row)
  const int64_t rows = H * N;
  const int mask_vec8 = key_mask != nullptr && (reinterpret_cast<uintptr_t>(key_mask) & 7u) == 0;
  pba::pba_pwa_lse_kernel<<<int((rows * 32 + 255) / 256), 256, 0, st>>>(static_cast<const uint16_t *>(bias), key_mask,
                                                                         mask_vec8, lse, int(N), rows);
  if (cudaGetLastError() != cudaSuccess) return PBA_ERR_CUDA;
  // second pass: the normalised weights times the values
  cudaError_t e = (D == 64) ? dispatch_pwa<64>(p, grid, gate != nullptr, st)
                            : dispatch_pwa<32>(p, grid, gate != nullptr, st);
  return e == cudaSuccess ? PBA_OK : PBA_ERR_CUDA;
}

pba_status pba_backward(const pba_attn_desc *d, const void *q, const void *k, const void *v, const void *bias,
                        const uint8_t *key_mask, const void *out, const float *lse, const void *dout, float *dq,
                        float *dk, float *dv, void *dbias, float *delta, void *stream_ptr) {
  pba_status s = check_desc(d);
  if (s != PBA_OK) return s;
  if (d->dtype != PBA_BF16) return PBA_ERR_UNSUPPORTED;
  const int64_t B = d->B, H = d->H, Nq = d->Nq, Nk = d->Nk, D = d->D;
  if (Nq == 0 || Nk == 0) return PBA_OK;  // no scores: nothing to write (a caller zero-fills dk, dv or dq)
  const void *ptrs[] = {q, k, v, bias, out, lse, dout, dq, dk, dv, dbias, delta};
  for (const void *x : ptrs)
    if (x == nullptr || !aligned16(x)) return PBA_ERR_INVALID_ARG;
  // contiguous [B][H][n][D] tensors (the output strides describe out and dout)
  if (!contiguous_bhnd(d->q_stride, B, H, Nq, D) || !contiguous_bhnd(d->k_stride, B, H, Nk, D) ||
      !contiguous_bhnd(d->v_stride, B, H, Nk, D) || !contiguous_bhnd(d->out_stride, B, H, Nq, D))
    return PBA_ERR_INVALID_ARG;
  if ((Nq > 1 && d->lse_stride[2] != 1) || (H > 1 && d->lse_stride[1] != Nq) ||
      (B > 1 && d->lse_stride[0] != H * Nq))
    return PBA_ERR_INVALID_ARG;
  if (d->bias_stride[2] % 8 != 0 || Nk % 8 != 0) return PBA_ERR_INVALID_ARG;  // 16-byte bias and dbias rows
  if (B * H * Nq > kMaxI32 || B * H * Nk > kMaxI32) return PBA_ERR_INVALID_ARG;
  s = check_device();
  if (s != PBA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream_ptr);
  pba::BwdParams p;
  std::memset(&p, 0, sizeof(p));
  const CUtensorMapSwizzle swz = (D == 64) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const uint32_t box[4] = {uint32_t(D), uint32_t(pba::kBwdTile), 1, 1};
  {
    const uint64_t dq_[4] = {uint64_t(D), uint64_t(Nq), uint64_t(H), uint64_t(B)};
    const uint64_t dk_[4] = {uint64_t(D), uint64_t(Nk), uint64_t(H), uint64_t(B)};
    const int64_t sq[3] = {D * 2, Nq * D * 2, H * Nq * D * 2}, sk[3] = {D * 2, Nk * D * 2, H * Nk * D * 2};
    if (!make_map(&p.tm_q, q, dq_, sq, box, swz) || !make_map(&p.tm_do, dout, dq_, sq, box, swz) ||
        !make_map(&p.tm_k, k, dk_, sk, box, swz) || !make_map(&p.tm_v, v, dk_, sk, box, swz))
      return PBA_ERR_INVALID_ARG;
  }
  const bool bh_bcast = d->bias_stride[1] == 0 && H > 1, bb_bcast = d->bias_stride[0] == 0 && B > 1;
  const uint64_t bdims[4] = {uint64_t(Nk), uint64_t(Nq), bh_bcast ? 1 : uint64_t(H), bb_bcast ? 1 : uint64_t(B)};
  const int64_t bst[3] = {d->bias_stride[2] * 2, d->bias_stride[1] * 2, d->bias_stride[0] * 2};
  p.bias_h_bcast = bh_bcast;
  p.bias_b_bcast = bb_bcast;
  p.B = int(B);
  p.H = int(H);
  p.Nq = int(Nq);
  p.Nk = int(Nk);
  p.tau = tau_of(d->softmax_scale, D);
  p.mask = key_mask;
  p.mask_sb = d->mask_stride_b;
  p.lse = lse;
  p.delta = delta;
  p.row_sb = H * Nq;
  p.row_sh = Nq;
  p.dbias = static_cast<uint16_t *>(dbias);
  p.db_sb = H * Nq * Nk;
  p.db_sh = Nq * Nk;
  p.db_sn = Nk;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.err = device_error_word();
  if (p.err == nullptr) return PBA_ERR_CUDA;
  p.timeout_ns = g_timeout_ns.load();
  // Delta = rowsum(dO * O)
  const int64_t rows = B * H * Nq;
  pba::pba_bwd_delta_kernel<<<int((rows * (D / 8) + 255) / 256), 256, 0, st>>>(
      static_cast<const uint16_t *>(dout), static_cast<const uint16_t *>(out), delta, rows, int(D));
  if (cudaGetLastError() != cudaSuccess) return PBA_ERR_CUDA;
  cudaError_t e;
  {
    // kernel A: dq and dbias, one CTA per (b, h, 128 query rows)
    pba::BwdParams a = p;
    const uint32_t bbox[4] = {64, uint32_t(pba::kBwdTile), 1, 1};
    if (!make_map(&a.tm_bias, bias, bdims, bst, bbox, CU_TENSOR_MAP_SWIZZLE_128B)) return PBA_ERR_INVALID_ARG;
    // dbias [B][H][Nq][Nk] (contiguous) as (Nk, Nq, H, B), one warp's 32 rows of 64 keys per store
    const uint64_t ddims[4] = {uint64_t(Nk), uint64_t(Nq), uint64_t(H), uint64_t(B)};
    const int64_t dst_[3] = {Nk * 2, Nq * Nk * 2, H * Nq * Nk * 2};
    const uint32_t dbox[4] = {64, 32, 1, 1};
    if (!make_map(&a.tm_dbias, dbias, ddims, dst_, dbox, CU_TENSOR_MAP_SWIZZLE_128B)) return PBA_ERR_INVALID_ARG;
    a.n_tiles = int((Nq + pba::kBwdTile - 1) / pba::kBwdTile);
    const int grid = int(B * H * a.n_tiles);
    e = (D == 64) ? launch_bwd<64, false>(a, grid, st) : launch_bwd<32, false>(a, grid, st);
    if (e != cudaSuccess) return PBA_ERR_CUDA;
  }
  {
    // kernel B: dk and dv, one CTA per (b, h, 128 key rows)
    pba::BwdParams bb = p;
    const uint32_t bbox[4] = {uint32_t(pba::kBwdTile), uint32_t(pba::kBwdTile), 1, 1};
    if (!make_map(&bb.tm_bias, bias, bdims, bst, bbox, CU_TENSOR_MAP_SWIZZLE_NONE)) return PBA_ERR_INVALID_ARG;
    bb.n_tiles = int((Nk + pba::kBwdTile - 1) / pba::kBwdTile);
    const int grid = int(B * H * bb.n_tiles);
    e = (D == 64) ? launch_bwd<64, true>(bb, grid, st) : launch_bwd<32, true>(bb, grid, st);
    if (e != cudaSuccess) return PBA_ERR_CUDA;
  }
  return PBA_OK;
}

}  // extern "C"

// ------------------------------------------------------------ pba_backward_noalloc
// The Delta rows of pba_backward_noalloc: a fixed array in every GPU that
// loads the library, shared by all its calls on that device.
static __device__ __align__(256) float g_bwd_noalloc_delta[PBA_BWD_NOALLOC_MAX_ROWS];

namespace {

constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mu;
float *g_noalloc_delta_ptr[kNoallocMaxDevices] = {};

// Device address of g_bwd_noalloc_delta on the current device.  In host code
// the array's name is a host-side stand-in, not a device address, so it is
// looked up once per device (with that device current) and kept.
pba_status noalloc_delta(float **ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PBA_ERR_CUDA;
  if (dev < 0 || dev >= kNoallocMaxDevices) return PBA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_delta_ptr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_noalloc_delta) != cudaSuccess || p == nullptr) return PBA_ERR_CUDA;
    g_noalloc_delta_ptr[dev] = static_cast<float *>(p);
  }
  *ptr = g_noalloc_delta_ptr[dev];
  return PBA_OK;
}

}  // namespace

extern "C" {

pba_status pba_backward_noalloc(const pba_attn_desc *d, const void *q, const void *k, const void *v,
                                const void *bias, const uint8_t *key_mask, const void *out, const float *lse,
                                const void *dout, float *dq, float *dk, float *dv, void *dbias, void *stream) {
  if (d == nullptr || d->B < 1 || d->H < 1 || d->Nq < 0) return PBA_ERR_INVALID_ARG;
  const int64_t cap = PBA_BWD_NOALLOC_MAX_ROWS;
  if (d->B > cap || d->H > cap || d->Nq > cap || d->B * d->H > cap || d->B * d->H * d->Nq > cap)
    return PBA_ERR_INVALID_ARG;  // more rows than the fixed Delta array holds
  pba_status s = check_device();
  if (s != PBA_OK) return s;
  float *delta = nullptr;
  s = noalloc_delta(&delta);
  if (s != PBA_OK) return s;
  return pba_backward(d, q, k, v, bias, key_mask, out, lse, dout, dq, dk, dv, dbias, delta, stream);
}

const char *pba_status_string(pba_status status) {
  switch (status) {
    case PBA_OK:
      return "PBA_OK";
    case PBA_ERR_INVALID_ARG:
      return "PBA_ERR_INVALID_ARG";
    case PBA_ERR_UNSUPPORTED:
      return "PBA_ERR_UNSUPPORTED";
    case PBA_ERR_CUDA:
      return "PBA_ERR_CUDA";
    case PBA_ERR_TIMEOUT:
      return "PBA_ERR_TIMEOUT";
  }
  return "PBA_ERR_UNKNOWN";
}

pba_status pba_last_device_error(void *stream_ptr) {
  static std::atomic<unsigned> next_slot{0};
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return PBA_ERR_CUDA;
  const int slot = int(next_slot.fetch_add(1) % kErrTakeSlots);
  pba_take_error_kernel<<<1, 1, 0, stream>>>(slot);
  int v = 0;
  if (cudaGetLastError() != cudaSuccess ||
      cudaMemcpyFromSymbolAsync(&v, g_pba_err_taken, sizeof(int), slot * sizeof(int), cudaMemcpyDeviceToHost,
                                stream) != cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return PBA_ERR_CUDA;
  return static_cast<pba_status>(v);
}

uint64_t pba_set_wait_timeout_ns(uint64_t timeout_ns) {
  return g_timeout_ns.exchange(timeout_ns == 0 ? kDefaultTimeoutNs : timeout_ns);
}

pba_status pba_selftest_wait_timeout(uint64_t timeout_ns, void *stream) {
  if (timeout_ns == 0 || timeout_ns > 10ull * kDefaultTimeoutNs) return PBA_ERR_INVALID_ARG;
  int *err = device_error_word();
  if (err == nullptr) return PBA_ERR_CUDA;
  pba::pba_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, timeout_ns);
  return cudaGetLastError() == cudaSuccess ? PBA_OK : PBA_ERR_CUDA;
}

pba_status pba_selftest_exp2(const float *in, float *out, int64_t n, void *stream) {
  if (n < 0 || (n > 0 && (in == nullptr || out == nullptr))) return PBA_ERR_INVALID_ARG;
  pba_status s = check_device();
  if (s != PBA_OK) return s;
  if (n == 0) return PBA_OK;
  pba::pba_exp2_selftest_kernel<<<148, 256, 0, static_cast<cudaStream_t>(stream)>>>(in, out, n);
  return cudaGetLastError() == cudaSuccess ? PBA_OK : PBA_ERR_CUDA;
}

}  // extern "C"
