/*
 * pba.h -- C ABI of libpba: pair-biased attention on NVIDIA B200 (sm_100a).
 *
 * The operation (all entry points): multi-head attention whose logits carry
 * an additive pair bias,
 *
 *     O = softmax_keys( tau * Q K^T + bias + mask ) V ,   tau = 1/sqrt(D),
 *
 * as named in "Fold-CP: A Context Parallelism Framework for Biomolecular
 * Modeling" (Table 1, rows "Attn Pair Bias (Ring)" and "Triangle Attention";
 * Figure 2 (a) and (c)).  The ring schemes there visit the keys block by
 * block; each block yields an online-softmax partial (O, m, l) and a
 * "tiled-softmax merge" combines them (the method of "Online normalizer
 * calculation for softmax" and "Self-attention Does Not Need O(n2) Memory",
 * both listed under "Builds on" on the page "Design-CP: Context Parallelism
 * for Design of Protein Nanoparticles").  On one GPU the ring's P steps are P
 * key blocks: pba_partial computes one block, softmax_merge combines them and
 * pba_forward does the whole pass at once.
 *
 * Conventions common to every entry point
 *   - Pointers marked "device" must be CUDA device memory of the current
 *     device; the caller owns every buffer.  Per call the library allocates
 *     nothing: it keeps one device error word and builds TMA descriptors on the
 *     host stack.
 *   - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).  Calls are thread-safe and keep no state
 *     between calls apart from the error word.
 *   - Natural logarithms throughout: lse = m + ln l, m = max of the scores.
 *   - A key takes part if its mask byte is nonzero and its bias is not -inf.
 *     A query row with no such key gets O = 0, lse = -inf (and m = -inf,
 *     l = 0 for partials); never NaN.  Values of K and V must be finite,
 *     masked keys included.  NaN or +inf in the inputs is outside the
 *     contract.
 *   - A pointer may be NULL when the tensor it stands for has no element
 *     (Nq = 0 or Nk = 0); every other required pointer must be non-NULL.
 *   - Return values: PBA_OK when the launch was enqueued.  PBA_ERR_INVALID_ARG
 *     for a NULL required pointer, a negative size, a misaligned pointer or
 *     stride (see below), or a size beyond the limits.  PBA_ERR_UNSUPPORTED for
 *     a head dimension or dtype without a kernel, or a device that is not
 *     sm_100.  PBA_ERR_CUDA when a CUDA runtime/driver call failed (the CUDA
 *     error is left for cudaGetLastError).  Nothing is thrown across the ABI.
 *   - Device-side faults are reported through pba_last_device_error(): every
 *     wait inside the kernels is bounded (pba_set_wait_timeout_ns); a wait that
 *     runs out records PBA_ERR_TIMEOUT and the kernel returns instead of
 *     hanging.
 *
 * Alignment rules of the bf16 path (its tiles are moved by the Tensor Memory
 * Accelerator): q, k, v and bias base addresses 16-byte aligned; every
 * non-unit stride of q, k, v and bias a multiple of 8 elements (16 bytes).
 * The bias row length may be ragged, but its row stride must be padded to a
 * multiple of 8 elements.  For pba_partial the caller points k, v, bias and
 * key_mask at the block's first key, so the block start must keep those rules
 * (a multiple of 8 keys).  The fp32 path has no alignment rule beyond natural
 * float alignment: calls whose q, k, v, bias and out bases are 16-byte
 * aligned and whose non-unit strides are multiples of 4 elements run on the
 * tensor cores, the others on the CUDA cores (same results to about 1e-5).
 */
#ifndef PBA_H
#define PBA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported from libpba.so (the library is built with hidden visibility). */
#if defined(__GNUC__)
#define PBA_API __attribute__((visibility("default")))
#else
#define PBA_API
#endif

typedef enum {
  PBA_OK = 0,
  PBA_ERR_INVALID_ARG = 1,
  PBA_ERR_UNSUPPORTED = 2,
  PBA_ERR_CUDA = 3,
  PBA_ERR_TIMEOUT = 4
} pba_status;

typedef enum { PBA_BF16 = 0, PBA_F32 = 1 } pba_dtype;

typedef enum { PBA_TRI_STARTING = 0, PBA_TRI_ENDING = 1 } pba_tri_orient;

/*
 * Shape and layout of one pair-biased attention problem.
 *   B, H       batch and heads (B, H >= 1)
 *   Nq, Nk     query rows and keys (>= 0; Nk = 0 makes every row empty)
 *   D          head dimension: 32 or 64 (bf16 and fp32)
 *   dtype      pba_dtype of q, k, v, bias and of pba_forward's `out`.  bf16
 *              runs on the tensor cores (kind::f16).  fp32 keeps fp32-level
 *              accuracy (about 1e-5 from the exact result): on the tensor
 *              cores as kind::tf32 with each operand split into a tf32 high
 *              and low part (three products per product, about six times
 *              slower than bf16 at size), or, for rows the tile loads cannot
 *              address, one warp per query row on the CUDA cores.
 *   softmax_scale  tau; 0 selects 1/sqrt(D).  The bias is added unscaled.
 *   *_stride   strides in ELEMENTS of the (b, h, n) axes; the d axis (and
 *              the key axis of the bias) has stride 1.
 *   bias_stride    (b, h, query row); a 0 in b or h broadcasts the bias over
 *              that axis.
 *   mask_stride_b  row stride of key_mask [B][Nk] (uint8, key stride 1).
 *   out_stride     (b, h, n) of `out` / `o_part`, d stride 1.
 *   lse_stride     (b, h, n) of `lse` / `m_part` / `l_part`.
 */
typedef struct {
  int64_t B, H, Nq, Nk, D;
  int32_t dtype;
  float softmax_scale;
  int64_t q_stride[3];
  int64_t k_stride[3];
  int64_t v_stride[3];
  int64_t bias_stride[3];
  int64_t mask_stride_b;
  int64_t out_stride[3];
  int64_t lse_stride[3];
} pba_attn_desc;

/*
 * pba_forward -- one full pass over all Nk keys (Fold-CP, Table 1 "Attn
 * Pair Bias"; the definition above).
 *   q [B,H,Nq,D], k/v [B,H,Nk,D], bias [B,H,Nq,Nk]   device, desc->dtype
 *   key_mask [B,Nk] uint8, device, or NULL (every key takes part)
 *   out [B,H,Nq,D] device, desc->dtype: O (normalised)
 *   lse [B,H,Nq] float, device, or NULL
 */
PBA_API pba_status pba_forward(const pba_attn_desc *desc, const void *q, const void *k, const void *v,
                       const void *bias, const uint8_t *key_mask, void *out, float *lse, void *stream);

/*
 * pba_partial -- one ring step (Fold-CP, Figure 2(c): local queries against
 * the key/value/bias block held): the online-softmax partial over the
 * desc->Nk keys that k, v, bias and key_mask point at.
 *   o_part [B,H,Nq,D] float: the block's output normalised by its own l
 *   m_part [B,H,Nq] float: maximum score in the block (natural units)
 *   l_part [B,H,Nq] float: sum over the block of exp(s - m_part)
 * A block with no valid key for a row gives exactly (0, -inf, 0) there.
 * bias_stride[2] is the row stride of the full bias matrix, so a block is a
 * column window of it.
 */
PBA_API pba_status pba_partial(const pba_attn_desc *desc, const void *q, const void *k, const void *v,
                       const void *bias, const uint8_t *key_mask, float *o_part, float *m_part, float *l_part,
                       void *stream);

/*
 * softmax_merge -- the tiled-softmax merge (Fold-CP, Figure 2 (a) and (c)).
 * P partials over disjoint key blocks, stacked in any order:
 *   o_parts [P][rows][D], m_parts [P][rows], l_parts [P][rows]  float, device
 * give, per row, M = max m_p over blocks with l_p > 0, w_p = l_p exp(m_p - M),
 *   out = sum_p w_p o_p / sum_p w_p        [rows][D], out_dtype (bf16 or fp32)
 *   lse = M + ln sum_p w_p                 [rows] float, or NULL
 * A row with no valid key in any block gives out = 0, lse = -inf.
 * P >= 1, rows >= 0, D a multiple of 4 up to 256; o_parts and out 16-byte
 * aligned.
 */
PBA_API pba_status softmax_merge(int32_t P, int64_t rows, int64_t D, const float *o_parts, const float *m_parts,
                         const float *l_parts, int32_t out_dtype, void *out, float *lse, void *stream);

/*
 * tri_attn_forward -- triangle attention on a pair tensor (Fold-CP, Table 1
 * "Triangle Attention"; Figure 2(a)), bf16, heads H, head dim D in {32, 64}.
 *   q, k, v, gate [N][N][H][D] (pair (i,j), then head, then d)  bf16, device
 *   bias [H][N][N] bf16, device: the triangular bias, shared by all rows
 *   pair_mask [N][N] uint8, device, or NULL
 * Starting node (orient = PBA_TRI_STARTING), for every pair (i, j), head h:
 *   o[i][j] = sum_k softmax_k( tau q[i][j].k[i][k] + b[h][j][k] ) v[i][k]
 *   over keys k with pair_mask[i][k] != 0.
 * Ending node (orient = PBA_TRI_ENDING):
 *   o[i][j] = sum_k softmax_k( tau q[i][j].k[k][j] + b[h][k][i] ) v[k][j]
 *   over keys k with pair_mask[k][j] != 0 -- the cross-axis transpose of
 *   Figure 2(a), done by the tile loads' strides, not by a copy.
 * out [N][N][H][D] bf16 = o * sigmoid(gate) (gate NULL: out = o);
 * lse [N][N][H] float or NULL.  softmax_scale 0 selects 1/sqrt(D).
 * N*H*D*2 bytes and H*D*2 bytes are the tile strides, so H*D must be a
 * multiple of 8 and N a multiple of 8.
 */
PBA_API pba_status tri_attn_forward(int64_t N, int64_t H, int64_t D, int32_t orient, float softmax_scale, const void *q,
                            const void *k, const void *v, const void *bias, const void *gate,
                            const uint8_t *pair_mask, void *out, float *lse, void *stream);

/*
 * tri_proj_forward -- the triangle projections of a pair tensor in one pass
 * (Fold-CP, Figure 2(a): triangle attention draws its queries, keys, values,
 * gate and per-head bias from the pair representation).
 *   z       [N][N][c]   bf16, device; pair row r = i*N + j, c in {64, 128}
 *   w_qkvg  [c][4*H*D]  bf16, device; column blocks W_q | W_k | W_v | W_g
 *   w_b     [c][H]      bf16, device
 * For every pair row r, in fp32 sums of the bf16 products, rounded once to bf16:
 *   q[r][:] = z[r] W_q,  k[r][:] = z[r] W_k,  v[r][:] = z[r] W_v,  g[r][:] = z[r] W_g
 *     (q, k, v, g [N][N][H][D] bf16, device: the layout tri_attn_forward takes;
 *      g is the gate before its sigmoid)
 *   bias[h][i][j] = z[i*N+j] W_b[:, h]   (bias [H][N][N] bf16, device)
 * Requires H*D = 128, H in {1, 2, 4, 8}, N <= 32768.  z, w_qkvg, q, k, v, g
 * must be 16-byte aligned, w_b and bias 2-byte aligned (else
 * PBA_ERR_INVALID_ARG); other shapes give PBA_ERR_UNSUPPORTED.  N = 0 does
 * nothing and accepts NULL buffers.  The caller
 * owns every buffer; nothing is allocated.  Asynchronous on `stream`.
 * The pages fix no layout for these maps; q|k|v|g as column blocks of one
 * weight is the plain reading of "projections of the pair representation".
 */
PBA_API pba_status tri_proj_forward(int64_t N, int64_t c, int64_t H, int64_t D, const void *z, const void *w_qkvg,
                                    const void *w_b, void *q, void *k, void *v, void *g, void *bias, void *stream);

/*
 * tri_out_proj_forward -- the output projection of triangle attention back
 * to the pair channels (Fold-CP, Figure 2(a): triangle attention reads the
 * pair representation and its result returns to it; the pages fix no layout
 * for this map, and a plain linear map of the concatenated heads is the
 * reading taken here):
 *   o     [N][N][H][D] bf16, device (tri_attn_forward's output; H*D = 128)
 *   w_o   [H*D][c]     bf16, device
 *   out   [N][N][c]    bf16, device
 * out[r][:] = o[r][:] W_o for every pair row r = i*N + j, in fp32 sums of the
 * bf16 products, rounded once to bf16.  Requires H*D = 128 and c in {64, 128}
 * (else PBA_ERR_UNSUPPORTED), N <= 32768 and o, w_o, out 16-byte aligned
 * (else PBA_ERR_INVALID_ARG).  N = 0 does nothing and accepts NULL buffers.
 * The caller owns every buffer; nothing is allocated.  Asynchronous on
 * `stream`.
 */
PBA_API pba_status tri_out_proj_forward(int64_t N, int64_t c, int64_t H, int64_t D, const void *o, const void *w_o,
                                        void *out, void *stream);

/*
 * pwa_forward -- pair weighted averaging (Fold-CP, Table 1 row "Pair
 * Weighted Avg.", serial time B*H*S*N^2*D, distributed as a "2D ring + tiled
 * softmax"; Figure 2 groups it with the ring attention, a softmax whose
 * per-block partials are merged).  The pages print no formula; the reading implemented here is a
 * softmax over the pair-bias logits alone, shared by the S sequences:
 *   w[h][i][:]    = softmax_j( bias[h][i][j] )  over keys j with key_mask[j] != 0
 *   o[s][i][h][:] = sum_j w[h][i][j] v[s][j][h][:]
 *   out = o * sigmoid(gate) (gate NULL: out = o);  lse[h][i] = natural log-sum-exp
 *   v, gate, out [S][N][H][D] bf16, device; bias [H][N][N] bf16, device;
 *   key_mask [N] uint8, device, or NULL; lse [H][N] float, device (required:
 *   the softmax is taken in two passes, lse first, then the weights
 *   exp(bias - lse) times the values).
 * A row with no valid key gives out = 0 and lse = -inf.  D in {32, 64}
 * (else PBA_ERR_UNSUPPORTED); N a multiple of 8, v, bias, gate, out 16-byte
 * aligned and lse 4-byte aligned (else PBA_ERR_INVALID_ARG).  S = 0 or N = 0
 * writes nothing and accepts NULL buffers.  The caller owns every buffer;
 * nothing is allocated.  Asynchronous on `stream`.
 */
PBA_API pba_status pwa_forward(int64_t S, int64_t N, int64_t H, int64_t D, const void *v, const void *bias,
                               const uint8_t *key_mask, const void *gate, void *out, float *lse, void *stream);

/*
 * pba_backward -- gradients of pba_forward (training is distributed too:
 * Fold-CP, Figure 3 right).  With s_ij = tau q_i.k_j + b_ij over valid keys,
 * P_ij = exp(s_ij - lse_i) recomputed from the forward's log-sum-exp, and
 * dout = dL/dO:
 *   delta_i = sum_d dout_id out_id          (written: delta [B][H][Nq] float)
 *   dS_ij   = P_ij (dout_i . v_j - delta_i) (written: dbias [B][H][Nq][Nk] bf16;
 *                                            0 for masked keys and -inf bias)
 *   dq_i = tau sum_j dS_ij k_j,  dk_j = tau sum_i dS_ij q_i,  dv_j = sum_i P_ij dout_i
 *                                           (written: dq, dk, dv float, contiguous
 *                                            [B][H][Nq or Nk][D])
 * `desc` describes q, k, v, bias, key_mask, out, lse as for pba_forward; the
 * output strides also describe dout.  bf16 only.  q, k, v, out, dout and the
 * outputs must be contiguous [B][H][n][D], lse contiguous [B][H][Nq], the
 * bias row stride and Nk multiples of 8, every pointer 16-byte aligned
 * (else PBA_ERR_INVALID_ARG).  Nq = 0 or Nk = 0 writes nothing.  The caller
 * owns every buffer, delta included; nothing is allocated.  Asynchronous on
 * `stream`: one delta kernel, then one kernel for dq and dbias and one for dk
 * and dv.
 */
PBA_API pba_status pba_backward(const pba_attn_desc *desc, const void *q, const void *k, const void *v,
                                const void *bias, const uint8_t *key_mask, const void *out, const float *lse,
                                const void *dout, float *dq, float *dk, float *dv, void *dbias, float *delta,
                                void *stream);

/*
 * pba_backward_noalloc -- pba_backward for callers that cannot allocate
 * device memory.  No counterpart on the pages: it exists for callers that
 * hold only the tensors they were handed and no device allocator of their
 * own (a plugin inside another runtime's memory manager, a C host program
 * that links this library alone), or that must not call cudaMalloc or
 * cudaFree on their path because those calls can synchronise the device and
 * stall the work of other streams.
 *
 * Same arguments, checks, results and launches as pba_backward, without the
 * `delta` argument: the per-row Delta = rowsum(dout * out) that pba_backward
 * writes to a caller buffer goes to a fixed array of
 * PBA_BWD_NOALLOC_MAX_ROWS floats (4 MiB) inside the library, which every
 * GPU that loads the library holds until the process exits.  The call
 * allocates nothing.
 *   - B * H * Nq above PBA_BWD_NOALLOC_MAX_ROWS: PBA_ERR_INVALID_ARG before
 *     anything else (use pba_backward with a delta buffer of your own).
 *   - The first call on a device looks up that device's address of the array
 *     (with the device current); make that first call before any stream
 *     capture.  Every later call on the device reuses the address.
 *   - Every call on a device shares the one array and leaves its Delta in it.
 *     Nothing in it must start at zero: each call writes every row it reads
 *     before reading it.  Calls whose kernels overlap on the GPU (different
 *     streams, no ordering between them) race on the array and may compute
 *     wrong gradients: order them on one stream or with events.
 */
#define PBA_BWD_NOALLOC_MAX_ROWS 1048576
PBA_API pba_status pba_backward_noalloc(const pba_attn_desc *desc, const void *q, const void *k, const void *v,
                                        const void *bias, const uint8_t *key_mask, const void *out,
                                        const float *lse, const void *dout, float *dq, float *dk, float *dv,
                                        void *dbias, void *stream);

/* Human-readable name of a status code (static storage). */
PBA_API const char *pba_status_string(pba_status status);

/*
 * pba_last_device_error -- synchronises `stream`, then returns and clears the
 * device error word of the current device (PBA_OK if no kernel recorded an
 * error since the last call; PBA_ERR_TIMEOUT if a bounded wait ran out).  The
 * read and the clear are one atomic exchange on the device, so an error that
 * a kernel on another stream records meanwhile is reported by this call or
 * the next, never lost.  Launches one single-thread kernel on `stream`.
 * Returns PBA_ERR_CUDA if the synchronisation itself failed.
 */
PBA_API pba_status pba_last_device_error(void *stream);

/*
 * pba_set_wait_timeout_ns -- limit of every wait inside the kernels, in
 * nanoseconds of GPU global time (default 1e9 = 1 s; 0 restores the default).
 * Applies to launches made after the call.  Returns the previous value.
 */
PBA_API uint64_t pba_set_wait_timeout_ns(uint64_t timeout_ns);

/*
 * pba_selftest_wait_timeout -- launches one block that waits on a barrier
 * that nothing will ever complete, with a wait limit of `timeout_ns`, so that
 * the bounded-wait path can be checked without hanging the GPU.  The kernel
 * records PBA_ERR_TIMEOUT in the device error word and returns; read it with
 * pba_last_device_error.  No counterpart on the pages: it tests this
 * library's failure detection.
 */
PBA_API pba_status pba_selftest_wait_timeout(uint64_t timeout_ns, void *stream);

/*
 * pba_selftest_exp2 -- applies the kernels' software 2^x (the share of the
 * exponentials computed on the FMA pipe instead of the exp2 unit) to n floats:
 * out[i] = 2^in[i], in and out device arrays.  Range reduction 2^n * 2^f with
 * a degree-4 polynomial for 2^f on [-1/2, 1/2]; relative error below 1e-5 for
 * inputs in [-126, 128); inputs at or below -127 (and -inf) give exactly 0.
 * No counterpart on the pages: it lets tests check that approximation.
 */
PBA_API pba_status pba_selftest_exp2(const float *in, float *out, int64_t n, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PBA_H */
