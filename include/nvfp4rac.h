/*
 * nvfp4rac.h -- C ABI of the NVFP4 W4A4 + Residual Activation Compensation (RAC) library
 * (sm_100a, B200).
 *
 * The operations follow the rollout-side hot path of QUADS:
 *   - "QUADS: Stabilizing NVFP4 Reinforcement Learning for MoE via QUantization-error
 *     Alignment across Dual Sides" (mlsanity.com), Abstract (arXiv): NVFP4 pairs fine-grained
 *     scaling with native W4A4 FP4 GEMMs; weights are aligned through a shared
 *     quantization-dequantization path; activations are recomputed (quantised) online.
 *   - "Why 4-bit RL rollout collapses - and it isn't the weights", section "Two fixes, on two
 *     different sides": Asymmetric QAT fake-quantizes weights only (trainer side); Residual
 *     Activation Compensation selects roughly the top 50% of activation channels by
 *     quantization error and runs a second, residual FP4 pass over just those channels,
 *     keeping the native W4A4 GEMM intact (rollout side).
 *   - same post, "The failure mode": E2M1 has 8 magnitude levels per sign.
 *
 * NVFP4 storage used by every call (the pages fix no layout; this is the library's):
 *   element codes  E2M1 (sign bit 3, magnitude index 0..7 = {0,.5,1,1.5,2,3,4,6}); two codes per
 *                  byte, element 2j in the low nibble, 2j+1 in the high nibble; a matrix of
 *                  rows x cols is stored row-major as rows_padded x cols/2 bytes.
 *   block scales   one E4M3 code per 16 consecutive elements of a row, stored in
 *                  "scale-factor atoms" of 512 bytes, each covering 128 rows x 64 columns:
 *                  atom(rb, kb) starts at byte (rb * (cols/64) + kb) * 512; inside it the
 *                  scale of row r (r % 128 = 32*i + j) and 16-column block c (c % 4) is byte
 *                  j*16 + i*4 + c.  This is the order the tcgen05 block-scaled MMA consumes.
 *   tensor scale   one FP32 s_g per tensor (per slab for batched weights), s_g = amax / 2688.
 *   value          x ~= e(code) * S(block) * s_g.
 * Quantisation (bit-exact contract, binary32 round-to-nearest-even, no FMA contraction):
 *   b = max|x_i| over the block; S = E4M3_RNE_satfinite(b / (6*s_g)); d = S*s_g;
 *   S == 0 -> all codes +0; else q_i = E2M1_RNE_satfinite(x_i * (1/d)), sign kept.
 *   The residual of the selected channels is r_i = x_i - e(q_i)*d, gathered into ascending
 *   channel order and quantised with the same s_g.  amax == 0 gives s_g = 0 and zero codes.
 *
 * Conventions (all calls):
 *   - Pointers are DEVICE pointers owned by the caller unless stated otherwise.  The library
 *     never allocates device memory; calls that need scratch take a caller workspace whose
 *     size the matching *_workspace_size() returns.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *     Host-detectable errors (null pointers, bad shapes, misalignment) return a status before
 *     anything is launched.  Errors found on the device (amax out of range, a wait that ran
 *     out, an invalid channel list) are written, first one wins, to the caller's int32
 *     *dev_status (device memory, zero on entry); read it after synchronising.
 *   - No C++ exception crosses this interface.  nvfp4_last_error_string() gives the text of
 *     the last host-side error of the calling thread.
 *   - Shapes: K % 64 == 0, 0 <= Kp <= K, Kp % 64 == 0, N % 128 == 0 for GEMM weights.
 *     16-byte alignment is required for every matrix base pointer and row pitch.
 *   - bf16 data is passed as uint16_t bit patterns.
 */
#ifndef NVFP4RAC_H
#define NVFP4RAC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,     /* null pointer, bad enum, bad channel list */
  NVFP4_ERR_UNSUPPORTED_SHAPE = 2,
  NVFP4_ERR_ALIGNMENT = 3,
  NVFP4_ERR_RANGE = 4,           /* non-finite input or nonzero amax outside [2^-100, 2^100] */
  NVFP4_ERR_CUDA = 5,            /* a CUDA runtime/driver call failed */
  NVFP4_ERR_TIMEOUT = 6          /* a bounded device-side wait ran out */
} nvfp4_status;

typedef enum { NVFP4_OUT_F32 = 0, NVFP4_OUT_BF16 = 1 } nvfp4_dtype;

typedef enum {
  NVFP4_EPI_NONE = 0,
  /* gate_up epilogue of an MoE expert: the packed weight holds gate/up rows interleaved in
   * 64-row chunks (pack_weights with gate_up_interleave = 1); the output is
   * h = bf16(silu(bf16(g)) * bf16(u)) with N/2 columns, and max|h| is folded into *amax_out. */
  NVFP4_EPI_SWIGLU_AMAX = 1
} nvfp4_epilogue;

/* Order of the block scales of a packed matrix.
 *   NVFP4_SF_ATOM128  the atom order above: rows in groups of 128 (rows_padded % 128 == 0);
 *                     sf holds rows_padded * cols/16 bytes.
 *   NVFP4_SF_SLAB16   decode activations: rows in slabs of 16 (rows_padded % 16 == 0); slab
 *                     s = row / 16 owns one whole atom per 64 columns, atom(s, kb) at byte
 *                     (s * (cols/64) + kb) * 512, and row r of the slab uses atom row r % 16 with
 *                     i = 0 (scale of block c at byte (r % 16)*16 + c % 4); the other bytes of the
 *                     atom are never read.  sf holds rows_padded/16 * cols/64 * 512 bytes.  The
 *                     decode GEMM reads one atom per slab as the scales of its 16-token operand. */
typedef enum { NVFP4_SF_ATOM128 = 0, NVFP4_SF_SLAB16 = 1 } nvfp4_sf_layout;

/* A packed NVFP4 matrix, or `slabs` equally shaped matrices (MoE experts) back to back.
 * codes: slabs * rows_padded * cols/2 bytes; sf: slabs * nvfp4_sf_bytes(...) bytes (atoms);
 * s_g: `slabs` floats.  rows <= rows_padded, cols % 64 == 0; rows_padded % 128 == 0 for
 * NVFP4_SF_ATOM128 (the default of a zero-initialised struct), % 16 == 0 for NVFP4_SF_SLAB16. */
typedef struct {
  uint8_t* codes;
  uint8_t* sf;
  float* s_g;
  int64_t slabs;
  int64_t rows;
  int64_t rows_padded;
  int64_t cols;
  int32_t sf_layout; /* nvfp4_sf_layout */
} nvfp4_tensor;

/* ---------------------------------------------------------------------------------------- */
/* housekeeping                                                                             */
/* ---------------------------------------------------------------------------------------- */
int32_t nvfp4_version(void);
const char* nvfp4_status_string(nvfp4_status s);
/* Text of the last host-side error on the calling thread ("" if none). */
const char* nvfp4_last_error_string(void);
/* Bytes of codes / scale atoms of one rows_padded x cols NVFP4 matrix. */
size_t nvfp4_codes_bytes(int64_t rows_padded, int64_t cols);
size_t nvfp4_sf_bytes(int64_t rows_padded, int64_t cols);
/* Bytes of scale atoms of one rows_padded x cols matrix in the given nvfp4_sf_layout. */
size_t nvfp4_sf_bytes_layout(int64_t rows_padded, int64_t cols, int32_t sf_layout);
/* K' = r*K rounded to the nearest multiple of 64 (ties up), clamped to [0, K].
 * "roughly top-50%" (Two fixes, on two different sides) -> r = 0.5 by default. */
int32_t nvfp4_kp_from_ratio(int64_t K, double r);
/* Upper bound of the wait inside every device-side spin loop, in nanoseconds (default 2e9).
 * A wait that runs out sets NVFP4_ERR_TIMEOUT in *dev_status and the kernel returns. */
void nvfp4_set_wait_limit_ns(uint64_t ns);
/* Tuning: N-tile of the GEMM kernels, 128 or 256 (0 = automatic choice per shape). */
void nvfp4_set_gemm_tile_n(int32_t n);
/* Tuning: 1 runs the W4A4 + RAC GEMMs whose N is a multiple of 256 on pairs of SMs (one
 * 256 x 256 tile per cluster of two CTAs); 0 (default) keeps one SM per 128-row tile. */
void nvfp4_set_gemm_pairs(int32_t on);
/* Tuning: 1 (default) runs weight_qdq on tensors of up to 4M elements in one pass over HBM
 * (groups of CTAs meet at a per-tensor counter in the workspace, then re-read the tensor from
 * L2); 0 keeps the two passes (amax, then the fake-quant).  Results are identical. */
void nvfp4_set_qdq_one_pass(int32_t on);
/* Tuning: rows per tile (1..16) and consumer warps (4, 6, 7 or 8) of the activation quantiser
 * (0 = automatic choice per shape).  A forced shape that does not fit shared memory makes the
 * quantise calls fall back to the row quantiser. */
void nvfp4_set_act_tile(int32_t rows, int32_t warps);

/* ---------------------------------------------------------------------------------------- */
/* nvfp4_quantize -- online activation quantisation with the RAC residual pass              */
/* (Abstract: activations are recomputed online; Two fixes: residual FP4 pass over the      */
/* selected channels).                                                                       */
/*   x          bf16 [M x K], row pitch ldx elements (ldx >= K, ldx % 8 == 0).               */
/*   row_gather optional int32 [M_out]: output row o is x row row_gather[o]; -1 (or >= M)   */
/*              gives a zero row.  NULL: M_out must equal M and row o is x row o.            */
/*   sel, Kp    ascending channel list [Kp] (Kp % 64 == 0); Kp == 0 disables the residual.   */
/*   amax_in    optional device float: use it as amax (e.g. from the SwiGLU epilogue); NULL  */
/*              computes amax over x rows [0, M).                                            */
/*   q          output: slabs = 1, rows = M_out, rows_padded >= M_out, cols = K; either      */
/*              scale layout; rows >= M_out are written as zeros; q->s_g receives s_g.       */
/*   q_res      output (Kp > 0), same rows and scale layout; its s_g receives the same s_g.  */
/*              cols = Kp: the method's residual, gathered into ascending channel order.     */
/*              cols = K (a variant of the method, "masked full-K residual"): the residual   */
/*              stays at its channel, zero off sel, in 16-blocks along K; the GEMM then      */
/*              takes the main packed weight as w_sel with Kp = K (no W_sel is stored).      */
/*   workspace  >= nvfp4_quantize_workspace_size() bytes, 16-byte aligned.                   */
/* ---------------------------------------------------------------------------------------- */
size_t nvfp4_quantize_workspace_size(int64_t M, int64_t K);
nvfp4_status nvfp4_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                            const int32_t* row_gather, int64_t M_out, const int32_t* sel, int32_t Kp,
                            const float* amax_in, const nvfp4_tensor* q, const nvfp4_tensor* q_res,
                            void* workspace, size_t workspace_bytes, int32_t* dev_status,
                            void* stream);

/* ---------------------------------------------------------------------------------------- */
/* The own-scale residual (a variant the pages leave open).  "Why 4-bit RL rollout collapses  */
/* ..." (Two fixes, on two different sides) gives the residual pass over the selected channels */
/* but not the tensor scale of the residual.  The method's reading here shares s_g of X (both  */
/* products then add in one accumulator).  With NVFP4_RAC_OWN_RES_SCALE in `flags`:            */
/*   the quantise calls (*_ex) give Q(R_sel) its own tensor scale s_r = amax(R_sel) / 2688,    */
/*   amax over every row the call quantises (one extra pass over x that only finds max|R_sel|), */
/*   and write s_r to q_res->s_g (q->s_g keeps s_g of x); the workspace is required.           */
/*   the GEMM calls (*_ex) keep the main and the residual products in two accumulators and      */
/*   compute y = s_a s_w (Q(X) Q(W)^T) + s_r s_w (Q(R_sel) Q(W_sel)^T) with s_r = *a_res->s_g  */
/*   (N-tile 128, the SwiGLU epilogue included).                                               */
/* Without the flag the *_ex calls are the calls without the suffix.                            */
/* ---------------------------------------------------------------------------------------- */
#define NVFP4_RAC_OWN_RES_SCALE 1u
nvfp4_status nvfp4_quantize_ex(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const int32_t* row_gather,
                               int64_t M_out, const int32_t* sel, int32_t Kp, const float* amax_in,
                               const nvfp4_tensor* q, const nvfp4_tensor* q_res, void* workspace,
                               size_t workspace_bytes, int32_t* dev_status, void* stream, uint32_t flags);

/* ---------------------------------------------------------------------------------------- */
/* nvfp4_quantize_scatter -- nvfp4_quantize for an MoE dispatch: each source row is quantised */
/* once and its codes / scales are written to up to `fanout` output rows.                    */
/*   row_scatter  int32 [M x fanout]: output rows of source row m (entries < 0 are skipped;  */
/*                an entry >= q->rows_padded is an error reported in *dev_status).            */
/*   Output rows that no entry names are left untouched: a caller that pads expert segments  */
/*   zero-fills q / q_res once, and the padding stays zero across calls.                     */
/*   Other arguments as nvfp4_quantize; s_g is computed over the M source rows.              */
/* ---------------------------------------------------------------------------------------- */
nvfp4_status nvfp4_quantize_scatter(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const int32_t* row_scatter,
                                    int32_t fanout, const int32_t* sel, int32_t Kp, const float* amax_in,
                                    const nvfp4_tensor* q, const nvfp4_tensor* q_res, void* workspace,
                                    size_t workspace_bytes, int32_t* dev_status, void* stream);

nvfp4_status nvfp4_quantize_scatter_ex(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                       const int32_t* row_scatter, int32_t fanout, const int32_t* sel, int32_t Kp,
                                       const float* amax_in, const nvfp4_tensor* q, const nvfp4_tensor* q_res,
                                       void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream,
                                       uint32_t flags);

/* ---------------------------------------------------------------------------------------- */
/* nvfp4_quantize_segments -- nvfp4_quantize of the token rows of an expert-grouped layout   */
/* only: the input of the down projection (h), whose expert segments are padded to 128 rows. */
/*   x              bf16 [M x K] in the padded expert-grouped row order (pitch ldx).          */
/*   expert_offsets int32 [E] (device): first row of each segment (moe_dispatch_plan's         */
/*                  offsets); expert_rows int32 [E] (device): token rows of each segment.      */
/*   Rows [expert_offsets[e], expert_offsets[e] + expert_rows[e]) of x are quantised into the  */
/*   same rows of q / q_res; every other row of q / q_res is left untouched (a caller zeroes   */
/*   them once if it wants the padding to stay zero; the grouped GEMM does not store the       */
/*   output boxes of padding rows when given the same expert_rows).  A segment reaching past  */
/*   row M is skipped and NVFP4_ERR_INVALID_ARG goes to *dev_status.                          */
/*   s_g is computed over all M rows unless amax_in is given (the SwiGLU epilogue's amax      */
/*   covers the token rows).  q.rows_padded >= M; 1 <= E <= 1024.  Other arguments as         */
/*   nvfp4_quantize (shared list, compact residual).                                          */
/* ---------------------------------------------------------------------------------------- */
nvfp4_status nvfp4_quantize_segments(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                     const int32_t* expert_offsets, const int32_t* expert_rows, int32_t E,
                                     const int32_t* sel, int32_t Kp, const float* amax_in, const nvfp4_tensor* q,
                                     const nvfp4_tensor* q_res, void* workspace, size_t workspace_bytes,
                                     int32_t* dev_status, void* stream);
nvfp4_status nvfp4_quantize_segments_ex(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                        const int32_t* expert_offsets, const int32_t* expert_rows, int32_t E,
                                        const int32_t* sel, int32_t Kp, const float* amax_in, const nvfp4_tensor* q,
                                        const nvfp4_tensor* q_res, void* workspace, size_t workspace_bytes,
                                        int32_t* dev_status, void* stream, uint32_t flags);

/* ---------------------------------------------------------------------------------------- */
/* nvfp4_quantize_grouped_sel -- nvfp4_quantize with one channel list per group of output    */
/* rows: the per-expert RAC variant for the down projection (the pages pick "the channels     */
/* with the largest quantization error" (Two fixes) without saying whether one list serves    */
/* every expert; this call takes one list per expert).                                        */
/*   row_group  int32 [q->rows_padded] (device): output row o uses list row_group[o]; a value */
/*              < 0 writes an all-zero residual row (padding); >= groups is an error reported */
/*              in *dev_status (the row's residual is then zero).  moe_row_groups makes it    */
/*              from expert offsets.                                                          */
/*   groups, sel  sel int32 [groups x Kp] (device, 16-byte aligned), each row ascending in    */
/*              [0, K) (checked on the device: NVFP4_ERR_INVALID_ARG in *dev_status).         */
/*   q_res      the compact residual only (cols == Kp > 0).  Other arguments as               */
/*              nvfp4_quantize; the main codes and s_g do not depend on the lists.             */
/* ---------------------------------------------------------------------------------------- */
nvfp4_status nvfp4_quantize_grouped_sel(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                        const int32_t* row_gather, int64_t M_out, const int32_t* row_group,
                                        int32_t groups, const int32_t* sel, int32_t Kp, const float* amax_in,
                                        const nvfp4_tensor* q, const nvfp4_tensor* q_res, void* workspace,
                                        size_t workspace_bytes, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------------------- */
/* rac_calibrate -- pick the Kp channels with the largest quantisation error                */
/* (Two fixes: "the roughly top-50% of activation channels with the largest quantization    */
/* error").  The calibration batch is quantised with its own s_g; e_k = sum_t r_{t,k}^2 in   */
/* binary64 with t ascending; the Kp largest e_k (ties -> lower k) are returned ascending.   */
/*   x_cal        bf16 [T x K] contiguous.                                                   */
/*   sel_out      int32 [Kp] (device).  chan_err_out: optional float64 [K] (device).         */
/* ---------------------------------------------------------------------------------------- */
size_t rac_calibrate_workspace_size(int64_t T, int64_t K);
nvfp4_status rac_calibrate(const uint16_t* x_cal, int64_t T, int64_t K, int32_t Kp, int32_t* sel_out,
                           double* chan_err_out, void* workspace, size_t workspace_bytes,
                           int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------------------- */
/* rac_calibrate_grouped -- one channel list per group of calibration rows (per-expert        */
/* variant).  x_cal rows are grouped: group g = rows [group_offsets[g], group_offsets[g+1])   */
/* (int32 [groups + 1], device, non-decreasing inside [0, T], else NVFP4_ERR_INVALID_ARG in   */
/* *dev_status).  The whole batch is quantised once with its own s_g (as rac_calibrate); e_k  */
/* of group g sums only its rows in binary64, t ascending; each group keeps its Kp largest    */
/* (ties -> lower k), ascending.  An empty group gets channels 0 .. Kp-1.                     */
/*   sel_out      int32 [groups x Kp]; chan_err_out optional float64 [groups x K] (device).    */
/*   workspace    >= rac_calibrate_grouped_workspace_size(T, K, groups) bytes.                */
/* ---------------------------------------------------------------------------------------- */
size_t rac_calibrate_grouped_workspace_size(int64_t T, int64_t K, int32_t groups);
nvfp4_status rac_calibrate_grouped(const uint16_t* x_cal, int64_t T, int64_t K, const int32_t* group_offsets,
                                   int32_t groups, int32_t Kp, int32_t* sel_out, double* chan_err_out,
                                   void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------------------- */
/* pack_weights -- rollout side of the shared weight QDQ path (Abstract: weights aligned by  */
/* a shared quantization-dequantization path), run once per trainer -> rollout sync.         */
/*   w        bf16 [E x N x K] contiguous (E experts, or E = 1).                             */
/*   sel, Kp  channel list of the layer input; W_sel = W[:, sel] (raw bf16 columns) is      */
/*            quantised with the slab's own s_gw.  Kp == 0: w_sel_q may be NULL.             */
/*   gate_up_interleave  0: packed rows in logical order.  1 (MoE gate_up, N/2 % 64 == 0):   */
/*            packed row 128q + j holds gate row 64q + j (j < 64) or up row N/2 + 64q + j-64. */
/*   w_q      output, slabs = E, rows = N, rows_padded = N (N % 128 == 0), cols = K.         */
/*   w_sel_q  output, slabs = E, rows = N, rows_padded = N, cols = Kp.                       */
/* ---------------------------------------------------------------------------------------- */
size_t pack_weights_workspace_size(int64_t E, int64_t N, int64_t K);
nvfp4_status pack_weights(const uint16_t* w, int64_t E, int64_t N, int64_t K, const int32_t* sel, int32_t Kp,
                          int32_t gate_up_interleave, const nvfp4_tensor* w_q, const nvfp4_tensor* w_sel_q,
                          void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/* pack_weights_grouped_sel -- pack_weights with one channel list per expert: sel int32        */
/* [E x Kp] (device, 16-byte aligned; each row ascending in [0, K), checked on the device);    */
/* W_sel of expert e = W_e[:, sel[e]] with e's own s_gw.  Other arguments as pack_weights.     */
nvfp4_status pack_weights_grouped_sel(const uint16_t* w, int64_t E, int64_t N, int64_t K, const int32_t* sel,
                                      int32_t Kp, int32_t gate_up_interleave, const nvfp4_tensor* w_q,
                                      const nvfp4_tensor* w_sel_q, void* workspace, size_t workspace_bytes,
                                      int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------------------- */
/* w4a4_rac_gemm -- Y = s_a*s_w*( Q(X) Q(W)^T + Q(R_sel) Q(W_sel)^T ) in one kernel with     */
/* one FP32 accumulator (tcgen05 block-scaled FP4 MMA; the residual K' loop follows the main */
/* K loop into the same tensor-memory accumulator).  "The native W4A4 GEMM path stays        */
/* intact" (Two fixes): with Kp == 0 this is the plain W4A4 GEMM.                            */
/*   a, a_res  from nvfp4_quantize (rows >= M, cols K / Kp).                                 */
/*   w, w_sel  from pack_weights with E = 1 (rows N).                                        */
/*   y         [M x N] FP32 or bf16, row pitch ldy elements (ldy % 8 == 0).                  */
/* ---------------------------------------------------------------------------------------- */
nvfp4_status w4a4_rac_gemm(const nvfp4_tensor* a, const nvfp4_tensor* a_res, const nvfp4_tensor* w,
                           const nvfp4_tensor* w_sel, int64_t M, int64_t N, int64_t K, int32_t Kp,
                           nvfp4_dtype out, void* y, int64_t ldy, int32_t* dev_status, void* stream);
/* w4a4_rac_gemm with flags (NVFP4_RAC_OWN_RES_SCALE: see the quantise calls above). */
nvfp4_status w4a4_rac_gemm_ex(const nvfp4_tensor* a, const nvfp4_tensor* a_res, const nvfp4_tensor* w,
                              const nvfp4_tensor* w_sel, int64_t M, int64_t N, int64_t K, int32_t Kp, nvfp4_dtype out,
                              void* y, int64_t ldy, int32_t* dev_status, void* stream, uint32_t flags);

/* ---------------------------------------------------------------------------------------- */
/* grouped_w4a4_rac_moe -- the GEMM above over token-sorted expert segments (MoE rollout).   */
/*   a, a_res         expert-sorted activations (nvfp4_quantize with row_gather); segment e  */
/*                    occupies rows [expert_offsets[e], expert_offsets[e+1]).                 */
/*   expert_offsets   device int32 [E+1], non-decreasing multiples of 128, offsets[0] = 0,   */
/*                    offsets[E] <= a->rows_padded.  Read on the device only.                */
/*   expert_rows      optional device int32 [E]: rows of segment e that hold tokens (the     */
/*                    rest is padding).  Output boxes of 32 rows that hold padding only are  */
/*                    not written (their contents stay as they were) and the SwiGLU amax     */
/*                    covers the counted rows.  NULL: every row is written (padding as 0).  */
/*   w, w_sel         pack_weights output with slabs = E.  alpha_e = a.s_g * w.s_g[e].        */
/*   ep               NVFP4_EPI_NONE: y [offsets[E] x N]; NVFP4_EPI_SWIGLU_AMAX: y bf16      */
/*                    [offsets[E] x N/2] and max|y| folded into *amax_out (device float, the  */
/*                    call zeroes it first).  Rows of padding come out as zeros.             */
/* ---------------------------------------------------------------------------------------- */
nvfp4_status grouped_w4a4_rac_moe(const nvfp4_tensor* a, const nvfp4_tensor* a_res, const int32_t* expert_offsets,
                                  const int32_t* expert_rows, int32_t E, const nvfp4_tensor* w,
                                  const nvfp4_tensor* w_sel, int64_t N, int64_t K, int32_t Kp, nvfp4_epilogue ep,
                                  nvfp4_dtype out, void* y, int64_t ldy, float* amax_out, int32_t* dev_status,
                                  void* stream);
/* grouped_w4a4_rac_moe with flags (NVFP4_RAC_OWN_RES_SCALE: see the quantise calls above). */
nvfp4_status grouped_w4a4_rac_moe_ex(const nvfp4_tensor* a, const nvfp4_tensor* a_res, const int32_t* expert_offsets,
                                     const int32_t* expert_rows, int32_t E, const nvfp4_tensor* w,
                                     const nvfp4_tensor* w_sel, int64_t N, int64_t K, int32_t Kp, nvfp4_epilogue ep,
                                     nvfp4_dtype out, void* y, int64_t ldy, float* amax_out, int32_t* dev_status,
                                     void* stream, uint32_t flags);

/* ---------------------------------------------------------------------------------------- */
/* grouped_w4a4_rac_moe_segments -- grouped_w4a4_rac_moe over arbitrary row segments, each   */
/* with its own weight slab: what an expert-parallel rank receives (one 128-padded segment per */
/* source rank and local expert, source-major), run without reordering the rows.             */
/*   seg_offsets int32 [n_seg + 1] (device): segment i is rows [seg_offsets[i],               */
/*               seg_offsets[i+1]) (multiples of 128); seg_rows optional int32 [n_seg]: token */
/*               rows of each segment (as expert_rows); seg_expert int32 [n_seg]: slab of w /  */
/*               w_sel used by segment i (0 <= seg_expert[i] < w->slabs, else                  */
/*               NVFP4_ERR_INVALID_ARG in *dev_status and slab 0 is read instead).              */
/*   Other arguments as grouped_w4a4_rac_moe (E there = n_seg here).                           */
/* ---------------------------------------------------------------------------------------- */
nvfp4_status grouped_w4a4_rac_moe_segments(const nvfp4_tensor* a, const nvfp4_tensor* a_res,
                                           const int32_t* seg_offsets, const int32_t* seg_rows,
                                           const int32_t* seg_expert, int32_t n_seg, const nvfp4_tensor* w,
                                           const nvfp4_tensor* w_sel, int64_t N, int64_t K, int32_t Kp,
                                           nvfp4_epilogue ep, nvfp4_dtype out, void* y, int64_t ldy,
                                           float* amax_out, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------------------- */
/* nvfp4_amax -- max |x| over a bf16 [M x K] matrix (pitch ldx) into *amax_out (device float): */
/* the input of the per-tensor scale s_g = amax / 2688.  An expert-parallel layer reduces it  */
/* over the ranks (a MAX all-reduce) and passes it to the quantise calls as amax_in, so that  */
/* every rank quantises with the scale of the whole batch.  workspace as nvfp4_quantize.       */
/* ---------------------------------------------------------------------------------------- */
nvfp4_status nvfp4_amax(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, float* amax_out, void* workspace,
                        size_t workspace_bytes, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------------------- */
/* grouped_w4a4_rac_moe_decode -- the grouped GEMM above for decode, where each expert sees   */
/* only a few tokens.  The expert's weight rows are streamed as the MMA's 128-row operand and  */
/* the expert's tokens, gathered into 16-row slabs, are the 16-column operand, so one pass     */
/* reads each touched expert's W and W_sel once per slab.  Same arithmetic as                 */
/* grouped_w4a4_rac_moe: y = alpha_e * (Q(X) Q(W_e)^T + Q(R_sel) Q(W_sel,e)^T), one FP32       */
/* accumulator, residual K' loop after the main K loop (Two fixes, on two different sides).    */
/*   a, a_res        activations in the NVFP4_SF_SLAB16 layout (nvfp4_quantize_scatter with    */
/*                   row_scatter naming rows 16*slot + j); rows_padded >= 16 * n_slots.        */
/*   slot_expert     device int32 [n_slots]: expert of each slab; e < 0 marks an unused slab  */
/*                   (skipped, its rows of y untouched); e >= E is NVFP4_ERR_INVALID_ARG in    */
/*                   *dev_status and the call stops.                                          */
/*   slot_count      device int32 [n_slots]: tokens in the slab (rows 16*slot + [0, count)    */
/*                   are results; the others are written as zeros).                           */
/*   w, w_sel, N, K, Kp, ep, amax_out  as grouped_w4a4_rac_moe (ep == SWIGLU_AMAX needs the   */
/*                   gate/up interleaved pack; amax covers the counted rows only).             */
/*   y               [16 * n_slots x N] (or N/2 with SwiGLU), FP32 or bf16, pitch ldy.         */
/* ---------------------------------------------------------------------------------------- */
nvfp4_status grouped_w4a4_rac_moe_decode(const nvfp4_tensor* a, const nvfp4_tensor* a_res,
                                         const int32_t* slot_expert, const int32_t* slot_count, int32_t n_slots,
                                         int32_t E, const nvfp4_tensor* w, const nvfp4_tensor* w_sel, int64_t N,
                                         int64_t K, int32_t Kp, nvfp4_epilogue ep, nvfp4_dtype out, void* y,
                                         int64_t ldy, float* amax_out, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------------------- */
/* The MoE block around the expert GEMMs, on the device, so that a step needs no host work.   */
/* The pages describe none of it (the method only names MoE rollout, Abstract); the readings: */
/* the top-k of softmax(logits) are the k largest logits, ties to the lower expert; a chosen  */
/* expert's weight is its probability renormalised over the k chosen,                          */
/* w_j = exp(l_j - l_max) / sum_i exp(l_i - l_max); pairs are grouped by expert with tokens   */
/* ascending; out[t] = sum_j w_tj * y[row(t, j)].                                             */
/* ---------------------------------------------------------------------------------------- */
/* moe_route_topk -- logits float32 [T x E] (finite, else NVFP4_ERR_RANGE in *dev_status),    */
/*   E <= 1024, k <= min(32, E).  topk_ids int32 [T x k] (best first), topk_w float32 [T x k]. */
nvfp4_status moe_route_topk(const float* logits, int64_t T, int32_t E, int32_t k, int32_t* topk_ids, float* topk_w,
                            int32_t* dev_status, void* stream);
/* Rows a dispatch plan can need at most (every routed expert wasting pad - 1 rows), rounded
 * up to a multiple of 128: size activation buffers with it (decode: rows / 16 slots). */
int64_t moe_rows_capacity(int64_t T, int32_t k, int32_t E, int32_t pad);
size_t moe_dispatch_workspace_size(int32_t E);
/* moe_dispatch_plan -- expert-grouped layout of the (token, expert) pairs of topk_ids [T x k]  */
/* (a token's experts must be distinct; k <= 128).                                            */
/*   pad            segment granularity, a multiple of 16: 128 for grouped_w4a4_rac_moe, 16 for */
/*                  the decode slabs.                                                          */
/*   expert_offsets int32 [E+1]: padded segment starts; offsets[E] = rows used, or -1 if they   */
/*                  would exceed rows_capacity (or the slot table), with NVFP4_ERR_INVALID_ARG */
/*                  in *dev_status; the GEMMs then do nothing.                                 */
/*   row_scatter    int32 [T x k]: row of pair (t, j), the row_scatter of                      */
/*                  nvfp4_quantize_scatter (fanout k) and of moe_combine; -1 if unrouted.     */
/*   expert_rows    optional int32 [E]: tokens routed to each expert (the expert_rows of       */
/*                  grouped_w4a4_rac_moe).                                                    */
/*   slot_expert, slot_count  optional int32 [n_slots] (pad == 16): the decode slot tables;    */
/*                  slots past the used ones get expert -1, which the decode GEMM skips.      */
nvfp4_status moe_dispatch_plan(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E, int32_t pad,
                               int64_t rows_capacity, int32_t* expert_offsets, int32_t* row_scatter,
                               int32_t* expert_rows, int32_t* slot_expert, int32_t* slot_count, int32_t n_slots,
                               void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);
/* moe_row_groups -- row_group[r] = e for rows r in [expert_offsets[e], expert_offsets[e+1])  */
/* of an expert-grouped layout (moe_dispatch_plan's offsets, any padding), -1 for rows at or  */
/* past expert_offsets[E] and for every row when expert_offsets[E] < 0 (a plan that did not   */
/* fit).  row_group: int32 [rows] (device).  Feeds nvfp4_quantize_grouped_sel.                */
nvfp4_status moe_row_groups(const int32_t* expert_offsets, int32_t E, int64_t rows, int32_t* row_group,
                            void* stream);

/* moe_combine -- out[t, :] = sum_j topk_w[t, j] * y[row_scatter[t, j], :] (binary32 sums in   */
/* j order, bf16 out); y bf16 with y_rows rows, pitch ldy; out bf16 [T x H], pitch ldo;       */
/* H % 8 == 0.  A row < 0 contributes nothing; a row >= y_rows is NVFP4_ERR_INVALID_ARG.      */
nvfp4_status moe_combine(const uint16_t* y, int64_t ldy, int64_t y_rows, const int32_t* row_scatter,
                         const float* topk_w, int64_t T, int32_t k, int64_t H, uint16_t* out, int64_t ldo,
                         int32_t* dev_status, void* stream);

/* moe_row_pairs -- the inverse of row_scatter: row_pair[r] = t * k + j where                 */
/*   row_scatter[t, j] = r, -1 on rows that hold no pair (padding).  row_pair int32 [rows]     */
/*   (device); a row_scatter entry >= rows is NVFP4_ERR_INVALID_ARG in *dev_status.            */
nvfp4_status moe_row_pairs(const int32_t* row_scatter, int64_t T, int32_t k, int64_t rows, int32_t* row_pair,
                           int32_t* dev_status, void* stream);
/* grouped_w4a4_rac_moe_combine -- the down projection of the MoE block with moe_combine in    */
/*   its epilogue (the expert rows are never written to memory):                               */
/*   out[t, :] = bf16( sum_j topk_w[t, j] * y_r ),  y_r = bf16(alpha_e * acc_r), r the row of   */
/*   pair (t, j), acc_r as in grouped_w4a4_rac_moe (NVFP4_EPI_NONE).  Each product            */
/*   RN(topk_w * y_r) is added into the binary32 row out32[t] by atomic vector adds, so the   */
/*   k terms of a token are summed in an unspecified order (reading: the same sum as          */
/*   moe_combine up to binary32 reassociation, |difference| <= k * 2^-23 * sum_j |w_j y_j|    */
/*   before the final bf16 rounding).                                                          */
/*   a, a_res, expert_offsets, expert_rows, E, w, w_sel, N, K, Kp  as grouped_w4a4_rac_moe.  */
/*   row_pair   int32 [a.rows_padded] (device, moe_row_pairs): the pair of each row, -1 none.  */
/*   topk_w     float32 [T x k] (device, moe_route_topk).                                      */
/*   out32      float32 [T x N] workspace, pitch N, 16-byte aligned; the call zeroes it.       */
/*   out        bf16 [T x N], pitch ldo (multiple of 8, 16-byte aligned).                      */
/*   Single-SM GEMM tiles only (NVFP4_ERR_UNSUPPORTED_SHAPE while CTA pairs are switched on). */
nvfp4_status grouped_w4a4_rac_moe_combine(const nvfp4_tensor* a, const nvfp4_tensor* a_res,
                                          const int32_t* expert_offsets, const int32_t* expert_rows, int32_t E,
                                          const nvfp4_tensor* w, const nvfp4_tensor* w_sel, int64_t N, int64_t K,
                                          int32_t Kp, const int32_t* row_pair, const float* topk_w, int64_t T,
                                          int32_t k, float* out32, uint16_t* out, int64_t ldo, int32_t* dev_status,
                                          void* stream);

/* ---------------------------------------------------------------------------------------- */
/* weight_qdq -- trainer-side Asymmetric QAT fake quantisation of weights only (Two fixes):  */
/* w_out = bf16(DQ(Q(w))) with one s_g per tensor; activations are not touched.  The         */
/* quantiser is the one pack_weights uses, so DQ(pack_weights(W)) == weight_qdq(W) bitwise.  */
/*   w, w_out         bf16 [n_tensors x elems_per_tensor] contiguous (elems % 16 == 0).       */
/*   s_g_out          optional device float [n_tensors].                                     */
/* ---------------------------------------------------------------------------------------- */
size_t weight_qdq_workspace_size(int64_t n_tensors, int64_t elems_per_tensor);
nvfp4_status weight_qdq(const uint16_t* w, int64_t n_tensors, int64_t elems_per_tensor, uint16_t* w_out,
                        float* s_g_out, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                        void* stream);

/* ---------------------------------------------------------------------------------------- */
/* weight_qdq_backward -- gradient of the trainer fake-quant (Two fixes: Asymmetric QAT       */
/* fake-quantises the weights only) under the straight-through estimator: the rounding of     */
/* W_fq = bf16(DQ(Q(W))) is treated as the identity, so dL/dW = dL/dW_fq.  (A reading: the    */
/* pages name QAT on weights without its backward rule; the straight-through estimator is the */
/* usual one, and with a per-tensor amax scale no element sits in a clipped range.)            */
/*   grad_fq   bf16 [n]: dL/dW_fq.                                                            */
/*   grad_w    optional bf16 [n]: receives dL/dW (== grad_fq bitwise; grad_w == grad_fq is    */
/*             allowed and launches nothing).                                                  */
/*   grad_acc  optional float32 [n]: the trainer's master gradient, grad_acc += dL/dW (one     */
/*             binary32 add per element).  At least one of grad_w / grad_acc.                 */
/*   All buffers 16-byte aligned.                                                              */
/* ---------------------------------------------------------------------------------------- */
nvfp4_status weight_qdq_backward(const uint16_t* grad_fq, int64_t n, uint16_t* grad_w, float* grad_acc,
                                 void* stream);

/* ---------------------------------------------------------------------------------------- */
/* nvfp4_unpack_logical -- a packed matrix in logical order (inspection and test helper).     */
/*   q          packed tensor (either scale layout); slab in [0, q->slabs) picks one matrix.  */
/*   codes_out  optional uint8 [q->rows x q->cols] (16-byte aligned): one E2M1 code per byte.  */
/*   sf_out     optional uint8 [q->rows x q->cols/16]: the E4M3 scale of (row, 16-block).      */
/*   Rows >= q->rows are not read.                                                             */
/* ---------------------------------------------------------------------------------------- */
nvfp4_status nvfp4_unpack_logical(const nvfp4_tensor* q, int64_t slab, uint8_t* codes_out, uint8_t* sf_out,
                                  void* stream);

/* ---------------------------------------------------------------------------------------- */
/* weight_qdq_noalloc -- weight_qdq for callers that cannot allocate device memory.          */
/* The paper has no counterpart: this is a library convenience.  Some callers of the         */
/* trainer-side fake-quant cannot call cudaMalloc: a training framework that owns all device */
/* memory through its own caching allocator (a raw cudaMalloc outside it fragments the pool  */
/* and can fail under memory pressure), a latency-bound loop that must not take the implicit  */
/* device synchronisation cudaMalloc/cudaFree may cause, or a plain C host program that links */
/* only this library and has no allocator plumbing.  This entry point needs no workspace: its */
/* amax scratch is a fixed 16 KiB array inside the library, resident on every GPU that loads  */
/* the library until the process exits.                                                      */
/*   Arguments, layout and results are those of weight_qdq (bitwise the same output).        */
/*   Limit: n_tensors * max(1, 512 / n_tensors) <= 4096 scratch floats, i.e. at most 4096     */
/*   tensors per call; larger calls return NVFP4_ERR_UNSUPPORTED_SHAPE with a message.        */
/*   The first call on a device looks up the scratch array's device address (once per        */
/*   device, with that device current); make that first call before any stream capture.      */
/*   The looked-up address is kept for the life of the process and is not refreshed: after   */
/*   cudaDeviceReset (or any other teardown of the device's primary context) it is stale, so  */
/*   do not call this entry point on that device again in the same process.                   */
/*   All calls share the one array, so calls that overlap on the GPU (different streams, or  */
/*   different host threads) race and may corrupt each other's scales: serialise them.        */
/*   Allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.            */
/* ---------------------------------------------------------------------------------------- */
nvfp4_status weight_qdq_noalloc(const uint16_t* w, int64_t n_tensors, int64_t elems_per_tensor, uint16_t* w_out,
                                float* s_g_out, int32_t* dev_status, void* stream);

/* ======================================================================================== */
/* FP8 comparison path.  The QUADS abstract reports the 4-bit rollouts about 16 % faster than */
/* FP8 rollouts but fixes no FP8 recipe; this is the block-scaled FP8 the tensor cores take   */
/* natively, run on the same shapes through the same GEMM kernel, so that the two formats     */
/* can be timed side by side.                                                                 */
/*   Format: E4M3 element codes (one byte each, row-major, sign kept), one power-of-two scale */
/*   2^X per 32 consecutive elements along K stored as the E8M0 code X + 127 in 512-byte     */
/*   atoms (128 rows x 4 blocks, the FP4 atom order with 32-element blocks); X is the         */
/*   smallest integer with 448 * 2^X >= max|x| of the block, clamped to [-127, 127], so no    */
/*   element saturates; q = E4M3_RNE_satfinite(RN(x * 2^-X)).  No tensor scale.              */
/*   Shape rules: K % 128 == 0, N % 128 == 0, rows_padded % 128 == 0.  A block holding an inf */
/*   or NaN is written as zero and NVFP4_ERR_RANGE goes to *dev_status.                       */
/* ======================================================================================== */
typedef struct mxfp8_tensor {
  uint8_t* codes;       /* device, slabs * rows_padded * cols bytes, 16-byte aligned */
  uint8_t* sf;          /* device, slabs * mxfp8_sf_bytes(rows_padded, cols) bytes, 16-byte aligned */
  int64_t slabs;        /* experts (weights) or 1 */
  int64_t rows;         /* logical rows per slab */
  int64_t rows_padded;  /* multiple of 128 */
  int64_t cols;         /* K */
} mxfp8_tensor;

size_t mxfp8_codes_bytes(int64_t rows_padded, int64_t cols);
size_t mxfp8_sf_bytes(int64_t rows_padded, int64_t cols);

/* mxfp8_quantize -- x bf16 [M x K] (pitch ldx, ldx % 8 == 0) -> q (rows >= M_out; rows past   */
/* M_out are written as zeros).  row_gather as in nvfp4_quantize.                              */
nvfp4_status mxfp8_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const int32_t* row_gather,
                            int64_t M_out, const mxfp8_tensor* q, int32_t* dev_status, void* stream);
/* mxfp8_quantize_scatter -- each x row quantised once and written to its row_scatter[m, :]    */
/* output rows (fanout <= 32; entries < 0 skipped; rows no entry names are left untouched).    */
nvfp4_status mxfp8_quantize_scatter(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const int32_t* row_scatter,
                                    int32_t fanout, const mxfp8_tensor* q, int32_t* dev_status, void* stream);
/* mxfp8_pack_weights -- w bf16 [E x N x K] -> w_q (slabs = E, rows = rows_padded = N);        */
/* gate_up_interleave as pack_weights.                                                         */
nvfp4_status mxfp8_pack_weights(const uint16_t* w, int64_t E, int64_t N, int64_t K, int32_t gate_up_interleave,
                                const mxfp8_tensor* w_q, int32_t* dev_status, void* stream);
/* mxfp8_gemm -- y [M x N] = A W^T over FP8 operands (one tensor-memory accumulator, K = 32    */
/* per block-scaled MMA); output and pitch rules as w4a4_rac_gemm.                             */
nvfp4_status mxfp8_gemm(const mxfp8_tensor* a, const mxfp8_tensor* w, int64_t M, int64_t N, int64_t K,
                        nvfp4_dtype out, void* y, int64_t ldy, int32_t* dev_status, void* stream);
/* grouped_mxfp8_moe -- grouped_w4a4_rac_moe over FP8 operands (no residual, alpha = 1);       */
/* amax_out is optional here (the FP8 format needs no tensor scale for h).                     */
nvfp4_status grouped_mxfp8_moe(const mxfp8_tensor* a, const int32_t* expert_offsets, const int32_t* expert_rows,
                               int32_t E, const mxfp8_tensor* w, int64_t N, int64_t K, nvfp4_epilogue ep,
                               nvfp4_dtype out, void* y, int64_t ldy, float* amax_out, int32_t* dev_status,
                               void* stream);

/* ---------------------------------------------------------------------------------------- */
/* test helpers (not part of the hot path)                                                   */
/* ---------------------------------------------------------------------------------------- */
/* The device E2M1 / E4M3 encoders applied to float32 inputs (v device [n], out device [n],
 * one code per byte; E4M3 takes non-negative inputs). */
nvfp4_status nvfp4_encode_e2m1(const float* v, int64_t n, uint8_t* out, void* stream);
nvfp4_status nvfp4_encode_e4m3(const float* v, int64_t n, uint8_t* out, void* stream);
/* Runs the bounded mbarrier wait used by every spin loop on a barrier that nothing completes,
 * with the given limit; expects *dev_status == NVFP4_ERR_TIMEOUT afterwards. */
nvfp4_status nvfp4_selftest_wait_timeout(uint64_t limit_ns, int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4RAC_H */
