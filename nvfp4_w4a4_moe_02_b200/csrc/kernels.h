// Internal launcher declarations shared by the kernel files and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4 {

enum { kModeAct = 0, kModePack = 1, kModeCal = 2 };
constexpr int64_t kMaxCalK = 16384;
constexpr int64_t kMaxK = 32768;

// Row quantiser arguments (one warp per output row).
struct RowArgs {
  int mode;                      // kModeAct, kModePack, kModeCal
  const uint16_t* src;           // bf16 rows
  int64_t src_rows;              // valid source rows (act: M; pack: N per slab; cal: T)
  int64_t ld;                    // source pitch (elements)
  int64_t K;                     // channels
  const int32_t* row_gather;     // act: optional output-row -> source-row map
  const int32_t* row_scatter;    // act: optional source-row -> fanout output rows (-1 = none)
  int fanout;
  int64_t rows_out;              // output rows to write (act: rows_padded; pack: slabs*rows_padded)
  int64_t rows_per_slab;         // pack: rows_padded per slab (== N); otherwise rows_out
  int64_t src_slab_stride;       // pack: N*K elements between slabs
  int interleave;                // pack: SwiGLU gate/up interleave
  int64_t N_half;                // pack: N/2
  const int32_t* sel;            // ascending channel list [Kp], or [sel_groups x Kp]
  int32_t Kp;
  int32_t sel_groups;            // 0: one shared list; G > 0: one list per group (per-expert variant)
  const int32_t* row_group;      // act with sel_groups: output row -> group (< 0: zero residual)
  // scale source
  const float* partial;          // amax partials [slabs x P]
  int P;
  const float* amax_in;          // act: given amax (overrides partials)
  float* s_g_out;                // per-slab s_g written by the first warp of each slab
  float* s_g_out2;               // second copy (residual tensor's s_g), may be null
  // outputs
  uint8_t* codes;                // [rows_out x K/2]
  uint8_t* sf;                   // atoms, K/64 groups per row
  int sf_slab16;                 // act: scales of codes/rcodes in the 16-row slab layout
  int masked_res;                // act: residual kept at its channel (zero off sel), K wide
  uint8_t* rcodes;               // [rows_out x Kp/2]
  uint8_t* rsf;                  // atoms, Kp/64 groups per row
  float* resid_all;              // cal: [rows_out x K] residual of every channel
  int32_t* status;
};

// Activation quantiser fed by bulk copies of row tiles (csrc/quant_act.cu): one shared channel
// list (or none); the masked and per-group residual variants use the row quantiser above.
enum { kMapRows = 0, kMapGather = 1, kMapScatter = 2, kMapSegments = 3 };
struct ActArgs {
  const uint16_t* src;           // bf16 rows, pitch ld elements
  int64_t src_rows;
  int64_t ld;
  int32_t K, Kp;                 // K % 64 == 0, Kp % 64 == 0
  int32_t map;                   // kMap*
  const int32_t* row_gather;     // gather: output row -> source row (< 0: zero row)
  const int32_t* row_scatter;    // scatter: [src_rows x fanout] output rows (< 0: none)
  int32_t fanout;                // 1 unless scatter
  const int32_t* seg_off;        // segments: first row of each segment [n_seg]
  const int32_t* seg_rows;       // segments: token rows of each segment [n_seg]
  int32_t n_seg;
  int64_t rows_out;              // rows (rows_padded) of the outputs
  int64_t rows_valid;            // rows / gather: output rows >= rows_valid are zero rows
  const int32_t* sel;            // ascending channel list [Kp]
  const float* partial;          // amax partials [P] (unless amax_in)
  int32_t P;
  const float* amax_in;
  float* s_g_out;
  float* s_g_out2;
  uint8_t* codes;
  uint8_t* sf;
  uint8_t* rcodes;
  uint8_t* rsf;
  int32_t sf_slab16;
  int32_t* status;
  uint64_t wait_limit_ns;
  int32_t R;                     // set by the launcher
  // residual tensor scale: 0 = the tensor scale of x (the method's reading); 1 = its own scale
  // from *res_amax_in; 2 = no output, max |R_sel| over the rows folded into *res_amax_out
  int32_t res_mode;
  const float* res_amax_in;
  float* res_amax_out;
};
bool act_plan_choose(int64_t K, int32_t Kp, int fanout, int32_t n_seg, int* R, int* W, int* smem, int force_R = 0,
                     int force_W = 0);
cudaError_t launch_act(ActArgs a, int num_sms, int force_R, int force_W, cudaStream_t st);

cudaError_t launch_amax(const uint16_t* x, int64_t segs, int64_t seg_rows, int64_t cols, int64_t ld, float* partial,
                        int P, int32_t* status, cudaStream_t st);
cudaError_t launch_reduce_amax(const float* partial, int P, float* out, cudaStream_t st);
cudaError_t launch_rows(const RowArgs& a, int num_sms, cudaStream_t st);
size_t rows_smem_bytes(int64_t K, int32_t Kp, int warps, bool masked = false);
cudaError_t launch_chan_err(const float* resid, int64_t T, int64_t K, const int32_t* off, int32_t groups,
                            double* err, int32_t* status, cudaStream_t st);
cudaError_t launch_select(const double* err, int32_t K, int32_t Kp, int32_t groups, int32_t* sel, double* err_out,
                          cudaStream_t st);
cudaError_t launch_qdq(const uint16_t* w, int64_t n_tensors, int64_t elems, uint16_t* out, const float* partial, int P,
                       float* s_g_out, int32_t* status, int num_sms, cudaStream_t st);
cudaError_t launch_unpack_logical(const uint8_t* codes, const uint8_t* sf, int64_t rows, int64_t cols, int slab16,
                                  uint8_t* codes_out, uint8_t* sf_out, int num_sms, cudaStream_t st);
int qdq_fused_group(int64_t n_tensors, int64_t elems, int grid);
cudaError_t launch_qdq_fused(const uint16_t* w, int64_t n_tensors, int64_t elems, uint16_t* out, uint32_t* sync_ws,
                             int GS, float* s_g_out, int32_t* status, uint64_t limit_ns, int num_sms, cudaStream_t st);
cudaError_t launch_qdq_backward(const uint16_t* g, int64_t n, uint16_t* gw, float* acc, int num_sms, cudaStream_t st);
cudaError_t launch_encode_e2m1(const float* v, int64_t n, uint8_t* out, cudaStream_t st);
cudaError_t launch_encode_e4m3(const float* v, int64_t n, uint8_t* out, cudaStream_t st);

// ---- FP8 comparison format: E4M3 codes, one E8M0 scale per 32 elements (atoms of 128 x 128)
struct Mx8RowArgs {
  const uint16_t* src;           // bf16 rows
  int64_t src_rows;              // valid source rows (act: M; pack: N per slab)
  int64_t ld;                    // source pitch (elements)
  int64_t K;                     // channels, K % 128 == 0
  const int32_t* row_gather;     // act: optional output-row -> source-row map
  const int32_t* row_scatter;    // act: optional source-row -> fanout output rows (-1 = none)
  int fanout;                    // <= 32
  int64_t rows_out;              // output rows (act: rows_padded; pack: slabs * N)
  int64_t rows_per_slab;         // pack: N; act: M_out
  int64_t src_slab_stride;       // pack: N*K elements between slabs
  int pack;                      // weight pack (slabs, optional gate/up interleave)
  int interleave;
  int64_t N_half;
  uint8_t* codes;                // [rows_out x K]
  uint8_t* sf;                   // atoms, K/128 per 128-row block
  int32_t* status;
};
cudaError_t launch_mx8_rows(const Mx8RowArgs& a, int num_sms, cudaStream_t st);

// ---- tcgen05 block-scaled GEMM (dense and grouped)
struct GemmArgs {
  const uint8_t* sfa;        // A scale atoms, rows_padded/128 x k64_main
  const uint8_t* sfa_res;    // A residual scale atoms, rows_padded/128 x k64_res
  const uint8_t* sfw;        // W scale atoms, per slab N/128 x k64_main
  const uint8_t* sfw_sel;    // W_sel scale atoms, per slab N/128 x k64_res
  int64_t sfw_slab_bytes;
  int64_t sfw_sel_slab_bytes;
  int32_t k64_main, k64_res; // K/64, Kp/64
  int32_t kt_main, kt_res;   // k-tiles of 256 elements (last may be partial)
  int32_t N;                 // output columns of the MMA (before the SwiGLU halving)
  int32_t n_blocks;          // N / BN
  const int32_t* offsets;    // grouped: device [E+1] segment starts; dense: nullptr
  const int32_t* expert_rows;  // grouped, optional device [E]: rows holding tokens per segment
  int32_t E;                 // grouped: segments (one per expert unless seg_expert is given)
  const int32_t* seg_expert; // grouped, optional device [E]: weight slab of each segment
  int32_t n_weights;         // grouped: weight slabs (bound of seg_expert)
  int64_t M;                 // dense: valid rows (stores masked beyond)
  int32_t m_blocks_dense;    // dense: ceil(M/128)
  int64_t rows_capacity;     // rows of the A / Y buffers
  const float* s_a;          // device scalar
  const float* s_w;          // device [E]
  void* y;
  int64_t ldy;
  int32_t out_bf16;
  int32_t epi;               // 0 none, 1 SwiGLU + amax, 2 weighted combine (row_pair, topk_w -> comb)
  float* amax_out;
  int32_t* status;
  uint64_t wait_limit_ns;
  int32_t fp8;               // 1: the FP8 comparison operands (E4M3, E8M0 per 32; kt_main = K/128, no residual)
  int32_t own_res_scale;     // 1: the residual has its own tensor scale *s_a_res (two accumulators, BN = 128)
  const float* s_a_res;      // own_res_scale: device scalar
  // epi == 2: row r's products topk_w[p] * bf16(alpha * acc) are added into comb[p / k_top]
  // (binary32, pitch ld_comb), p = row_pair[r] (< 0: no pair; >= n_pairs: reported)
  const int32_t* row_pair;
  const float* topk_w;
  int32_t k_top;
  int64_t n_pairs;
  float* comb;
  int64_t ld_comb;
};

// bn: 128 or 256
cudaError_t launch_gemm(int bn, const CUtensorMap& tm_a, const CUtensorMap& tm_ar, const CUtensorMap& tm_w,
                        const CUtensorMap& tm_ws, const CUtensorMap& tm_y, const GemmArgs& args, int grid,
                        cudaStream_t st);
size_t gemm_smem_bytes(int bn);
// CTA-pair form (csrc/gemm2.cu): FP4, N % 256 == 0, W tensor maps with 128-row boxes; grid of
// n_pairs clusters of two CTAs
cudaError_t launch_gemm_pair(const CUtensorMap& tm_a, const CUtensorMap& tm_ar, const CUtensorMap& tm_w,
                             const CUtensorMap& tm_ws, const CUtensorMap& tm_y, const GemmArgs& args, int n_pairs,
                             cudaStream_t st);
size_t gemm_pair_smem_bytes();

// ---- swap-AB decode GEMM (weights = MMA A, 16-token slabs = MMA B)
struct DecodeArgs {
  const uint8_t* sfx;        // activation scale atoms, slab layout, n_slots x k64_main
  const uint8_t* sfx_res;    // residual activation scale atoms, slab layout, n_slots x k64_res
  const uint8_t* sfw;        // W scale atoms, per slab N/128 x k64_main
  const uint8_t* sfw_sel;    // W_sel scale atoms, per slab N/128 x k64_res
  int64_t sfw_slab_bytes;
  int64_t sfw_sel_slab_bytes;
  int32_t k64_main, k64_res;
  int32_t kt_main, kt_res;
  int32_t m_tiles;           // N / 128
  const int32_t* slot_expert;  // device [n_slots]
  const int32_t* slot_count;   // device [n_slots], tokens of the slab (<= 16)
  int32_t n_slots;
  int32_t E;
  const float* s_x;          // device scalar
  const float* s_w;          // device [E]
  void* y;
  int64_t ldy;
  int32_t out_bf16;
  int32_t epi;               // 0 none, 1 SwiGLU + amax, 2 weighted combine (row_pair, topk_w -> comb)
  float* amax_out;
  int32_t* status;
  uint64_t wait_limit_ns;
};
cudaError_t launch_decode(const CUtensorMap& tm_w, const CUtensorMap& tm_ws, const CUtensorMap& tm_x,
                          const CUtensorMap& tm_xr, const DecodeArgs& args, int grid, cudaStream_t st);
size_t decode_smem_bytes();

// ---- MoE block around the GEMMs (csrc/moe.cu)
constexpr int kMaxRouteExperts = 1024;
cudaError_t launch_route_topk(const float* logits, int64_t T, int E, int k, int32_t* ids, float* w, int32_t* status,
                              cudaStream_t st);
cudaError_t launch_dispatch_plan(const int32_t* ids, int64_t T, int k, int E, int pad, int64_t rows_capacity,
                                 int32_t* counts, int32_t* offsets, int32_t* row_scatter, int32_t* expert_rows,
                                 int32_t* slot_expert, int32_t* slot_count, int n_slots, int num_sms,
                                 int32_t* status, cudaStream_t st);
cudaError_t launch_row_groups(const int32_t* off, int E, int64_t rows, int32_t* group, int num_sms, cudaStream_t st);
cudaError_t launch_row_pairs(const int32_t* row_scatter, int64_t n, int64_t rows, int32_t* row_pair, int num_sms,
                             int32_t* status, cudaStream_t st);
cudaError_t launch_combine_finalize(const float* acc, int64_t T, int64_t H, uint16_t* out, int64_t ldo, int num_sms,
                                    cudaStream_t st);
cudaError_t launch_combine(const uint16_t* y, int64_t ldy, int64_t y_rows, const int32_t* rows, const float* w,
                           int64_t T, int k, int64_t H, uint16_t* out, int64_t ldo, int num_sms, int32_t* status,
                           cudaStream_t st);

cudaError_t launch_wait_selftest(uint64_t limit_ns, int32_t* status, cudaStream_t st);

}  // namespace nvfp4
