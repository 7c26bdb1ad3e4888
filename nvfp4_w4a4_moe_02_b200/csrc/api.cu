// C-ABI entry points of the NVFP4 W4A4 + RAC library: argument checks, tensor-map encoding
// and kernel launches.  Nothing here allocates device memory; everything is enqueued on the
// caller's stream.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "common.cuh"
#include "kernels.h"
#include "nvfp4rac.h"

namespace {

thread_local std::string g_last_error;
std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};
std::atomic<int> g_tile_n{0};  // 0: automatic
std::atomic<int> g_act_rows{0}, g_act_warps{0};  // activation quantiser tile: 0 = automatic
std::atomic<int> g_gemm_pair{0};  // CTA-pair GEMM where the shape allows it
std::atomic<int> g_qdq_fused{1};  // one-pass fake-quant where the tensors fit

nvfp4_status fail(nvfp4_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

nvfp4_status cuda_fail(cudaError_t e, const char* what) {
  return fail(NVFP4_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Packed FP4 codes viewed as bytes: [slabs][rows][inner_bytes], 128-byte boxes of box_rows rows,
// 128-byte swizzle (the layout the tcgen05 descriptors expect).
nvfp4_status make_code_map(CUtensorMap* m, const void* base, uint64_t inner_bytes, uint64_t rows, uint64_t slabs,
                           uint32_t box_rows, cuuint32_t rank, const char* what) {
  auto fn = encode_fn();
  if (!fn) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[3] = {inner_bytes, rows, slabs};
  cuuint64_t strides[2] = {inner_bytes, inner_bytes * rows};
  cuuint32_t box[3] = {128, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(NVFP4_ERR_CUDA, "tensor map for %s failed (error %d, inner %llu bytes, rows %llu, slabs %llu)", what,
                (int)r, (unsigned long long)inner_bytes, (unsigned long long)rows, (unsigned long long)slabs);
  return NVFP4_OK;
}

// Output matrix [rows x cols] (bf16 or fp32, row pitch ld elements) stored by the GEMM epilogue
// in boxes of 32 rows x 128 bytes, 128-byte swizzle.  Rows beyond `rows` are clipped.
// kOutNarrow: boxes of 32 rows x 64 bytes without swizzle (the SwiGLU stores of the own-scale
// mode); kOutNarrow64: 32 rows x 64 bytes, 64-byte swizzle (the four-stage BN = 256 kernel)
enum OutBox { kOutWide = 0, kOutNarrow = 1, kOutNarrow64 = 2 };
nvfp4_status make_out_map(CUtensorMap* m, void* base, bool bf16, uint64_t cols, uint64_t rows, uint64_t ld,
                          OutBox mode = kOutWide) {
  const bool narrow = mode != kOutWide;
  auto fn = encode_fn();
  if (!fn) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  const uint64_t esz = bf16 ? 2 : 4;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * esz};
  cuuint32_t box[2] = {(cuuint32_t)((narrow ? 64 : 128) / esz), 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  mode == kOutNarrow    ? CU_TENSOR_MAP_SWIZZLE_NONE
                  : mode == kOutNarrow64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                         : CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(NVFP4_ERR_CUDA, "tensor map for the output failed (error %d, cols %llu, rows %llu)", (int)r,
                (unsigned long long)cols, (unsigned long long)rows);
  return NVFP4_OK;
}

// layouts: bit mask of the accepted nvfp4_sf_layout values (1 << layout)
constexpr int kAtom128Only = 1 << NVFP4_SF_ATOM128;
constexpr int kSlab16Only = 1 << NVFP4_SF_SLAB16;
constexpr int kAnyLayout = kAtom128Only | kSlab16Only;

nvfp4_status check_tensor(const nvfp4_tensor* t, const char* name, int64_t cols, int64_t min_rows, int64_t slabs,
                          int layouts = kAtom128Only) {
  if (!t) return fail(NVFP4_ERR_INVALID_ARG, "%s is NULL", name);
  if (!t->codes || !t->sf || !t->s_g) return fail(NVFP4_ERR_INVALID_ARG, "%s has a NULL buffer", name);
  if (t->cols != cols) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "%s.cols = %lld, expected %lld", name, (long long)t->cols, (long long)cols);
  if (t->slabs != slabs) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "%s.slabs = %lld, expected %lld", name, (long long)t->slabs, (long long)slabs);
  if (t->sf_layout != NVFP4_SF_ATOM128 && t->sf_layout != NVFP4_SF_SLAB16)
    return fail(NVFP4_ERR_INVALID_ARG, "%s.sf_layout = %d is not a scale layout", name, (int)t->sf_layout);
  if (((1 << t->sf_layout) & layouts) == 0)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "%s.sf_layout = %d is not accepted by this call", name, (int)t->sf_layout);
  const int64_t group = t->sf_layout == NVFP4_SF_SLAB16 ? 16 : 128;
  if (t->rows_padded % group != 0 || t->rows_padded < min_rows || t->rows < 0 || t->rows > t->rows_padded)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "%s rows %lld / rows_padded %lld invalid (need >= %lld, multiple of %lld)", name,
                (long long)t->rows, (long long)t->rows_padded, (long long)min_rows, (long long)group);
  if (!aligned16(t->codes) || !aligned16(t->sf)) return fail(NVFP4_ERR_ALIGNMENT, "%s buffers must be 16-byte aligned", name);
  return NVFP4_OK;
}

int act_partials(int64_t M, int64_t K) {
  int64_t p = (M * K) / 16384;
  if (p < 1) p = 1;
  if (p > 1024) p = 1024;
  return (int)p;
}
int slab_partials(int64_t slabs) {
  int64_t p = 512 / (slabs > 0 ? slabs : 1);
  return (int)(p < 1 ? 1 : p);
}
size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// N-tile of the GEMM: 256 (one accumulator, best MMA / scale-copy ratio) unless forced or N
// is not a multiple of 256.
int choose_tile_n(int64_t N, int64_t K, int64_t Kp) {
  (void)K;
  (void)Kp;
  const int forced = g_tile_n.load();
  if (forced == 128) return 128;
  if (forced == 256 && N % 256 == 0) return 256;
  return (N % 256 == 0) ? 256 : 128;
}

}  // namespace

using namespace nvfp4;

extern "C" {

int32_t nvfp4_version(void) { return 100; }

const char* nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case NVFP4_ERR_ALIGNMENT: return "misaligned pointer or pitch";
    case NVFP4_ERR_RANGE: return "value out of range";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* nvfp4_last_error_string(void) { return g_last_error.c_str(); }

size_t nvfp4_codes_bytes(int64_t rows_padded, int64_t cols) { return (size_t)rows_padded * (size_t)(cols / 2); }
size_t nvfp4_sf_bytes(int64_t rows_padded, int64_t cols) { return (size_t)rows_padded * (size_t)(cols / 16); }
size_t nvfp4_sf_bytes_layout(int64_t rows_padded, int64_t cols, int32_t sf_layout) {
  if (sf_layout == NVFP4_SF_SLAB16) return (size_t)(rows_padded / 16) * (size_t)(cols / 64) * 512;
  return nvfp4_sf_bytes(rows_padded, cols);
}

int32_t nvfp4_kp_from_ratio(int64_t K, double r) {
  if (!(r > 0.0)) return 0;
  double q = r * (double)K / 64.0;
  int64_t kp = (int64_t)(q + 0.5) * 64;
  if (kp > K) kp = K / 64 * 64;
  if (kp < 0) kp = 0;
  return (int32_t)kp;
}

void nvfp4_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns); }

void nvfp4_set_gemm_tile_n(int32_t n) { g_tile_n.store((n == 128 || n == 256) ? n : 0); }

void nvfp4_set_gemm_pairs(int32_t on) { g_gemm_pair.store(on ? 1 : 0); }

void nvfp4_set_qdq_one_pass(int32_t on) { g_qdq_fused.store(on ? 1 : 0); }

void nvfp4_set_act_tile(int32_t rows, int32_t warps) {
  g_act_rows.store(rows >= 1 && rows <= 16 ? rows : 0);
  g_act_warps.store((warps == 4 || warps == 6 || warps == 7 || warps == 8) ? warps : 0);
}

// ------------------------------------------------------------------------------------------ quantize
size_t nvfp4_quantize_workspace_size(int64_t M, int64_t K) {
  (void)M;
  (void)K;
  return 1024 * sizeof(float) + 256;  // amax partials, then the residual's amax (own-scale variant)
}

}  // extern "C"

namespace {
// The bulk-copy activation quantiser serves the method's compact residual with one shared list
// (and no residual); the masked and per-group variants keep the row quantiser.
bool use_act_kernel(int64_t K, int32_t Kp, int fanout, int32_t n_seg, bool masked, int32_t groups) {
  int R, W, smem;
  return !masked && groups == 0 &&
         act_plan_choose(K, Kp, fanout, n_seg, &R, &W, &smem, g_act_rows.load(), g_act_warps.load());
}

nvfp4::ActArgs act_args(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const int32_t* sel, int32_t Kp,
                        const float* partial, int P, const float* amax_in, const nvfp4_tensor* q,
                        const nvfp4_tensor* q_res, int32_t* dev_status) {
  nvfp4::ActArgs a;
  memset(&a, 0, sizeof(a));
  a.src = x;
  a.src_rows = M;
  a.ld = ldx;
  a.K = (int32_t)K;
  a.Kp = Kp;
  a.fanout = 1;
  a.rows_out = q->rows_padded;
  a.sel = sel;
  a.partial = partial;
  a.P = P;
  a.amax_in = amax_in;
  a.s_g_out = q->s_g;
  a.s_g_out2 = Kp > 0 ? q_res->s_g : nullptr;
  a.codes = q->codes;
  a.sf = q->sf;
  a.rcodes = Kp > 0 ? q_res->codes : nullptr;
  a.rsf = Kp > 0 ? q_res->sf : nullptr;
  a.sf_slab16 = q->sf_layout == NVFP4_SF_SLAB16;
  a.status = dev_status;
  a.wait_limit_ns = g_wait_limit_ns.load();
  return a;
}

// One activation quantisation: a single launch, or for the own-scale residual (flag
// NVFP4_RAC_OWN_RES_SCALE, Kp > 0) a pass that folds max |R_sel| into the workspace float after
// the amax partials, then the quantisation with the residual's own scale.
nvfp4_status run_act(nvfp4::ActArgs b, uint32_t flags, void* workspace, cudaStream_t s) {
  if ((flags & NVFP4_RAC_OWN_RES_SCALE) && b.Kp > 0) {
    float* res_amax = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + 1024 * sizeof(float));
    cudaError_t e = cudaMemsetAsync(res_amax, 0, sizeof(float), s);
    if (e != cudaSuccess) return cuda_fail(e, "residual amax reset");
    nvfp4::ActArgs pass = b;
    pass.res_mode = 2;
    pass.res_amax_out = res_amax;
    pass.s_g_out = nullptr;
    pass.s_g_out2 = nullptr;
    e = launch_act(pass, num_sms(), g_act_rows.load(), g_act_warps.load(), s);
    if (e != cudaSuccess) return cuda_fail(e, "residual amax launch");
    b.res_mode = 1;
    b.res_amax_in = res_amax;
  }
  cudaError_t e = launch_act(b, num_sms(), g_act_rows.load(), g_act_warps.load(), s);
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "quantize launch");
}

}  // namespace

namespace {
// nvfp4_quantize and its per-group form: groups == 0 -> one shared list sel [Kp]; groups > 0 ->
// sel [groups x Kp] and output row o takes the list of group row_group[o].
nvfp4_status quantize_rows(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const int32_t* row_gather,
                           int64_t M_out, const int32_t* row_group, int32_t groups, const int32_t* sel, int32_t Kp,
                           const float* amax_in, const nvfp4_tensor* q, const nvfp4_tensor* q_res, void* workspace,
                           size_t workspace_bytes, int32_t* dev_status, void* stream, uint32_t flags = 0) {
  if (!x && M > 0) return fail(NVFP4_ERR_INVALID_ARG, "x is NULL");
  if (M < 0 || M_out < 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "negative row count");
  if (K <= 0 || K % 64 != 0 || K > kMaxK) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "K = %lld must be a positive multiple of 64 <= %lld", (long long)K, (long long)kMaxK);
  if (ldx < K || ldx % 8 != 0) return fail(NVFP4_ERR_ALIGNMENT, "ldx = %lld must be >= K and a multiple of 8", (long long)ldx);
  if (x && !aligned16(x)) return fail(NVFP4_ERR_ALIGNMENT, "x must be 16-byte aligned");
  if (!row_gather && M_out != M) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "without row_gather M_out must equal M");
  if (Kp < 0 || Kp % 64 != 0 || Kp > K) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "Kp = %d must be a multiple of 64 in [0, K]", Kp);
  nvfp4_status st = check_tensor(q, "q", K, M_out, 1, kAnyLayout);
  if (st != NVFP4_OK) return st;
  if (Kp > 0) {
    if (!sel) return fail(NVFP4_ERR_INVALID_ARG, "sel is NULL with Kp > 0");
    const int64_t res_cols = (q_res && q_res->cols == K && Kp < K) ? K : Kp;  // K: masked residual
    st = check_tensor(q_res, "q_res", res_cols, M_out, 1, kAnyLayout);
    if (st != NVFP4_OK) return st;
    if (q_res->rows_padded != q->rows_padded || q_res->sf_layout != q->sf_layout)
      return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "q_res must have q's rows_padded and sf_layout");
  }
  if (groups > 0) {
    if (Kp == 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "per-group channel lists need Kp > 0");
    if (q_res->cols != Kp) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "per-group lists take the compact residual (q_res cols == Kp)");
    if (!row_group && q->rows_padded > 0) return fail(NVFP4_ERR_INVALID_ARG, "row_group is NULL");
    if (!aligned16(sel)) return fail(NVFP4_ERR_ALIGNMENT, "sel must be 16-byte aligned");
  }
  const int P = act_partials(M, K);
  const bool own = (flags & NVFP4_RAC_OWN_RES_SCALE) && Kp > 0;
  if (!amax_in || own) {
    if (!workspace || workspace_bytes < nvfp4_quantize_workspace_size(M, K))
      return fail(NVFP4_ERR_INVALID_ARG, "workspace too small");
    if (!aligned16(workspace)) return fail(NVFP4_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  }
  const bool masked = Kp > 0 && Kp < K && q_res->cols == K;
  const bool act_kernel = q->rows_padded > 0 && use_act_kernel(K, Kp, 1, 0, masked, groups);
  if (own && !act_kernel)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "the own-scale residual takes the compact residual with one list");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* partial = reinterpret_cast<float*>(workspace);
  if (!amax_in) {
    cudaError_t e = launch_amax(x, 1, M, K, ldx, partial, P, dev_status, s);
    if (e != cudaSuccess) return cuda_fail(e, "amax launch");
  }
  if (act_kernel) {
    nvfp4::ActArgs b = act_args(x, M, K, ldx, sel, Kp, partial, P, amax_in, q, q_res, dev_status);
    b.map = row_gather ? kMapGather : kMapRows;
    b.row_gather = row_gather;
    b.rows_valid = M_out;
    return run_act(b, flags, workspace, s);
  }
  RowArgs a;
  memset(&a, 0, sizeof(a));
  a.mode = kModeAct;
  a.src = x;
  a.src_rows = M;
  a.ld = ldx;
  a.K = K;
  a.row_gather = row_gather;
  a.rows_out = q->rows_padded;
  a.rows_per_slab = M_out;
  a.src_slab_stride = 0;
  a.sel = sel;
  a.Kp = Kp;
  a.sel_groups = groups;
  a.row_group = row_group;
  a.partial = partial;
  a.P = P;
  a.amax_in = amax_in;
  a.s_g_out = q->s_g;
  a.s_g_out2 = Kp > 0 ? q_res->s_g : nullptr;
  a.codes = q->codes;
  a.sf = q->sf;
  a.sf_slab16 = q->sf_layout == NVFP4_SF_SLAB16;
  a.masked_res = (Kp > 0 && Kp < K && q_res->cols == K) ? 1 : 0;
  a.rcodes = Kp > 0 ? q_res->codes : nullptr;
  a.rsf = Kp > 0 ? q_res->sf : nullptr;
  a.status = dev_status;
  if (a.rows_out == 0) return NVFP4_OK;
  cudaError_t e = launch_rows(a, num_sms(), s);
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  return NVFP4_OK;
}
}  // namespace

extern "C" {

nvfp4_status nvfp4_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const int32_t* row_gather,
                            int64_t M_out, const int32_t* sel, int32_t Kp, const float* amax_in, const nvfp4_tensor* q,
                            const nvfp4_tensor* q_res, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                            void* stream) {
  g_last_error.clear();
  return quantize_rows(x, M, K, ldx, row_gather, M_out, nullptr, 0, sel, Kp, amax_in, q, q_res, workspace,
                       workspace_bytes, dev_status, stream);
}

nvfp4_status nvfp4_quantize_ex(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const int32_t* row_gather,
                               int64_t M_out, const int32_t* sel, int32_t Kp, const float* amax_in,
                               const nvfp4_tensor* q, const nvfp4_tensor* q_res, void* workspace,
                               size_t workspace_bytes, int32_t* dev_status, void* stream, uint32_t flags) {
  g_last_error.clear();
  return quantize_rows(x, M, K, ldx, row_gather, M_out, nullptr, 0, sel, Kp, amax_in, q, q_res, workspace,
                       workspace_bytes, dev_status, stream, flags);
}

nvfp4_status nvfp4_quantize_grouped_sel(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                        const int32_t* row_gather, int64_t M_out, const int32_t* row_group,
                                        int32_t groups, const int32_t* sel, int32_t Kp, const float* amax_in,
                                        const nvfp4_tensor* q, const nvfp4_tensor* q_res, void* workspace,
                                        size_t workspace_bytes, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (groups <= 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "groups must be positive");
  if (!sel) return fail(NVFP4_ERR_INVALID_ARG, "sel is NULL");
  return quantize_rows(x, M, K, ldx, row_gather, M_out, row_group, groups, sel, Kp, amax_in, q, q_res, workspace,
                       workspace_bytes, dev_status, stream);
}

}  // extern "C"

namespace {
nvfp4_status scatter_rows(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const int32_t* row_scatter,
                          int32_t fanout, const int32_t* sel, int32_t Kp, const float* amax_in, const nvfp4_tensor* q,
                          const nvfp4_tensor* q_res, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                          void* stream, uint32_t flags) {
  if (!x && M > 0) return fail(NVFP4_ERR_INVALID_ARG, "x is NULL");
  if (!row_scatter && M > 0) return fail(NVFP4_ERR_INVALID_ARG, "row_scatter is NULL");
  if (M < 0 || fanout <= 0 || fanout > 64) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "M >= 0 and 1 <= fanout <= 64 required");
  if (K <= 0 || K % 64 != 0 || K > kMaxK) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "K = %lld must be a positive multiple of 64 <= %lld", (long long)K, (long long)kMaxK);
  if (ldx < K || ldx % 8 != 0) return fail(NVFP4_ERR_ALIGNMENT, "ldx = %lld must be >= K and a multiple of 8", (long long)ldx);
  if (x && !aligned16(x)) return fail(NVFP4_ERR_ALIGNMENT, "x must be 16-byte aligned");
  if (Kp < 0 || Kp % 64 != 0 || Kp > K) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "Kp = %d must be a multiple of 64 in [0, K]", Kp);
  nvfp4_status st = check_tensor(q, "q", K, 0, 1, kAnyLayout);
  if (st != NVFP4_OK) return st;
  if (Kp > 0) {
    if (!sel) return fail(NVFP4_ERR_INVALID_ARG, "sel is NULL with Kp > 0");
    const int64_t res_cols = (q_res && q_res->cols == K && Kp < K) ? K : Kp;  // K: masked residual
    st = check_tensor(q_res, "q_res", res_cols, 0, 1, kAnyLayout);
    if (st != NVFP4_OK) return st;
    if (q_res->rows_padded != q->rows_padded || q_res->sf_layout != q->sf_layout)
      return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "q_res must have q's rows_padded and sf_layout");
  }
  const int P = act_partials(M, K);
  const bool own = (flags & NVFP4_RAC_OWN_RES_SCALE) && Kp > 0;
  if (!amax_in || own) {
    if (!workspace || workspace_bytes < nvfp4_quantize_workspace_size(M, K))
      return fail(NVFP4_ERR_INVALID_ARG, "workspace too small");
    if (!aligned16(workspace)) return fail(NVFP4_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  }
  const bool masked = Kp > 0 && Kp < K && q_res->cols == K;
  const bool act_kernel = use_act_kernel(K, Kp, fanout, 0, masked, 0);
  if (own && !act_kernel)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "the own-scale residual takes the compact residual with one list");
  if (M == 0) return NVFP4_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* partial = reinterpret_cast<float*>(workspace);
  if (!amax_in) {
    cudaError_t e = launch_amax(x, 1, M, K, ldx, partial, P, dev_status, s);
    if (e != cudaSuccess) return cuda_fail(e, "amax launch");
  }
  if (act_kernel) {
    nvfp4::ActArgs b = act_args(x, M, K, ldx, sel, Kp, partial, P, amax_in, q, q_res, dev_status);
    b.map = kMapScatter;
    b.row_scatter = row_scatter;
    b.fanout = fanout;
    return run_act(b, flags, workspace, s);
  }
  RowArgs a;
  memset(&a, 0, sizeof(a));
  a.mode = kModeAct;
  a.src = x;
  a.src_rows = M;
  a.ld = ldx;
  a.K = K;
  a.row_scatter = row_scatter;
  a.fanout = fanout;
  a.rows_out = q->rows_padded;
  a.rows_per_slab = M;
  a.sel = sel;
  a.Kp = Kp;
  a.partial = partial;
  a.P = P;
  a.amax_in = amax_in;
  a.s_g_out = q->s_g;
  a.s_g_out2 = Kp > 0 ? q_res->s_g : nullptr;
  a.codes = q->codes;
  a.sf = q->sf;
  a.sf_slab16 = q->sf_layout == NVFP4_SF_SLAB16;
  a.masked_res = (Kp > 0 && Kp < K && q_res->cols == K) ? 1 : 0;
  a.rcodes = Kp > 0 ? q_res->codes : nullptr;
  a.rsf = Kp > 0 ? q_res->sf : nullptr;
  a.status = dev_status;
  cudaError_t e = launch_rows(a, num_sms(), s);
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  return NVFP4_OK;
}

nvfp4_status segments_rows(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const int32_t* expert_offsets,
                           const int32_t* expert_rows, int32_t E, const int32_t* sel, int32_t Kp,
                           const float* amax_in, const nvfp4_tensor* q, const nvfp4_tensor* q_res, void* workspace,
                           size_t workspace_bytes, int32_t* dev_status, void* stream, uint32_t flags) {
  if (!x && M > 0) return fail(NVFP4_ERR_INVALID_ARG, "x is NULL");
  if (!expert_offsets || !expert_rows) return fail(NVFP4_ERR_INVALID_ARG, "expert_offsets / expert_rows is NULL");
  if (E < 1 || E > kMaxRouteExperts) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "E must be in [1, %d]", kMaxRouteExperts);
  if (M < 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "negative row count");
  if (K <= 0 || K % 64 != 0 || K > kMaxK) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "K = %lld must be a positive multiple of 64 <= %lld", (long long)K, (long long)kMaxK);
  if (ldx < K || ldx % 8 != 0) return fail(NVFP4_ERR_ALIGNMENT, "ldx = %lld must be >= K and a multiple of 8", (long long)ldx);
  if (x && !aligned16(x)) return fail(NVFP4_ERR_ALIGNMENT, "x must be 16-byte aligned");
  if (Kp < 0 || Kp % 64 != 0 || Kp > K) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "Kp = %d must be a multiple of 64 in [0, K]", Kp);
  nvfp4_status st = check_tensor(q, "q", K, M, 1, kAnyLayout);
  if (st != NVFP4_OK) return st;
  if (Kp > 0) {
    if (!sel) return fail(NVFP4_ERR_INVALID_ARG, "sel is NULL with Kp > 0");
    st = check_tensor(q_res, "q_res", Kp, M, 1, kAnyLayout);
    if (st != NVFP4_OK) return st;
    if (q_res->rows_padded != q->rows_padded || q_res->sf_layout != q->sf_layout)
      return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "q_res must have q's rows_padded and sf_layout");
  }
  if (!use_act_kernel(K, Kp, 1, E, false, 0))
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "K = %lld, Kp = %d too large for the segment quantiser", (long long)K, Kp);
  const int P = act_partials(M, K);
  if (!amax_in || ((flags & NVFP4_RAC_OWN_RES_SCALE) && Kp > 0)) {
    if (!workspace || workspace_bytes < nvfp4_quantize_workspace_size(M, K))
      return fail(NVFP4_ERR_INVALID_ARG, "workspace too small");
    if (!aligned16(workspace)) return fail(NVFP4_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  }
  if (M == 0) return NVFP4_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* partial = reinterpret_cast<float*>(workspace);
  if (!amax_in) {
    cudaError_t e = launch_amax(x, 1, M, K, ldx, partial, P, dev_status, s);
    if (e != cudaSuccess) return cuda_fail(e, "amax launch");
  }
  nvfp4::ActArgs b = act_args(x, M, K, ldx, sel, Kp, partial, P, amax_in, q, q_res, dev_status);
  b.map = kMapSegments;
  b.seg_off = expert_offsets;
  b.seg_rows = expert_rows;
  b.n_seg = E;
  b.rows_valid = M;
  b.src_rows = M;
  return run_act(b, flags, workspace, s);
}
}  // namespace

extern "C" {

nvfp4_status nvfp4_quantize_scatter(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const int32_t* row_scatter,
                                    int32_t fanout, const int32_t* sel, int32_t Kp, const float* amax_in,
                                    const nvfp4_tensor* q, const nvfp4_tensor* q_res, void* workspace,
                                    size_t workspace_bytes, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  return scatter_rows(x, M, K, ldx, row_scatter, fanout, sel, Kp, amax_in, q, q_res, workspace, workspace_bytes,
                      dev_status, stream, 0);
}

nvfp4_status nvfp4_quantize_scatter_ex(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                       const int32_t* row_scatter, int32_t fanout, const int32_t* sel, int32_t Kp,
                                       const float* amax_in, const nvfp4_tensor* q, const nvfp4_tensor* q_res,
                                       void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream,
                                       uint32_t flags) {
  g_last_error.clear();
  return scatter_rows(x, M, K, ldx, row_scatter, fanout, sel, Kp, amax_in, q, q_res, workspace, workspace_bytes,
                      dev_status, stream, flags);
}

nvfp4_status nvfp4_quantize_segments(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                     const int32_t* expert_offsets, const int32_t* expert_rows, int32_t E,
                                     const int32_t* sel, int32_t Kp, const float* amax_in, const nvfp4_tensor* q,
                                     const nvfp4_tensor* q_res, void* workspace, size_t workspace_bytes,
                                     int32_t* dev_status, void* stream) {
  g_last_error.clear();
  return segments_rows(x, M, K, ldx, expert_offsets, expert_rows, E, sel, Kp, amax_in, q, q_res, workspace,
                       workspace_bytes, dev_status, stream, 0);
}

nvfp4_status nvfp4_quantize_segments_ex(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                        const int32_t* expert_offsets, const int32_t* expert_rows, int32_t E,
                                        const int32_t* sel, int32_t Kp, const float* amax_in, const nvfp4_tensor* q,
                                        const nvfp4_tensor* q_res, void* workspace, size_t workspace_bytes,
                                        int32_t* dev_status, void* stream, uint32_t flags) {
  g_last_error.clear();
  return segments_rows(x, M, K, ldx, expert_offsets, expert_rows, E, sel, Kp, amax_in, q, q_res, workspace,
                       workspace_bytes, dev_status, stream, flags);
}

// ------------------------------------------------------------------------------------------ calibrate
size_t rac_calibrate_workspace_size(int64_t T, int64_t K) { return rac_calibrate_grouped_workspace_size(T, K, 1); }

size_t rac_calibrate_grouped_workspace_size(int64_t T, int64_t K, int32_t groups) {
  const size_t G = (size_t)(groups > 0 ? groups : 1);
  return round_up(1024 * sizeof(float), 256) + round_up((size_t)T * (size_t)K * sizeof(float), 256) +
         round_up(G * (size_t)K * sizeof(double), 256);
}

}  // extern "C"

namespace {
// rac_calibrate and its per-group form (offsets == nullptr: one group of all T rows)
nvfp4_status calibrate_rows(const uint16_t* x_cal, int64_t T, int64_t K, const int32_t* offsets, int32_t groups,
                            int32_t Kp, int32_t* sel_out, double* chan_err_out, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, void* stream) {
  if (!x_cal || (!sel_out && Kp > 0)) return fail(NVFP4_ERR_INVALID_ARG, "x_cal / sel_out is NULL");
  if (T <= 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "T must be positive");
  if (K <= 0 || K % 64 != 0 || K > kMaxCalK) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "K = %lld must be a positive multiple of 64 <= %lld", (long long)K, (long long)kMaxCalK);
  if (Kp < 0 || Kp > K) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "Kp out of range");
  if (groups < 1 || groups > 65535) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "groups must be in [1, 65535]");
  if (!aligned16(x_cal)) return fail(NVFP4_ERR_ALIGNMENT, "x_cal must be 16-byte aligned");
  if (!workspace || workspace_bytes < rac_calibrate_grouped_workspace_size(T, K, groups))
    return fail(NVFP4_ERR_INVALID_ARG, "workspace too small");
  if (!aligned16(workspace)) return fail(NVFP4_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* ws = reinterpret_cast<char*>(workspace);
  float* partial = reinterpret_cast<float*>(ws);
  float* resid = reinterpret_cast<float*>(ws + round_up(1024 * sizeof(float), 256));
  double* err = reinterpret_cast<double*>(ws + round_up(1024 * sizeof(float), 256) +
                                          round_up((size_t)T * (size_t)K * sizeof(float), 256));
  const int P = act_partials(T, K);
  cudaError_t e = launch_amax(x_cal, 1, T, K, K, partial, P, dev_status, s);
  if (e != cudaSuccess) return cuda_fail(e, "amax launch");
  RowArgs a;
  memset(&a, 0, sizeof(a));
  a.mode = kModeCal;
  a.src = x_cal;
  a.src_rows = T;
  a.ld = K;
  a.K = K;
  a.rows_out = T;
  a.rows_per_slab = T;
  a.Kp = 0;
  a.partial = partial;
  a.P = P;
  a.resid_all = resid;
  a.status = dev_status;
  e = launch_rows(a, num_sms(), s);
  if (e != cudaSuccess) return cuda_fail(e, "calibration residual launch");
  e = launch_chan_err(resid, T, K, offsets, groups, err, dev_status, s);
  if (e != cudaSuccess) return cuda_fail(e, "channel error launch");
  if (Kp > 0 || chan_err_out) {
    e = launch_select(err, (int32_t)K, Kp, groups, sel_out, chan_err_out, s);
    if (e != cudaSuccess) return cuda_fail(e, "selection launch");
  }
  return NVFP4_OK;
}

// pack_weights and its per-expert form (sel [E x Kp] when per_expert)
nvfp4_status pack_rows(const uint16_t* w, int64_t E, int64_t N, int64_t K, const int32_t* sel, int32_t Kp,
                       bool per_expert, int32_t gate_up_interleave, const nvfp4_tensor* w_q,
                       const nvfp4_tensor* w_sel_q, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                       void* stream) {
  if (!w) return fail(NVFP4_ERR_INVALID_ARG, "w is NULL");
  if (E <= 0 || N <= 0 || N % 128 != 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "E > 0 and N %% 128 == 0 required");
  if (K <= 0 || K % 64 != 0 || K > kMaxK) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "K must be a positive multiple of 64");
  if (Kp < 0 || Kp % 64 != 0 || Kp > K) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "Kp must be a multiple of 64 in [0, K]");
  if (gate_up_interleave != 0 && gate_up_interleave != 1) return fail(NVFP4_ERR_INVALID_ARG, "gate_up_interleave must be 0 or 1");
  if (!aligned16(w)) return fail(NVFP4_ERR_ALIGNMENT, "w must be 16-byte aligned");
  nvfp4_status st = check_tensor(w_q, "w_q", K, N, E);
  if (st != NVFP4_OK) return st;
  if (w_q->rows_padded != N || w_q->rows != N) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "w_q rows / rows_padded must equal N");
  if (Kp > 0) {
    if (!sel) return fail(NVFP4_ERR_INVALID_ARG, "sel is NULL with Kp > 0");
    if (per_expert && !aligned16(sel)) return fail(NVFP4_ERR_ALIGNMENT, "sel must be 16-byte aligned");
    st = check_tensor(w_sel_q, "w_sel_q", Kp, N, E);
    if (st != NVFP4_OK) return st;
    if (w_sel_q->rows_padded != N) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "w_sel_q rows_padded must equal N");
  }
  if (!workspace || workspace_bytes < pack_weights_workspace_size(E, N, K)) return fail(NVFP4_ERR_INVALID_ARG, "workspace too small");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* partial = reinterpret_cast<float*>(workspace);
  const int P = slab_partials(E);
  cudaError_t e = launch_amax(w, E, N, K, K, partial, P, dev_status, s);
  if (e != cudaSuccess) return cuda_fail(e, "amax launch");
  RowArgs a;
  memset(&a, 0, sizeof(a));
  a.mode = kModePack;
  a.src = w;
  a.src_rows = N;
  a.ld = K;
  a.K = K;
  a.rows_out = E * N;
  a.rows_per_slab = N;
  a.src_slab_stride = N * K;
  a.interleave = gate_up_interleave;
  a.N_half = N / 2;
  a.sel = sel;
  a.Kp = Kp;
  a.sel_groups = (per_expert && Kp > 0) ? (int32_t)E : 0;
  a.partial = partial;
  a.P = P;
  a.s_g_out = w_q->s_g;
  a.s_g_out2 = (Kp > 0 && w_sel_q->s_g != w_q->s_g) ? w_sel_q->s_g : nullptr;
  a.codes = w_q->codes;
  a.sf = w_q->sf;
  a.rcodes = Kp > 0 ? w_sel_q->codes : nullptr;
  a.rsf = Kp > 0 ? w_sel_q->sf : nullptr;
  a.status = dev_status;
  e = launch_rows(a, num_sms(), s);
  if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  return NVFP4_OK;
}
}  // namespace

extern "C" {

nvfp4_status rac_calibrate(const uint16_t* x_cal, int64_t T, int64_t K, int32_t Kp, int32_t* sel_out,
                           double* chan_err_out, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                           void* stream) {
  g_last_error.clear();
  return calibrate_rows(x_cal, T, K, nullptr, 1, Kp, sel_out, chan_err_out, workspace, workspace_bytes, dev_status,
                        stream);
}

nvfp4_status rac_calibrate_grouped(const uint16_t* x_cal, int64_t T, int64_t K, const int32_t* group_offsets,
                                   int32_t groups, int32_t Kp, int32_t* sel_out, double* chan_err_out,
                                   void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (!group_offsets) return fail(NVFP4_ERR_INVALID_ARG, "group_offsets is NULL");
  return calibrate_rows(x_cal, T, K, group_offsets, groups, Kp, sel_out, chan_err_out, workspace, workspace_bytes,
                        dev_status, stream);
}

// ------------------------------------------------------------------------------------------ pack
size_t pack_weights_workspace_size(int64_t E, int64_t N, int64_t K) {
  (void)N;
  (void)K;
  return round_up((size_t)(E > 0 ? E : 1) * (size_t)slab_partials(E) * sizeof(float), 256);
}

nvfp4_status pack_weights(const uint16_t* w, int64_t E, int64_t N, int64_t K, const int32_t* sel, int32_t Kp,
                          int32_t gate_up_interleave, const nvfp4_tensor* w_q, const nvfp4_tensor* w_sel_q,
                          void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  return pack_rows(w, E, N, K, sel, Kp, false, gate_up_interleave, w_q, w_sel_q, workspace, workspace_bytes,
                   dev_status, stream);
}

nvfp4_status pack_weights_grouped_sel(const uint16_t* w, int64_t E, int64_t N, int64_t K, const int32_t* sel,
                                      int32_t Kp, int32_t gate_up_interleave, const nvfp4_tensor* w_q,
                                      const nvfp4_tensor* w_sel_q, void* workspace, size_t workspace_bytes,
                                      int32_t* dev_status, void* stream) {
  g_last_error.clear();
  return pack_rows(w, E, N, K, sel, Kp, true, gate_up_interleave, w_q, w_sel_q, workspace, workspace_bytes,
                   dev_status, stream);
}

// ------------------------------------------------------------------------------------------ GEMMs
static nvfp4_status gemm_common(const nvfp4_tensor* a, const nvfp4_tensor* a_res, const nvfp4_tensor* w,
                                const nvfp4_tensor* w_sel, int64_t rows_needed, int64_t N, int64_t K, int32_t Kp,
                                int64_t E, nvfp4_dtype out, void* y, int64_t ldy, int64_t y_cols, int64_t y_rows,
                                int bn, CUtensorMap* maps, GemmArgs* g, int w_box_rows = 0, bool own = false,
                                bool swiglu = false, bool pair_kernel = false) {
  if (w_box_rows == 0) w_box_rows = bn;
  if (K <= 0 || K % 64 != 0 || K > kMaxK) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "K must be a positive multiple of 64");
  if (Kp < 0 || Kp % 64 != 0 || Kp > K) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "Kp must be a multiple of 64 in [0, K]");
  if (N <= 0 || N % 128 != 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "N must be a positive multiple of 128");
  if (out != NVFP4_OUT_F32 && out != NVFP4_OUT_BF16) return fail(NVFP4_ERR_INVALID_ARG, "bad output dtype");
  if (!y) return fail(NVFP4_ERR_INVALID_ARG, "y is NULL");
  if (!aligned16(y)) return fail(NVFP4_ERR_ALIGNMENT, "y must be 16-byte aligned");
  if (ldy < y_cols || (out == NVFP4_OUT_BF16 ? ldy % 8 : ldy % 4) != 0)
    return fail(NVFP4_ERR_ALIGNMENT, "ldy = %lld must be >= %lld and keep rows 16-byte aligned", (long long)ldy, (long long)y_cols);
  nvfp4_status st = check_tensor(a, "a", K, rows_needed, 1);
  if (st != NVFP4_OK) return st;
  st = check_tensor(w, "w", K, N, E);
  if (st != NVFP4_OK) return st;
  if (w->rows_padded != N) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "w.rows_padded must equal N");
  if (Kp > 0) {
    st = check_tensor(a_res, "a_res", Kp, rows_needed, 1);
    if (st != NVFP4_OK) return st;
    if (a_res->rows_padded != a->rows_padded) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "a_res.rows_padded must equal a.rows_padded");
    st = check_tensor(w_sel, "w_sel", Kp, N, E);
    if (st != NVFP4_OK) return st;
    if (w_sel->rows_padded != N) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "w_sel.rows_padded must equal N");
  }
  memset(maps, 0, 5 * sizeof(CUtensorMap));
  if (y_rows > 0) {
    // the single-SM FP4 kernel at BN = 256 stages its stores in 64-byte boxes
    const OutBox box = (own && swiglu) ? kOutNarrow : (!own && !pair_kernel && bn == 256) ? kOutNarrow64 : kOutWide;
    st = make_out_map(&maps[4], y, out == NVFP4_OUT_BF16, (uint64_t)y_cols, (uint64_t)y_rows, (uint64_t)ldy, box);
    if (st != NVFP4_OK) return st;
  }
  st = make_code_map(&maps[0], a->codes, (uint64_t)K / 2, (uint64_t)a->rows_padded, 1, 128, 2, "A");
  if (st != NVFP4_OK) return st;
  st = make_code_map(&maps[2], w->codes, (uint64_t)K / 2, (uint64_t)N, (uint64_t)E, (uint32_t)w_box_rows, 3, "W");
  if (st != NVFP4_OK) return st;
  if (Kp > 0) {
    st = make_code_map(&maps[1], a_res->codes, (uint64_t)Kp / 2, (uint64_t)a_res->rows_padded, 1, 128, 2, "A_res");
    if (st != NVFP4_OK) return st;
    st = make_code_map(&maps[3], w_sel->codes, (uint64_t)Kp / 2, (uint64_t)N, (uint64_t)E, (uint32_t)w_box_rows, 3,
                       "W_sel");
    if (st != NVFP4_OK) return st;
  } else {
    maps[1] = maps[0];
    maps[3] = maps[2];
  }
  memset(g, 0, sizeof(*g));
  g->sfa = a->sf;
  g->sfa_res = Kp > 0 ? a_res->sf : a->sf;
  g->sfw = w->sf;
  g->sfw_sel = Kp > 0 ? w_sel->sf : w->sf;
  g->sfw_slab_bytes = (int64_t)nvfp4_sf_bytes(N, K);
  g->sfw_sel_slab_bytes = Kp > 0 ? (int64_t)nvfp4_sf_bytes(N, Kp) : 0;
  g->k64_main = (int32_t)(K / 64);
  g->k64_res = Kp / 64;
  g->kt_main = (int32_t)((K + 255) / 256);
  g->kt_res = (Kp + 255) / 256;
  g->N = (int32_t)N;
  g->n_blocks = (int32_t)(N / bn);
  g->rows_capacity = a->rows_padded;
  g->s_a = a->s_g;
  g->s_w = w->s_g;
  g->y = y;
  g->ldy = ldy;
  g->out_bf16 = out == NVFP4_OUT_BF16;
  g->wait_limit_ns = g_wait_limit_ns.load();
  g->own_res_scale = own ? 1 : 0;
  g->s_a_res = (own && Kp > 0) ? a_res->s_g : a->s_g;
  return NVFP4_OK;
}

static nvfp4_status dense_gemm(const nvfp4_tensor* a, const nvfp4_tensor* a_res, const nvfp4_tensor* w,
                               const nvfp4_tensor* w_sel, int64_t M, int64_t N, int64_t K, int32_t Kp, nvfp4_dtype out,
                               void* y, int64_t ldy, int32_t* dev_status, void* stream, uint32_t flags) {
  if (M < 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "M must be >= 0");
  const bool own = (flags & NVFP4_RAC_OWN_RES_SCALE) != 0;
  const bool pairs = !own && g_gemm_pair.load() != 0 && N % 256 == 0 && g_tile_n.load() != 128;
  const int bn = own ? 128 : pairs ? 256 : choose_tile_n(N, K, Kp);
  CUtensorMap maps[5];
  GemmArgs g;
  nvfp4_status st =
      gemm_common(a, a_res, w, w_sel, M, N, K, Kp, 1, out, y, ldy, N, M, bn, maps, &g, pairs ? 128 : bn, own, false,
                  pairs);
  if (st != NVFP4_OK) return st;
  if (M == 0) return NVFP4_OK;
  g.offsets = nullptr;
  g.E = 1;
  g.M = M;
  g.m_blocks_dense = (int32_t)((M + 127) / 128);
  g.epi = 0;
  g.status = dev_status;
  int64_t tiles = (int64_t)g.m_blocks_dense * g.n_blocks;
  cudaError_t e;
  if (pairs) {
    const int64_t pair_tiles = (int64_t)((g.m_blocks_dense + 1) / 2) * g.n_blocks;
    const int n_pairs = (int)(pair_tiles < num_sms() / 2 ? pair_tiles : num_sms() / 2);
    e = launch_gemm_pair(maps[0], maps[1], maps[2], maps[3], maps[4], g, n_pairs, reinterpret_cast<cudaStream_t>(stream));
  } else {
    int grid = (int)(tiles < num_sms() ? tiles : num_sms());
    e = launch_gemm(bn, maps[0], maps[1], maps[2], maps[3], maps[4], g, grid, reinterpret_cast<cudaStream_t>(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  return NVFP4_OK;
}

nvfp4_status w4a4_rac_gemm(const nvfp4_tensor* a, const nvfp4_tensor* a_res, const nvfp4_tensor* w,
                           const nvfp4_tensor* w_sel, int64_t M, int64_t N, int64_t K, int32_t Kp, nvfp4_dtype out,
                           void* y, int64_t ldy, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  return dense_gemm(a, a_res, w, w_sel, M, N, K, Kp, out, y, ldy, dev_status, stream, 0);
}

nvfp4_status w4a4_rac_gemm_ex(const nvfp4_tensor* a, const nvfp4_tensor* a_res, const nvfp4_tensor* w,
                              const nvfp4_tensor* w_sel, int64_t M, int64_t N, int64_t K, int32_t Kp, nvfp4_dtype out,
                              void* y, int64_t ldy, int32_t* dev_status, void* stream, uint32_t flags) {
  g_last_error.clear();
  return dense_gemm(a, a_res, w, w_sel, M, N, K, Kp, out, y, ldy, dev_status, stream, flags);
}

}  // extern "C"

namespace {
// The weighted combine of the down projection's epilogue (grouped_w4a4_rac_moe_combine).
struct CombineSpec {
  const int32_t* row_pair;
  const float* topk_w;
  int64_t T;
  int32_t k;
};

// The grouped GEMM over n_seg row segments; segment i uses weight slab seg_expert[i] (or i).
// With `comb`, y is the binary32 [T x N] combine accumulator (zeroed here) instead of the rows.
nvfp4_status grouped_common(const nvfp4_tensor* a, const nvfp4_tensor* a_res, const int32_t* offsets,
                            const int32_t* seg_rows, const int32_t* seg_expert, int32_t n_seg, const nvfp4_tensor* w,
                            const nvfp4_tensor* w_sel, int64_t N, int64_t K, int32_t Kp, nvfp4_epilogue ep,
                            nvfp4_dtype out, void* y, int64_t ldy, float* amax_out, int32_t* dev_status,
                            void* stream, uint32_t flags = 0, const CombineSpec* comb = nullptr) {
  if (!offsets) return fail(NVFP4_ERR_INVALID_ARG, "expert_offsets is NULL");
  if (n_seg <= 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "the segment count must be positive");
  if (ep != NVFP4_EPI_NONE && ep != NVFP4_EPI_SWIGLU_AMAX) return fail(NVFP4_ERR_INVALID_ARG, "bad epilogue");
  if (ep == NVFP4_EPI_SWIGLU_AMAX) {
    if (out != NVFP4_OUT_BF16) return fail(NVFP4_ERR_INVALID_ARG, "the SwiGLU epilogue writes bf16");
    if (!amax_out) return fail(NVFP4_ERR_INVALID_ARG, "amax_out is NULL with the SwiGLU epilogue");
  }
  if (ep == NVFP4_EPI_SWIGLU_AMAX && N % 256 != 0)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "the SwiGLU epilogue needs N %% 256 == 0");
  if (!w) return fail(NVFP4_ERR_INVALID_ARG, "w is NULL");
  const int64_t E = seg_expert ? w->slabs : n_seg;
  const bool own = (flags & NVFP4_RAC_OWN_RES_SCALE) != 0;
  const bool pairs =
      !own && g_gemm_pair.load() != 0 && N % 256 == 0 && g_tile_n.load() != 128 && n_seg <= kMaxRouteExperts;
  const int bn = own ? 128 : (pairs || ep == NVFP4_EPI_SWIGLU_AMAX) ? 256 : choose_tile_n(N, K, Kp);
  CUtensorMap maps[5];
  GemmArgs g;
  const int64_t y_cols = ep == NVFP4_EPI_SWIGLU_AMAX ? N / 2 : N;
  const int64_t y_rows = comb ? comb->T : (a ? a->rows_padded : 0);
  nvfp4_status st = gemm_common(a, a_res, w, w_sel, 0, N, K, Kp, E, out, y, ldy, y_cols, y_rows, bn, maps, &g,
                                pairs ? 128 : bn, own, ep == NVFP4_EPI_SWIGLU_AMAX, pairs && !comb);
  if (st != NVFP4_OK) return st;
  g.offsets = offsets;
  g.expert_rows = seg_rows;
  g.E = n_seg;
  g.seg_expert = seg_expert;
  g.n_weights = (int32_t)E;
  g.M = a->rows_padded;
  g.m_blocks_dense = 0;
  g.epi = ep == NVFP4_EPI_SWIGLU_AMAX ? 1 : comb ? 2 : 0;
  g.amax_out = amax_out;
  g.status = dev_status;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (ep == NVFP4_EPI_SWIGLU_AMAX) {
    cudaError_t e = cudaMemsetAsync(amax_out, 0, sizeof(float), s);
    if (e != cudaSuccess) return cuda_fail(e, "amax reset");
  }
  if (comb) {
    g.row_pair = comb->row_pair;
    g.topk_w = comb->topk_w;
    g.k_top = comb->k;
    g.n_pairs = comb->T * comb->k;
    g.comb = reinterpret_cast<float*>(y);
    g.ld_comb = ldy;
    cudaError_t e = cudaMemsetAsync(y, 0, (size_t)comb->T * (size_t)ldy * sizeof(float), s);
    if (e != cudaSuccess) return cuda_fail(e, "combine accumulator reset");
    if (comb->T == 0) return NVFP4_OK;
  }
  cudaError_t e = (pairs && !comb) ? launch_gemm_pair(maps[0], maps[1], maps[2], maps[3], maps[4], g, num_sms() / 2, s)
                                   : launch_gemm(bn, maps[0], maps[1], maps[2], maps[3], maps[4], g, num_sms(), s);
  if (e != cudaSuccess) return cuda_fail(e, "grouped gemm launch");
  return NVFP4_OK;
}
}  // namespace

extern "C" {

nvfp4_status grouped_w4a4_rac_moe(const nvfp4_tensor* a, const nvfp4_tensor* a_res, const int32_t* expert_offsets,
                                  const int32_t* expert_rows, int32_t E, const nvfp4_tensor* w,
                                  const nvfp4_tensor* w_sel, int64_t N, int64_t K,
                                  int32_t Kp, nvfp4_epilogue ep, nvfp4_dtype out, void* y, int64_t ldy,
                                  float* amax_out, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (E <= 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "E must be positive");
  return grouped_common(a, a_res, expert_offsets, expert_rows, nullptr, E, w, w_sel, N, K, Kp, ep, out, y, ldy,
                        amax_out, dev_status, stream);
}

nvfp4_status grouped_w4a4_rac_moe_ex(const nvfp4_tensor* a, const nvfp4_tensor* a_res, const int32_t* expert_offsets,
                                     const int32_t* expert_rows, int32_t E, const nvfp4_tensor* w,
                                     const nvfp4_tensor* w_sel, int64_t N, int64_t K, int32_t Kp, nvfp4_epilogue ep,
                                     nvfp4_dtype out, void* y, int64_t ldy, float* amax_out, int32_t* dev_status,
                                     void* stream, uint32_t flags) {
  g_last_error.clear();
  if (E <= 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "E must be positive");
  return grouped_common(a, a_res, expert_offsets, expert_rows, nullptr, E, w, w_sel, N, K, Kp, ep, out, y, ldy,
                        amax_out, dev_status, stream, flags);
}

nvfp4_status grouped_w4a4_rac_moe_segments(const nvfp4_tensor* a, const nvfp4_tensor* a_res,
                                           const int32_t* seg_offsets, const int32_t* seg_rows,
                                           const int32_t* seg_expert, int32_t n_seg, const nvfp4_tensor* w,
                                           const nvfp4_tensor* w_sel, int64_t N, int64_t K, int32_t Kp,
                                           nvfp4_epilogue ep, nvfp4_dtype out, void* y, int64_t ldy,
                                           float* amax_out, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (!seg_expert) return fail(NVFP4_ERR_INVALID_ARG, "seg_expert is NULL");
  return grouped_common(a, a_res, seg_offsets, seg_rows, seg_expert, n_seg, w, w_sel, N, K, Kp, ep, out, y, ldy,
                        amax_out, dev_status, stream);
}

nvfp4_status grouped_w4a4_rac_moe_combine(const nvfp4_tensor* a, const nvfp4_tensor* a_res,
                                          const int32_t* expert_offsets, const int32_t* expert_rows, int32_t E,
                                          const nvfp4_tensor* w, const nvfp4_tensor* w_sel, int64_t N, int64_t K,
                                          int32_t Kp, const int32_t* row_pair, const float* topk_w, int64_t T,
                                          int32_t k, float* out32, uint16_t* out, int64_t ldo, int32_t* dev_status,
                                          void* stream) {
  g_last_error.clear();
  if (E <= 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "E must be positive");
  if (T < 0 || k <= 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "T >= 0 and k > 0 required");
  if (T > 0 && (!row_pair || !topk_w || !out32 || !out)) return fail(NVFP4_ERR_INVALID_ARG, "NULL buffer");
  if (ldo < N || ldo % 8 != 0 || (out && !aligned16(out)))
    return fail(NVFP4_ERR_ALIGNMENT, "out must be 16-byte aligned with a pitch >= N, a multiple of 8");
  if (T == 0) return NVFP4_OK;
  if (g_gemm_pair.load() != 0 && N % 256 == 0 && g_tile_n.load() != 128)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "the combine epilogue runs on single-SM tiles (CTA pairs are on)");
  const CombineSpec comb{row_pair, topk_w, T, k};
  nvfp4_status st = grouped_common(a, a_res, expert_offsets, expert_rows, nullptr, E, w, w_sel, N, K, Kp,
                                   NVFP4_EPI_NONE, NVFP4_OUT_F32, out32, N, nullptr, dev_status, stream, 0, &comb);
  if (st != NVFP4_OK) return st;
  cudaError_t e = launch_combine_finalize(out32, T, N, out, ldo, num_sms(), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "combine finalize launch");
}

nvfp4_status moe_row_pairs(const int32_t* row_scatter, int64_t T, int32_t k, int64_t rows, int32_t* row_pair,
                           int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (T < 0 || k <= 0 || rows < 0 || rows > INT32_MAX) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "T >= 0, k > 0, 0 <= rows <= INT32_MAX");
  if (T * k > INT32_MAX) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "T * k must fit in int32");
  if (rows == 0) return NVFP4_OK;
  if (!row_pair || (T > 0 && !row_scatter)) return fail(NVFP4_ERR_INVALID_ARG, "NULL buffer");
  cudaError_t e = launch_row_pairs(row_scatter, T * k, rows, row_pair, num_sms(), dev_status,
                                   reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "row pairs launch");
}

nvfp4_status nvfp4_amax(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, float* amax_out, void* workspace,
                        size_t workspace_bytes, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (!amax_out || (!x && M > 0)) return fail(NVFP4_ERR_INVALID_ARG, "x / amax_out is NULL");
  if (M < 0 || K <= 0 || K % 8 != 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "M >= 0 and K a positive multiple of 8");
  if (ldx < K || ldx % 8 != 0) return fail(NVFP4_ERR_ALIGNMENT, "ldx must be >= K and a multiple of 8");
  if (x && !aligned16(x)) return fail(NVFP4_ERR_ALIGNMENT, "x must be 16-byte aligned");
  if (!workspace || workspace_bytes < nvfp4_quantize_workspace_size(M, K))
    return fail(NVFP4_ERR_INVALID_ARG, "workspace too small");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (M == 0) {
    cudaError_t e = cudaMemsetAsync(amax_out, 0, sizeof(float), s);
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "amax reset");
  }
  float* partial = reinterpret_cast<float*>(workspace);
  const int P = act_partials(M, K);
  cudaError_t e = launch_amax(x, 1, M, K, ldx, partial, P, dev_status, s);
  if (e == cudaSuccess) e = launch_reduce_amax(partial, P, amax_out, s);
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "amax launch");
}

nvfp4_status grouped_w4a4_rac_moe_decode(const nvfp4_tensor* a, const nvfp4_tensor* a_res,
                                         const int32_t* slot_expert, const int32_t* slot_count, int32_t n_slots,
                                         int32_t E, const nvfp4_tensor* w, const nvfp4_tensor* w_sel, int64_t N,
                                         int64_t K, int32_t Kp, nvfp4_epilogue ep, nvfp4_dtype out, void* y,
                                         int64_t ldy, float* amax_out, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (n_slots < 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "n_slots must be >= 0");
  if (n_slots > 0 && (!slot_expert || !slot_count)) return fail(NVFP4_ERR_INVALID_ARG, "slot_expert / slot_count is NULL");
  if (E <= 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "E must be positive");
  if (K <= 0 || K % 64 != 0 || K > kMaxK) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "K must be a positive multiple of 64");
  if (Kp < 0 || Kp % 64 != 0 || Kp > K) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "Kp must be a multiple of 64 in [0, K]");
  if (N <= 0 || N % 128 != 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "N must be a positive multiple of 128");
  if (ep != NVFP4_EPI_NONE && ep != NVFP4_EPI_SWIGLU_AMAX) return fail(NVFP4_ERR_INVALID_ARG, "bad epilogue");
  if (ep == NVFP4_EPI_SWIGLU_AMAX && !amax_out) return fail(NVFP4_ERR_INVALID_ARG, "amax_out is NULL with the SwiGLU epilogue");
  if (out != NVFP4_OUT_F32 && out != NVFP4_OUT_BF16) return fail(NVFP4_ERR_INVALID_ARG, "bad output dtype");
  const int64_t y_cols = ep == NVFP4_EPI_SWIGLU_AMAX ? N / 2 : N;
  if (!y && n_slots > 0) return fail(NVFP4_ERR_INVALID_ARG, "y is NULL");
  if (ldy < y_cols) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "ldy = %lld must be >= %lld", (long long)ldy, (long long)y_cols);
  const int64_t rows = 16 * (int64_t)n_slots;
  nvfp4_status st = check_tensor(a, "a", K, rows, 1, kSlab16Only);
  if (st != NVFP4_OK) return st;
  st = check_tensor(w, "w", K, N, E);
  if (st != NVFP4_OK) return st;
  if (w->rows_padded != N) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "w.rows_padded must equal N");
  if (Kp > 0) {
    st = check_tensor(a_res, "a_res", Kp, rows, 1, kSlab16Only);
    if (st != NVFP4_OK) return st;
    st = check_tensor(w_sel, "w_sel", Kp, N, E);
    if (st != NVFP4_OK) return st;
    if (w_sel->rows_padded != N) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "w_sel.rows_padded must equal N");
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (ep == NVFP4_EPI_SWIGLU_AMAX) {
    cudaError_t e = cudaMemsetAsync(amax_out, 0, sizeof(float), s);
    if (e != cudaSuccess) return cuda_fail(e, "amax reset");
  }
  if (n_slots == 0) return NVFP4_OK;
  CUtensorMap maps[4];
  memset(maps, 0, sizeof(maps));
  st = make_code_map(&maps[0], w->codes, (uint64_t)K / 2, (uint64_t)N, (uint64_t)E, 128, 3, "W");
  if (st != NVFP4_OK) return st;
  st = make_code_map(&maps[2], a->codes, (uint64_t)K / 2, (uint64_t)a->rows_padded, 1, 16, 2, "X");
  if (st != NVFP4_OK) return st;
  if (Kp > 0) {
    st = make_code_map(&maps[1], w_sel->codes, (uint64_t)Kp / 2, (uint64_t)N, (uint64_t)E, 128, 3, "W_sel");
    if (st != NVFP4_OK) return st;
    st = make_code_map(&maps[3], a_res->codes, (uint64_t)Kp / 2, (uint64_t)a_res->rows_padded, 1, 16, 2, "X_res");
    if (st != NVFP4_OK) return st;
  } else {
    maps[1] = maps[0];
    maps[3] = maps[2];
  }
  DecodeArgs d;
  memset(&d, 0, sizeof(d));
  d.sfx = a->sf;
  d.sfx_res = Kp > 0 ? a_res->sf : a->sf;
  d.sfw = w->sf;
  d.sfw_sel = Kp > 0 ? w_sel->sf : w->sf;
  d.sfw_slab_bytes = (int64_t)nvfp4_sf_bytes(N, K);
  d.sfw_sel_slab_bytes = Kp > 0 ? (int64_t)nvfp4_sf_bytes(N, Kp) : 0;
  d.k64_main = (int32_t)(K / 64);
  d.k64_res = Kp / 64;
  d.kt_main = (int32_t)((K + 255) / 256);
  d.kt_res = (Kp + 255) / 256;
  d.m_tiles = (int32_t)(N / 128);
  d.slot_expert = slot_expert;
  d.slot_count = slot_count;
  d.n_slots = n_slots;
  d.E = E;
  d.s_x = a->s_g;
  d.s_w = w->s_g;
  d.y = y;
  d.ldy = ldy;
  d.out_bf16 = out == NVFP4_OUT_BF16;
  d.epi = ep == NVFP4_EPI_SWIGLU_AMAX ? 1 : 0;
  d.amax_out = amax_out;
  d.status = dev_status;
  d.wait_limit_ns = g_wait_limit_ns.load();
  const int64_t units = (int64_t)n_slots * d.m_tiles;
  const int grid = (int)(units < num_sms() ? units : num_sms());
  cudaError_t e = launch_decode(maps[0], maps[1], maps[2], maps[3], d, grid, s);
  if (e != cudaSuccess) return cuda_fail(e, "decode gemm launch");
  return NVFP4_OK;
}

// ------------------------------------------------------------------------------------------ MoE block
nvfp4_status moe_route_topk(const float* logits, int64_t T, int32_t E, int32_t k, int32_t* topk_ids, float* topk_w,
                            int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (T < 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "T must be >= 0");
  if (E <= 0 || E > kMaxRouteExperts) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "E = %d must be in [1, %d]", E, kMaxRouteExperts);
  if (k <= 0 || k > 32 || k > E) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "k = %d must be in [1, min(32, E)]", k);
  if (T > 0 && (!logits || !topk_ids || !topk_w)) return fail(NVFP4_ERR_INVALID_ARG, "NULL buffer");
  if (T == 0) return NVFP4_OK;
  cudaError_t e = launch_route_topk(logits, T, E, k, topk_ids, topk_w, dev_status, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "router launch");
}

int64_t moe_rows_capacity(int64_t T, int32_t k, int32_t E, int32_t pad) {
  if (T < 0 || k <= 0 || E <= 0 || pad <= 0) return 0;
  // at most min(E, T*k) experts are routed to, and each wastes at most pad - 1 rows of padding
  const int64_t pairs = T * k;
  const int64_t used = pairs < (int64_t)E ? pairs : (int64_t)E;
  const int64_t worst = pairs + used * (pad - 1);
  return (worst + 127) / 128 * 128;
}

size_t moe_dispatch_workspace_size(int32_t E) { return round_up((size_t)(E > 0 ? E : 1) * sizeof(int32_t), 256); }

nvfp4_status moe_dispatch_plan(const int32_t* topk_ids, int64_t T, int32_t k, int32_t E, int32_t pad,
                               int64_t rows_capacity, int32_t* expert_offsets, int32_t* row_scatter,
                               int32_t* expert_rows, int32_t* slot_expert, int32_t* slot_count, int32_t n_slots,
                               void* workspace,
                               size_t workspace_bytes, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (T < 0 || k <= 0 || k > 128 || E <= 0)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "T >= 0, 0 < k <= 128 and E > 0 required");
  if (pad <= 0 || pad % 16 != 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "pad = %d must be a positive multiple of 16", pad);
  if (rows_capacity < 0 || rows_capacity > INT32_MAX) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "rows_capacity out of range");
  if (!expert_offsets || (T > 0 && (!topk_ids || !row_scatter))) return fail(NVFP4_ERR_INVALID_ARG, "NULL buffer");
  if ((slot_expert == nullptr) != (slot_count == nullptr))
    return fail(NVFP4_ERR_INVALID_ARG, "slot_expert and slot_count go together");
  if (slot_expert && (pad != 16 || n_slots < 0)) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "slot tables need pad == 16");
  if (!workspace || workspace_bytes < moe_dispatch_workspace_size(E)) return fail(NVFP4_ERR_INVALID_ARG, "workspace too small");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_dispatch_plan(topk_ids, T, k, E, pad, rows_capacity, reinterpret_cast<int32_t*>(workspace),
                                       expert_offsets, row_scatter, expert_rows, slot_expert, slot_count, n_slots,
                                       num_sms(), dev_status, s);
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "dispatch plan launch");
}

nvfp4_status moe_row_groups(const int32_t* expert_offsets, int32_t E, int64_t rows, int32_t* row_group,
                            void* stream) {
  g_last_error.clear();
  if (E <= 0 || rows < 0 || rows > INT32_MAX) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "E > 0 and 0 <= rows <= INT32_MAX required");
  if (rows == 0) return NVFP4_OK;
  if (!expert_offsets || !row_group) return fail(NVFP4_ERR_INVALID_ARG, "NULL buffer");
  cudaError_t e = launch_row_groups(expert_offsets, E, rows, row_group, num_sms(), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "row groups launch");
}

nvfp4_status moe_combine(const uint16_t* y, int64_t ldy, int64_t y_rows, const int32_t* row_scatter,
                         const float* topk_w, int64_t T, int32_t k, int64_t H, uint16_t* out, int64_t ldo,
                         int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (T < 0 || k <= 0 || H <= 0 || H % 8 != 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "T >= 0, k > 0, H %% 8 == 0 required");
  if (T == 0) return NVFP4_OK;
  if (!y || !row_scatter || !topk_w || !out) return fail(NVFP4_ERR_INVALID_ARG, "NULL buffer");
  if (ldy < H || ldo < H || ldy % 8 != 0 || ldo % 8 != 0 || !aligned16(y) || !aligned16(out))
    return fail(NVFP4_ERR_ALIGNMENT, "y / out must be 16-byte aligned with pitches >= H, multiples of 8");
  cudaError_t e = launch_combine(y, ldy, y_rows, row_scatter, topk_w, T, k, H, out, ldo, num_sms(), dev_status,
                                 reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "combine launch");
}

// ------------------------------------------------------------------------------------------ qdq
size_t weight_qdq_workspace_size(int64_t n_tensors, int64_t elems_per_tensor) {
  (void)elems_per_tensor;
  const size_t n = (size_t)(n_tensors > 0 ? n_tensors : 1);
  const size_t partials = n * (size_t)slab_partials(n_tensors) * sizeof(float);
  const size_t words = n * 2 * sizeof(uint32_t);  // one-pass form: amax and arrival count per tensor
  return round_up(partials > words ? partials : words, 256);
}

nvfp4_status weight_qdq(const uint16_t* w, int64_t n_tensors, int64_t elems_per_tensor, uint16_t* w_out,
                        float* s_g_out, void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (!w || !w_out) return fail(NVFP4_ERR_INVALID_ARG, "w / w_out is NULL");
  if (n_tensors <= 0 || elems_per_tensor <= 0 || elems_per_tensor % 16 != 0)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "n_tensors > 0 and elems_per_tensor %% 16 == 0 required");
  if (!aligned16(w) || !aligned16(w_out)) return fail(NVFP4_ERR_ALIGNMENT, "w / w_out must be 16-byte aligned");
  if (!workspace || workspace_bytes < weight_qdq_workspace_size(n_tensors, elems_per_tensor))
    return fail(NVFP4_ERR_INVALID_ARG, "workspace too small");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // one pass over HBM when two tensors per CTA group fit in L2 next to each other: tensors of up
  // to 4M elements (8 MB of bf16); larger ones take the two passes (amax, then the fake-quant)
  if (g_qdq_fused.load() && elems_per_tensor <= (4ll << 20)) {
    uint32_t* sync_ws = reinterpret_cast<uint32_t*>(workspace);
    cudaError_t e = cudaMemsetAsync(sync_ws, 0, (size_t)n_tensors * 2 * sizeof(uint32_t), s);
    if (e == cudaSuccess)
      e = launch_qdq_fused(w, n_tensors, elems_per_tensor, w_out, sync_ws, 0, s_g_out, dev_status,
                           g_wait_limit_ns.load(), num_sms(), s);
    if (e == cudaSuccess) return NVFP4_OK;
    cudaGetLastError();  // a grid that cannot be co-resident: the two-pass form below
  }
  float* partial = reinterpret_cast<float*>(workspace);
  const int P = slab_partials(n_tensors);
  cudaError_t e = launch_amax(w, n_tensors, 1, elems_per_tensor, elems_per_tensor, partial, P, dev_status, s);
  if (e != cudaSuccess) return cuda_fail(e, "amax launch");
  e = launch_qdq(w, n_tensors, elems_per_tensor, w_out, partial, P, s_g_out, dev_status, num_sms(), s);
  if (e != cudaSuccess) return cuda_fail(e, "qdq launch");
  return NVFP4_OK;
}

nvfp4_status weight_qdq_backward(const uint16_t* grad_fq, int64_t n, uint16_t* grad_w, float* grad_acc,
                                 void* stream) {
  g_last_error.clear();
  if (n < 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "n must be >= 0");
  if (n > 0 && !grad_fq) return fail(NVFP4_ERR_INVALID_ARG, "grad_fq is NULL");
  if (!grad_w && !grad_acc) return fail(NVFP4_ERR_INVALID_ARG, "grad_w and grad_acc are both NULL");
  if ((grad_fq && !aligned16(grad_fq)) || (grad_w && !aligned16(grad_w)) || (grad_acc && !aligned16(grad_acc)))
    return fail(NVFP4_ERR_ALIGNMENT, "gradient buffers must be 16-byte aligned");
  if (grad_w == grad_fq) grad_w = nullptr;  // in place: the identity needs no copy
  if (n == 0 || (!grad_w && !grad_acc)) return NVFP4_OK;
  cudaError_t e = launch_qdq_backward(grad_fq, n, grad_w, grad_acc, num_sms(), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "qdq backward launch");
}

nvfp4_status nvfp4_unpack_logical(const nvfp4_tensor* q, int64_t slab, uint8_t* codes_out, uint8_t* sf_out,
                                  void* stream) {
  g_last_error.clear();
  if (!q) return fail(NVFP4_ERR_INVALID_ARG, "q is NULL");
  if (!codes_out && !sf_out) return fail(NVFP4_ERR_INVALID_ARG, "codes_out and sf_out are both NULL");
  if (q->slabs < 1 || slab < 0 || slab >= q->slabs) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "slab out of range");
  nvfp4_status st = check_tensor(q, "q", q->cols, q->rows, q->slabs, kAnyLayout);
  if (st != NVFP4_OK) return st;
  if (q->cols <= 0 || q->cols % 64 != 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "q.cols must be a positive multiple of 64");
  if (codes_out && !aligned16(codes_out)) return fail(NVFP4_ERR_ALIGNMENT, "codes_out must be 16-byte aligned");
  if (q->rows == 0) return NVFP4_OK;
  const int64_t cb = q->rows_padded * q->cols / 2;
  const int64_t sb = (int64_t)nvfp4_sf_bytes_layout(q->rows_padded, q->cols, q->sf_layout);
  cudaError_t e = launch_unpack_logical(q->codes + slab * cb, q->sf + slab * sb, q->rows, q->cols,
                                        q->sf_layout == NVFP4_SF_SLAB16, codes_out, sf_out, num_sms(),
                                        reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "unpack launch");
}

// ------------------------------------------------------------------------------------------ helpers
nvfp4_status nvfp4_encode_e2m1(const float* v, int64_t n, uint8_t* out, void* stream) {
  g_last_error.clear();
  if (n < 0 || (n > 0 && (!v || !out))) return fail(NVFP4_ERR_INVALID_ARG, "bad arguments");
  if (n == 0) return NVFP4_OK;
  cudaError_t e = launch_encode_e2m1(v, n, out, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "encode launch");
}

nvfp4_status nvfp4_encode_e4m3(const float* v, int64_t n, uint8_t* out, void* stream) {
  g_last_error.clear();
  if (n < 0 || (n > 0 && (!v || !out))) return fail(NVFP4_ERR_INVALID_ARG, "bad arguments");
  if (n == 0) return NVFP4_OK;
  cudaError_t e = launch_encode_e4m3(v, n, out, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "encode launch");
}

nvfp4_status nvfp4_selftest_wait_timeout(uint64_t limit_ns, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (!dev_status) return fail(NVFP4_ERR_INVALID_ARG, "dev_status is NULL");
  cudaError_t e = launch_wait_selftest(limit_ns, dev_status, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "self-test launch");
}

// ------------------------------------------------------------------------------------------ FP8 comparison path
size_t mxfp8_codes_bytes(int64_t rows_padded, int64_t cols) { return (size_t)rows_padded * (size_t)cols; }
size_t mxfp8_sf_bytes(int64_t rows_padded, int64_t cols) { return (size_t)rows_padded * (size_t)(cols / 32); }

}  // extern "C"

namespace {
nvfp4_status check_mx8(const mxfp8_tensor* t, const char* name, int64_t cols, int64_t min_rows, int64_t slabs) {
  if (!t) return fail(NVFP4_ERR_INVALID_ARG, "%s is NULL", name);
  if (!t->codes || !t->sf) return fail(NVFP4_ERR_INVALID_ARG, "%s has a NULL buffer", name);
  if (t->cols != cols) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "%s.cols = %lld, expected %lld", name, (long long)t->cols, (long long)cols);
  if (t->slabs != slabs) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "%s.slabs = %lld, expected %lld", name, (long long)t->slabs, (long long)slabs);
  if (t->rows_padded % 128 != 0 || t->rows_padded < min_rows || t->rows < 0 || t->rows > t->rows_padded)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "%s rows %lld / rows_padded %lld invalid (need >= %lld, multiple of 128)", name,
                (long long)t->rows, (long long)t->rows_padded, (long long)min_rows);
  if (!aligned16(t->codes) || !aligned16(t->sf)) return fail(NVFP4_ERR_ALIGNMENT, "%s buffers must be 16-byte aligned", name);
  return NVFP4_OK;
}

nvfp4_status mx8_check_k(int64_t K) {
  if (K <= 0 || K % 128 != 0 || K > kMaxK)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "K = %lld must be a positive multiple of 128 <= %lld", (long long)K, (long long)kMaxK);
  return NVFP4_OK;
}

nvfp4_status mx8_gemm_setup(const mxfp8_tensor* a, const mxfp8_tensor* w, int64_t rows_needed, int64_t N, int64_t K,
                            int64_t E, nvfp4_dtype out, void* y, int64_t ldy, int64_t y_cols, int64_t y_rows, int bn,
                            CUtensorMap* maps, GemmArgs* g) {
  nvfp4_status st = mx8_check_k(K);
  if (st != NVFP4_OK) return st;
  if (N <= 0 || N % 128 != 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "N must be a positive multiple of 128");
  if (out != NVFP4_OUT_F32 && out != NVFP4_OUT_BF16) return fail(NVFP4_ERR_INVALID_ARG, "bad output dtype");
  if (!y) return fail(NVFP4_ERR_INVALID_ARG, "y is NULL");
  if (!aligned16(y)) return fail(NVFP4_ERR_ALIGNMENT, "y must be 16-byte aligned");
  if (ldy < y_cols || (out == NVFP4_OUT_BF16 ? ldy % 8 : ldy % 4) != 0)
    return fail(NVFP4_ERR_ALIGNMENT, "ldy = %lld must be >= %lld and keep rows 16-byte aligned", (long long)ldy, (long long)y_cols);
  st = check_mx8(a, "a", K, rows_needed, 1);
  if (st != NVFP4_OK) return st;
  st = check_mx8(w, "w", K, N, E);
  if (st != NVFP4_OK) return st;
  if (w->rows_padded != N) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "w.rows_padded must equal N");
  memset(maps, 0, 5 * sizeof(CUtensorMap));
  if (y_rows > 0) {
    st = make_out_map(&maps[4], y, out == NVFP4_OUT_BF16, (uint64_t)y_cols, (uint64_t)y_rows, (uint64_t)ldy);
    if (st != NVFP4_OK) return st;
  }
  st = make_code_map(&maps[0], a->codes, (uint64_t)K, (uint64_t)a->rows_padded, 1, 128, 2, "A");
  if (st != NVFP4_OK) return st;
  st = make_code_map(&maps[2], w->codes, (uint64_t)K, (uint64_t)N, (uint64_t)E, (uint32_t)bn, 3, "W");
  if (st != NVFP4_OK) return st;
  maps[1] = maps[0];
  maps[3] = maps[2];
  memset(g, 0, sizeof(*g));
  g->fp8 = 1;
  g->sfa = a->sf;
  g->sfa_res = a->sf;
  g->sfw = w->sf;
  g->sfw_sel = w->sf;
  g->sfw_slab_bytes = (int64_t)mxfp8_sf_bytes(N, K);
  g->k64_main = (int32_t)(K / 64);
  g->kt_main = (int32_t)(K / 128);
  g->kt_res = 0;
  g->N = (int32_t)N;
  g->n_blocks = (int32_t)(N / bn);
  g->rows_capacity = a->rows_padded;
  g->y = y;
  g->ldy = ldy;
  g->out_bf16 = out == NVFP4_OUT_BF16;
  g->wait_limit_ns = g_wait_limit_ns.load();
  return NVFP4_OK;
}

nvfp4_status mx8_rows(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const int32_t* row_gather,
                      const int32_t* row_scatter, int32_t fanout, int64_t M_out, const mxfp8_tensor* q,
                      int32_t* dev_status, void* stream) {
  if (!x && M > 0) return fail(NVFP4_ERR_INVALID_ARG, "x is NULL");
  if (M < 0 || M_out < 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "negative row count");
  nvfp4_status st = mx8_check_k(K);
  if (st != NVFP4_OK) return st;
  if (ldx < K || ldx % 8 != 0) return fail(NVFP4_ERR_ALIGNMENT, "ldx = %lld must be >= K and a multiple of 8", (long long)ldx);
  if (x && !aligned16(x)) return fail(NVFP4_ERR_ALIGNMENT, "x must be 16-byte aligned");
  st = check_mx8(q, "q", K, row_scatter ? 0 : M_out, 1);
  if (st != NVFP4_OK) return st;
  Mx8RowArgs a;
  memset(&a, 0, sizeof(a));
  a.src = x;
  a.src_rows = M;
  a.ld = ldx;
  a.K = K;
  a.row_gather = row_gather;
  a.row_scatter = row_scatter;
  a.fanout = fanout;
  a.rows_out = q->rows_padded;
  a.rows_per_slab = row_scatter ? M : M_out;
  a.codes = q->codes;
  a.sf = q->sf;
  a.status = dev_status;
  if ((row_scatter ? M : a.rows_out) == 0) return NVFP4_OK;
  cudaError_t e = launch_mx8_rows(a, num_sms(), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "fp8 quantize launch");
}
}  // namespace

extern "C" {

nvfp4_status mxfp8_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const int32_t* row_gather,
                            int64_t M_out, const mxfp8_tensor* q, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (!row_gather && M_out != M) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "without row_gather M_out must equal M");
  return mx8_rows(x, M, K, ldx, row_gather, nullptr, 1, M_out, q, dev_status, stream);
}

nvfp4_status mxfp8_quantize_scatter(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const int32_t* row_scatter,
                                    int32_t fanout, const mxfp8_tensor* q, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (!row_scatter && M > 0) return fail(NVFP4_ERR_INVALID_ARG, "row_scatter is NULL");
  if (fanout <= 0 || fanout > 32) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "1 <= fanout <= 32 required");
  return mx8_rows(x, M, K, ldx, nullptr, row_scatter, fanout, 0, q, dev_status, stream);
}

nvfp4_status mxfp8_pack_weights(const uint16_t* w, int64_t E, int64_t N, int64_t K, int32_t gate_up_interleave,
                                const mxfp8_tensor* w_q, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (!w) return fail(NVFP4_ERR_INVALID_ARG, "w is NULL");
  if (E <= 0 || N <= 0 || N % 128 != 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "E > 0 and N %% 128 == 0 required");
  nvfp4_status st = mx8_check_k(K);
  if (st != NVFP4_OK) return st;
  if (gate_up_interleave != 0 && gate_up_interleave != 1) return fail(NVFP4_ERR_INVALID_ARG, "gate_up_interleave must be 0 or 1");
  if (!aligned16(w)) return fail(NVFP4_ERR_ALIGNMENT, "w must be 16-byte aligned");
  st = check_mx8(w_q, "w_q", K, N, E);
  if (st != NVFP4_OK) return st;
  if (w_q->rows_padded != N || w_q->rows != N) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "w_q rows / rows_padded must equal N");
  Mx8RowArgs a;
  memset(&a, 0, sizeof(a));
  a.src = w;
  a.src_rows = N;
  a.ld = K;
  a.K = K;
  a.rows_out = E * N;
  a.rows_per_slab = N;
  a.src_slab_stride = N * K;
  a.pack = 1;
  a.interleave = gate_up_interleave;
  a.N_half = N / 2;
  a.codes = w_q->codes;
  a.sf = w_q->sf;
  a.status = dev_status;
  cudaError_t e = launch_mx8_rows(a, num_sms(), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "fp8 pack launch");
}

nvfp4_status mxfp8_gemm(const mxfp8_tensor* a, const mxfp8_tensor* w, int64_t M, int64_t N, int64_t K,
                        nvfp4_dtype out, void* y, int64_t ldy, int32_t* dev_status, void* stream) {
  g_last_error.clear();
  if (M < 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "M must be >= 0");
  const int bn = choose_tile_n(N, K, 0);
  CUtensorMap maps[5];
  GemmArgs g;
  nvfp4_status st = mx8_gemm_setup(a, w, M, N, K, 1, out, y, ldy, N, M, bn, maps, &g);
  if (st != NVFP4_OK) return st;
  if (M == 0) return NVFP4_OK;
  g.E = 1;
  g.M = M;
  g.m_blocks_dense = (int32_t)((M + 127) / 128);
  g.status = dev_status;
  const int64_t tiles = (int64_t)g.m_blocks_dense * g.n_blocks;
  const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
  cudaError_t e = launch_gemm(bn, maps[0], maps[1], maps[2], maps[3], maps[4], g, grid,
                              reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "fp8 gemm launch");
}

nvfp4_status grouped_mxfp8_moe(const mxfp8_tensor* a, const int32_t* expert_offsets, const int32_t* expert_rows,
                               int32_t E, const mxfp8_tensor* w, int64_t N, int64_t K, nvfp4_epilogue ep,
                               nvfp4_dtype out, void* y, int64_t ldy, float* amax_out, int32_t* dev_status,
                               void* stream) {
  g_last_error.clear();
  if (!expert_offsets) return fail(NVFP4_ERR_INVALID_ARG, "expert_offsets is NULL");
  if (E <= 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "E must be positive");
  if (ep != NVFP4_EPI_NONE && ep != NVFP4_EPI_SWIGLU_AMAX) return fail(NVFP4_ERR_INVALID_ARG, "bad epilogue");
  if (ep == NVFP4_EPI_SWIGLU_AMAX) {
    if (out != NVFP4_OUT_BF16) return fail(NVFP4_ERR_INVALID_ARG, "the SwiGLU epilogue writes bf16");
    if (N % 256 != 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "the SwiGLU epilogue needs N %% 256 == 0");
  }
  const int bn = ep == NVFP4_EPI_SWIGLU_AMAX ? 256 : choose_tile_n(N, K, 0);
  CUtensorMap maps[5];
  GemmArgs g;
  const int64_t y_cols = ep == NVFP4_EPI_SWIGLU_AMAX ? N / 2 : N;
  nvfp4_status st = mx8_gemm_setup(a, w, 0, N, K, E, out, y, ldy, y_cols, a ? a->rows_padded : 0, bn, maps, &g);
  if (st != NVFP4_OK) return st;
  g.offsets = expert_offsets;
  g.expert_rows = expert_rows;
  g.E = E;
  g.M = a->rows_padded;
  g.epi = ep == NVFP4_EPI_SWIGLU_AMAX ? 1 : 0;
  g.amax_out = amax_out;
  g.status = dev_status;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (ep == NVFP4_EPI_SWIGLU_AMAX && amax_out) {
    cudaError_t e = cudaMemsetAsync(amax_out, 0, sizeof(float), s);
    if (e != cudaSuccess) return cuda_fail(e, "amax reset");
  }
  cudaError_t e = launch_gemm(bn, maps[0], maps[1], maps[2], maps[3], maps[4], g, num_sms(), s);
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "grouped fp8 gemm launch");
}

}  // extern "C"

// Helpers for entry points defined in other files of the library.
namespace nvfp4 {
nvfp4_status record_host_error(nvfp4_status s, const char* msg) { return fail(s, "%s", msg); }
void clear_host_error() { g_last_error.clear(); }
int qdq_partial_count(int64_t n_tensors) { return slab_partials(n_tensors); }
int device_sm_count() { return num_sms(); }
}  // namespace nvfp4
