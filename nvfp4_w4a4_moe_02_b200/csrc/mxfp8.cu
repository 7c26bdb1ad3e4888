// FP8 comparison path: the row quantiser of the block-scaled FP8 format the FP4 + RAC path is
// measured against (the pages set their 4-bit rollouts against FP8 without fixing an FP8 recipe).
//
// Format: E4M3 elements, one power-of-two scale 2^X per 32 consecutive elements along K, stored
// as the E8M0 code X + 127 in the same 512-byte atoms the FP4 scales use (128 rows x 4 blocks, so
// one atom covers 128 K-elements = one 128-byte k-tile of the GEMM); no tensor scale.  X is the
// smallest integer with 448 * 2^X >= max|x| of the block (clamped to [-127, 127]), so no element
// saturates; q = E4M3_RNE_satfinite(RN(x * 2^-X)) with the sign kept.
//
// One warp per row; lane l owns the 32-element block [it*1024 + 32l, +32): four 16-byte loads,
// one exponent, sixteen paired conversions, two 16-byte code stores and one scale byte per
// destination row.  No amax pass: the format has no tensor scale.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {

__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// smallest X in [-127, 127] with 448 * 2^X >= b (b finite, >= 0)
__device__ __forceinline__ int mx8_exponent(float b) {
  if (b == 0.0f) return -127;
  int E;
  frexpf(b, &E);  // b = m 2^E, m in [0.5, 1): 448 * 2^(E-9) = 0.875 * 2^E is the first candidate
  int X = E - 9;
  if (X < -127) return -127;
  if (ldexpf(448.0f, X) < b) ++X;  // 448 * 2^(E-8) = 1.75 * 2^E > b always holds
  return X > 127 ? 127 : X;
}

__global__ void __launch_bounds__(256) mx8_rows_kernel(const Mx8RowArgs a) {
  const int lane = threadIdx.x & 31;
  const int32_t K = (int32_t)a.K;
  const int64_t kt = K / 128;  // scale atoms per 128-row block
  const int64_t row_first = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t row_step = (int64_t)gridDim.x * (blockDim.x >> 5);
  const bool scatter = a.row_scatter != nullptr;
  const int64_t n_rows = scatter ? a.src_rows : a.rows_out;
  for (int64_t row = row_first; row < n_rows; row += row_step) {
    const int64_t slab = a.pack ? row / a.rows_per_slab : 0;
    const int64_t r_in = row - slab * a.rows_per_slab;
    int64_t src_row = r_in;
    if (!scatter && !a.pack && a.row_gather != nullptr) src_row = r_in < a.rows_per_slab ? a.row_gather[r_in] : -1;
    if (a.pack && a.interleave) {
      const int64_t q = r_in >> 7, j = r_in & 127;
      src_row = (j < 64) ? (q * 64 + j) : (a.N_half + q * 64 + (j - 64));
    }
    const bool valid = src_row >= 0 && src_row < a.src_rows;
    const uint16_t* srow = a.src + slab * a.src_slab_stride + (valid ? src_row : 0) * a.ld;
    // destinations: the row itself, or the source row's fanout rows (lane j holds entry j)
    const int fan = scatter ? a.fanout : 1;
    const int32_t mine = (scatter && lane < fan) ? __ldg(a.row_scatter + row * a.fanout + lane) : -1;
    for (int32_t base = 0; base < K; base += 1024) {
      const int32_t e = base + 32 * lane;
      const bool h = e < K;
      float x[32];
      uint4 u[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        u[q] = (h && valid) ? __ldg(reinterpret_cast<const uint4*>(srow + e) + q) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t w[4] = {u[q].x, u[q].y, u[q].z, u[q].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          x[8 * q + 2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
          x[8 * q + 2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
        }
      }
      float b = 0.0f;
#pragma unroll
      for (int i = 0; i < 32; ++i) b = fmaxf(b, fabsf(x[i]));
      if (!(b <= 3.4028234663852886e38f)) {  // inf or NaN: reported, the block is written as zero
        report_status(a.status, kErrRange);
        b = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = 0.0f;
      }
      const int X = mx8_exponent(b);
      const float inv = ldexpf(1.0f, -X);  // a normal binary32 power of two: the product is RN(x 2^-X)
      uint32_t c[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        c[i] = e4m3x2(__fmul_rn(x[4 * i], inv), __fmul_rn(x[4 * i + 1], inv)) |
               (e4m3x2(__fmul_rn(x[4 * i + 2], inv), __fmul_rn(x[4 * i + 3], inv)) << 16);
      const uint8_t sbyte = (uint8_t)(X + 127);
      const int32_t kb = e >> 5;
      for (int j = 0; j < fan; ++j) {
        const int64_t drow = scatter ? (int64_t)__shfl_sync(0xffffffffu, mine, j) : row;
        if (drow < 0 || !h) continue;
        if (drow >= a.rows_out) {
          report_status(a.status, kErrInvalid);
          continue;
        }
        uint4* cp = reinterpret_cast<uint4*>(a.codes + drow * K + e);
        cp[0] = make_uint4(c[0], c[1], c[2], c[3]);
        cp[1] = make_uint4(c[4], c[5], c[6], c[7]);
        a.sf[(drow >> 7) * kt * 512 + (drow & 31) * 16 + ((drow >> 5) & 3) * 4 + (kb >> 2) * 512 + (kb & 3)] = sbyte;
      }
    }
  }
}

cudaError_t launch_mx8_rows(const Mx8RowArgs& a, int num_sms, cudaStream_t st) {
  const int64_t rows = a.row_scatter ? a.src_rows : a.rows_out;
  int64_t grid = (rows + 7) / 8;
  if (grid > (int64_t)num_sms * 8) grid = (int64_t)num_sms * 8;
  if (grid < 1) grid = 1;
  mx8_rows_kernel<<<(unsigned)grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace nvfp4
