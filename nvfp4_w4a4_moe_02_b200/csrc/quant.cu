// Quantisation kernels: per-tensor amax, the row quantiser (activation + RAC residual,
// weight pack, calibration residuals), calibration reduction/selection and trainer QDQ.
//
// All of them are HBM-streaming kernels: 128-bit loads of 8 bf16, two lanes per 16-element
// block (one shuffle for the block max), packed e2m1 stores that stay contiguous across the
// warp, and scales written straight into the 512-byte scale atoms the tcgen05 MMA reads.
#include "common.cuh"
#include <algorithm>
#include <climits>

#include "kernels.h"

namespace nvfp4 {

// ----------------------------------------------------------------------------------------
// K1: segmented amax.  Segment s = rows [s*seg_rows, (s+1)*seg_rows) of a [rows x cols]
// bf16 matrix with pitch ld.  Grid (P, segments); CTA p writes partial[s*P + p].
// ----------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* __restrict__ x, int64_t seg_rows, int64_t cols,
                                                   int64_t ld, float* __restrict__ partial, int32_t* status) {
  const int P = gridDim.x;
  const int64_t seg = blockIdx.y;
  float m = 0.0f;
  bool bad = false;
  const uint16_t* base = x + seg * seg_rows * ld;
  if (ld == cols) {
    // contiguous segment: flat vector loop, eight independent 16-byte loads in flight per thread
    // (a partial covers 16K elements: one round of loads)
    const int64_t nvec = seg_rows * cols / 8;
    const uint4* v = reinterpret_cast<const uint4*>(base);
    const int64_t stride = (int64_t)P * blockDim.x;
    for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < nvec; i0 += 8 * stride) {
      uint4 q[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) q[u] = (i0 + u * stride < nvec) ? __ldg(v + i0 + u * stride) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float a = fabsf(bf16_bits_to_f32(w[j] & 0xFFFFu));
          float b = fabsf(bf16_bits_to_f32(w[j] >> 16));
          bad |= !(a <= 3.4e38f) || !(b <= 3.4e38f);
          m = fmaxf(m, fmaxf(a, b));
        }
      }
    }
  } else {
    const int64_t vpr = cols / 8;
    for (int64_t r = blockIdx.x; r < seg_rows; r += P) {
      const uint4* v = reinterpret_cast<const uint4*>(base + r * ld);
      for (int64_t i = threadIdx.x; i < vpr; i += blockDim.x) {
        uint4 q = __ldg(v + i);
        uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float a = fabsf(bf16_bits_to_f32(w[j] & 0xFFFFu));
          float b = fabsf(bf16_bits_to_f32(w[j] >> 16));
          bad |= !(a <= 3.4e38f) || !(b <= 3.4e38f);
          m = fmaxf(m, fmaxf(a, b));
        }
      }
    }
  }
  if (bad) report_status(status, kErrRange);
  __shared__ float red[8];
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.0f;
    v = warp_max(v);
    if (threadIdx.x == 0) partial[seg * P + blockIdx.x] = v;
  }
}

// max over P partials of one segment, by one warp (all lanes return the result)
__device__ __forceinline__ float reduce_partials(const float* partial, int P) {
  float m = 0.0f;
  for (int i = threadIdx.x & 31; i < P; i += 32) m = fmaxf(m, partial[i]);
  return warp_max(m);
}

// amax of one tensor from its partials, written to a device float (one warp)
__global__ void reduce_amax_kernel(const float* __restrict__ partial, int P, float* out) {
  const float m = reduce_partials(partial, P);
  if (threadIdx.x == 0) *out = m;
}

// ----------------------------------------------------------------------------------------
// K2 / K7 / calibration: the row quantiser.  One warp per row, 512 elements per warp
// iteration: lane l owns the 16-element block [it*512 + 16l, +16), so a block's scale is
// computed once, by one lane, with no shuffles; its 8 bytes of codes and its scale byte are
// stored by that lane.
//
// The residual pass over the selected channels (activation mode) or the raw selected columns
// (weight pack) runs after the main pass: each lane takes 16 consecutive compact positions, reads
// their channel numbers, gathers x from the row again (it was just read: the loads hit L1) and
// re-derives its code and DQ = e*d from a per-warp stash of each block's (d, 1/d).  Keeping only
// the block scales in shared memory, not the row, leaves room for more warps per SM.
//
// Masked residual (activation mode, a variant of the method): the residual stays at its channel,
// zero off the selection, and is quantised in 16-blocks along K in the main pass itself (each
// lane knows which of its 16 channels are selected from a CTA-shared bitmap); there is no
// residual pass, and the GEMM reuses the main packed weights for it.
//
// SPLIT (activations with few rows, e.g. the tokens of one decode step): a whole CTA works on
// one row; warp w takes the 512-element chunks w, w + nwarps, ... of both passes and the stash
// is shared by the CTA, so a 64-token batch still occupies every warp of 64 CTAs.
// ----------------------------------------------------------------------------------------

// destinations of the current row: the row itself, or up to `fanout` (<= 64) rows in scatter
// mode, read once per row into the warp's registers (lane l holds entries l and l + 32) so that
// the per-chunk store loops pick them with a shuffle instead of a dependent global load
struct Dests {
  bool scatter;
  int n;
  int64_t row;
  int32_t mine0, mine1;
  __device__ __forceinline__ void load(const int32_t* list, int fanout) {
    const int lane = threadIdx.x & 31;
    scatter = true;
    n = fanout;
    mine0 = lane < fanout ? __ldg(list + lane) : -1;
    mine1 = lane + 32 < fanout ? __ldg(list + 32 + lane) : -1;
  }
  // all lanes call get(j) with the same j
  __device__ __forceinline__ int64_t get(int j) const {
    if (!scatter) return row;
    const int32_t v0 = __shfl_sync(0xffffffffu, mine0, j & 31);
    const int32_t v1 = __shfl_sync(0xffffffffu, mine1, j & 31);
    return (int64_t)(j < 32 ? v0 : v1);
  }
};

__device__ __forceinline__ void unpack8(const uint4 raw, float x[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    x[2 * j] = bf16_bits_to_f32(w[j] & 0xFFFFu);
    x[2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
  }
}

template <int MODE, bool SPLIT>
__global__ void __launch_bounds__(256, 4) quant_rows_kernel(const RowArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int32_t K = (int32_t)a.K;  // <= 32768: offsets inside a row fit in 32 bits
  const int32_t Kp = a.Kp;
  constexpr bool kHasSel = (MODE == kModeAct || MODE == kModePack);
  const bool masked = MODE == kModeAct && a.masked_res != 0 && Kp > 0;
  const bool use_sel = kHasSel && Kp > 0 && !masked;  // compact residual pass
  // per-group channel lists (pack: group = slab; act: group = row_group[row]) are read from
  // global memory (L1-resident) in the residual pass instead of the CTA-shared copy
  const bool grouped = use_sel && a.sel_groups > 0;

  // CTA-shared channel list (int16), then per warp (per CTA when SPLIT) each block's (d, 1/d);
  // the masked variant keeps a bitmap of the selected channels instead
  int16_t* sel_s = reinterpret_cast<int16_t*>(smem_raw);
  uint32_t* mask_s = reinterpret_cast<uint32_t*>(smem_raw);
  const size_t sel_bytes = (use_sel && !grouped) ? (((size_t)Kp * 2 + 15) / 16) * 16 : 0;
  const size_t warp_bytes = use_sel ? (size_t)(K / 16) * 8 : 0;
  float2* dinv_s = reinterpret_cast<float2*>(smem_raw + sel_bytes + (SPLIT ? 0 : warp) * warp_bytes);
  if ((use_sel && !grouped) || masked) {
    if (masked) {
      for (int32_t w = threadIdx.x; w < (K + 31) / 32; w += blockDim.x) mask_s[w] = 0u;
      __syncthreads();
    }
    for (int32_t j = threadIdx.x; j < Kp; j += blockDim.x) {
      int32_t c = a.sel[j];
      bool ok = (c >= 0 && c < K) && (j == 0 || a.sel[j - 1] < c);
      if (!ok) {
        report_status(a.status, kErrInvalid);
        c = 0;
      }
      if (masked) atomicOr(mask_s + (c >> 5), 1u << (c & 31));
      else sel_s[j] = (int16_t)c;
    }
    __syncthreads();
  }

  const int64_t k64 = K / 64;
  const int64_t kp64 = Kp / 64;
  const bool scatter = (MODE == kModeAct && a.row_scatter != nullptr);
  const int64_t n_rows = scatter ? a.src_rows : a.rows_out;
  const bool slab16 = a.sf_slab16 != 0;
  int64_t cached_slab = -1;
  float s_g = 0.0f, t6 = 0.0f;

  // byte offset of a row's part of a scale-atom array, and of a block's part (see sf_offset)
  auto sf_row = [&](int64_t r, int64_t groups) -> int64_t {
    return slab16 ? (r >> 4) * groups * 512 + (r & 15) * 16
                  : (r >> 7) * groups * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4;
  };
  auto sf_blk = [](int32_t kb) -> int32_t { return (kb >> 2) * 512 + (kb & 3); };

  const int64_t row_first = SPLIT ? (int64_t)blockIdx.x : (int64_t)blockIdx.x * nwarps + warp;
  const int64_t row_step = SPLIT ? (int64_t)gridDim.x : (int64_t)gridDim.x * nwarps;
  const int32_t chunk0 = SPLIT ? 512 * warp : 0;          // this warp's first chunk of a row
  const int32_t chunk_step = SPLIT ? 512 * nwarps : 512;  // distance to its next chunk
  for (int64_t row = row_first; row < n_rows; row += row_step) {
    // ---- source row, destinations, scale
    int64_t slab = (MODE == kModePack) ? row / a.rows_per_slab : 0;
    int64_t r_in_slab = row - slab * a.rows_per_slab;
    int64_t src_row = r_in_slab;
    Dests dst{false, 1, row, -1, -1};
    if (scatter) {
      dst.load(a.row_scatter + row * a.fanout, a.fanout);
    } else if (MODE == kModeAct && a.row_gather != nullptr) {
      src_row = (r_in_slab < a.rows_per_slab) ? a.row_gather[r_in_slab] : -1;
    }
    if (MODE == kModePack && a.interleave) {
      int64_t q = r_in_slab >> 7, j = r_in_slab & 127;
      src_row = (j < 64) ? (q * 64 + j) : (a.N_half + q * 64 + (j - 64));
    }
    const bool valid = (src_row >= 0 && src_row < a.src_rows);
    // this row's channel list when the lists are per group (nullptr: the residual row is zero)
    const int32_t* gsel = nullptr;
    if (grouped) {
      const int64_t g = (MODE == kModePack) ? slab : (int64_t)a.row_group[row];
      if (g >= a.sel_groups) {
        if (lane == 0) report_status(a.status, kErrInvalid);
      } else if (g >= 0) {
        gsel = a.sel + g * Kp;
      }
    }
    if (slab != cached_slab) {
      float amax = (MODE == kModeAct && a.amax_in != nullptr) ? *a.amax_in : reduce_partials(a.partial + slab * a.P, a.P);
      s_g = scale_from_amax(amax, a.status);
      t6 = __fmul_rn(6.0f, s_g);
      cached_slab = slab;
      if (row == slab * a.rows_per_slab && lane == 0 && (!SPLIT || warp == 0)) {
        // exactly one warp writes each slab's scale: the one owning the slab's first row
        if (a.s_g_out) a.s_g_out[slab] = s_g;
        if (a.s_g_out2) a.s_g_out2[slab] = s_g;
      }
    }
    const uint16_t* srow = a.src + slab * a.src_slab_stride + (valid ? src_row : 0) * a.ld;

    // ---- main pass: lane l owns the 16-element block starting at chunk + 16 l (the next
    // chunk's loads are issued before this block's arithmetic)
    auto load16 = [&](int32_t e, uint4& u0, uint4& u1) {
      const bool ok = valid && e < K;
      u0 = ok ? __ldg(reinterpret_cast<const uint4*>(srow + e)) : make_uint4(0, 0, 0, 0);
      u1 = ok ? __ldg(reinterpret_cast<const uint4*>(srow + e + 8)) : make_uint4(0, 0, 0, 0);
    };
    uint4 n0, n1;
    load16(chunk0 + 16 * lane, n0, n1);
    for (int32_t base = chunk0; base < K; base += chunk_step) {
      const int32_t e = base + 16 * lane;
      const bool h = e < K;  // K % 16 == 0: a block is wholly inside or outside
      const uint4 r0 = n0, r1 = n1;
      if (base + chunk_step < K) load16(e + chunk_step, n0, n1);
      float x[16];
      unpack8(r0, x);
      unpack8(r1, x + 8);
      float b = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) b = fmaxf(b, fabsf(x[i]));
      const BlockScale bs = block_scale(b, s_g, t6);
      if (MODE == kModeCal) {
        float dq[16];
        quant8(x, bs, dq);
        quant8(x + 8, bs, dq + 8);
        if (h) {
          float* rr = a.resid_all + row * K + e;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<float4*>(rr + 4 * q) =
                make_float4(__fsub_rn(x[4 * q], dq[4 * q]), __fsub_rn(x[4 * q + 1], dq[4 * q + 1]),
                            __fsub_rn(x[4 * q + 2], dq[4 * q + 2]), __fsub_rn(x[4 * q + 3], dq[4 * q + 3]));
        }
        continue;
      }
      const int32_t kb = e >> 4;
      uint2 c, mc = make_uint2(0u, 0u);
      uint32_t mS = 0;
      if (masked) {
        // residual of the selected channels of this block, zero elsewhere, quantised in place
        float dq[16], m[16];
        c = make_uint2(quant8(x, bs, dq), quant8(x + 8, bs, dq + 8));
        const uint32_t bits = h ? (mask_s[e >> 5] >> (e & 31)) & 0xFFFFu : 0u;
        float bm = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          m[i] = ((bits >> i) & 1u) ? __fsub_rn(x[i], dq[i]) : 0.0f;
          bm = fmaxf(bm, fabsf(m[i]));
        }
        const BlockScale ms = block_scale(bm, s_g, t6);
        mc = make_uint2(quant8_codes(m, ms), quant8_codes(m + 8, ms));
        mS = ms.S;
      } else {
        c = make_uint2(quant8_codes(x, bs), quant8_codes(x + 8, bs));
      }
      if (use_sel && h) dinv_s[kb] = make_float2(bs.d, bs.inv);  // block scales for the residual pass
      const int32_t blk = sf_blk(kb);
      for (int j = 0; j < dst.n; ++j) {
        const int64_t drow = dst.get(j);
        if (drow < 0 || !h) continue;
        if (drow >= a.rows_out) {
          report_status(a.status, kErrInvalid);
          continue;
        }
        *reinterpret_cast<uint2*>(a.codes + drow * (K / 2) + e / 2) = c;
        a.sf[sf_row(drow, k64) + blk] = (uint8_t)bs.S;
        if (masked) {
          *reinterpret_cast<uint2*>(a.rcodes + drow * (K / 2) + e / 2) = mc;
          a.rsf[sf_row(drow, k64) + blk] = (uint8_t)mS;
        }
      }
    }

    // ---- residual pass: lane l owns the compact 16 positions starting at chunk + 16 l
    if (use_sel) {
      if (SPLIT) __syncthreads(); else __syncwarp();  // every block's scale is stashed
      for (int32_t base = chunk0; base < Kp; base += chunk_step) {
        const int32_t p = base + 16 * lane;
        const bool h = p < Kp;
        int32_t ch[16];
        bool rvalid = valid;
        if (!grouped) {
          const uint4 c0 = h ? *reinterpret_cast<const uint4*>(sel_s + p) : make_uint4(0, 0, 0, 0);
          const uint4 c1 = h ? *reinterpret_cast<const uint4*>(sel_s + p + 8) : make_uint4(0, 0, 0, 0);
          const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            ch[2 * q] = (int32_t)(int16_t)(w[q] & 0xFFFFu);
            ch[2 * q + 1] = (int32_t)(int16_t)(w[q] >> 16);
          }
        } else {
          rvalid = valid && gsel != nullptr;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int4 c = (h && gsel) ? __ldg(reinterpret_cast<const int4*>(gsel + p) + q) : make_int4(0, 0, 0, 0);
            ch[4 * q] = c.x;
            ch[4 * q + 1] = c.y;
            ch[4 * q + 2] = c.z;
            ch[4 * q + 3] = c.w;
          }
          // the list must be ascending and inside [0, K): checked where it is used
          bool bad = false;
          int32_t prev = (h && gsel && p > 0) ? __ldg(gsel + p - 1) : -1;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            bad |= (ch[i] <= prev) || (ch[i] >= K);
            prev = ch[i];
          }
          if (h && gsel && bad) {
            report_status(a.status, kErrInvalid);
#pragma unroll
            for (int i = 0; i < 16; ++i) ch[i] = 0;
          }
        }
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = (h && rvalid) ? bf16_bits_to_f32(__ldg(srow + ch[i])) : 0.0f;
        if (MODE != kModePack) {
          // re-derive each channel's code under its own block scale, then r = x - e*d
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float sc[8], d[8], ev[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 di = dinv_s[ch[8 * hh + i] >> 4];
              d[i] = di.x;
              sc[i] = __fmul_rn(v[8 * hh + i], di.y);
            }
            e2m1_decode8(e2m1_encode8(sc), ev);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              v[8 * hh + i] = __fsub_rn(v[8 * hh + i], d[i] == 0.0f ? 0.0f : __fmul_rn(ev[i], d[i]));
          }
        }
        float b = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) b = fmaxf(b, fabsf(v[i]));
        const BlockScale bs = block_scale(b, s_g, t6);
        const uint2 c = make_uint2(quant8_codes(v, bs), quant8_codes(v + 8, bs));
        const int32_t blk = sf_blk(p >> 4);
        for (int j = 0; j < dst.n; ++j) {
          const int64_t drow = dst.get(j);
          if (drow < 0 || drow >= a.rows_out || !h) continue;
          *reinterpret_cast<uint2*>(a.rcodes + drow * (Kp / 2) + p / 2) = c;
          a.rsf[sf_row(drow, kp64) + blk] = (uint8_t)bs.S;
        }
      }
      if (SPLIT) __syncthreads(); else __syncwarp();  // stash reads done before the next row
    }
  }
}

// ----------------------------------------------------------------------------------------
// calibration: e_k = sum_t r_{t,k}^2 in binary64, t ascending (one thread per channel), then
// selection of the Kp largest (ties -> lower k), written ascending.
// ----------------------------------------------------------------------------------------
// Grouped form (one channel list per expert): blockIdx.y = group g sums rows [off[g], off[g+1])
// into err[g * K + k]; off == nullptr is the single group [0, T).
__global__ void __launch_bounds__(256) chan_err_kernel(const float* __restrict__ resid, int64_t T, int64_t K,
                                                       const int32_t* __restrict__ off, double* __restrict__ err,
                                                       int32_t* status) {
  int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const int64_t g = blockIdx.y;
  int64_t t0 = off ? (int64_t)off[g] : 0, t1 = off ? (int64_t)off[g + 1] : T;
  if (t0 < 0 || t1 < t0 || t1 > T) {  // offsets must be non-decreasing inside [0, T]
    if (k == 0) report_status(status, kErrInvalid);
    t0 = t1 = 0;
  }
  double e = 0.0;
  for (int64_t t = t0; t < t1; ++t) {
    double v = (double)resid[t * K + k];
    e = __dadd_rn(e, __dmul_rn(v, v));
  }
  err[g * K + k] = e;
}

// One CTA of 1024 threads per group (blockIdx.x = g selects from err + g K into sel_out + g Kp);
// K <= kMaxCalK.
__global__ void __launch_bounds__(1024) select_topk_kernel(const double* __restrict__ err, int32_t K, int32_t Kp,
                                                           int32_t* __restrict__ sel_out, double* __restrict__ err_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  err += (int64_t)blockIdx.x * K;
  sel_out += (int64_t)blockIdx.x * Kp;
  if (err_out) err_out += (int64_t)blockIdx.x * K;
  double* e = reinterpret_cast<double*>(smem_raw);
  int32_t* flag = reinterpret_cast<int32_t*>(e + K);
  __shared__ int32_t warp_sums[32];
  for (int32_t k = threadIdx.x; k < K; k += blockDim.x) {
    e[k] = err[k];
    if (err_out) err_out[k] = err[k];
  }
  __syncthreads();
  for (int32_t k = threadIdx.x; k < K; k += blockDim.x) {
    const double ek = e[k];
    int32_t rank = 0;
    for (int32_t j = 0; j < K; ++j) {
      const double ej = e[j];
      rank += (ej > ek) || (ej == ek && j < k);
    }
    flag[k] = rank < Kp;
  }
  __syncthreads();
  // ascending compaction: chunked exclusive scan over K flags
  int32_t carry = 0;
  for (int32_t base = 0; base < K; base += blockDim.x) {
    int32_t k = base + threadIdx.x;
    int32_t f = (k < K) ? flag[k] : 0;
    int32_t lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int32_t incl = f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int32_t n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane == 31) warp_sums[w] = incl;
    __syncthreads();
    if (w == 0) {
      int32_t v = warp_sums[lane];
      int32_t s = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int32_t n = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += n;
      }
      warp_sums[lane] = s - v;  // exclusive prefix of warp totals
    }
    __syncthreads();
    int32_t excl = carry + warp_sums[w] + incl - f;
    if (f) sel_out[excl] = k;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) warp_sums[0] = excl + f;  // chunk total (with carry)
    __syncthreads();
    carry = warp_sums[0];
    __syncthreads();
  }
}

// ----------------------------------------------------------------------------------------
// K8: trainer fake quantisation, bf16(DQ(Q(w))), one scale per tensor.  Same lane layout as
// the row quantiser over the flat array of all tensors (lane pairs hold the two halves of a
// 16-block).  Each warp takes a contiguous run of 512-element chunks, so it streams sequential
// memory, changes tensor (and recomputes the tensor's scale) rarely, and finds the tensor of a
// chunk by counting instead of dividing; the next chunk's loads are issued before this
// chunk's arithmetic.
// ----------------------------------------------------------------------------------------
struct QdqScale {
  int64_t t;  // tensor whose scale is cached (-1: none)
  float s_g, t6;
};

__device__ __forceinline__ void qdq_scale_for(QdqScale& c, int64_t t, const float* __restrict__ partial, int P,
                                              int32_t* status) {
  if (t == c.t) return;
  float am = 0.0f;
  for (int i = 0; i < P; ++i) am = fmaxf(am, __ldg(partial + t * P + i));
  c.s_g = scale_from_amax(am, status);
  c.t6 = __fmul_rn(6.0f, c.s_g);
  c.t = t;
}

__device__ __forceinline__ void qdq_half(const uint4 q, float s_g, float t6, uint4& o) {
  // the block's max |w| from the bf16 patterns (non-negative bf16 values order as their bits),
  // over this lane's 8 elements, then with the lane holding the other half of the block
  uint32_t m = __vmaxu2(__vmaxu2(q.x & 0x7FFF7FFFu, q.y & 0x7FFF7FFFu), __vmaxu2(q.z & 0x7FFF7FFFu, q.w & 0x7FFF7FFFu));
  m = max(m >> 16, m & 0xFFFFu);
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
  float x[8];
  unpack8(q, x);
  const BlockScale b = block_scale(__uint_as_float(m << 16), s_g, t6);
  float dq[8];
  quant8(x, b, dq);
  uint32_t r[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    __nv_bfloat162 p = __floats2bfloat162_rn(dq[2 * j], dq[2 * j + 1]);
    r[j] = *reinterpret_cast<uint32_t*>(&p);
  }
  o = make_uint4(r[0], r[1], r[2], r[3]);
}

__global__ void __launch_bounds__(256) qdq_kernel(const uint16_t* __restrict__ w, int64_t n_tensors, int64_t elems,
                                                  uint16_t* __restrict__ out, const float* __restrict__ partial, int P,
                                                  float* s_g_out, int32_t* status) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t total = n_tensors * elems;
  const int64_t nchunks = (total + 511) / 512;
  const int64_t c_begin = nchunks * warp_global / nwarps, c_end = nchunks * (warp_global + 1) / nwarps;
  if (c_begin >= c_end) return;
  // tensor of each lane's two half-blocks (lane pairs agree: elems % 16 == 0), kept by counting
  int64_t e0 = c_begin * 512 + 8 * lane, e1 = e0 + 256;
  int64_t t0 = min(e0 / elems, n_tensors - 1), t1 = min(e1 / elems, n_tensors - 1);  // once per warp
  int64_t b0 = t0 * elems, b1 = t1 * elems;        // first element of each lane's current tensor
  QdqScale sc0{-1, 0.f, 0.f}, sc1{-1, 0.f, 0.f};
  uint4 n0 = e0 < total ? __ldg(reinterpret_cast<const uint4*>(w + e0)) : make_uint4(0, 0, 0, 0);
  uint4 n1 = e1 < total ? __ldg(reinterpret_cast<const uint4*>(w + e1)) : make_uint4(0, 0, 0, 0);
  for (int64_t ch = c_begin; ch < c_end; ++ch) {
    const uint4 q0 = n0, q1 = n1;
    const bool h0 = e0 < total, h1 = e1 < total;
    if (ch + 1 < c_end) {
      n0 = e0 + 512 < total ? __ldg(reinterpret_cast<const uint4*>(w + e0 + 512)) : make_uint4(0, 0, 0, 0);
      n1 = e1 + 512 < total ? __ldg(reinterpret_cast<const uint4*>(w + e1 + 512)) : make_uint4(0, 0, 0, 0);
    }
    while (t0 + 1 < n_tensors && e0 >= b0 + elems) { ++t0; b0 += elems; }
    while (t1 + 1 < n_tensors && e1 >= b1 + elems) { ++t1; b1 += elems; }
    qdq_scale_for(sc0, t0, partial, P, status);
    qdq_scale_for(sc1, t1, partial, P, status);
    if (s_g_out) {
      if (h0 && e0 == b0) s_g_out[t0] = sc0.s_g;
      if (h1 && e1 == b1) s_g_out[t1] = sc1.s_g;
    }
    uint4 o0, o1;
    qdq_half(q0, sc0.s_g, sc0.t6, o0);
    qdq_half(q1, sc1.s_g, sc1.t6, o1);
    if (h0) *reinterpret_cast<uint4*>(out + e0) = o0;
    if (h1) *reinterpret_cast<uint4*>(out + e1) = o1;
    e0 += 512;
    e1 += 512;
  }
}

// ----------------------------------------------------------------------------------------
// K8 in one pass over HBM: groups of GS co-resident CTAs (a cooperative launch) take tensors
// group, group + n_groups, ...  A CTA reduces max|w| over its slice of a tensor, folds it into
// the tensor's word of the workspace and counts itself in; once all GS are in (a bounded wait on
// the counter) it reads the tensor scale and fake-quantises its slice, reading it a second time,
// now from L2.  The wait on tensor t comes after the amax pass over the group's next tensor, so
// the meeting is hidden behind HBM reads; two tensors per group are in flight, which the host
// keeps well inside L2.  HBM sees each weight read once and written once: 4 bytes per element.
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ uint64_t l2_policy_keep() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_stream() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint4 ld_hint(const uint16_t* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}
__device__ __forceinline__ void st_hint(uint16_t* p, const uint4 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w), "l"(pol)
               : "memory");
}

// |w| of two bf16 as their bit patterns (non-negative bf16 values order as their bits), a NaN as
// 0 (a binary32 max ignores it); flags collects the halves that are infinite or NaN
__device__ __forceinline__ uint32_t bf16x2_abs_bits(uint32_t w, uint32_t& flags) {
  const uint32_t v = w & 0x7FFF7FFFu;
  flags |= __vcmpgeu2(v, 0x7F807F80u);
  return v & ~__vcmpgtu2(v, 0x7F807F80u);
}

// max |w| over elements [v_lo*8, v_hi*8) of one tensor, four 16-byte loads in flight per thread;
// the maximum is taken on the bf16 bit patterns, two per instruction
__device__ __forceinline__ float slice_amax(const uint16_t* wt, int64_t v_lo, int64_t v_hi, uint64_t pol,
                                            bool& nonfinite) {
  uint32_t m = 0, flags = 0;
  const int64_t stride = blockDim.x;
  for (int64_t i0 = v_lo + threadIdx.x; i0 < v_hi; i0 += 4 * stride) {
    uint4 q[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      q[u] = (i0 + u * stride < v_hi) ? ld_hint(wt + 8 * (i0 + u * stride), pol) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      m = __vmaxu2(m, __vmaxu2(bf16x2_abs_bits(q[u].x, flags), bf16x2_abs_bits(q[u].y, flags)));
      m = __vmaxu2(m, __vmaxu2(bf16x2_abs_bits(q[u].z, flags), bf16x2_abs_bits(q[u].w, flags)));
    }
  }
  nonfinite |= flags != 0;
  return __uint_as_float(max(m >> 16, m & 0xFFFFu) << 16);
}

// qdq_half with (d, 1/d) looked up per scale code in a table made for the tensor's scale
__device__ __forceinline__ void qdq_half_tab(const uint4 q, float s_g, float t6, const float2* tab, uint4& o) {
  uint32_t m = __vmaxu2(__vmaxu2(q.x & 0x7FFF7FFFu, q.y & 0x7FFF7FFFu), __vmaxu2(q.z & 0x7FFF7FFFu, q.w & 0x7FFF7FFFu));
  m = max(m >> 16, m & 0xFFFFu);
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
  float x[8];
  unpack8(q, x);
  BlockScale b;
  b.S = s_g > 0.0f ? e4m3_encode(__fdiv_rn(__uint_as_float(m << 16), t6)) : 0u;
  const float2 di = tab[b.S];
  b.d = di.x;
  b.inv = di.y;
  float dq[8];
  quant8(x, b, dq);
  uint32_t r[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    __nv_bfloat162 p = __floats2bfloat162_rn(dq[2 * j], dq[2 * j + 1]);
    r[j] = *reinterpret_cast<uint32_t*>(&p);
  }
  o = make_uint4(r[0], r[1], r[2], r[3]);
}

__global__ void __launch_bounds__(256, 4) qdq_fused_kernel(const uint16_t* __restrict__ w, int64_t n_tensors,
                                                           int64_t elems, uint16_t* __restrict__ out,
                                                           uint32_t* __restrict__ sync_ws, int GS, float* s_g_out,
                                                           int32_t* status, uint64_t limit_ns) {
  __shared__ float red[8];
  __shared__ float sg_sh;
  __shared__ int bad_sh;
  __shared__ float2 tab[128];  // (d, 1/d) of the 128 E4M3 codes for the current tensor's scale
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (int)(blockDim.x >> 5);
  const int n_groups = (int)(gridDim.x / GS);
  const int group = (int)(blockIdx.x / GS), rank = (int)(blockIdx.x % GS);
  if (group >= n_groups) return;  // a CTA beyond the last whole group has no tensor
  const int64_t chunks = (elems + 511) / 512;  // 512-element chunks (one warp step of the fake-quant)
  const int64_t c_lo = chunks * rank / GS, c_hi = chunks * (rank + 1) / GS;
  const int64_t v_lo = c_lo * 64, v_hi = min(c_hi * 64, elems / 8);
  const uint64_t keep = l2_policy_keep(), stream = l2_policy_stream();
  bool nonfinite = false;

  // amax pass over tensor t, then this CTA's arrival at the tensor's counter
  auto amax_and_arrive = [&](int64_t t) {
    float m = warp_max(slice_amax(w + t * elems, v_lo, v_hi, keep, nonfinite));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
      float mm = 0.0f;
      for (int i = 0; i < nw; ++i) mm = fmaxf(mm, red[i]);
      atomicMax(sync_ws + 2 * t, __float_as_uint(mm));  // non-negative floats order as their bits
      __threadfence();
      atomicAdd(sync_ws + 2 * t + 1, 1u);
    }
  };

  int64_t t = group;
  if (t < n_tensors) amax_and_arrive(t);
  for (; t < n_tensors; t += n_groups) {
    if (t + n_groups < n_tensors) amax_and_arrive(t + n_groups);
    if (threadIdx.x == 0) {
      const uint32_t* count = sync_ws + 2 * t + 1;
      bool ok = false;
      const uint64_t t0 = globaltimer_ns();
      while (true) {
        uint32_t c;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(c) : "l"(count) : "memory");
        if (c >= (uint32_t)GS) {
          ok = true;
          break;
        }
        if (globaltimer_ns() - t0 > limit_ns) break;
        __nanosleep(100);
      }
      if (!ok) report_status(status, kErrTimeout);
      uint32_t am;
      asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(am) : "l"(sync_ws + 2 * t) : "memory");
      const float s_g = scale_from_amax(__uint_as_float(am), status);
      if (ok && rank == 0 && s_g_out) s_g_out[t] = s_g;
      sg_sh = s_g;
      bad_sh = ok ? 0 : 1;
    }
    __syncthreads();
    if (bad_sh) break;
    const float s_g = sg_sh, t6 = __fmul_rn(6.0f, s_g);
    if (threadIdx.x < 128) {
      const uint32_t S = threadIdx.x;
      const float d = __fmul_rn(e4m3_decode(S), s_g);
      tab[S] = make_float2(d, (S != 0 && S < 0x7F) ? __frcp_rn(d) : 0.0f);
    }
    __syncthreads();
    // the fake-quant of this CTA's chunks, one warp per 512-element chunk (lane pairs hold the two
    // halves of a 16-block), the next chunk's loads issued before this one's arithmetic
    const uint16_t* wt = w + t * elems;
    uint16_t* ot = out + t * elems;
    int64_t ch = c_lo + warp;
    int64_t e0 = ch * 512 + 8 * lane, e1 = e0 + 256;
    uint4 n0 = (ch < c_hi && e0 < elems) ? ld_hint(wt + e0, stream) : make_uint4(0, 0, 0, 0);
    uint4 n1 = (ch < c_hi && e1 < elems) ? ld_hint(wt + e1, stream) : make_uint4(0, 0, 0, 0);
    for (; ch < c_hi; ch += nw) {
      const uint4 q0 = n0, q1 = n1;
      const int64_t f0 = e0, f1 = e1;
      e0 += 512 * nw;
      e1 += 512 * nw;
      if (ch + nw < c_hi) {
        n0 = e0 < elems ? ld_hint(wt + e0, stream) : make_uint4(0, 0, 0, 0);
        n1 = e1 < elems ? ld_hint(wt + e1, stream) : make_uint4(0, 0, 0, 0);
      }
      uint4 o0, o1;
      qdq_half_tab(q0, s_g, t6, tab, o0);
      qdq_half_tab(q1, s_g, t6, tab, o1);
      if (f0 < elems) st_hint(ot + f0, o0, stream);
      if (f1 < elems) st_hint(ot + f1, o1, stream);
    }
  }
  if (nonfinite) report_status(status, kErrRange);
}

// ----------------------------------------------------------------------------------------
// logical view of a packed matrix: one code per byte, scales row-major [rows x cols/16]
// ----------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) unpack_logical_kernel(const uint8_t* __restrict__ codes,
                                                             const uint8_t* __restrict__ sf, int64_t rows,
                                                             int64_t cols, int slab16, uint8_t* __restrict__ codes_out,
                                                             uint8_t* __restrict__ sf_out) {
  const int64_t nblk = cols / 16;
  const int64_t k64 = cols / 64;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows * nblk;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / nblk, kb = i - r * nblk;
    if (codes_out) {
      const uint2 c = *reinterpret_cast<const uint2*>(codes + r * (cols / 2) + kb * 8);
      const uint32_t w[2] = {c.x, c.y};
      uint32_t o[4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // bytes of 4 nibble pairs -> 8 bytes: low nibble first
        const uint32_t lo = w[h] & 0x0F0F0F0Fu, hi = (w[h] >> 4) & 0x0F0F0F0Fu;
        o[2 * h] = __byte_perm(lo, hi, 0x5140);
        o[2 * h + 1] = __byte_perm(lo, hi, 0x7362);
      }
      *reinterpret_cast<uint4*>(codes_out + r * cols + kb * 16) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (sf_out) sf_out[r * nblk + kb] = sf[sf_offset_any(r, kb, k64, slab16 != 0)];
  }
}

// ----------------------------------------------------------------------------------------
// trainer fake-quant backward (straight-through): grad_w = grad_fq, grad_acc += grad_fq
// ----------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) qdq_backward_kernel(const uint16_t* __restrict__ g, int64_t n,
                                                           uint16_t* __restrict__ gw, float* __restrict__ acc) {
  const int64_t n8 = n / 8;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(g) + i);
    if (gw) reinterpret_cast<uint4*>(gw)[i] = v;
    if (acc) {
      float x[8];
      unpack8(v, x);
      float4* a = reinterpret_cast<float4*>(acc) + 2 * i;
      const float4 a0 = a[0], a1 = a[1];
      a[0] = make_float4(__fadd_rn(a0.x, x[0]), __fadd_rn(a0.y, x[1]), __fadd_rn(a0.z, x[2]), __fadd_rn(a0.w, x[3]));
      a[1] = make_float4(__fadd_rn(a1.x, x[4]), __fadd_rn(a1.y, x[5]), __fadd_rn(a1.z, x[6]), __fadd_rn(a1.w, x[7]));
    }
  }
  // the tail (n % 8 elements), one thread each
  const int64_t t = n8 * 8 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t < n) {
    if (gw) gw[t] = g[t];
    if (acc) acc[t] = __fadd_rn(acc[t], bf16_bits_to_f32(g[t]));
  }
}

// ----------------------------------------------------------------------------------------
// codec test kernels
// ----------------------------------------------------------------------------------------
__global__ void encode_e2m1_kernel(const float* v, int64_t n, uint8_t* out) {
  int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (i >= n) return;
  float x[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) x[j] = (i + j < n) ? v[i + j] : 0.0f;
  uint32_t c = e2m1_encode8(x);
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (i + j < n) out[i + j] = (c >> (4 * j)) & 0xF;
}

__global__ void encode_e4m3_kernel(const float* v, int64_t n, uint8_t* out) {
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = (uint8_t)e4m3_encode(v[i]);
}

// ----------------------------------------------------------------------------------------
// host launchers
// ----------------------------------------------------------------------------------------
cudaError_t launch_amax(const uint16_t* x, int64_t segs, int64_t seg_rows, int64_t cols, int64_t ld, float* partial,
                        int P, int32_t* status, cudaStream_t st) {
  dim3 grid(P, (unsigned)segs);
  amax_kernel<<<grid, 256, 0, st>>>(x, seg_rows, cols, ld, partial, status);
  return cudaGetLastError();
}

cudaError_t launch_reduce_amax(const float* partial, int P, float* out, cudaStream_t st) {
  reduce_amax_kernel<<<1, 32, 0, st>>>(partial, P, out);
  return cudaGetLastError();
}

size_t rows_smem_bytes(int64_t K, int32_t Kp, int warps, bool masked) {
  if (Kp <= 0) return 16;
  if (masked) return (size_t)((K + 31) / 32) * 4;
  return (size_t)((Kp * 2 + 15) / 16) * 16 + (size_t)warps * (size_t)(K / 16) * 8;
}

cudaError_t launch_rows(const RowArgs& a, int num_sms, cudaStream_t st) {
  int warps = 8;
  const int64_t rows = a.row_scatter ? a.src_rows : a.rows_out;
  // few activation rows: one CTA of 8 warps per row (SPLIT), so that every warp of the grid
  // has work; otherwise one warp per row with as many warps per CTA as the stashes allow
  const bool split = a.mode == kModeAct && rows * 2 < (int64_t)num_sms * warps;
  const bool masked = a.mode == kModeAct && a.masked_res != 0;
  size_t smem = rows_smem_bytes(a.K, a.Kp, split ? 1 : warps, masked);
  while (!split && smem > 200 * 1024 && warps > 1) {
    warps /= 2;
    smem = rows_smem_bytes(a.K, a.Kp, warps, masked);
  }
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  int64_t ctas_needed = split ? rows : (rows + warps - 1) / warps;
  int per_sm = (int)((220 * 1024) / (smem + 1024));
  if (per_sm < 1) per_sm = 1;
  if (per_sm > 8) per_sm = 8;
  int64_t grid = (int64_t)num_sms * per_sm;
  if (grid > ctas_needed) grid = ctas_needed;
  if (grid < 1) grid = 1;
  cudaError_t e = cudaSuccess;
  switch (a.mode) {
    case kModeAct:
      if (split) {
        e = cudaFuncSetAttribute(quant_rows_kernel<kModeAct, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e == cudaSuccess) quant_rows_kernel<kModeAct, true><<<(unsigned)grid, warps * 32, smem, st>>>(a);
      } else {
        e = cudaFuncSetAttribute(quant_rows_kernel<kModeAct, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e == cudaSuccess) quant_rows_kernel<kModeAct, false><<<(unsigned)grid, warps * 32, smem, st>>>(a);
      }
      break;
    case kModePack:
      e = cudaFuncSetAttribute(quant_rows_kernel<kModePack, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
      if (e == cudaSuccess) quant_rows_kernel<kModePack, false><<<(unsigned)grid, warps * 32, smem, st>>>(a);
      break;
    case kModeCal:
      e = cudaFuncSetAttribute(quant_rows_kernel<kModeCal, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
      if (e == cudaSuccess) quant_rows_kernel<kModeCal, false><<<(unsigned)grid, warps * 32, smem, st>>>(a);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_chan_err(const float* resid, int64_t T, int64_t K, const int32_t* off, int32_t groups,
                            double* err, int32_t* status, cudaStream_t st) {
  const dim3 grid((unsigned)((K + 255) / 256), (unsigned)(off ? groups : 1));
  chan_err_kernel<<<grid, 256, 0, st>>>(resid, T, K, off, err, status);
  return cudaGetLastError();
}

cudaError_t launch_select(const double* err, int32_t K, int32_t Kp, int32_t groups, int32_t* sel, double* err_out,
                          cudaStream_t st) {
  size_t smem = (size_t)K * 8 + (size_t)K * 4;
  cudaError_t e = cudaFuncSetAttribute(select_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  select_topk_kernel<<<(unsigned)groups, 1024, smem, st>>>(err, K, Kp, sel, err_out);
  return cudaGetLastError();
}

cudaError_t launch_qdq(const uint16_t* w, int64_t n_tensors, int64_t elems, uint16_t* out, const float* partial, int P,
                       float* s_g_out, int32_t* status, int num_sms, cudaStream_t st) {
  int64_t total = n_tensors * elems;
  int64_t warps_needed = (total + 511) / 512;
  int64_t grid = (warps_needed + 7) / 8;
  int64_t cap = (int64_t)num_sms * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  qdq_kernel<<<(unsigned)grid, 256, 0, st>>>(w, n_tensors, elems, out, partial, P, s_g_out, status);
  return cudaGetLastError();
}

cudaError_t launch_unpack_logical(const uint8_t* codes, const uint8_t* sf, int64_t rows, int64_t cols, int slab16,
                                  uint8_t* codes_out, uint8_t* sf_out, int num_sms, cudaStream_t st) {
  const int64_t work = rows * (cols / 16);
  int64_t grid = (work + 255) / 256;
  if (grid > (int64_t)num_sms * 16) grid = (int64_t)num_sms * 16;
  if (grid < 1) grid = 1;
  unpack_logical_kernel<<<(unsigned)grid, 256, 0, st>>>(codes, sf, rows, cols, slab16, codes_out, sf_out);
  return cudaGetLastError();
}

// CTAs per group for the one-pass fake-quant on `grid` co-resident CTAs: the fewest slice-steps
// per CTA (rounds of tensors x 512-element chunks per slice) while the two tensors per group in
// flight stay within 128 MB (about the L2); ties go to the smaller group (fewer CTAs meet per
// tensor).  Measured on 1024 tensors of 2M elements: 16 groups of 37 CTAs 2.09 ms, 8 of 74
// 2.21 ms, 4 of 147 2.41 ms (the meetings of larger groups wait on more CTAs).
int qdq_fused_group(int64_t n_tensors, int64_t elems, int grid) {
  const int64_t chunks = (elems + 511) / 512;
  const double budget = 128.0 * (1 << 20);
  int best = 0;
  int64_t best_cost = INT64_MAX;
  for (int gs = 1; gs <= grid; ++gs) {
    const int64_t ng = grid / gs;
    if ((double)std::min<int64_t>(ng, n_tensors) * 2.0 * (double)elems * 2.0 > budget) continue;
    const int64_t cost = ((n_tensors + ng - 1) / ng) * ((chunks + gs - 1) / gs);
    if (cost < best_cost) {
      best_cost = cost;
      best = gs;
    }
  }
  return best;
}

// Grid of the fused fake-quant: co-resident CTAs (occupancy x SMs, at most 4 per SM) in whole
// groups of GS CTAs (GS <= 0: chosen by qdq_fused_group).
cudaError_t launch_qdq_fused(const uint16_t* w, int64_t n_tensors, int64_t elems, uint16_t* out, uint32_t* sync_ws,
                             int GS, float* s_g_out, int32_t* status, uint64_t limit_ns, int num_sms,
                             cudaStream_t st) {
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, qdq_fused_kernel, 256, 0);
  if (e != cudaSuccess) return e;
  if (per_sm > 4) per_sm = 4;
  const int grid_max = num_sms * per_sm;
  if (GS <= 0) GS = qdq_fused_group(n_tensors, elems, grid_max);
  if (GS <= 0 || GS > grid_max) return cudaErrorInvalidValue;
  int grid = grid_max / GS * GS;
  void* args[] = {(void*)&w, (void*)&n_tensors, (void*)&elems, (void*)&out, (void*)&sync_ws, (void*)&GS,
                  (void*)&s_g_out, (void*)&status, (void*)&limit_ns};
  e = cudaLaunchCooperativeKernel((const void*)qdq_fused_kernel, dim3((unsigned)grid), dim3(256), args, 0, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_qdq_backward(const uint16_t* g, int64_t n, uint16_t* gw, float* acc, int num_sms, cudaStream_t st) {
  int64_t grid = (n / 8 + 255) / 256;
  if (grid > (int64_t)num_sms * 8) grid = (int64_t)num_sms * 8;
  if (grid < 1) grid = 1;
  qdq_backward_kernel<<<(unsigned)grid, 256, 0, st>>>(g, n, gw, acc);
  return cudaGetLastError();
}

cudaError_t launch_encode_e2m1(const float* v, int64_t n, uint8_t* out, cudaStream_t st) {
  int64_t threads = (n + 7) / 8;
  encode_e2m1_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(v, n, out);
  return cudaGetLastError();
}

cudaError_t launch_encode_e4m3(const float* v, int64_t n, uint8_t* out, cudaStream_t st) {
  encode_e4m3_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(v, n, out);
  return cudaGetLastError();
}

}  // namespace nvfp4
