// The MoE block around the expert GEMMs, on the device: router top-k, the expert-grouped
// dispatch layout of the (token, expert) pairs, and the weighted combine of expert outputs.
//
// Readings (the pages fix none of this): the top-k of softmax(logits) are the k largest logits,
// ties to the lower expert; a chosen expert's weight is its probability renormalised over the
// k chosen, exp(l_j - l_max) / sum_i exp(l_i - l_max); pairs are grouped by expert with tokens
// ascending, each expert segment padded to a multiple of `pad` rows; out[t] = sum_j w_tj y_row(t,j).
#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {

// ----------------------------------------------------------------------------------------
// router: one warp per token; lane l holds logits l, l + 32, ...; k rounds of a warp arg-max
// ordered by (value descending, expert ascending)
// ----------------------------------------------------------------------------------------

// V = logits per lane (E <= 32 V): the scan loops are compiled for the expert count's bracket.
template <int V>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits, int64_t T, int E, int k,
                                                         int32_t* __restrict__ ids, float* __restrict__ w,
                                                         int32_t* status) {
  const int lane = threadIdx.x & 31;
  const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  float v[V];
  bool bad = false;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? __ldg(logits + t * E + e) : -INFINITY;
    if (e < E && !(fabsf(v[i]) <= 3.4e38f)) bad = true;
  }
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0) report_status(status, kErrRange);
    return;
  }
  float lmax = 0.0f, sum = 0.0f;
  float chosen_v = 0.0f;  // lane j keeps the value of the j-th choice
  int chosen_e = 0;
  for (int j = 0; j < k; ++j) {
    // local best: the first maximum over this lane's experts (ascending); experts already
    // chosen hold -inf and lose to every finite logit
    float bv = -INFINITY;
    int be = 0x7FFFFFFF;
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const int e = lane + 32 * i;
      if (e < E && (be == 0x7FFFFFFF || v[i] > bv)) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    // every lane now holds the winner; its owner takes it out of the running
    if ((be & 31) == lane) {
#pragma unroll
      for (int i = 0; i < V; ++i)
        if (lane + 32 * i == be) v[i] = -INFINITY;
    }
    if (j == 0) lmax = bv;
    const float p = expf(__fsub_rn(bv, lmax));
    sum = __fadd_rn(sum, p);
    if (lane == j) {
      chosen_v = p;
      chosen_e = be;
    }
  }
  if (lane < k) {
    ids[t * k + lane] = chosen_e;
    w[t * k + lane] = __fdiv_rn(chosen_v, sum);
  }
}

// ----------------------------------------------------------------------------------------
// dispatch plan
// ----------------------------------------------------------------------------------------
__global__ void count_kernel(const int32_t* __restrict__ ids, int64_t n, int E, int32_t* __restrict__ counts,
                             int32_t* status) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int e = __ldg(ids + i);
    if (e < 0 || e >= E) {
      report_status(status, kErrInvalid);
      continue;
    }
    atomicAdd(counts + e, 1);
  }
}

// the same counts through a per-CTA histogram in shared memory (E <= kCountSmemExperts): one
// global atomic per CTA and expert instead of one per pair
constexpr int kCountSmemExperts = 8192;
__global__ void __launch_bounds__(1024) count_smem_kernel(const int32_t* __restrict__ ids, int64_t n, int E,
                                                          int32_t* __restrict__ counts, int32_t* status) {
  extern __shared__ int hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  bool bad = false;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int e = __ldg(ids + i);
    if (e < 0 || e >= E) {
      bad = true;
      continue;
    }
    atomicAdd(hist + e, 1);
  }
  if (bad) report_status(status, kErrInvalid);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (hist[e] != 0) atomicAdd(counts + e, hist[e]);
}

// one CTA: padded segment starts (exclusive scan), then the decode slot tables
__global__ void __launch_bounds__(1024) offsets_kernel(const int32_t* __restrict__ counts, int E, int pad,
                                                       int64_t rows_capacity, int32_t* __restrict__ offsets,
                                                       int32_t* expert_rows, int32_t* slot_expert,
                                                       int32_t* slot_count, int n_slots, int32_t* status) {
  __shared__ int64_t part[1024];
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = threadIdx.x * per;
  int64_t mine = 0;
  for (int e = e0; e < min(E, e0 + per); ++e) mine += (int64_t)(counts[e] + pad - 1) / pad * pad;
  part[threadIdx.x] = mine;
  __syncthreads();
  // inclusive scan over the threads' sums (Hillis-Steele)
  for (int o = 1; o < (int)blockDim.x; o <<= 1) {
    const int64_t add = threadIdx.x >= (unsigned)o ? part[threadIdx.x - o] : 0;
    __syncthreads();
    part[threadIdx.x] += add;
    __syncthreads();
  }
  int64_t run = part[threadIdx.x] - mine;
  const int64_t total = part[blockDim.x - 1];
  const bool fits = total <= rows_capacity && (slot_expert == nullptr || total / 16 <= n_slots);
  if (!fits && threadIdx.x == 0) report_status(status, kErrInvalid);
  for (int e = e0; e < min(E, e0 + per); ++e) {
    offsets[e] = fits ? (int32_t)run : 0;
    const int c = counts[e];
    if (expert_rows != nullptr) expert_rows[e] = fits ? c : 0;
    if (slot_expert != nullptr && fits) {
      const int s0 = (int)(run / 16);
      for (int s = 0; 16 * s < c; ++s) {
        slot_expert[s0 + s] = e;
        slot_count[s0 + s] = min(16, c - 16 * s);
      }
    }
    run += (int64_t)(c + pad - 1) / pad * pad;
  }
  // an unusable plan is marked by offsets[E] = -1: no pair gets a row, the GEMMs do nothing
  if (threadIdx.x == 0) offsets[E] = fits ? (int32_t)total : -1;
  if (slot_expert != nullptr) {
    const int used = fits ? (int)(total / 16) : 0;
    for (int s = used + threadIdx.x; s < n_slots; s += blockDim.x) {
      slot_expert[s] = -1;  // unused slot: the decode GEMM skips it
      slot_count[s] = 0;
    }
  }
}

// one CTA per expert: the rank of each of its tokens (ascending) -> row of the pair.  Thread i
// takes kRankTpt consecutive tokens of a chunk of kRankThreads * kRankTpt; the CTA's exclusive
// scan of the per-thread hit counts gives each hit its rank within the chunk.
constexpr int kRankThreads = 1024;
constexpr int kRankTpt = 4;
__global__ void __launch_bounds__(kRankThreads) rank_kernel(const int32_t* __restrict__ ids, int64_t T, int k,
                                                            const int32_t* __restrict__ offsets, int E,
                                                            int32_t* __restrict__ row_scatter) {
  __shared__ int warp_sum[kRankThreads / 32];
  __shared__ int chunk_total;
  const int e = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (offsets[E] < 0) return;  // unusable plan (reported): every pair stays unrouted (-1)
  int64_t run = offsets[e];
  const bool vec = (reinterpret_cast<uintptr_t>(ids) & 15u) == 0;
  static_assert(kRankTpt == 4, "four tokens per thread: 16-byte groups of ids and one byte of `hits` each");
  for (int64_t base = 0; base < T; base += (int64_t)kRankThreads * kRankTpt) {
    const int64_t t0 = base + (int64_t)threadIdx.x * kRankTpt;
    // byte i of `hits`: 0x80 | slot j for token t0 + i when ids[t0 + i][j] == e (a token's experts
    // are distinct), else 0.  The thread's kRankTpt * k ids are contiguous: with 16-byte aligned
    // ids they come in k 16-byte loads, eight in flight at a time.
    uint32_t hits = 0;
    if (vec && t0 + kRankTpt <= T) {
      const int4* src = reinterpret_cast<const int4*>(ids + t0 * k);
      for (int v0 = 0; v0 < k; v0 += 8) {
        int4 q[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (v0 + u < k) q[u] = __ldg(src + v0 + u);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (v0 + u >= k) break;
          const int w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
          for (int c = 0; c < 4; ++c)
            if (w[c] == e) {
              const int idx = 4 * (v0 + u) + c, tok = idx / k;
              hits |= (uint32_t)(0x80 | (idx - tok * k)) << (8 * tok);
            }
        }
      }
    } else {
      for (int i = 0; i < kRankTpt; ++i)
        if (t0 + i < T)
          for (int j = 0; j < k; ++j)
            if (__ldg(ids + (t0 + i) * k + j) == e) hits |= (uint32_t)(0x80 | j) << (8 * i);
    }
    const int mine = __popc(hits & 0x80808080u);
    // exclusive scan of `mine` over the CTA: in the warp by shuffles, then over the warps
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int up = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += up;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int ws = warp_sum[lane];
      int wi = ws;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int up = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += up;
      }
      warp_sum[lane] = wi - ws;  // exclusive prefix of the warps
      if (lane == 31) chunk_total = wi;
    }
    __syncthreads();
    int64_t r = run + warp_sum[warp] + (incl - mine);
#pragma unroll
    for (int i = 0; i < kRankTpt; ++i) {
      const uint32_t h = (hits >> (8 * i)) & 0xFFu;
      if (h & 0x80u) row_scatter[(t0 + i) * k + (int)(h & 0x7Fu)] = (int32_t)(r++);
    }
    run += chunk_total;
    __syncthreads();  // warp_sum and chunk_total are rewritten by the next chunk
  }
}

// ----------------------------------------------------------------------------------------
// combine: thread = 8 consecutive features of one token; binary32 accumulation in j order
// ----------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ y, int64_t ldy, int64_t y_rows,
                                                      const int32_t* __restrict__ rows, const float* __restrict__ w,
                                                      int64_t T, int k, int64_t H, uint16_t* __restrict__ out,
                                                      int64_t ldo, int32_t* status) {
  const int64_t per_tok = H / 8;
  const int64_t n = T * per_tok;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / per_tok;
    const int64_t h = (i - t * per_tok) * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
      const int32_t r = __ldg(rows + t * k + j);
      if (r < 0) continue;  // an unrouted pair contributes nothing
      if (r >= y_rows) {
        report_status(status, kErrInvalid);
        continue;
      }
      const float wj = __ldg(w + t * k + j);
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(y + r * ldy + h));
      const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc[2 * c] = fmaf(wj, bf16_bits_to_f32(u[c] & 0xFFFFu), acc[2 * c]);
        acc[2 * c + 1] = fmaf(wj, bf16_bits_to_f32(u[c] >> 16), acc[2 * c + 1]);
      }
    }
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      __nv_bfloat162 p = __floats2bfloat162_rn(acc[2 * c], acc[2 * c + 1]);
      ow[c] = *reinterpret_cast<uint32_t*>(&p);
    }
    *reinterpret_cast<uint4*>(out + t * ldo + h) = o;
  }
}

// ----------------------------------------------------------------------------------------
// row -> expert of an expert-grouped layout: row r of segment [off[e], off[e+1]) gets e, rows at or
// past off[E] get -1 (padding capacity); off[E] < 0 (a plan that did not fit) gives -1 everywhere.
// Used to pick each row's channel list when the down projection has one list per expert.
// ----------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) row_groups_kernel(const int32_t* __restrict__ off, int E, int64_t rows,
                                                         int32_t* __restrict__ group) {
  const int32_t end = __ldg(off + E);
  for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < rows; r += (int64_t)gridDim.x * blockDim.x) {
    int32_t g = -1;
    if (end >= 0 && r < end && r >= __ldg(off)) {
      // largest e with off[e] <= r (segments are non-decreasing); empty segments are skipped over
      int lo = 0, hi = E - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((int64_t)__ldg(off + mid) <= r) lo = mid;
        else hi = mid - 1;
      }
      g = lo;
    }
    group[r] = g;
  }
}

// ----------------------------------------------------------------------------------------
// inverse of the pair -> row map: row_pair[row_scatter[p]] = p for every routed pair p = t*k + j
// (the caller's memset leaves -1 on the other rows); a row past `rows` is reported
// ----------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) row_pairs_kernel(const int32_t* __restrict__ row_scatter, int64_t n,
                                                        int64_t rows, int32_t* __restrict__ row_pair,
                                                        int32_t* status) {
  for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < n; p += (int64_t)gridDim.x * blockDim.x) {
    const int32_t r = __ldg(row_scatter + p);
    if (r < 0) continue;
    if (r >= rows) {
      report_status(status, kErrInvalid);
      continue;
    }
    row_pair[r] = (int32_t)p;
  }
}

// binary32 combine sums -> bf16 rows (8 features per thread)
__global__ void __launch_bounds__(256) combine_finalize_kernel(const float* __restrict__ acc, int64_t T, int64_t H,
                                                               uint16_t* __restrict__ out, int64_t ldo) {
  const int64_t per_tok = H / 8;
  const int64_t n = T * per_tok;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / per_tok;
    const int64_t h = (i - t * per_tok) * 8;
    const float4 a = __ldg(reinterpret_cast<const float4*>(acc + t * H + h));
    const float4 b = __ldg(reinterpret_cast<const float4*>(acc + t * H + h + 4));
    const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      __nv_bfloat162 p = __floats2bfloat162_rn(v[2 * c], v[2 * c + 1]);
      ow[c] = *reinterpret_cast<uint32_t*>(&p);
    }
    *reinterpret_cast<uint4*>(out + t * ldo + h) = o;
  }
}

// ----------------------------------------------------------------------------------------
// launchers
// ----------------------------------------------------------------------------------------
cudaError_t launch_row_pairs(const int32_t* row_scatter, int64_t n, int64_t rows, int32_t* row_pair, int num_sms,
                             int32_t* status, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(row_pair, 0xFF, sizeof(int32_t) * (size_t)rows, st);  // -1: no pair
  if (e != cudaSuccess || n == 0) return e;
  int64_t blocks = (n + 255) / 256;
  if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
  row_pairs_kernel<<<(unsigned)blocks, 256, 0, st>>>(row_scatter, n, rows, row_pair, status);
  return cudaGetLastError();
}

cudaError_t launch_combine_finalize(const float* acc, int64_t T, int64_t H, uint16_t* out, int64_t ldo, int num_sms,
                                    cudaStream_t st) {
  const int64_t n = T * (H / 8);
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > (int64_t)num_sms * 16) blocks = (int64_t)num_sms * 16;
  combine_finalize_kernel<<<(unsigned)blocks, 256, 0, st>>>(acc, T, H, out, ldo);
  return cudaGetLastError();
}
cudaError_t launch_row_groups(const int32_t* off, int E, int64_t rows, int32_t* group, int num_sms, cudaStream_t st) {
  int64_t blocks = (rows + 255) / 256;
  if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
  if (blocks < 1) blocks = 1;
  row_groups_kernel<<<(unsigned)blocks, 256, 0, st>>>(off, E, rows, group);
  return cudaGetLastError();
}

cudaError_t launch_route_topk(const float* logits, int64_t T, int E, int k, int32_t* ids, float* w, int32_t* status,
                              cudaStream_t st) {
  const unsigned blocks = (unsigned)((T + 7) / 8);
  const int v = (E + 31) / 32;
  if (v <= 1) route_topk_kernel<1><<<blocks, 256, 0, st>>>(logits, T, E, k, ids, w, status);
  else if (v <= 2) route_topk_kernel<2><<<blocks, 256, 0, st>>>(logits, T, E, k, ids, w, status);
  else if (v <= 4) route_topk_kernel<4><<<blocks, 256, 0, st>>>(logits, T, E, k, ids, w, status);
  else if (v <= 8) route_topk_kernel<8><<<blocks, 256, 0, st>>>(logits, T, E, k, ids, w, status);
  else if (v <= 16) route_topk_kernel<16><<<blocks, 256, 0, st>>>(logits, T, E, k, ids, w, status);
  else route_topk_kernel<kMaxRouteExperts / 32><<<blocks, 256, 0, st>>>(logits, T, E, k, ids, w, status);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_plan(const int32_t* ids, int64_t T, int k, int E, int pad, int64_t rows_capacity,
                                 int32_t* counts, int32_t* offsets, int32_t* row_scatter, int32_t* expert_rows,
                                 int32_t* slot_expert, int32_t* slot_count, int n_slots, int num_sms,
                                 int32_t* status, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * (size_t)E, st);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(row_scatter, 0xFF, sizeof(int32_t) * (size_t)(T * k), st);  // -1: unrouted
  if (e != cudaSuccess) return e;
  const int64_t n = T * k;
  if (E <= kCountSmemExperts) {
    // about 4096 pairs per CTA
    int64_t blocks = (n + 4095) / 4096;
    if (blocks > (int64_t)num_sms) blocks = num_sms;
    if (blocks < 1) blocks = 1;
    const size_t smem = sizeof(int) * (size_t)E;
    if (smem > 48 * 1024) {
      e = cudaFuncSetAttribute(count_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    count_smem_kernel<<<(unsigned)blocks, 1024, smem, st>>>(ids, n, E, counts, status);
  } else {
    int64_t blocks = (n + 255) / 256;
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    if (blocks < 1) blocks = 1;
    count_kernel<<<(unsigned)blocks, 256, 0, st>>>(ids, n, E, counts, status);
  }
  offsets_kernel<<<1, 1024, 0, st>>>(counts, E, pad, rows_capacity, offsets, expert_rows, slot_expert, slot_count,
                                     n_slots, status);
  rank_kernel<<<(unsigned)E, kRankThreads, 0, st>>>(ids, T, k, offsets, E, row_scatter);
  return cudaGetLastError();
}

cudaError_t launch_combine(const uint16_t* y, int64_t ldy, int64_t y_rows, const int32_t* rows, const float* w,
                           int64_t T, int k, int64_t H, uint16_t* out, int64_t ldo, int num_sms, int32_t* status,
                           cudaStream_t st) {
  const int64_t n = T * (H / 8);
  int64_t blocks = (n + 255) / 256;
  if (blocks > (int64_t)num_sms * 16) blocks = (int64_t)num_sms * 16;
  if (blocks < 1) blocks = 1;
  combine_kernel<<<(unsigned)blocks, 256, 0, st>>>(y, ldy, y_rows, rows, w, T, k, H, out, ldo, status);
  return cudaGetLastError();
}

}  // namespace nvfp4
