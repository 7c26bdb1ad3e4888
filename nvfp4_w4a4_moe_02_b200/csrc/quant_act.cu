// Online activation quantiser with the RAC residual pass, fed by bulk copies of row tiles.
//
// "Why 4-bit RL rollout collapses - and it isn't the weights", Two fixes, on two different
// sides: the selected channels get "a second, residual FP4 pass"; the QUADS abstract: the
// activations are quantised online, every step.  Per element this is a handful of binary32
// operations on 2 bytes read and ~0.84 bytes written, so the kernel is built to keep HBM busy:
//
//   * one producer warp streams tiles of R source rows (R * K * 2 bytes, up to 16 KB) into a
//     3-stage shared-memory ring with cp.async.bulk, completing on mbarriers, and writes each
//     stage's row metadata (destination rows, byte offsets of codes and scales);
//   * 4 to 8 consumer warps quantise the stage: thread = one 16-element block (its block max,
//     its E4M3 scale by one IEEE division and one reciprocal, eight E2M1 conversions), stores
//     of 8 code bytes per destination row and its scale byte (one destination) or, with several
//     destinations, the scale word of four neighbouring blocks from one lane of the four;
//   * in the same pass each thread writes the block's residual r = x - e*d (binary32) into a
//     shared buffer whose 16-float blocks sit 17 words apart (the consumer warps' stores and
//     the residual pass's gathers then spread over the banks), and after a barrier the
//     residual pass reads the selected channels in ascending order, 16 compact positions per
//     thread, and quantises them with the same tensor scale.
//
// Row maps: plain rows (output row = source row, rows past the valid count are zero), a
// gather list, a scatter list (each source row to up to `fanout` output rows: the MoE
// dispatch), or expert segments (only the token rows of each padded segment).
//
// Every mbarrier wait is bounded; a wait that runs out records NVFP4_ERR_TIMEOUT, all
// consumer warps leave together (barrier with an OR-reduction), and the producer waits
// (bounded) for its own copies before the CTA exits.
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace nvfp4 {
namespace act {

constexpr int kStages = 2;
constexpr int kMaxMeta = 128;              // R * fanout entries of one stage
constexpr int kPitch = 17;                 // words per 16-block in the residual buffer

// shared-memory plan of one launch (host and device agree through these)
struct Plan {
  int R;             // source rows per tile
  int fanout;        // destinations per row (1 unless scatter)
  int mc;            // metadata entries per stage: R * fanout
  int stage_bytes;   // R * K * 2
  int off_stage;     // S stages of rows
  int off_meta;      // S stages of metadata
  int meta_bytes;    // one stage: 4 x mc int64 offsets, R int32 valid flags, the slot count
  int off_rbuf;      // R x (K/16) x 17 floats (residual mode)
  int off_sel;       // Kp uint16 word offsets, transposed [16][Kp/16]
  int off_seg;       // segments mode: n_seg + 1 int32 tile prefix, then each segment's first row and rows
  int off_bar;       // full[S], empty[S]
  int off_misc;      // s_g, t6, n_tiles, abort
  int off_tab;       // float2 [128]: (d, 1/d) per E4M3 code
  int smem;
};

__host__ __device__ inline int round16(int v) { return (v + 15) & ~15; }

__host__ __device__ inline Plan make_plan(int K, int Kp, int fanout, int n_seg, int R) {
  Plan p;
  p.R = R;
  p.fanout = fanout;
  p.mc = R * fanout;
  p.stage_bytes = R * K * 2;
  p.off_stage = 0;
  p.meta_bytes = round16(p.mc * 4 * 8 + R * 4 + 4);
  p.off_meta = p.off_stage + kStages * p.stage_bytes;
  p.off_rbuf = p.off_meta + kStages * p.meta_bytes;
  const int rbuf = Kp > 0 ? R * (K / 16) * kPitch * 4 : 0;
  p.off_sel = p.off_rbuf + round16(rbuf);
  p.off_seg = p.off_sel + round16(Kp * 2);
  p.off_bar = p.off_seg + round16(n_seg > 0 ? (3 * n_seg + 1) * 4 : 0);
  p.off_misc = p.off_bar + 2 * kStages * 8;
  p.off_tab = p.off_misc + 64;     // (d, 1/d) of the 128 E4M3 codes, for s_g and for the residual
  p.smem = p.off_tab + 2 * 128 * 8;
  return p;
}

// metadata of one stage: per (slot, destination) the byte offsets of the code row and of the
// scale-atom row of the main and the residual outputs (code offset -1: no destination), per
// slot whether its source row was loaded (else the row is zero), and the number of slots
struct MetaView {
  int64_t* code;
  int64_t* sfrow;
  int64_t* rcode;
  int64_t* rsfrow;
  int32_t* valid;
  int32_t* n_slots;
  __device__ __forceinline__ MetaView(unsigned char* base, int mc, int R) {
    code = reinterpret_cast<int64_t*>(base);
    sfrow = code + mc;
    rcode = sfrow + mc;
    rsfrow = rcode + mc;
    valid = reinterpret_cast<int32_t*>(rsfrow + mc);
    n_slots = valid + R;
  }
};

__device__ __forceinline__ int64_t sf_row_off(int64_t r, int64_t groups, bool slab16) {
  return slab16 ? (r >> 4) * groups * 512 + (r & 15) * 16
                : (r >> 7) * groups * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4;
}
__device__ __forceinline__ int32_t sf_blk_off(int32_t kb) { return (kb >> 2) * 512 + (kb & 3); }

// barrier of the NC consumer threads with an OR vote, and the plain one
template <int NC>
__device__ __forceinline__ bool consumers_sync_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(NC)
      : "memory");
  return r != 0;
}
template <int NC>
__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 2, %0;" ::"n"(NC) : "memory");
}

// max |x| over 16 bf16 (exact: the maximum of non-negative bf16 patterns compared as integers)
__device__ __forceinline__ float absmax16(const uint4 a, const uint4 b) {
  uint32_t m = __vmaxu2(a.x & 0x7FFF7FFFu, a.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, a.z & 0x7FFF7FFFu);
  m = __vmaxu2(m, a.w & 0x7FFF7FFFu);
  m = __vmaxu2(m, b.x & 0x7FFF7FFFu);
  m = __vmaxu2(m, b.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, b.z & 0x7FFF7FFFu);
  m = __vmaxu2(m, b.w & 0x7FFF7FFFu);
  const uint32_t top = max(m >> 16, m & 0xFFFFu);
  return __uint_as_float(top << 16);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 u, float x[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    x[2 * j] = __uint_as_float(w[j] << 16);
    x[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}

// codes of 8 values under (S, inv): RN(x * inv) converted to E2M1; S == 0 -> all +0
__device__ __forceinline__ uint32_t codes8(const float x[8], const BlockScale& bs) {
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 p = __fmul2_rn(make_float2(x[i], x[i + 1]), make_float2(bs.inv, bs.inv));
    v[i] = p.x;
    v[i + 1] = p.y;
  }
  const uint32_t c = e2m1_encode8(v);
  return bs.S == 0 ? 0u : c;
}

// r = RN(x - RN(e(c) * d)) for 8 values
__device__ __forceinline__ void resid8(const float x[8], uint32_t c, float d, float r[8]) {
  float e[8];
  e2m1_decode8(c, e);
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 dq = __fmul2_rn(make_float2(e[i], e[i + 1]), make_float2(d, d));
    const float2 rr = __fadd2_rn(make_float2(x[i], x[i + 1]), make_float2(-dq.x, -dq.y));
    r[i] = rr.x;
    r[i + 1] = rr.y;
  }
}

// The scale bytes of four neighbouring blocks of one row (lanes 4g .. 4g+3, blocks 4m .. 4m+3)
// form one 32-bit word of each destination's scale row (byte i = block 4m + i); every lane of the
// group gets the whole word.  The four lanes of a group are on the same row and trip count in
// both passes: K and K' are multiples of 64 (blocks per row a multiple of 4) and the consumer count
// a multiple of 32, so lane l's block index within the tile is l mod 4 plus a multiple of 4.
__device__ __forceinline__ uint32_t scale_word4(uint32_t S, int lane) {
  const uint32_t gm = 0xFu << (lane & ~3);
  uint32_t w = S << (8u * (uint32_t)(lane & 3));
  w |= __shfl_xor_sync(gm, w, 1);
  w |= __shfl_xor_sync(gm, w, 2);
  return w;
}

// W consumer warps (4..8, chosen per shape so that both passes divide evenly) + 1 producer warp
// The block scale with (d, 1/d) looked up per E4M3 code: for a fixed tensor scale s_g the 127
// codes give 127 (d, 1/d) pairs, computed once per CTA with the same operations as block_scale.
__device__ __forceinline__ BlockScale block_scale_tab(float b, float s_g, float t6, const float2* tab) {
  BlockScale bs;
  bs.S = s_g > 0.0f ? e4m3_encode(__fdiv_rn(b, t6)) : 0u;
  const float2 di = tab[bs.S];
  bs.d = di.x;
  bs.inv = di.y;
  return bs;
}

template <bool RES, int W>
__global__ void __launch_bounds__(32 * W + 32) act_quant_kernel(const ActArgs a) {
  constexpr int kConsumerWarps = W;
  constexpr int kConsumers = 32 * W;
  extern __shared__ __align__(128) unsigned char smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int K = a.K, Kp = a.Kp;
  const int KB = K / 16, QB = Kp / 16;
  const Plan p = make_plan(K, Kp, a.fanout, a.map == kMapSegments ? a.n_seg : 0, a.R);
  const uint32_t sb = tc::smem_u32(smem);
  auto bar_full = [&](int s) { return sb + (uint32_t)p.off_bar + 8u * s; };
  auto bar_empty = [&](int s) { return sb + (uint32_t)p.off_bar + 8u * (kStages + s); };
  float* misc_f = reinterpret_cast<float*>(smem + p.off_misc);
  int32_t* misc_i = reinterpret_cast<int32_t*>(smem + p.off_misc);
  // misc: [0] s_g, [1] t6, [2] n_tiles, [3] abort
  volatile int32_t* abort_flag = misc_i + 3;
  int32_t* seg_prefix = reinterpret_cast<int32_t*>(smem + p.off_seg);
  uint16_t* sel_off = reinterpret_cast<uint16_t*>(smem + p.off_sel);
  const bool slab16 = a.sf_slab16 != 0;
  const int64_t k64 = K / 64, kp64 = Kp / 64;
  const int R = p.R;

  // ---------------------------------------------------------------- set-up (all threads)
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(bar_full(s), 1);
      tc::mbar_init(bar_empty(s), kConsumerWarps);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (RES) {
    // channel list -> word offsets of the channels in the residual buffer's row, transposed so
    // that position j of residual block q sits at [j][q] (consecutive q for consecutive lanes)
    // four entries per thread and round, their loads issued before any is used
    for (int j0 = threadIdx.x; j0 < Kp; j0 += 4 * blockDim.x) {
      int c[4], prev[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = j0 + u * blockDim.x;
        c[u] = j < Kp ? __ldg(a.sel + j) : 0;
        prev[u] = (j < Kp && j > 0) ? __ldg(a.sel + j - 1) : -1;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = j0 + u * blockDim.x;
        if (j >= Kp) break;
        int cc = c[u];
        if (!(cc >= 0 && cc < K && prev[u] < cc)) {
          report_status(a.status, kErrInvalid);
          cc = 0;
        }
        sel_off[(j & 15) * QB + (j >> 4)] = (uint16_t)((cc >> 4) * kPitch + (cc & 15));
      }
    }
  }
  if (warp == 0) {
    // tensor scale (the amax kernel or the caller's amax)
    float am;
    if (a.amax_in != nullptr) {
      am = *a.amax_in;
    } else {
      am = 0.0f;
      for (int i = lane; i < a.P; i += 32) am = fmaxf(am, a.partial[i]);
      am = warp_max(am);
    }
    const float s_g = scale_from_amax(am, lane == 0 ? a.status : nullptr);
    if (lane == 0) {
      misc_f[0] = s_g;
      misc_f[1] = __fmul_rn(6.0f, s_g);
      if (blockIdx.x == 0 && a.res_mode != 2) {
        if (a.s_g_out) *a.s_g_out = s_g;
        if (a.s_g_out2 && a.res_mode == 0) *a.s_g_out2 = s_g;
      }
    }
  }
  if (warp == kConsumerWarps) {
    // number of tiles (segments: prefix over the segments' tiles)
    int64_t n_tiles;
    if (a.map == kMapSegments) {
      // each segment's first row and row count, kept in shared memory for the producer's tiles
      // (all of a lane's loads issued before any is used)
      int32_t* seg_first_s = seg_prefix + a.n_seg + 1;
      int32_t* seg_rows_s = seg_first_s + a.n_seg;
      for (int e = lane; e < a.n_seg; e += 32) {
        seg_first_s[e] = __ldg(a.seg_off + e);
        seg_rows_s[e] = __ldg(a.seg_rows + e);
      }
      __syncwarp();
      int carry = 0;
      for (int base = 0; base < a.n_seg; base += 32) {
        const int e = base + lane;
        int t = 0;
        if (e < a.n_seg) {
          const int rows = seg_rows_s[e];
          t = rows > 0 ? (rows + R - 1) / R : 0;
        }
        int incl = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        if (e < a.n_seg) seg_prefix[e] = carry + incl - t;
        carry += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) seg_prefix[a.n_seg] = carry;
      n_tiles = carry;
    } else if (a.map == kMapScatter) {
      n_tiles = (a.src_rows + R - 1) / R;
    } else {
      n_tiles = (a.rows_out + R - 1) / R;
    }
    if (lane == 0) misc_i[2] = (int32_t)n_tiles;
  }
  __syncthreads();
  const int n_tiles = misc_i[2];
  const float s_g = misc_f[0], t6 = misc_f[1];
  float2* dtab = reinterpret_cast<float2*>(smem + p.off_tab);
  // the residual's tensor scale: that of x, or its own (own-scale variant)
  const float s_r = a.res_mode == 1 ? scale_from_amax(*a.res_amax_in, nullptr) : s_g;
  const float t6_r = __fmul_rn(6.0f, s_r);
  float2* dtab_r = a.res_mode == 1 ? dtab + 128 : dtab;
  if (threadIdx.x < 128) {
    const uint32_t S = threadIdx.x;
    const float d = __fmul_rn(e4m3_decode(S), s_g);
    dtab[S] = make_float2(d, (S != 0 && S < 0x7F) ? __frcp_rn(d) : 0.0f);
    if (a.res_mode == 1) {
      const float dr = __fmul_rn(e4m3_decode(S), s_r);
      dtab_r[S] = make_float2(dr, (S != 0 && S < 0x7F) ? __frcp_rn(dr) : 0.0f);
    }
  }
  if (a.res_mode == 1 && blockIdx.x == 0 && threadIdx.x == 0 && a.s_g_out2) *a.s_g_out2 = s_r;
  __syncthreads();
  const bool amax_only = a.res_mode == 2;
  float res_max = 0.0f;
  const uint64_t limit = a.wait_limit_ns;

  if (warp == kConsumerWarps) {
    // ============================================================ producer
    // Per tile: its rows and the global reads of its row map are issued first, then the wait for
    // a free stage (which hides their latency), then the stage's metadata and the row copies.
    int j = 0;
    const int32_t* seg_first_s = seg_prefix + a.n_seg + 1;
    const int32_t* seg_rows_s = seg_first_s + a.n_seg;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++j) {
      const int s = j % kStages;
      // rows of this tile
      int64_t r0;      // first source row (rows / segments / scatter) or first output row (gather)
      int n;           // slots in use
      int64_t out0;    // first output row (rows / gather / segments)
      if (a.map == kMapSegments) {
        int lo = 0, hi = a.n_seg - 1;
        while (lo < hi) {  // last segment whose first tile is <= t
          const int mid = (lo + hi + 1) >> 1;
          if (seg_prefix[mid] <= t) lo = mid;
          else hi = mid - 1;
        }
        const int c = t - seg_prefix[lo];
        const int rows = seg_rows_s[lo];
        r0 = (int64_t)seg_first_s[lo] + (int64_t)c * R;
        n = min(R, rows - c * R);
        out0 = r0;
        if (r0 < 0 || r0 + n > a.src_rows || r0 + n > a.rows_out) {  // a segment outside the rows
          if (lane == 0) report_status(a.status, kErrInvalid);
          n = 0;
        }
      } else if (a.map == kMapScatter) {
        r0 = (int64_t)t * R;
        n = (int)min((int64_t)R, a.src_rows - r0);
        out0 = -1;
      } else {
        out0 = (int64_t)t * R;
        n = (int)min((int64_t)R, a.rows_out - out0);
        r0 = out0;
      }
      // per slot: source row (or -1 for a zero row); scatter: up to 4 destinations per lane
      int64_t my_src = -1;
      if (lane < n) {
        if (a.map == kMapGather) {
          const int64_t o = out0 + lane;
          if (o < a.rows_valid) {
            const int64_t g = __ldg(a.row_gather + o);
            my_src = (g >= 0 && g < a.src_rows) ? g : -1;
          }
        } else if (a.map == kMapRows) {
          my_src = (r0 + lane < a.rows_valid && r0 + lane < a.src_rows) ? r0 + lane : -1;
        } else {
          my_src = r0 + lane;
        }
      }
      const int fo = p.fanout;
      int32_t dpre[kMaxMeta / 32];
#pragma unroll
      for (int q = 0; q < kMaxMeta / 32; ++q) {
        const int e = lane + 32 * q;
        const int slot = e / fo, jj = e - slot * fo;
        dpre[q] = (a.map == kMapScatter && e < R * fo && slot < n) ? __ldg(a.row_scatter + (r0 + slot) * fo + jj) : -1;
      }
      if (j >= kStages) {
        bool ok = true;
        if (lane == 0) ok = tc::mbar_wait(bar_empty(s), (uint32_t)(((j / kStages) - 1) & 1), limit, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) {
            if (!*abort_flag) report_status(a.status, kErrTimeout);
            *abort_flag = 1;
          }
          break;
        }
      }
      MetaView m(smem + p.off_meta + s * p.meta_bytes, p.mc, R);
      if (lane < R) m.valid[lane] = (lane < n && my_src >= 0) ? 1 : 0;
      // per (slot, destination): output row and its byte offsets
#pragma unroll
      for (int q = 0; q < kMaxMeta / 32; ++q) {
        const int e = lane + 32 * q;
        if (e >= R * fo) break;
        const int slot = e / fo, jj = e - slot * fo;
        (void)jj;
        int64_t drow = -1;
        if (slot < n) {
          if (a.map == kMapScatter) {
            drow = dpre[q];
            if (drow >= a.rows_out) {
              report_status(a.status, kErrInvalid);
              drow = -1;
            }
          } else {
            drow = out0 + slot;
          }
        }
        m.code[e] = drow >= 0 ? drow * (K / 2) : -1;
        m.sfrow[e] = drow >= 0 ? sf_row_off(drow, k64, slab16) : 0;
        if (RES) {
          m.rcode[e] = drow >= 0 ? drow * (Kp / 2) : -1;
          m.rsfrow[e] = drow >= 0 ? sf_row_off(drow, kp64, slab16) : 0;
        }
      }
      if (lane == 0) *m.n_slots = n;
      __threadfence_block();
      __syncwarp();
      // bytes of this stage: contiguous source rows come in one copy, gathered rows one by one
      const uint32_t dst = sb + (uint32_t)(p.off_stage + s * p.stage_bytes);
      const uint32_t row_bytes = (uint32_t)K * 2u;
      const bool contiguous = (a.map != kMapGather) && (a.ld == K);
      int n_loaded;
      if (a.map == kMapGather || a.map == kMapRows) {
        n_loaded = __popc(__ballot_sync(0xffffffffu, my_src >= 0));
      } else {
        n_loaded = n;
      }
      if (lane == 0) tc::mbar_expect_tx(bar_full(s), (uint32_t)n_loaded * row_bytes);
      __syncwarp();
      if (contiguous && a.map != kMapGather) {
        // the loaded rows of a plain / scatter / segment tile are a prefix of its slots
        if (lane == 0 && n_loaded > 0)
          tc::bulk_load(dst, a.src + r0 * a.ld, (uint32_t)n_loaded * row_bytes, bar_full(s));
      } else if (my_src >= 0) {
        tc::bulk_load(dst + (uint32_t)lane * row_bytes, a.src + my_src * a.ld, row_bytes, bar_full(s));
      }
    }
    // every copy this warp issued has landed before the CTA can exit: the last use of each stage
    // (tile i < j issued into stage i % kStages, phase (i / kStages) & 1)
    if (lane == 0) {
      for (int i = max(0, j - kStages); i < j; ++i)
        tc::mbar_wait(bar_full(i % kStages), (uint32_t)((i / kStages) & 1), limit, nullptr);
    }
    return;
  }

  // ============================================================== consumers
  const int tid = threadIdx.x;  // 0 .. kConsumers-1
  // when kConsumers is a multiple of QB a thread works on the same residual block q = tid % QB in
  // every tile: its 16 channel offsets are read once, into registers
  const bool fixed_q = RES && QB > 0 && kConsumers % QB == 0;
  uint32_t my_off[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) my_off[i] = 0;
  if (fixed_q) {
    const int q = tid % QB;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      my_off[i] = (uint32_t)sel_off[(2 * i) * QB + q] | ((uint32_t)sel_off[(2 * i + 1) * QB + q] << 16);
  }
  float* rbuf = reinterpret_cast<float*>(smem + p.off_rbuf);
  const int rpitch = KB * kPitch;  // words per row of the residual buffer
  int j = 0;
  for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++j) {
    const int s = j % kStages;
    bool ok = tc::mbar_wait(bar_full(s), (uint32_t)((j / kStages) & 1), limit, abort_flag);
    // all consumers waited for this stage and finished the previous tile's residual pass
    const bool bad = RES ? consumers_sync_or<kConsumers>(!ok) : __any_sync(0xffffffffu, !ok);
    if (bad) {
      if (tid == 0 || !ok) {
        if (!*abort_flag) report_status(a.status, kErrTimeout);
        *abort_flag = 1;
      }
      break;
    }
    const MetaView m(smem + p.off_meta + s * p.meta_bytes, p.mc, R);
    const unsigned char* stage = smem + p.off_stage + s * p.stage_bytes;
    const int n = *m.n_slots;
    const int fo = p.fanout;
    // ---- main pass: one 16-element block per thread and step
    int slot = tid / KB, kb = tid - (tid / KB) * KB;
    const int dslot = kConsumers / KB, dkb = kConsumers - (kConsumers / KB) * KB;
    for (; slot < n; slot += dslot, kb += dkb) {
      if (kb >= KB) {
        kb -= KB;
        ++slot;
        if (slot >= n) break;
      }
      uint4 u0 = make_uint4(0, 0, 0, 0), u1 = make_uint4(0, 0, 0, 0);
      if (m.valid[slot]) {
        const uint4* src = reinterpret_cast<const uint4*>(stage + ((size_t)slot * K + (size_t)kb * 16) * 2);
        u0 = src[0];
        u1 = src[1];
      }
      const BlockScale bs = block_scale_tab(absmax16(u0, u1), s_g, t6, dtab);
      float x[16];
      bf16x8_to_f32(u0, x);
      bf16x8_to_f32(u1, x + 8);
      const uint2 c = make_uint2(codes8(x, bs), codes8(x + 8, bs));
      if (fo == 1) {
        const int64_t co = m.code[slot];
        if (!amax_only && co >= 0) {
          *reinterpret_cast<uint2*>(a.codes + co + kb * 8) = c;
          a.sf[m.sfrow[slot] + sf_blk_off(kb)] = (uint8_t)bs.S;
        }
      } else if (!amax_only) {
        // several destinations: lane p of a four-lane group stores the group's scale word of
        // destinations p, p + 4, ... (one 32-bit store instead of four byte stores per row)
        const uint32_t sw = scale_word4(bs.S, lane);
        for (int jj = 0; jj < fo; ++jj) {
          const int64_t co = m.code[slot * fo + jj];
          if (co >= 0) *reinterpret_cast<uint2*>(a.codes + co + kb * 8) = c;
        }
        const int32_t wblk = sf_blk_off(kb & ~3);
        for (int jj = lane & 3; jj < fo; jj += 4) {
          const int e = slot * fo + jj;
          if (m.code[e] >= 0) *reinterpret_cast<uint32_t*>(a.sf + m.sfrow[e] + wblk) = sw;
        }
      }
      if (RES) {
        float r[16];
        resid8(x, c.x, bs.d, r);
        resid8(x + 8, c.y, bs.d, r + 8);
        float* rb = rbuf + slot * rpitch + kb * kPitch;
#pragma unroll
        for (int i = 0; i < 16; ++i) rb[i] = r[i];
      }
    }
    if (RES) {
      consumers_sync<kConsumers>();  // the residual buffer of this tile is complete
      // ---- residual pass: 16 compact positions (one residual block) per thread and step
      int rs = tid / QB, q = tid - (tid / QB) * QB;
      const int drs = kConsumers / QB, dq = kConsumers - (kConsumers / QB) * QB;
      for (; rs < n; rs += drs, q += dq) {
        if (q >= QB) {
          q -= QB;
          ++rs;
          if (rs >= n) break;
        }
        const float* rrow = rbuf + rs * rpitch;
        float v[16];
        if (fixed_q) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            v[2 * i] = rrow[my_off[i] & 0xFFFFu];
            v[2 * i + 1] = rrow[my_off[i] >> 16];
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = rrow[sel_off[i * QB + q]];
        }
        float b = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) b = fmaxf(b, fabsf(v[i]));
        if (amax_only) {
          res_max = fmaxf(res_max, b);
          continue;
        }
        const BlockScale bs = block_scale_tab(b, s_r, t6_r, dtab_r);
        const uint2 c = make_uint2(codes8(v, bs), codes8(v + 8, bs));
        if (fo == 1) {
          const int64_t co = m.rcode[rs];
          if (co >= 0) {
            *reinterpret_cast<uint2*>(a.rcodes + co + q * 8) = c;
            a.rsf[m.rsfrow[rs] + sf_blk_off(q)] = (uint8_t)bs.S;
          }
        } else {
          const uint32_t sw = scale_word4(bs.S, lane);
          for (int jj = 0; jj < fo; ++jj) {
            const int64_t co = m.rcode[rs * fo + jj];
            if (co >= 0) *reinterpret_cast<uint2*>(a.rcodes + co + q * 8) = c;
          }
          const int32_t wblk = sf_blk_off(q & ~3);
          for (int jj = lane & 3; jj < fo; jj += 4) {
            const int e = rs * fo + jj;
            if (m.rcode[e] >= 0) *reinterpret_cast<uint32_t*>(a.rsf + m.rsfrow[e] + wblk) = sw;
          }
        }
      }
    }
    // this stage (rows and metadata) is free for the producer
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(bar_empty(s));
  }
  if (amax_only) {
    res_max = warp_max(res_max);
    if (lane == 0 && res_max > 0.0f)
      atomicMax(reinterpret_cast<unsigned int*>(a.res_amax_out), __float_as_uint(res_max));
  }
}

}  // namespace act

// Launch shape: rows per tile R (stages of at most ~16 KB) and consumer warps W.  Chosen so that
// the main pass (R * K/16 blocks) and the residual pass (R * Kp/16 blocks) leave the fewest idle
// thread steps, discounted when fewer than 18 consumer warps fit on an SM, then for the most
// bytes in flight per SM (CTAs per SM x the two stages ahead, up to 96 KB), then for more CTAs per
// SM.  force_R / force_W (> 0) override the choice.
bool act_plan_choose(int64_t K, int32_t Kp, int fanout, int32_t n_seg, int* R_out, int* W_out, int* smem_out,
                     int force_R, int force_W) {
  if (K <= 0 || K % 64 != 0 || fanout < 1 || fanout > act::kMaxMeta) return false;
  if (n_seg > kMaxRouteExperts) return false;
  const int KB = (int)(K / 16), QB = Kp / 16;
  double best = -1.0;
  int bR = 0, bW = 0, bsm = 0;
  const int warps[4] = {4, 6, 7, 8};
  for (int R = 1; R <= 16; ++R) {
    if (force_R > 0 && R != force_R) continue;
    if ((int64_t)R * K * 2 > 16384 && R > 1 && force_R <= 0) break;
    if (R * fanout > act::kMaxMeta) break;
    const act::Plan p = act::make_plan((int)K, Kp, fanout, n_seg, R);
    if (p.smem > 200 * 1024) continue;
    const int per_sm = (227 * 1024) / (p.smem + 1024);
    if (per_sm < 1) continue;
    const double inflight = (double)min(per_sm, 8) * (act::kStages - 1) * p.stage_bytes;
    for (int wi = 0; wi < 4; ++wi) {
      if (force_W > 0 && warps[wi] != force_W) continue;
      const int T = 32 * warps[wi];
      const int steps = (R * KB + T - 1) / T + (QB > 0 ? (R * QB + T - 1) / T : 0);
      const double eff = (double)R * (KB + QB) / ((double)steps * T);
      // consumer warps resident per SM: below ~18 the dependent chains of a block are not hidden
      const int ctas = min(per_sm, 64 / (warps[wi] + 1));
      const double occ = min(1.0, (double)(ctas * warps[wi]) / 18.0);
      const double score = (double)(int)(eff * occ * 100.0) * 1e9 + min(inflight, 96.0 * 1024) * 100.0 + per_sm;
      if (score > best) {
        best = score;
        bR = R;
        bW = warps[wi];
        bsm = p.smem;
      }
    }
  }
  if (bR == 0) return false;
  *R_out = bR;
  *W_out = bW;
  *smem_out = bsm;
  return true;
}

template <bool RES, int W>
static cudaError_t launch_act_t(const ActArgs& a, int grid, int smem, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(act::act_quant_kernel<RES, W>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  act::act_quant_kernel<RES, W><<<(unsigned)grid, 32 * W + 32, smem, st>>>(a);
  return cudaGetLastError();
}

template <bool RES>
static cudaError_t launch_act_w(const ActArgs& a, int W, int grid, int smem, cudaStream_t st) {
  switch (W) {
    case 4: return launch_act_t<RES, 4>(a, grid, smem, st);
    case 6: return launch_act_t<RES, 6>(a, grid, smem, st);
    case 7: return launch_act_t<RES, 7>(a, grid, smem, st);
    case 8: return launch_act_t<RES, 8>(a, grid, smem, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_act(ActArgs a, int num_sms, int force_R, int force_W, cudaStream_t st) {
  int R = 0, W = 0, smem = 0;
  if (!act_plan_choose(a.K, a.Kp, a.fanout, a.map == kMapSegments ? a.n_seg : 0, &R, &W, &smem, force_R, force_W))
    return cudaErrorInvalidValue;
  a.R = R;
  // tiles (segments: an upper bound; the kernel counts them)
  const int64_t tiles = a.map == kMapScatter ? (a.src_rows + R - 1) / R : (a.rows_out + R - 1) / R;
  int per_sm = (int)((227 * 1024) / (smem + 1024));
  if (per_sm < 1) per_sm = 1;
  if (per_sm > 8) per_sm = 8;
  int64_t grid = (int64_t)num_sms * per_sm;
  if (grid > tiles) grid = tiles;
  if (grid < 1) grid = 1;
  return a.Kp > 0 ? launch_act_w<true>(a, W, (int)grid, smem, st) : launch_act_w<false>(a, W, (int)grid, smem, st);
}

}  // namespace nvfp4
