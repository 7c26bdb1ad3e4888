// W4A4 + RAC grouped GEMM for MoE decode (a few tokens per expert), sm_100a.
//
// At decode the rows routed to one expert are a handful of tokens, so the roles of the two
// operands are swapped: the expert's weight rows are the MMA's A operand (M = 128 weight rows
// per unit) and the expert's tokens, held in a 16-row "slab", are the B operand (N = 16).  The
// kernel is then a weight stream: every unit (slab, 128-row weight tile) reads its
// 128 x (K + K') weight codes once through a deep TMA ring; the tensor cores need only a small
// share of their peak.
//
// The method is the prefill GEMM's ("Why 4-bit RL rollout collapses - and it isn't the
// weights", section "Two fixes, on two different sides": the native W4A4 GEMM stays as it is
// and the residual FP4 pass over the selected channels is added to it): the residual K' loop
// accumulates into the same tensor-memory accumulator as the main K loop.
//
// Roles: warp 0 TMA producer; warp 1 TMEM allocation + MMA issue; warps 2..5 epilogue, one per
// TMEM lane quadrant (32 weight rows each); warps 6..9 scale warps, one per quadrant, which store
// each k-tile's scale atoms (shared -> registers -> tensor memory, tcgen05.st, the four-way
// replicated layout) into a two-slot ring, so the tensor pipe runs only the MMAs (a scale copy on
// the tensor pipe costs about as much as an N = 16 MMA, and each MMA needs two).  A unit's
// accumulator is 128 lanes x 16 columns (weight rows x tokens); four accumulator buffers let the
// epilogue trail the MMAs.
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace nvfp4 {
namespace tc {

namespace dec {
constexpr int BM = 128;       // weight rows per unit
constexpr int BT = 16;        // tokens per slab (MMA N)
constexpr int KT_BYTES = 128; // 256 FP4 codes per row per k-tile
constexpr int STAGES = 9;
constexpr int A_BYTES = BM * KT_BYTES;  // 16 KB
constexpr int B_BYTES = BT * KT_BYTES;  // 2 KB
constexpr int SFA_BYTES = 4 * 512;
constexpr int SFB_BYTES = 4 * 512;
constexpr int ACC_BUFS = 4;
constexpr int SF_KT = 32;               // a stored k-tile: A scales of its 4 blocks, then B's (4 + 4 columns each)
constexpr int SF_BASE = ACC_BUFS * BT;  // 64
constexpr int TMEM_COLS = 128;
constexpr int NUM_THREADS = 320;
constexpr int SF_WARP0 = 6;
constexpr int XCH_BYTES = 64 * BT * 4;  // SwiGLU exchange: 64 up rows x 16 tokens, fp32
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
constexpr int OFF_XCH = OFF_SFB + STAGES * SFB_BYTES;  // two exchange buffers
constexpr int OFF_BAR = OFF_XCH + 2 * XCH_BYTES;
// full[STAGES] empty[STAGES] accf[ACC_BUFS] acce[ACC_BUFS] drain xfull[2] xempty[2] sf_full[2]
// sf_landed[STAGES]
constexpr int NUM_BARS = 3 * STAGES + 2 * ACC_BUFS + 1 + 4 + 2;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM = OFF_MISC + 32;
static_assert(SMEM <= 232448, "shared memory budget");
static_assert(SF_BASE + 2 * SF_KT <= TMEM_COLS, "tensor memory budget");
static_assert(OFF_B % 1024 == 0 && B_BYTES % 1024 == 0, "swizzled tiles need 1024-byte alignment");
}  // namespace dec

// 32 lanes x 16 columns of 32-bit accumulator -> 16 registers per thread
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void store_out(void* y, bool bf16, int64_t idx, float v) {
  if (bf16) {
    reinterpret_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
  } else {
    reinterpret_cast<float*>(y)[idx] = v;
  }
}

__global__ void __launch_bounds__(dec::NUM_THREADS, 1)
    w4a4_rac_decode_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_ws,
                           const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_xr,
                           const DecodeArgs args) {
  using namespace dec;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  unsigned char* smem = smem_raw;
  if ((sbase & 1023u) != 0) {
    if (threadIdx.x == 0) report_status(args.status, kErrAlign);
    return;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto bar_full = [&](int s) { return sbase + OFF_BAR + 8u * s; };
  auto bar_empty = [&](int s) { return sbase + OFF_BAR + 8u * (STAGES + s); };
  auto bar_accf = [&](int a) { return sbase + OFF_BAR + 8u * (2 * STAGES + a); };
  auto bar_acce = [&](int a) { return sbase + OFF_BAR + 8u * (2 * STAGES + ACC_BUFS + a); };
  const uint32_t bar_drain = sbase + OFF_BAR + 8u * (2 * STAGES + 2 * ACC_BUFS);
  auto bar_xfull = [&](int b) { return sbase + OFF_BAR + 8u * (2 * STAGES + 2 * ACC_BUFS + 1 + b); };
  auto bar_xempty = [&](int b) { return sbase + OFF_BAR + 8u * (2 * STAGES + 2 * ACC_BUFS + 3 + b); };
  auto bar_sff = [&](int b) { return sbase + OFF_BAR + 8u * (2 * STAGES + 2 * ACC_BUFS + 5 + b); };
  // a stage's scale atoms landed (apart from its operands, so the scale warps can start first)
  auto bar_sfl = [&](int s) { return sbase + OFF_BAR + 8u * (2 * STAGES + 2 * ACC_BUFS + 7 + s); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  volatile int* prod_issued = reinterpret_cast<volatile int*>(smem + OFF_MISC + 8);
  volatile int* mma_taken = reinterpret_cast<volatile int*>(smem + OFF_MISC + 12);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
      mbar_init(bar_sfl(s), 1);
    }
    for (int a = 0; a < ACC_BUFS; ++a) {
      mbar_init(bar_accf(a), 1);
      mbar_init(bar_acce(a), 4);
    }
    mbar_init(bar_drain, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_xfull(b), 2);
      mbar_init(bar_xempty(b), 2);
      mbar_init(bar_sff(b), 4);
    }
    *abort_flag = 0;
    *prod_issued = 0;
    *mma_taken = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t total_units = (int64_t)args.n_slots * args.m_tiles;
  const int kt_total = args.kt_main + args.kt_res;
  const uint64_t limit = args.wait_limit_ns;
  // every role reads the same slot table: a negative expert marks an unused slot that all of
  // them skip; an expert index >= E stops all of them at the same unit (nothing is loaded for it)
  constexpr int kSkip = -1, kBad = -2;
  auto unit_expert = [&](int slot) -> int {
    const int e = __ldg(args.slot_expert + slot);
    return e < 0 ? kSkip : (e < args.E ? e : kBad);
  };

  if (warp == 0) {
    // ===================================================================== TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int64_t u = blockIdx.x; u < total_units && !*abort_flag; u += gridDim.x) {
        const int slot = (int)(u / args.m_tiles);
        const int mt = (int)(u - (int64_t)slot * args.m_tiles);
        const int e = unit_expert(slot);
        if (e == kSkip) continue;
        if (e == kBad) {
          report_status(args.status, kErrInvalid);
          *abort_flag = 1;
          break;
        }
        bool ok = true;
        for (int kt = 0; kt < kt_total; ++kt) {
          if (!mbar_wait(bar_empty(stage), phase ^ 1u, limit, abort_flag)) {
            ok = false;
            break;
          }
          const bool res = kt >= args.kt_main;
          const int kk = res ? kt - args.kt_main : kt;
          const int k64 = res ? args.k64_res : args.k64_main;
          const int nk64 = min(4, k64 - kk * 4);
          const uint32_t sf_bytes = (uint32_t)nk64 * 512u;
          mbar_expect_tx(bar_sfl(stage), 2u * sf_bytes);
          mbar_expect_tx(bar_full(stage), (uint32_t)(A_BYTES + B_BYTES));
          tma_load_3d(sbase + OFF_A + stage * A_BYTES, res ? &tm_ws : &tm_w, kk * KT_BYTES, mt * BM, e,
                      bar_full(stage));
          tma_load_2d(sbase + OFF_B + stage * B_BYTES, res ? &tm_xr : &tm_x, kk * KT_BYTES, slot * BT,
                      bar_full(stage));
          const uint8_t* sfw = res ? args.sfw_sel + (int64_t)e * args.sfw_sel_slab_bytes
                                   : args.sfw + (int64_t)e * args.sfw_slab_bytes;
          bulk_load(sbase + OFF_SFA + stage * SFA_BYTES, sfw + ((int64_t)mt * k64 + kk * 4) * 512, sf_bytes,
                    bar_sfl(stage));
          // slab layout: slab `slot` owns one scale atom per 64 columns
          const uint8_t* sfx = res ? args.sfx_res : args.sfx;
          bulk_load(sbase + OFF_SFB + stage * SFB_BYTES, sfx + ((int64_t)slot * k64 + kk * 4) * 512, sf_bytes,
                    bar_sfl(stage));
          ++issued;
          *prod_issued = issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) {
          report_status(args.status, kErrTimeout);
          *abort_flag = 1;
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ===================================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_fp4(BM, BT);
      int stage = 0;
      uint32_t phase = 0;
      int taken = 0;
      uint32_t mma_count = 0;
      bool ok = true;
      int64_t uidx = 0;  // units processed by this CTA (skipped slots not counted)
      uint32_t g = 0;    // k-tiles taken (the scale ring's sequence)
      for (int64_t u = blockIdx.x; u < total_units && !*abort_flag; u += gridDim.x) {
        const int slot = (int)(u / args.m_tiles);
        const int eu = unit_expert(slot);
        if (eu == kSkip) continue;
        if (eu == kBad) break;  // reported by the producer
        const int buf = (int)(uidx % ACC_BUFS);
        const int64_t use = uidx / ACC_BUFS;
        if (use >= 1 && !mbar_wait(bar_acce(buf), (uint32_t)((use - 1) & 1), limit, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BT);
        for (int kt = 0; kt < kt_total; ++kt) {
          if (!mbar_wait(bar_full(stage), phase, limit, abort_flag) ||
              !mbar_wait(bar_sff(g & 1), (g >> 1) & 1u, limit, abort_flag)) {
            ok = false;
            break;
          }
          ++taken;
          *mma_taken = taken;
          tc_fence_after();
          const bool res = kt >= args.kt_main;
          const int kk = res ? kt - args.kt_main : kt;
          const int k64 = res ? args.k64_res : args.k64_main;
          const int nk64 = min(4, k64 - kk * 4);
          const uint32_t a_s = sbase + OFF_A + stage * A_BYTES;
          const uint32_t b_s = sbase + OFF_B + stage * B_BYTES;
          // scales of block j: A at +4j, B at +16 + 4j of slot g & 1 (stored by the scale warps)
          const uint32_t sf_t = tmem_base + (uint32_t)(SF_BASE + (int)(g & 1) * SF_KT);
          for (int j = 0; j < nk64; ++j, ++mma_count)
            tc_mma_fp4(d_tmem, desc_sw128(a_s + 32 * j), desc_sw128(b_s + 32 * j), idesc, sf_t + 4 * j,
                       sf_t + 16 + 4 * j, (kt | j) != 0 ? 1u : 0u);
          tc_commit(bar_empty(stage));
          ++g;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(bar_accf(buf));
        ++uidx;
      }
      if (!ok) {
        report_status(args.status, kErrTimeout);
        *abort_flag = 1;
      }
    }
  } else if (warp >= SF_WARP0) {
    // ===================================================================== scale warps
    // Warp w stores lanes [32 (w % 4), +32): lane j takes the 16 bytes at 16 j of each 512-byte
    // atom into 4 columns.  Per k-tile g: its stage has landed, slot g & 1 is free (the commit that
    // empties the stage of k-tile g - 2 has arrived, so its MMAs are complete), then the 4 A and
    // 4 B atoms -> 32 columns, wait for the stores, arrive on sf_full.
    const int quad = warp & 3;
    const uint32_t t_lane = tmem_base + ((uint32_t)(quad * 32) << 16);
    uint32_t g = 0;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < total_units && ok && !*abort_flag; u += gridDim.x) {
      const int e = unit_expert((int)(u / args.m_tiles));
      if (e == kSkip) continue;
      if (e == kBad) break;
      for (int kt = 0; kt < kt_total; ++kt) {
        bool w_ok = mbar_wait(bar_sfl(stage), phase, limit, abort_flag);
        if (w_ok && g >= 2) {
          const uint32_t gp = g - 2;
          w_ok = mbar_wait(bar_empty((int)(gp % STAGES)), (gp / STAGES) & 1u, limit, abort_flag);
        }
        if (!__all_sync(0xffffffffu, w_ok)) {
          if (lane == 0) {
            if (!*abort_flag) report_status(args.status, kErrTimeout);
            *abort_flag = 1;
          }
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sl = t_lane + (uint32_t)(SF_BASE + (int)(g & 1) * SF_KT);
        const uint32_t sfa_s = sbase + OFF_SFA + stage * SFA_BYTES + lane * 16;
        const uint32_t sfb_s = sbase + OFF_SFB + stage * SFB_BYTES + lane * 16;
        uint32_t r[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) ld_shared_v4(sfa_s + j * 512, r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
        tmem_st16(sl, r);
#pragma unroll
        for (int j = 0; j < 4; ++j) ld_shared_v4(sfb_s + j * 512, r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
        tmem_st16(sl + 16, r);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_sff((int)(g & 1)));
        ++g;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else {
    // ===================================================================== epilogue
    const int quad = warp & 3;  // TMEM lanes [32*quad, +32) = weight rows of the unit
    const bool swiglu = args.epi != 0;
    const bool bf16 = args.out_bf16 != 0;
    float* xch = reinterpret_cast<float*>(smem + OFF_XCH);
    float amax = 0.0f;
    int64_t uidx = 0;  // units processed by this CTA, as counted by the MMA issuer
    for (int64_t u = blockIdx.x; u < total_units && !*abort_flag; u += gridDim.x) {
      const int slot = (int)(u / args.m_tiles);
      const int mt = (int)(u - (int64_t)slot * args.m_tiles);
      const int e = unit_expert(slot);
      if (e == kSkip) continue;
      if (e == kBad) break;
      const int cnt = min(BT, max(0, (int)__ldg(args.slot_count + slot)));
      const int buf = (int)(uidx % ACC_BUFS);
      const uint32_t parity = (uint32_t)((uidx / ACC_BUFS) & 1);
      bool ok = __all_sync(0xffffffffu, mbar_wait(bar_accf(buf), parity, limit, abort_flag));
      uint32_t v[16];
      if (ok) {
        tc_fence_after();
        tmem_ld16(tmem_base + (uint32_t)(buf * BT) + ((uint32_t)(quad * 32) << 16), v);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_acce(buf));
      }
      const float alpha = __fmul_rn(__ldg(args.s_x), __ldg(args.s_w + e));
      const int64_t row0 = (int64_t)slot * BT;
      if (ok && !swiglu) {
        // weight row f = mt*128 + 32*quad + lane is output column f; token j of the slab is
        // output row slot*16 + j.  Rows past the slab's count are written as zeros.
        const int64_t f = (int64_t)mt * BM + quad * 32 + lane;
#pragma unroll
        for (int j = 0; j < BT; ++j)
          store_out(args.y, bf16, (row0 + j) * args.ldy + f, j < cnt ? __fmul_rn(__uint_as_float(v[j]), alpha) : 0.0f);
      } else if (ok) {
        // SwiGLU: lanes 0..63 of the unit hold gate rows, lanes 64..127 the matching up rows
        // (64-row gate/up interleave of the packed weight).  The up warps hand their values to
        // the gate warps through one of two shared-memory buffers.
        const int xb = (int)(uidx & 1);
        const int64_t xuse = uidx >> 1;
        float* xbuf = xch + xb * (XCH_BYTES / 4);
        if (quad >= 2) {
          if (xuse >= 1)
            ok = __all_sync(0xffffffffu, mbar_wait(bar_xempty(xb), (uint32_t)((xuse - 1) & 1), limit, abort_flag));
          if (ok) {
#pragma unroll
            for (int j = 0; j < BT; ++j) xbuf[j * 64 + (quad - 2) * 32 + lane] = __uint_as_float(v[j]);
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_xfull(xb));
          }
        } else {
          ok = __all_sync(0xffffffffu, mbar_wait(bar_xfull(xb), (uint32_t)(xuse & 1), limit, abort_flag));
          if (ok) {
            float up[BT];
#pragma unroll
            for (int j = 0; j < BT; ++j) up[j] = xbuf[j * 64 + quad * 32 + lane];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_xempty(xb));
            const int64_t f = (int64_t)mt * 64 + quad * 32 + lane;  // output feature of h
#pragma unroll
            for (int j = 0; j < BT; ++j) {
              float hv = 0.0f;
              if (j < cnt) {
                const float gv = bf16_round(__fmul_rn(__uint_as_float(v[j]), alpha));
                const float uv = bf16_round(__fmul_rn(up[j], alpha));
                // silu(g) = g / (1 + e^-g); e^-g overflowing to inf gives -0 (the limit)
                const float sg = __fdividef(gv, 1.0f + __expf(-gv));
                hv = bf16_round(sg * uv);
                amax = fmaxf(amax, fabsf(hv));
              }
              store_out(args.y, bf16, (row0 + j) * args.ldy + f, hv);
            }
          }
        }
      }
      if (!ok) {
        if (lane == 0) {
          report_status(args.status, kErrTimeout);
          *abort_flag = 1;
        }
        break;
      }
      ++uidx;
    }
    if (swiglu && args.amax_out != nullptr) {
      amax = warp_max(amax);
      if (lane == 0 && amax > 0.0f) atomicMax(reinterpret_cast<unsigned int*>(args.amax_out), __float_as_uint(amax));
    }
  }

  // ---- teardown
  __syncthreads();
  if (*abort_flag) {
    if (warp == 1 && lane == 0) {
      // all MMAs issued by this thread complete before the commit arrives
      tc_commit(bar_drain);
      mbar_wait(bar_drain, 0, limit, nullptr);
    }
    if (warp == 0 && lane == 0) {
      // tensor copies still in flight land before the shared memory is released
      for (int i = *mma_taken; i < *prod_issued; ++i) {
        mbar_wait(bar_full(i % STAGES), (uint32_t)((i / STAGES) & 1), limit, nullptr);
        mbar_wait(bar_sfl(i % STAGES), (uint32_t)((i / STAGES) & 1), limit, nullptr);
      }
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"((uint32_t)TMEM_COLS)
                 : "memory");
  }
}

}  // namespace tc

size_t decode_smem_bytes() { return (size_t)tc::dec::SMEM; }

cudaError_t launch_decode(const CUtensorMap& tm_w, const CUtensorMap& tm_ws, const CUtensorMap& tm_x,
                          const CUtensorMap& tm_xr, const DecodeArgs& args, int grid, cudaStream_t st) {
  cudaError_t e =
      cudaFuncSetAttribute(tc::w4a4_rac_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::dec::SMEM);
  if (e != cudaSuccess) return e;
  tc::w4a4_rac_decode_kernel<<<grid, tc::dec::NUM_THREADS, tc::dec::SMEM, st>>>(tm_w, tm_ws, tm_x, tm_xr, args);
  return cudaGetLastError();
}

}  // namespace nvfp4
