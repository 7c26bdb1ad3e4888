// W4A4 + RAC GEMM on the 5th-generation tensor cores (sm_100a).
//
//   Y = s_a * s_w * ( Q(X) Q(W)^T + Q(R_sel) Q(W_sel)^T )
//
// "The native W4A4 GEMM path stays intact; only the highest-error channels get a correction
// pass layered on top" ("Why 4-bit RL rollout collapses - and it isn't the weights", Two
// fixes, on two different sides).  Here the correction pass is a second K loop (K' = Kp
// columns of the residual and of the gathered weight columns) that accumulates into the
// same tensor-memory accumulator as the main loop, so one epilogue applies the scale.
//
// Structure (one CTA per SM, persistent over output tiles of 128 x BN; four warpgroups whose
// register shares are moved with setmaxnreg: 128 x (56 + 72) + 256 x 192 = 65536 registers):
//   warp 0      TMA producer: A/B code tiles (128-byte swizzle) by tensor-map copies, the
//               scale atoms (512 B each) by bulk copies, into a STAGES-deep shared ring.
//   warp 1      tensor-memory allocation and the single MMA-issuing thread:
//               tcgen05.mma.kind::mxf4nvf4.block_scale (K = 64 per instruction); commits
//               free the shared stage and, at the end of a tile, publish the accumulator.
//   warps 4..7  scale warps (one per tensor-memory lane quadrant): each k-tile's scale atoms,
//               shared -> registers -> tensor memory (tcgen05.st, the four-way replicated
//               layout the MMA reads), into a two-slot ring.  Measured: a 512-byte atom copy
//               on the tensor pipe (tcgen05.cp 32x128b.warpx4) costs about 55 cycles there,
//               serialised with the MMAs (three per K = 64 MMA at BN = 256, about as much
//               time as the MMA itself); stores by warps run beside the MMAs.  The FP8 and
//               own-scale modes keep the copies on the tensor pipe.
//   warps 8..15 epilogue: tcgen05.ld of the FP32 accumulator (two warps per lane quadrant,
//               one column half each) into registers, release, then scale by alpha and
//               store bf16/FP32 rows (or SwiGLU + amax) while the next tile's MMAs run.
// Every mbarrier wait is bounded by a wall-clock limit; on expiry the kernel records
// NVFP4_ERR_TIMEOUT, drains its own copies and MMAs, frees tensor memory and returns.
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace nvfp4 {
namespace tc {

constexpr int BM = 128;
constexpr int KT_BYTES = 128;  // bytes of one row per k-tile: 256 FP4 elements
constexpr int NUM_THREADS = 512;  // producer, MMA, 2 idle | 4 scale warps | 8 epilogue warps
constexpr int EPI_WARP0 = 8;      // first epilogue warp
constexpr int SF_WARP0 = 4;       // first scale warp
// per-thread registers after the split (warpgroups 0, 1, 2-3): 128 x (56 + 72) + 256 x 192
constexpr int REG_CTRL = 56, REG_SF = 72, REG_EPI = 192;
static_assert(128 * (REG_CTRL + REG_SF) + 256 * REG_EPI <= 65536, "register split over the launch's total");

// Weight slab of grouped segment `seg`: the segment itself, or seg_expert[seg] (segments of
// several sources that share an expert, as an expert-parallel rank receives them).  An index
// outside the weight slabs is reported and replaced by slab 0, so no load leaves the weights.
__device__ __forceinline__ int segment_weight(const GemmArgs& args, int seg) {
  if (args.seg_expert == nullptr) return seg;
  const int e = __ldg(args.seg_expert + seg);
  if (e < 0 || e >= args.n_weights) {
    report_status(args.status, kErrInvalid);
    return 0;
  }
  return e;
}

// OWN: the residual operand carries its own tensor scale (the own-scale RAC variant), so the main
// and the residual products go to two accumulators (columns [0, BN) and [BN, 2 BN) of a buffer)
// and the epilogue adds them with their own scales; only BN = 128 (the two halves then take the
// tensor memory of one BN = 256 accumulator).
// SFST: the scale warps store each k-tile's scale factors into a two-slot ring of tensor memory
// (FP4 without the own-scale mode); otherwise the MMA thread copies them per MMA (two slots).
template <int BN, bool OWN = false, bool SFST = false>
struct Cfg {
  static constexpr int ACC_W = OWN ? 2 * BN : BN;  // accumulator columns per tile
  // NARROW (scale-warp mode at BN = 256): 32-row x 64-byte staging boxes (64-byte swizzle), so
  // that the shared memory holds a fourth operand stage
  static constexpr bool NARROW = SFST && BN == 256;
  static constexpr int STAGES = (BN == 256) ? (NARROW ? 4 : 3) : 5;
  // scale atoms: in scale-warp mode a ring of their own, SFR k-tiles deep (filled by a second
  // producer thread ahead of the operand ring, so the scale warps finish before the operands
  // land); otherwise part of each operand stage
  static constexpr int SFR = SFST ? (NARROW ? 3 : 6) : STAGES;
  // epilogue staging: per epilogue warp, STG boxes of 32 rows x 128 bytes for TMA stores (one in
  // scale-warp mode, whose scale ring takes the shared memory of the second; one of 32 rows x 64
  // bytes in the NARROW mode)
  static constexpr int STG = SFST ? 1 : (BN == 256) ? 2 : 1;
  static constexpr int BOX_BYTES = NARROW ? 32 * 64 : 32 * 128;
  static constexpr int A_BYTES = BM * KT_BYTES;
  static constexpr int B_BYTES = BN * KT_BYTES;
  static constexpr int SFA_BYTES = 4 * 512;
  static constexpr int SFB_BYTES = (BN / 128) * 4 * 512;
  // Tensor memory: two accumulator buffers and two per-MMA scale slots (A: 4 columns, B: 4
  // per 128 columns of N).  The tensor pipe executes copies and MMAs of one thread in order,
  // so a scale slot can be rewritten for the next-but-one MMA.  When 2 accumulators and the slots
  // exceed the 512 columns, the buffers overlap: buffer 1 starts ACC_OVERLAP columns before
  // buffer 0 ends, and the epilogue drains that strip first and releases it early.
  static constexpr int SF_SLOT = 4 + 4 * (BN / 128);
  // a stored k-tile: the A scales of its four K = 64 blocks (4 columns each), then their B scales
  // (4 columns per 128 rows of B each)
  static constexpr int SF_KT = 4 * 4 + 4 * 4 * (BN / 128);
  static constexpr int SF_COLS = SFST ? 2 * SF_KT : 2 * SF_SLOT;
  static constexpr int TMEM_COLS = 512;
  static constexpr int ACC_OVERLAP = (2 * ACC_W + SF_COLS > TMEM_COLS) ? (2 * ACC_W + SF_COLS - TMEM_COLS) : 0;
  static constexpr int ACC1_BASE = ACC_W - ACC_OVERLAP;
  static constexpr int SF_BASE = ACC1_BASE + ACC_W;
  static_assert(SF_BASE + SF_COLS <= TMEM_COLS, "tensor memory budget");
  static_assert(ACC_OVERLAP % 32 == 0 || ACC_OVERLAP < 32, "the shared strip is whole 32-column chunks");
  static_assert(ACC_OVERLAP <= 96, "at most three chunks of a half are shared");
  // chunks of a half (of BN / 2 columns) in the strip shared by the two buffers
  static constexpr int OVL_CHUNKS = (ACC_OVERLAP + 31) / 32;
  static_assert(!OWN || BN == 128, "two accumulators only at BN = 128");
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_SFB = OFF_SFA + SFR * SFA_BYTES;
  static constexpr int OFF_STG = OFF_SFB + SFR * SFB_BYTES;  // 1024-aligned
  static constexpr int OFF_BAR = OFF_STG + 8 * STG * BOX_BYTES;
  static_assert(OFF_STG % 1024 == 0, "staging boxes start on a swizzle-pattern boundary");
  // full[S], empty[S], accf[2], acce[2], ovf[2], drain, sf_full[2], sf_landed[SFR], sf_free[SFR]
  static constexpr int NUM_BARS = 2 * STAGES + 9 + 2 * SFR;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  // the dynamic shared window starts 1024-byte aligned (checked in the kernel)
  static constexpr int SMEM = OFF_MISC + 32;
  static_assert(SMEM <= 232448, "shared memory budget");
};

// ---------------------------------------------------------------------------------------- kernel
// FP8: the comparison operands (E4M3 codes, one E8M0 scale per 32 elements): a 128-byte k-tile
// holds 128 elements and one scale atom per 128 rows, copied once per k-tile; its four K = 32
// MMAs pick their scale byte by id.  No residual loop, no tensor scales (alpha = 1).
template <int BN, bool FP8, bool OWN = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    w4a4_rac_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_ar,
                         const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_ws,
                         const __grid_constant__ CUtensorMap tm_y, const GemmArgs args) {
  constexpr bool SFST = !FP8 && !OWN;  // scale factors stored by the scale warps
  using C = Cfg<BN, OWN, SFST>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  unsigned char* smem = smem_raw;
  if ((sbase & 1023u) != 0) {  // the swizzled tiles need a 1024-byte aligned window
    if (threadIdx.x == 0) report_status(args.status, kErrAlign);
    return;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  auto bar_full = [&](int s) { return sbase + C::OFF_BAR + 8u * s; };
  auto bar_empty = [&](int s) { return sbase + C::OFF_BAR + 8u * (C::STAGES + s); };
  auto bar_accf = [&](int a) { return sbase + C::OFF_BAR + 8u * (2 * C::STAGES + a); };      // accumulator ready
  auto bar_acce = [&](int a) { return sbase + C::OFF_BAR + 8u * (2 * C::STAGES + 2 + a); };  // fully drained
  auto bar_ovf = [&](int a) { return sbase + C::OFF_BAR + 8u * (2 * C::STAGES + 4 + a); };   // shared strip drained
  const uint32_t bar_drain = sbase + C::OFF_BAR + 8u * (2 * C::STAGES + 6);
  auto bar_sff = [&](int i) { return sbase + C::OFF_BAR + 8u * (2 * C::STAGES + 7 + i); };  // scale slot stored
  // scale-warp mode: a slot of the scale ring landed / was read by the four scale warps
  auto bar_sfl = [&](int s) { return sbase + C::OFF_BAR + 8u * (2 * C::STAGES + 9 + s); };
  auto bar_sfe = [&](int s) { return sbase + C::OFF_BAR + 8u * (2 * C::STAGES + 9 + C::SFR + s); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  volatile int* prod_issued = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  volatile int* mma_taken = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 12);
  volatile int* sf_issued = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 16);  // scale ring
  volatile int* sf_seen = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 20);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar_accf(a), 1);
      mbar_init(bar_acce(a), 8);
      mbar_init(bar_ovf(a), 4);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_sff(0), 4);
    mbar_init(bar_sff(1), 4);
    for (int s = 0; s < C::SFR; ++s) {
      mbar_init(bar_sfl(s), 1);
      mbar_init(bar_sfe(s), 4);
    }
    *abort_flag = 0;
    *prod_issued = 0;
    *mma_taken = 0;
    *sf_issued = 0;
    *sf_seen = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // ---- tile space
  const bool grouped = args.offsets != nullptr;
  int64_t m_blocks;
  int64_t row_limit;
  if (grouped) {
    const int64_t rows = __ldg(args.offsets + args.E);
    m_blocks = rows / BM;
    row_limit = rows;
    if (rows % BM != 0 || rows > args.rows_capacity || rows < 0) {
      if (threadIdx.x == 0) report_status(args.status, kErrInvalid);
      m_blocks = 0;
    }
  } else {
    m_blocks = args.m_blocks_dense;
    row_limit = args.M;
  }
  const int64_t total_tiles = m_blocks * args.n_blocks;
  const int kt_total = args.kt_main + args.kt_res;
  const uint64_t limit = args.wait_limit_ns;

  // Roles by warpgroup; each first moves its register share (every warp of a warpgroup executes
  // the same setmaxnreg), so the code of each role is compiled within that share.
  if (warp < SF_WARP0) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_CTRL));
  if (warp == 0) {
    // ===================================================================== TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int64_t t = blockIdx.x; t < total_tiles && !*abort_flag; t += gridDim.x) {
        const int64_t mb = t / args.n_blocks;
        const int nb = (int)(t - mb * args.n_blocks);
        const int e = grouped ? segment_weight(args, find_expert(args.offsets, args.E, mb * BM)) : 0;
        for (int kt = 0; kt < kt_total; ++kt) {
          if (!mbar_wait(bar_empty(stage), phase ^ 1u, limit, abort_flag)) {
            report_status(args.status, kErrTimeout);
            *abort_flag = 1;
            break;
          }
          const bool res = kt >= args.kt_main;
          const int kk = res ? kt - args.kt_main : kt;
          // scale atoms of this k-tile: FP4 one per 64 elements (fewer in a partial last tile),
          // FP8 one per 128 elements; at_row = atoms per 128-row block of the operand
          const int k64 = res ? args.k64_res : args.k64_main;
          const int n_at = FP8 ? 1 : min(4, k64 - kk * 4);
          const int64_t at_row = FP8 ? (int64_t)args.kt_main : (int64_t)k64;
          const int64_t at0 = FP8 ? (int64_t)kk : (int64_t)kk * 4;
          const uint32_t sf_bytes = (uint32_t)n_at * 512u;
          mbar_expect_tx(bar_full(stage),
                         (uint32_t)(C::A_BYTES + C::B_BYTES) + (SFST ? 0u : sf_bytes * (1u + BN / 128)));
          tma_load_2d(sbase + C::OFF_A + stage * C::A_BYTES, res ? &tm_ar : &tm_a, kk * KT_BYTES, (int32_t)(mb * BM),
                      bar_full(stage));
          tma_load_3d(sbase + C::OFF_B + stage * C::B_BYTES, res ? &tm_ws : &tm_w, kk * KT_BYTES, nb * BN, e,
                      bar_full(stage));
          if constexpr (!SFST) {
            const uint8_t* sfa = (res ? args.sfa_res : args.sfa) + (mb * at_row + at0) * 512;
            bulk_load(sbase + C::OFF_SFA + stage * C::SFA_BYTES, sfa, sf_bytes, bar_full(stage));
            const uint8_t* sfw = res ? args.sfw_sel + (int64_t)e * args.sfw_sel_slab_bytes
                                     : args.sfw + (int64_t)e * args.sfw_slab_bytes;
#pragma unroll
            for (int rb = 0; rb < BN / 128; ++rb) {
              const uint8_t* src = sfw + ((int64_t)(nb * (BN / 128) + rb) * at_row + at0) * 512;
              bulk_load(sbase + C::OFF_SFB + stage * C::SFB_BYTES + rb * 2048, src, sf_bytes, bar_full(stage));
            }
          }
          ++issued;
          *prod_issued = issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 2) {
    // ===================================================================== scale-ring producer
    // Scale-warp mode: the scale atoms of k-tile g go to ring slot g % SFR once the four scale
    // warps have read that slot's previous contents; the ring runs up to SFR k-tiles ahead.
    if (SFST && lane == 0) {
      int slot = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int64_t t = blockIdx.x; t < total_tiles && !*abort_flag; t += gridDim.x) {
        const int64_t mb = t / args.n_blocks;
        const int nb = (int)(t - mb * args.n_blocks);
        const int e = grouped ? segment_weight(args, find_expert(args.offsets, args.E, mb * BM)) : 0;
        for (int kt = 0; kt < kt_total; ++kt) {
          if (!mbar_wait(bar_sfe(slot), phase ^ 1u, limit, abort_flag)) {
            report_status(args.status, kErrTimeout);
            *abort_flag = 1;
            break;
          }
          const bool res = kt >= args.kt_main;
          const int kk = res ? kt - args.kt_main : kt;
          const int k64 = res ? args.k64_res : args.k64_main;
          const int n_at = min(4, k64 - kk * 4);
          const uint32_t sf_bytes = (uint32_t)n_at * 512u;
          mbar_expect_tx(bar_sfl(slot), sf_bytes * (1u + BN / 128));
          const uint8_t* sfa = (res ? args.sfa_res : args.sfa) + (mb * (int64_t)k64 + kk * 4) * 512;
          bulk_load(sbase + C::OFF_SFA + slot * C::SFA_BYTES, sfa, sf_bytes, bar_sfl(slot));
          const uint8_t* sfw = res ? args.sfw_sel + (int64_t)e * args.sfw_sel_slab_bytes
                                   : args.sfw + (int64_t)e * args.sfw_slab_bytes;
#pragma unroll
          for (int rb = 0; rb < BN / 128; ++rb) {
            const uint8_t* src = sfw + ((int64_t)(nb * (BN / 128) + rb) * k64 + kk * 4) * 512;
            bulk_load(sbase + C::OFF_SFB + slot * C::SFB_BYTES + rb * 2048, src, sf_bytes, bar_sfl(slot));
          }
          ++issued;
          *sf_issued = issued;
          if (++slot == C::SFR) {
            slot = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ===================================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = FP8 ? idesc_fp8(BM, BN) : idesc_fp4(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int taken = 0;
      uint32_t mma_count = 0;
      bool ok = true;
      int64_t tile_idx = 0;
      uint32_t g = 0;  // k-tiles taken so far (the scale ring's sequence)
      for (int64_t t = blockIdx.x; t < total_tiles && ok && !*abort_flag; t += gridDim.x, ++tile_idx) {
        const int acc = (int)(tile_idx & 1);
        const int64_t use = tile_idx >> 1;  // how many times buffer `acc` was used before
        // buffer `acc` fully drained by the epilogue of its previous tile
        if (use >= 1 && !mbar_wait(bar_acce(acc), (uint32_t)((use - 1) & 1), limit, abort_flag)) {
          ok = false;
          break;
        }
        // the strip shared with the other buffer drained by the epilogue of the previous tile
        if (C::ACC_OVERLAP > 0 && tile_idx >= 1 &&
            !mbar_wait(bar_ovf(acc ^ 1), (uint32_t)(((tile_idx - 1) >> 1) & 1), limit, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc ? C::ACC1_BASE : 0);
        for (int kt = 0; kt < kt_total; ++kt) {
          if (!mbar_wait(bar_full(stage), phase, limit, abort_flag)) {
            ok = false;
            break;
          }
          // the scale warps stored this k-tile's scales into slot g & 1
          if (SFST && !mbar_wait(bar_sff(g & 1), (g >> 1) & 1u, limit, abort_flag)) {
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
          const uint32_t a_s = sbase + C::OFF_A + stage * C::A_BYTES;
          const uint32_t b_s = sbase + C::OFF_B + stage * C::B_BYTES;
          const uint32_t sfa_s = sbase + C::OFF_SFA + stage * C::SFA_BYTES;
          const uint32_t sfb_s = sbase + C::OFF_SFB + stage * C::SFB_BYTES;
          if constexpr (FP8) {
            // one scale atom per operand block covers the whole k-tile: copy once, then the
            // four K = 32 MMAs take scale byte j of each row
            const uint32_t sfa_t = tmem_base + (uint32_t)(C::SF_BASE + (mma_count & 1) * C::SF_SLOT);
            const uint32_t sfb_t = sfa_t + 4;
            ++mma_count;
            tc_copy_sf(sfa_t, desc_sf(sfa_s));
#pragma unroll
            for (int rb = 0; rb < BN / 128; ++rb) tc_copy_sf(sfb_t + 4 * rb, desc_sf(sfb_s + rb * 2048));
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tc_mma_fp8(d_tmem, desc_sw128(a_s + 32 * j), desc_sw128(b_s + 32 * j),
                         idesc | idesc_sf_ids((uint32_t)j, (uint32_t)j), sfa_t, sfb_t, (kt | j) != 0 ? 1u : 0u);
          }
          // FP4: each MMA's scale atoms are copied right before it (into alternating slots): the
          // tensor pipe overlaps the copies with the preceding MMA
          // own-scale variant: the residual k-tiles go to the second accumulator, which starts
          // fresh at the first of them
          const uint32_t d_k = d_tmem + ((OWN && res) ? (uint32_t)BN : 0u);
          const int kt_first = (OWN && res) ? args.kt_main : 0;
          if constexpr (SFST) {
            // scales already in tensor memory: A of block j at +4j, B at +16 + 4 (BN / 128) j
            const uint32_t slot = tmem_base + (uint32_t)(C::SF_BASE + (int)(g & 1) * C::SF_KT);
            for (int j = 0; j < nk64; ++j)
              tc_mma_fp4(d_k, desc_sw128(a_s + 32 * j), desc_sw128(b_s + 32 * j), idesc, slot + 4 * j,
                         slot + 16 + 4 * (BN / 128) * j, (kt != kt_first || j != 0) ? 1u : 0u);
          }
          for (int j = 0; j < ((FP8 || SFST) ? 0 : nk64); ++j, ++mma_count) {
            const uint32_t sfa_t = tmem_base + (uint32_t)(C::SF_BASE + (mma_count & 1) * C::SF_SLOT);
            const uint32_t sfb_t = sfa_t + 4;
            tc_copy_sf(sfa_t, desc_sf(sfa_s + j * 512));
#pragma unroll
            for (int rb = 0; rb < BN / 128; ++rb) tc_copy_sf(sfb_t + 4 * rb, desc_sf(sfb_s + rb * 2048 + j * 512));
            tc_mma_fp4(d_k, desc_sw128(a_s + 32 * j), desc_sw128(b_s + 32 * j), idesc, sfa_t, sfb_t,
                       (kt != kt_first || j != 0) ? 1u : 0u);
          }
          tc_commit(bar_empty(stage));
          ++g;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(bar_accf(acc));
      }
      if (!ok) {
        report_status(args.status, kErrTimeout);
        *abort_flag = 1;
      }
    }
  }
  } else if (warp < EPI_WARP0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_SF));
    // ===================================================================== scale warps
    // Warp w stores into lanes [32 (w % 4), +32): lane j takes 16 bytes at 16 j of each 512-byte
    // atom (the scales of rows j, 32 + j, 64 + j, 96 + j) into 4 columns, as the replicating
    // copy would.  Per k-tile g: its stage has landed (full), slot g & 1 is free (the MMAs of
    // k-tile g - 2 are complete: the commit that empties their stage), then 12 atoms -> 48
    // (BN = 256) or 8 atoms -> 32 columns, wait for the stores, arrive on sf_full.
    if constexpr (SFST) {
      const int quad = warp & 3;
      const uint32_t t_lane = tmem_base + ((uint32_t)(quad * 32) << 16);
      uint32_t g = 0;
      int rslot = 0;  // scale-ring slot of k-tile g, and its phase
      uint32_t rphase = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        for (int kt = 0; kt < kt_total; ++kt) {
          // the atoms of k-tile g landed in ring slot rslot: read them into registers and release
          // the slot before waiting for tensor memory, so only the stores follow that wait
          bool w_ok = __all_sync(0xffffffffu, mbar_wait(bar_sfl(rslot), rphase, limit, abort_flag));
          if (w_ok && warp == SF_WARP0 && lane == 0) *sf_seen = (int)g + 1;
          uint32_t r[16 + 16 * (BN / 128)];
          if (w_ok) {
            const uint32_t sfa_s = sbase + C::OFF_SFA + rslot * C::SFA_BYTES + lane * 16;
            const uint32_t sfb_s = sbase + C::OFF_SFB + rslot * C::SFB_BYTES + lane * 16;
            // A scales of the four K = 64 blocks -> columns 0..15; B scales: block j, 128-row group
            // rb -> column 16 + 4 (BN / 128) j + 4 rb
#pragma unroll
            for (int j = 0; j < 4; ++j) ld_shared_v4(sfa_s + j * 512, r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
#pragma unroll
            for (int q = 0; q < 4 * (BN / 128); ++q) {
              const int jb = q / (BN / 128), rb = q % (BN / 128);
              ld_shared_v4(sfb_s + rb * 2048 + jb * 512, r[16 + 4 * q], r[17 + 4 * q], r[18 + 4 * q], r[19 + 4 * q]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_sfe(rslot));
          }
          // tensor-memory slot g & 1 is free once the MMAs of k-tile g - 2 are complete
          if (w_ok && g >= 2) {
            const uint32_t gp = g - 2;
            w_ok = mbar_wait(bar_empty((int)(gp % C::STAGES)), (gp / C::STAGES) & 1u, limit, abort_flag);
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
          const uint32_t slot = t_lane + (uint32_t)(C::SF_BASE + (int)(g & 1) * C::SF_KT);
#pragma unroll
          for (int h = 0; h < 1 + BN / 128; ++h) {
            uint32_t q16[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) q16[i] = r[16 * h + i];
            tmem_st16(slot + 16 * h, q16);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_sff((int)(g & 1)));
          ++g;
          if (++rslot == C::SFR) {
            rslot = 0;
            rphase ^= 1u;
          }
        }
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REG_EPI));
    // ===================================================================== epilogue
    // Eight warps: two per tensor-memory lane quadrant, each owning half of the tile's
    // columns.  A warp drains its columns into registers, releases the accumulator, and only
    // then converts and stores, so the math overlaps the next tile's MMAs.
    constexpr int NCH = C::ACC_W / 64;      // 32-column chunks per warp
    const int quad = warp & 3;              // tensor-memory lanes [32*quad, 32*quad + 32)
    const int half = (warp - EPI_WARP0) >> 2;  // which half of the tile's columns
    float amax = 0.0f;
    int64_t tile_idx = 0;
    for (int64_t t = blockIdx.x; t < total_tiles; t += gridDim.x, ++tile_idx) {
      const int acc = (int)(tile_idx & 1);
      const uint32_t acc_phase = (uint32_t)((tile_idx >> 1) & 1);
      const int64_t mb = t / args.n_blocks;
      const int nb = (int)(t - mb * args.n_blocks);
      const int seg = grouped ? find_expert(args.offsets, args.E, mb * BM) : 0;
      const int e = grouped ? segment_weight(args, seg) : 0;
      // every lane polls (acquire), and all lanes agree on the outcome before the
      // warp-collective tensor-memory loads
      const bool got = __all_sync(0xffffffffu, mbar_wait(bar_accf(acc), acc_phase, limit, abort_flag));
      if (!got) {
        if (lane == 0) {
          report_status(args.status, kErrTimeout);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const int64_t row = mb * BM + quad * 32 + lane;
      // with per-expert row counts, rows past the expert's tokens are padding: a 32-row output
      // box that holds no token row is not stored
      const int64_t rows_e = (grouped && args.expert_rows != nullptr)
                                 ? (int64_t)__ldg(args.offsets + seg) + __ldg(args.expert_rows + seg)
                                 : row_limit;
      const bool row_ok = row < row_limit && row < args.rows_capacity && row < rows_e;
      const float alpha = FP8 ? 1.0f : __fmul_rn(__ldg(args.s_a), __ldg(args.s_w + e));
      // own-scale variant: the residual product's scale (0 when there is no residual loop, so the
      // second accumulator, never written, is not read)
      const bool has_res = OWN && args.kt_res > 0;
      const float alpha_r = has_res ? __fmul_rn(__ldg(args.s_a_res), __ldg(args.s_w + e)) : 0.0f;
      const uint32_t t_row = tmem_base + (uint32_t)(acc ? C::ACC1_BASE : 0) + ((uint32_t)(quad * 32) << 16);
      // chunk i of this warp: plain -> columns half*BN/2 + 32i; SwiGLU -> output features
      // [half*BN/4, ...): chunks 0..NCH/2-1 gate (column (f/64)*128 + f%64), NCH/2.. the up
      // columns 64 further (gate/up interleave of the packed weight).  Own-scale variant: the
      // same for the main accumulator in chunks 0..NCH/2-1 and the residual one (columns + BN)
      // in chunks NCH/2..NCH-1.
      auto chunk_col = [&](int i) -> int {
        if (OWN) {
          const int base = i >= NCH / 2 ? BN : 0;
          const int ii = i % (NCH / 2);
          if (args.epi != 1) return base + half * (BN / 2) + 32 * ii;
          const int f = half * (BN / 4);
          return base + (f / 64) * 128 + (f % 64) + (ii == 1 ? 64 : 0);
        }
        if (args.epi != 1) return half * (BN / 2) + 32 * i;
        const int ii = i % (NCH / 2);
        const int f = half * (BN / 4) + 32 * ii;
        return (f / 64) * 128 + (f % 64) + (i >= NCH / 2 ? 64 : 0);
      };
      // the chunks holding the strip shared with the other buffer are drained and released first:
      // buffer 0's last columns (the last OVL_CHUNKS chunks of half 1), buffer 1's first ones
      // (the first OVL_CHUNKS chunks of half 0)
      auto in_strip = [&](int i) -> bool {
        if (C::ACC_OVERLAP == 0) return false;
        if (acc == 0) return half == 1 && i >= NCH - C::OVL_CHUNKS;
        return half == 0 && i < C::OVL_CHUNKS;
      };
      const bool holds_strip = C::ACC_OVERLAP > 0 && ((acc == 0 && half == 1) || (acc == 1 && half == 0));
      uint32_t v[NCH][32];
      if (holds_strip) {
#pragma unroll
        for (int i = 0; i < NCH; ++i)
          if (in_strip(i)) tmem_ld32(t_row + chunk_col(i), v[i]);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_ovf(acc));
      }
#pragma unroll
      for (int i = 0; i < NCH; ++i)
        if (!in_strip(i)) tmem_ld32(t_row + chunk_col(i), v[i]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_acce(acc));
      if (OWN) {
        // y = alpha * main + alpha_r * residual, the sum in binary32; the values of the
        // SwiGLU / store paths below then come from chunks 0..NCH/2-1 with alpha 1
#pragma unroll
        for (int i = 0; i < NCH / 2; ++i)
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const float m = __fmul_rn(__uint_as_float(v[i][k]), alpha);
            const float r = has_res ? __fmul_rn(__uint_as_float(v[NCH / 2 + i][k]), alpha_r) : 0.0f;
            v[i][k] = __float_as_uint(__fadd_rn(m, r));
          }
      }
      const float alpha_out = OWN ? 1.0f : alpha;
      // ---- output through shared memory: each box is 32 rows x 128 bytes in the 128-byte
      // swizzled layout (16-byte chunk c of row r at chunk c ^ (r % 8)), stored by one TMA copy
      const uint32_t stg = sbase + C::OFF_STG + (uint32_t)((warp - EPI_WARP0) * C::STG * C::BOX_BYTES);
      const int32_t y0 = (int32_t)(mb * BM + quad * 32);
      const bool box_live = (int64_t)y0 < rows_e;
      auto put_box = [&](int slot, const uint32_t (&w)[32], int32_t x) {
        if constexpr (C::NARROW) {
          // the 128-byte row in two boxes of 32 rows x 64 bytes (64-byte swizzle: 16-byte chunk c
          // of row r at chunk c ^ ((r / 2) % 4)); x advances by 64 bytes of elements
          const int32_t dx = args.out_bf16 ? 32 : 16;
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            if (lane == 0) bulk_wait_group_read<0>();
            __syncwarp();
            const uint32_t rowp = stg + (uint32_t)(lane * 64);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              st_shared_v4(rowp + (uint32_t)((c ^ ((lane >> 1) & 3)) * 16), w[16 * hb + 4 * c],
                           w[16 * hb + 4 * c + 1], w[16 * hb + 4 * c + 2], w[16 * hb + 4 * c + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tm_y, stg, x + hb * dx, y0);
              bulk_commit_group();
            }
          }
          return;
        }
        // at most STG - 1 earlier stores of this warp may still be reading the staging boxes
        if (lane == 0) bulk_wait_group_read<C::STG - 1>();
        __syncwarp();
        const uint32_t rowp = stg + (uint32_t)(slot * C::BOX_BYTES + lane * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(rowp + (uint32_t)(((c ^ (lane & 7)) * 16)), w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_y, stg + (uint32_t)(slot * C::BOX_BYTES), x, y0);
          bulk_commit_group();
        }
      };
      // output chunks: all NCH of the plain accumulator; the first NCH / 2 in the own-scale
      // variant (already combined above)
      constexpr int NOUT = OWN ? NCH / 2 : NCH;
      if (!box_live) {
        // padding only: nothing to store
      } else if (args.epi == 2) {
        // weighted combine: this row's products w * bf16(alpha * acc) go into its token's binary32
        // row by vector atomic adds (the order of a token's k terms is not fixed)
        const int32_t pair = row_ok ? __ldg(args.row_pair + row) : -1;
        if (pair >= 0 && (int64_t)pair >= args.n_pairs) report_status(args.status, kErrInvalid);
        if (pair >= 0 && (int64_t)pair < args.n_pairs) {
          const float wt = __ldg(args.topk_w + pair);
          float* dst = args.comb + (int64_t)(pair / args.k_top) * args.ld_comb + (int64_t)nb * BN;
#pragma unroll
          for (int i = 0; i < NOUT; ++i)
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              float o[4];
#pragma unroll
              for (int z = 0; z < 4; ++z)
                o[z] = __fmul_rn(wt, bf16_round(__fmul_rn(__uint_as_float(v[i][4 * q + z]), alpha_out)));
              red_add_v4(dst + chunk_col(i) + 4 * q, o);
            }
        }
      } else if (args.epi == 0 && args.out_bf16) {
        // 64 columns per box
#pragma unroll
        for (int b = 0; b < NOUT / 2; ++b) {
          uint32_t w[32];
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int k = 0; k < 16; ++k)
              w[16 * h + k] = pack_bf16x2(__fmul_rn(__uint_as_float(v[2 * b + h][2 * k]), alpha_out),
                                          __fmul_rn(__uint_as_float(v[2 * b + h][2 * k + 1]), alpha_out));
          put_box(b % C::STG, w, (int32_t)(nb * BN + half * (BN / 2) + 64 * b));
        }
      } else if (args.epi == 0) {
        // fp32: 32 columns per box
#pragma unroll
        for (int b = 0; b < NOUT; ++b) {
          uint32_t w[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) w[k] = __float_as_uint(__fmul_rn(__uint_as_float(v[b][k]), alpha_out));
          put_box(b % C::STG, w, (int32_t)(nb * BN + half * (BN / 2) + 32 * b));
        }
      } else if (!OWN) {
        // SwiGLU (BN = 256): this warp's 64 output features form one box
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < NCH / 2; ++i)
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            float hv[2];
#pragma unroll
            for (int z = 0; z < 2; ++z) {
              const int j = 2 * k + z;
              const float gv = bf16_round(__fmul_rn(__uint_as_float(v[i][j]), alpha));
              const float uv = bf16_round(__fmul_rn(__uint_as_float(v[NCH / 2 + i][j]), alpha));
              // silu(g) = g / (1 + e^-g); e^-g overflowing to inf gives -0 (the limit)
              const float sg = __fdividef(gv, 1.0f + __expf(-gv));
              hv[z] = bf16_round(sg * uv);
              if (row_ok) amax = fmaxf(amax, fabsf(hv[z]));
            }
            w[16 * i + k] = pack_bf16x2(hv[0], hv[1]);
          }
        put_box(0, w, (int32_t)(nb * (BN / 2) + half * (BN / 4)));
      } else {
        // SwiGLU of the own-scale variant (BN = 128): this warp's 32 output features (gate in
        // chunk 0, up in chunk 1) form one box of 32 rows x 64 bytes, row-major (the output
        // tensor map of this mode has 64-byte boxes and no swizzle)
        uint32_t w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          float hv[2];
#pragma unroll
          for (int z = 0; z < 2; ++z) {
            const int j = 2 * k + z;
            const float gv = bf16_round(__uint_as_float(v[0][j]));
            const float uv = bf16_round(__uint_as_float(v[1][j]));
            const float sg = __fdividef(gv, 1.0f + __expf(-gv));
            hv[z] = bf16_round(sg * uv);
            if (row_ok) amax = fmaxf(amax, fabsf(hv[z]));
          }
          w[k] = pack_bf16x2(hv[0], hv[1]);
        }
        if (lane == 0) bulk_wait_group_read<C::STG - 1>();
        __syncwarp();
        const uint32_t rowp = stg + (uint32_t)(lane * 64);
#pragma unroll
        for (int c = 0; c < 4; ++c) st_shared_v4(rowp + 16u * c, w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_y, stg, (int32_t)(nb * (BN / 2) + half * (BN / 4)), y0);
          bulk_commit_group();
        }
      }
    }
    if (lane == 0) bulk_wait_group_all();  // this warp's stores complete before exit
    if (args.epi != 0 && args.amax_out != nullptr) {
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
      // copies issued but never consumed by the MMA thread
      for (int i = *mma_taken; i < *prod_issued; ++i)
        mbar_wait(bar_full(i % C::STAGES), (uint32_t)((i / C::STAGES) & 1), limit, nullptr);
    }
    if (SFST && warp == 2 && lane == 0) {
      // scale-ring copies issued but never seen landed by the scale warps
      for (int i = *sf_seen; i < *sf_issued; ++i)
        mbar_wait(bar_sfl(i % C::SFR), (uint32_t)((i / C::SFR) & 1), limit, nullptr);
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
  }
}

// A kernel that only runs the bounded wait on a barrier nothing completes (self-test of the
// timeout path: it must come back with NVFP4_ERR_TIMEOUT in *status).
__global__ void wait_selftest_kernel(uint64_t limit_ns, int32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (!mbar_wait(b, 0, limit_ns, nullptr)) report_status(status, kErrTimeout);
  }
}

}  // namespace tc

size_t gemm_smem_bytes(int bn) {
  return bn == 256 ? (size_t)tc::Cfg<256, false, true>::SMEM : (size_t)tc::Cfg<128, false, true>::SMEM;
}

template <int BN, bool FP8, bool OWN = false>
static cudaError_t launch_gemm_t(const CUtensorMap& tm_a, const CUtensorMap& tm_ar, const CUtensorMap& tm_w,
                                 const CUtensorMap& tm_ws, const CUtensorMap& tm_y, const GemmArgs& args, int grid,
                                 cudaStream_t st) {
  constexpr int smem = tc::Cfg<BN, OWN, !FP8 && !OWN>::SMEM;
  cudaError_t e =
      cudaFuncSetAttribute(tc::w4a4_rac_gemm_kernel<BN, FP8, OWN>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // the warpgroups' setmaxnreg shares are drawn from the registers the CTA is launched with: a
  // build whose launch count falls short would leave setmaxnreg.inc waiting, so it is refused
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, tc::w4a4_rac_gemm_kernel<BN, FP8, OWN>);
  if (e != cudaSuccess) return e;
  if ((int64_t)fa.numRegs * tc::NUM_THREADS < 128ll * (tc::REG_CTRL + tc::REG_SF) + 256ll * tc::REG_EPI)
    return cudaErrorInvalidConfiguration;
  tc::w4a4_rac_gemm_kernel<BN, FP8, OWN><<<grid, tc::NUM_THREADS, smem, st>>>(tm_a, tm_ar, tm_w, tm_ws, tm_y, args);
  return cudaGetLastError();
}

cudaError_t launch_gemm(int bn, const CUtensorMap& tm_a, const CUtensorMap& tm_ar, const CUtensorMap& tm_w,
                        const CUtensorMap& tm_ws, const CUtensorMap& tm_y, const GemmArgs& args, int grid,
                        cudaStream_t st) {
  if (args.own_res_scale) {
    if (bn != 128 || args.fp8) return cudaErrorInvalidValue;
    return launch_gemm_t<128, false, true>(tm_a, tm_ar, tm_w, tm_ws, tm_y, args, grid, st);
  }
  if (bn == 256)
    return args.fp8 ? launch_gemm_t<256, true>(tm_a, tm_ar, tm_w, tm_ws, tm_y, args, grid, st)
                    : launch_gemm_t<256, false>(tm_a, tm_ar, tm_w, tm_ws, tm_y, args, grid, st);
  if (bn == 128)
    return args.fp8 ? launch_gemm_t<128, true>(tm_a, tm_ar, tm_w, tm_ws, tm_y, args, grid, st)
                    : launch_gemm_t<128, false>(tm_a, tm_ar, tm_w, tm_ws, tm_y, args, grid, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, int32_t* status, cudaStream_t st) {
  tc::wait_selftest_kernel<<<1, 32, 0, st>>>(limit_ns, status);
  return cudaGetLastError();
}

}  // namespace nvfp4
