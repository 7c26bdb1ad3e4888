// W4A4 + RAC GEMM on CTA pairs: one tcgen05 MMA covers a 256 x 256 output tile over the two
// SMs of a cluster (cta_group::2).
//
//   Y = s_a * s_w * ( Q(X) Q(W)^T + Q(R_sel) Q(W_sel)^T )      (same arithmetic as gemm.cu)
//
// Why pairs: per k-tile a single-SM 128 x 256 tile needs 48 KB of operands (A 16 KB, B 32 KB);
// with two SMs sharing the B tile each SM brings A 16 KB and half of B (16 KB) for the same
// 128 x 256 share of the work, so the same shared memory holds four stages instead of three and
// every stage covers as much work with a third fewer bytes from L2 / HBM.  The pair's MMAs, the
// scale-factor copies into tensor memory and the commits are issued by one thread of the leader
// CTA for both SMs.
//
// Structure (both CTAs of a pair run the same warp roles, 320 threads):
//   warp 0      TMA producer of its own CTA: its 128 rows of A, its 128 rows of the pair's 256
//               B rows, its A scale atoms and the B scale atoms of all 256 rows (each SM's tensor
//               memory holds the scales of the whole N tile), into a STAGES-deep ring; the copies
//               complete on its own CTA's barrier.
//   warp 1      leader: tensor memory (allocated for the pair) and the MMA-issuing thread, which
//               waits for its own stage and the follower's, copies the scale atoms of both CTAs
//               (tcgen05.cp.cta_group::2) and issues the pair MMA (M = 256, N = 256, K = 64);
//               commits go to both CTAs' barriers (multicast).  follower: relays "stage full" to
//               the leader with a remote mbarrier arrive, so each CTA only ever waits for its own
//               copies.
//   warps 2..9  epilogue of the CTA's 128 rows, as in gemm.cu; "accumulator drained" goes to the
//               leader's barriers (remote arrive from the follower).
// Grouped (MoE) tiles pair two 128-row blocks of the same expert segment; where a segment has an
// odd number of blocks the follower's half runs past the segment and its rows are not stored.
// Every wait is bounded by a wall-clock limit; on expiry the kernel records NVFP4_ERR_TIMEOUT and
// both CTAs leave through the same teardown: drain their own copies, the leader its MMAs, a
// cluster barrier, then the pair frees tensor memory.
// No load in this file uses cluster multicast: each CTA loads its own operands.
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace nvfp4 {
namespace tc2 {

using namespace tc;

constexpr int BM = 128;        // rows per CTA
constexpr int BN = 256;        // columns of the pair tile
constexpr int KT_BYTES = 128;  // bytes of one row per k-tile: 256 FP4 elements
constexpr int NUM_THREADS = 320;
constexpr int STAGES = 4;
constexpr int STG = 2;                    // epilogue staging boxes per warp
constexpr int BOX_BYTES = 32 * 128;
constexpr int A_BYTES = BM * KT_BYTES;    // 16 KB
constexpr int B_BYTES = (BN / 2) * KT_BYTES;  // 16 KB: this CTA's half of the B rows
constexpr int SFA_BYTES = 4 * 512;
constexpr int SFB_BYTES = 2 * 4 * 512;    // scale atoms of all 256 B rows
constexpr int SF_SLOT = 4 + 8;
constexpr int SF_COLS = 2 * SF_SLOT;
constexpr int TMEM_COLS = 512;
constexpr int ACC_OVERLAP = 2 * BN + SF_COLS - TMEM_COLS;  // 24
constexpr int ACC1_BASE = BN - ACC_OVERLAP;
constexpr int SF_BASE = ACC1_BASE + BN;
static_assert(SF_BASE + SF_COLS <= TMEM_COLS, "tensor memory budget");
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
constexpr int OFF_STG = OFF_SFB + STAGES * SFB_BYTES;  // 1024-aligned
constexpr int OFF_BAR = OFF_STG + 8 * STG * BOX_BYTES;
// full[S], peer_full[S], empty[S], accf[2], acce[2], ovf[2], drain
constexpr int NUM_BARS = 3 * STAGES + 7;
constexpr int OFF_SEG = OFF_BAR + NUM_BARS * 8;          // pair-tile prefix over the segments
constexpr int OFF_MISC = OFF_SEG + (kMaxRouteExperts + 1) * 4;
constexpr int SMEM = OFF_MISC + 32;
static_assert(SMEM <= 232448, "shared memory budget");
static_assert(OFF_STG % 1024 == 0, "staging boxes need 1024-byte alignment");

__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
// bounded wait on a barrier that other CTAs of the cluster arrive on (cluster-scope acquire)
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                                  volatile int* abort_flag) {
  const uint32_t hint = limit_ns < 1000000ull ? (uint32_t)limit_ns : 1000000u;
  if (mbar_try_wait_cluster(bar, parity, hint)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity, hint)) return true;
    if (abort_flag != nullptr && *abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc2_copy_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tc2_mma_fp4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                            uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}
// arrive on the barrier at this shared-memory offset in both CTAs of the pair once every MMA and
// copy issued so far by this thread has completed
__device__ __forceinline__ void tc2_commit_both(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
          bar)
      : "memory");
}
__device__ __forceinline__ void tc2_commit_local(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// weight slab of a segment (segment_weight in gemm.cu)
__device__ __forceinline__ int seg_weight(const GemmArgs& args, int seg) {
  if (args.seg_expert == nullptr) return seg;
  const int e = __ldg(args.seg_expert + seg);
  if (e < 0 || e >= args.n_weights) {
    report_status(args.status, kErrInvalid);
    return 0;
  }
  return e;
}

// A pair tile: rows [r0, r0 + 256) of segment `seg` (rows below row_end are stored), N block nb.
struct PairTile {
  int64_t r0;
  int64_t row_end;  // first row not to store (segment end, or past the token rows)
  int seg;
  int e;
  int nb;
};

__global__ void __launch_bounds__(NUM_THREADS, 1)
    w4a4_rac_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_ar,
                              const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_ws,
                              const __grid_constant__ CUtensorMap tm_y, const GemmArgs args) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  unsigned char* smem = smem_raw;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank();  // 0: leader, 1: follower
  const bool leader = rank == 0;
  const bool aligned = (sbase & 1023u) == 0;  // same in both CTAs of the pair

  auto bar_full = [&](int s) { return sbase + OFF_BAR + 8u * s; };
  auto bar_peer = [&](int s) { return sbase + OFF_BAR + 8u * (STAGES + s); };
  auto bar_empty = [&](int s) { return sbase + OFF_BAR + 8u * (2 * STAGES + s); };
  auto bar_accf = [&](int a) { return sbase + OFF_BAR + 8u * (3 * STAGES + a); };
  auto bar_acce = [&](int a) { return sbase + OFF_BAR + 8u * (3 * STAGES + 2 + a); };
  auto bar_ovf = [&](int a) { return sbase + OFF_BAR + 8u * (3 * STAGES + 4 + a); };
  const uint32_t bar_drain = sbase + OFF_BAR + 8u * (3 * STAGES + 6);
  int32_t* seg_prefix = reinterpret_cast<int32_t*>(smem + OFF_SEG);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  volatile int* prod_issued = reinterpret_cast<volatile int*>(smem + OFF_MISC + 8);
  volatile int* n_tiles_s = reinterpret_cast<volatile int*>(smem + OFF_MISC + 16);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_peer(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar_accf(a), 1);
      mbar_init(bar_acce(a), 16);  // 8 epilogue warps in each CTA
      mbar_init(bar_ovf(a), 8);    // 4 in each CTA
    }
    mbar_init(bar_drain, 1);
    *abort_flag = aligned ? 0 : 1;
    *prod_issued = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (!aligned) report_status(args.status, kErrAlign);
  }
  // ---- tile space (every CTA computes it; both CTAs of a pair get the same answer)
  const bool grouped = args.offsets != nullptr;
  int64_t row_limit;
  int n_tiles = 0;
  if (grouped) {
    const int64_t rows = __ldg(args.offsets + args.E);
    row_limit = rows;
    const bool ok = rows % BM == 0 && rows <= args.rows_capacity && rows >= 0 && args.E <= kMaxRouteExperts;
    if (warp == 2) {
      // pair tiles of each segment: ceil(blocks / 2); prefix in shared memory
      int carry = 0;
      for (int base = 0; ok && base < args.E; base += 32) {
        const int i = base + lane;
        int t = 0;
        if (i < args.E) {
          const int64_t a0 = __ldg(args.offsets + i), a1 = __ldg(args.offsets + i + 1);
          const bool good = a0 >= 0 && a1 >= a0 && a1 <= rows && a0 % BM == 0;
          if (!good) report_status(args.status, kErrInvalid);
          t = good ? (int)(((a1 - a0) / BM + 1) / 2) : 0;
        }
        int incl = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        if (i < args.E) seg_prefix[i] = carry + incl - t;
        carry += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) {
        if (!ok) report_status(args.status, kErrInvalid);
        *n_tiles_s = ok ? carry * args.n_blocks : 0;
      }
    }
  } else {
    row_limit = args.M;
    if (threadIdx.x == 64) *n_tiles_s = ((args.m_blocks_dense + 1) / 2) * args.n_blocks;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  n_tiles = *n_tiles_s;
  const int kt_total = args.kt_main + args.kt_res;
  const uint64_t limit = args.wait_limit_ns;
  const int pair = (int)(blockIdx.x >> 1);
  const int n_pairs = (int)(gridDim.x >> 1);

  auto tile_of = [&](int t) -> PairTile {
    PairTile pt;
    const int pm = t / args.n_blocks;
    pt.nb = t - pm * args.n_blocks;
    if (grouped) {
      int lo = 0, hi = args.E - 1;
      while (lo < hi) {  // last segment whose first pair tile is <= pm
        const int mid = (lo + hi + 1) >> 1;
        if (seg_prefix[mid] <= pm) lo = mid;
        else hi = mid - 1;
      }
      pt.seg = lo;
      pt.e = seg_weight(args, lo);
      const int64_t a0 = __ldg(args.offsets + lo), a1 = __ldg(args.offsets + lo + 1);
      pt.r0 = a0 + (int64_t)(pm - seg_prefix[lo]) * (2 * BM);
      int64_t end = a1;  // the segment's end, or its last token row
      if (args.expert_rows != nullptr) end = min(end, a0 + (int64_t)__ldg(args.expert_rows + lo));
      pt.row_end = end;
    } else {
      pt.seg = 0;
      pt.e = 0;
      pt.r0 = (int64_t)pm * (2 * BM);
      pt.row_end = row_limit;
    }
    return pt;
  };

  if (warp == 0) {
    // ===================================================================== TMA producer (own CTA)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int t = pair; t < n_tiles && !*abort_flag; t += n_pairs) {
        const PairTile pt = tile_of(t);
        const int64_t my_row = pt.r0 + (int64_t)rank * BM;
        for (int kt = 0; kt < kt_total; ++kt) {
          if (!mbar_wait_cluster(bar_empty(stage), phase ^ 1u, limit, abort_flag)) {
            if (!*abort_flag) report_status(args.status, kErrTimeout);
            *abort_flag = 1;
            break;
          }
          const bool res = kt >= args.kt_main;
          const int kk = res ? kt - args.kt_main : kt;
          const int k64 = res ? args.k64_res : args.k64_main;
          const int n_at = min(4, k64 - kk * 4);
          const uint32_t sf_bytes = (uint32_t)n_at * 512u;
          mbar_expect_tx(bar_full(stage), (uint32_t)(A_BYTES + B_BYTES) + sf_bytes * 3u);
          tma_load_2d(sbase + OFF_A + stage * A_BYTES, res ? &tm_ar : &tm_a, kk * KT_BYTES, (int32_t)my_row,
                      bar_full(stage));
          tma_load_3d(sbase + OFF_B + stage * B_BYTES, res ? &tm_ws : &tm_w, kk * KT_BYTES,
                      pt.nb * BN + (int)rank * (BN / 2), pt.e, bar_full(stage));
          // A scales of this CTA's 128 rows (a whole atom row of the activation layout)
          const int64_t a_block = my_row / BM;
          const uint8_t* sfa = (res ? args.sfa_res : args.sfa) + (a_block * k64 + kk * 4) * 512;
          if (a_block < args.rows_capacity / BM) {
            bulk_load(sbase + OFF_SFA + stage * SFA_BYTES, sfa, sf_bytes, bar_full(stage));
          } else {
            // past the buffer (the follower's half of a last pair): no scales to read, but the
            // byte count must still complete: load this CTA's first rows' atoms instead (never used)
            bulk_load(sbase + OFF_SFA + stage * SFA_BYTES, (res ? args.sfa_res : args.sfa) + kk * 4 * 512, sf_bytes,
                      bar_full(stage));
          }
          const uint8_t* sfw = res ? args.sfw_sel + (int64_t)pt.e * args.sfw_sel_slab_bytes
                                   : args.sfw + (int64_t)pt.e * args.sfw_slab_bytes;
#pragma unroll
          for (int rb = 0; rb < 2; ++rb) {
            const uint8_t* src = sfw + ((int64_t)(pt.nb * 2 + rb) * k64 + kk * 4) * 512;
            bulk_load(sbase + OFF_SFB + stage * SFB_BYTES + rb * 2048, src, sf_bytes, bar_full(stage));
          }
          ++issued;
          *prod_issued = issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1 && !leader) {
    // ===================================================================== follower relay
    if (lane == 0) {
      const uint32_t peer_bar0 = map_to_rank(bar_peer(0), 0);
      int stage = 0;
      uint32_t phase = 0;
      for (int t = pair; t < n_tiles && !*abort_flag; t += n_pairs) {
        bool ok = true;
        for (int kt = 0; kt < kt_total; ++kt) {
          if (!mbar_wait(bar_full(stage), phase, limit, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_remote(peer_bar0 + 8u * stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) {
          if (!*abort_flag) report_status(args.status, kErrTimeout);
          *abort_flag = 1;
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ===================================================================== MMA issuer (leader)
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_fp4(2 * BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t mma_count = 0;
      bool ok = true;
      int64_t tile_idx = 0;
      for (int t = pair; t < n_tiles && ok && !*abort_flag; t += n_pairs, ++tile_idx) {
        const int acc = (int)(tile_idx & 1);
        const int64_t use = tile_idx >> 1;
        if (use >= 1 && !mbar_wait_cluster(bar_acce(acc), (uint32_t)((use - 1) & 1), limit, abort_flag)) {
          ok = false;
          break;
        }
        if (tile_idx >= 1 &&
            !mbar_wait_cluster(bar_ovf(acc ^ 1), (uint32_t)(((tile_idx - 1) >> 1) & 1), limit, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc ? ACC1_BASE : 0);
        for (int kt = 0; kt < kt_total; ++kt) {
          if (!mbar_wait(bar_full(stage), phase, limit, abort_flag) ||
              !mbar_wait_cluster(bar_peer(stage), phase, limit, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const bool res = kt >= args.kt_main;
          const int kk = res ? kt - args.kt_main : kt;
          const int k64 = res ? args.k64_res : args.k64_main;
          const int nk64 = min(4, k64 - kk * 4);
          const uint32_t a_s = sbase + OFF_A + stage * A_BYTES;
          const uint32_t b_s = sbase + OFF_B + stage * B_BYTES;
          const uint32_t sfa_s = sbase + OFF_SFA + stage * SFA_BYTES;
          const uint32_t sfb_s = sbase + OFF_SFB + stage * SFB_BYTES;
          for (int j = 0; j < nk64; ++j, ++mma_count) {
            const uint32_t sfa_t = tmem_base + (uint32_t)(SF_BASE + (mma_count & 1) * SF_SLOT);
            const uint32_t sfb_t = sfa_t + 4;
            tc2_copy_sf(sfa_t, desc_sf(sfa_s + j * 512));
            tc2_copy_sf(sfb_t, desc_sf(sfb_s + j * 512));
            tc2_copy_sf(sfb_t + 4, desc_sf(sfb_s + 2048 + j * 512));
            tc2_mma_fp4(d_tmem, desc_sw128(a_s + 32 * j), desc_sw128(b_s + 32 * j), idesc, sfa_t, sfb_t,
                        (kt | j) != 0 ? 1u : 0u);
          }
          tc2_commit_both(bar_empty(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc2_commit_both(bar_accf(acc));
      }
      if (!ok) {
        if (!*abort_flag) report_status(args.status, kErrTimeout);
        *abort_flag = 1;
      }
    }
  } else {
    // ===================================================================== epilogue (own rows)
    constexpr int NCH = BN / 64;      // 32-column chunks per warp
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t acce_leader = map_to_rank(bar_acce(0), 0);
    const uint32_t ovf_leader = map_to_rank(bar_ovf(0), 0);
    float amax = 0.0f;
    int64_t tile_idx = 0;
    for (int t = pair; t < n_tiles; t += n_pairs, ++tile_idx) {
      const PairTile pt = tile_of(t);
      const int acc = (int)(tile_idx & 1);
      const uint32_t acc_phase = (uint32_t)((tile_idx >> 1) & 1);
      const bool got = __all_sync(0xffffffffu, mbar_wait_cluster(bar_accf(acc), acc_phase, limit, abort_flag));
      if (!got) {
        if (lane == 0) {
          if (!*abort_flag) report_status(args.status, kErrTimeout);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const int64_t base_row = pt.r0 + (int64_t)rank * BM;
      const int64_t row = base_row + quad * 32 + lane;
      const bool row_ok = row < pt.row_end && row < row_limit && row < args.rows_capacity;
      const float alpha = __fmul_rn(__ldg(args.s_a), __ldg(args.s_w + pt.e));
      const uint32_t t_row = tmem_base + (uint32_t)(acc ? ACC1_BASE : 0) + ((uint32_t)(quad * 32) << 16);
      auto chunk_col = [&](int i) -> int {
        if (args.epi == 0) return half * (BN / 2) + 32 * i;
        const int ii = i % (NCH / 2);
        const int f = half * (BN / 4) + 32 * ii;
        return (f / 64) * 128 + (f % 64) + (i >= NCH / 2 ? 64 : 0);
      };
      int ovl_i = -1;
      if (acc == 0 && half == 1) ovl_i = NCH - 1;
      if (acc == 1 && half == 0) ovl_i = 0;
      uint32_t v[NCH][32];
      if (ovl_i >= 0) {
#pragma unroll
        for (int i = 0; i < NCH; ++i)
          if (i == ovl_i) tmem_ld32(t_row + chunk_col(i), v[i]);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(ovf_leader + 8u * acc);
      }
#pragma unroll
      for (int i = 0; i < NCH; ++i)
        if (i != ovl_i) tmem_ld32(t_row + chunk_col(i), v[i]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acce_leader + 8u * acc);
      const uint32_t stg = sbase + OFF_STG + (uint32_t)((warp - 2) * STG * BOX_BYTES);
      const int32_t y0 = (int32_t)(base_row + quad * 32);
      // segments are 128-row aligned and boxes 32-row aligned, so a box lies wholly inside or
      // wholly past its segment: the follower's half past a segment's end stores nothing
      const bool box_live = (int64_t)y0 < pt.row_end && (int64_t)y0 < row_limit;
      auto put_box = [&](int slot, const uint32_t (&w)[32], int32_t x) {
        if (lane == 0) bulk_wait_group_read<STG - 1>();
        __syncwarp();
        const uint32_t rowp = stg + (uint32_t)(slot * BOX_BYTES + lane * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(rowp + (uint32_t)(((c ^ (lane & 7)) * 16)), w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_y, stg + (uint32_t)(slot * BOX_BYTES), x, y0);
          bulk_commit_group();
        }
      };
      if (!box_live) {
      } else if (args.epi == 0 && args.out_bf16) {
#pragma unroll
        for (int b = 0; b < NCH / 2; ++b) {
          uint32_t w[32];
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int k = 0; k < 16; ++k)
              w[16 * h + k] = pack_bf16x2(__fmul_rn(__uint_as_float(v[2 * b + h][2 * k]), alpha),
                                          __fmul_rn(__uint_as_float(v[2 * b + h][2 * k + 1]), alpha));
          put_box(b % STG, w, (int32_t)(pt.nb * BN + half * (BN / 2) + 64 * b));
        }
      } else if (args.epi == 0) {
#pragma unroll
        for (int b = 0; b < NCH; ++b) {
          uint32_t w[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) w[k] = __float_as_uint(__fmul_rn(__uint_as_float(v[b][k]), alpha));
          put_box(b % STG, w, (int32_t)(pt.nb * BN + half * (BN / 2) + 32 * b));
        }
      } else {
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
              const float sg = __fdividef(gv, 1.0f + __expf(-gv));
              hv[z] = bf16_round(sg * uv);
              if (row_ok) amax = fmaxf(amax, fabsf(hv[z]));
            }
            w[16 * i + k] = pack_bf16x2(hv[0], hv[1]);
          }
        put_box(0, w, (int32_t)(pt.nb * (BN / 2) + half * (BN / 4)));
      }
    }
    if (lane == 0) bulk_wait_group_all();
    if (args.epi != 0 && args.amax_out != nullptr) {
      amax = warp_max(amax);
      if (lane == 0 && amax > 0.0f) atomicMax(reinterpret_cast<unsigned int*>(args.amax_out), __float_as_uint(amax));
    }
  }

  // ---- teardown (both CTAs take the same steps)
  __syncthreads();
  if (*abort_flag) {
    if (warp == 1 && lane == 0 && leader) {
      tc2_commit_local(bar_drain);  // every pair MMA and copy issued by this thread has completed
      mbar_wait(bar_drain, 0, limit, nullptr);
    }
    if (warp == 0 && lane == 0) {
      // this CTA's copies that no role consumed: the last use of each stage it issued into
      const int issued = *prod_issued;
      for (int i = max(0, issued - STAGES); i < issued; ++i)
        mbar_wait(bar_full(i % STAGES), (uint32_t)((i / STAGES) & 1), limit, nullptr);
    }
    __syncthreads();
  }
  tc_fence_before();
  cluster_sync();  // no remote arrive or multicast commit can still target either CTA
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"((uint32_t)TMEM_COLS)
                 : "memory");
  }
}

}  // namespace tc2

size_t gemm_pair_smem_bytes() { return (size_t)tc2::SMEM; }

cudaError_t launch_gemm_pair(const CUtensorMap& tm_a, const CUtensorMap& tm_ar, const CUtensorMap& tm_w,
                             const CUtensorMap& tm_ws, const CUtensorMap& tm_y, const GemmArgs& args, int n_pairs,
                             cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(tc2::w4a4_rac_gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       tc2::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * n_pairs), 1, 1);
  cfg.blockDim = dim3(tc2::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = tc2::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, tc2::w4a4_rac_gemm_pair_kernel, tm_a, tm_ar, tm_w, tm_ws, tm_y, args);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace nvfp4
