// NVFP4 / MXFP4 W4A4 GEMM with the fused low-rank up projection (sm_100a, CTA pairs).
//
// One kernel, two scale flavours: NVFP4 (E4M3 scales per 16 elements, kind::mxf4nvf4
// block16) and MXFP4 (E8M0 power-of-two scales per 32 elements, kind::mxf4 block32).  The
// scales of both sit in the same 128-row x 4-group blocked layout; an MXFP4 block covers
// 128 K elements, so a step carries half as many scale blocks, and each 64-element MMA uses
// two of the four bytes of a TMEM scale column, picked by the scale-factor id of its
// instruction descriptor (and the top bits of its scale addresses).
//
// "SVDQuant 阅读笔记：用少量高精度计算保护 4-bit 扩散模型", §6.1 "算法 2"
// steps 4-8 and eq.(7): the 4-bit product Q(X_hat) Q(R) and the 16-bit branch
// Z L2 are merged before the single write of Y.
//
// B200 design:
//   * clusters of two CTAs on neighbouring SMs compute 256 x 256 output tiles
//     with tcgen05 cta_group::2 MMAs (M = 256: each CTA holds 128 rows of A and
//     128 rows of B; the pair's tensor cores share the B halves, which halves
//     the shared-memory operand traffic per SM against a one-CTA 128 x 256 tile);
//   * persistent clusters each take a contiguous run of tiles, N fastest.  The
//     operands travel through a 3-deep ring of double steps: one slot holds two
//     K steps of 256 E2M1 elements (128 bytes per row) of A and of B, and each
//     operand arrives with ONE 3-D TMA load ([K/256 chunks][rows][128 bytes],
//     two chunks per box).  A TMA load costs the SM's TMA engine a fixed time
//     of the order of a hundred cycles on top of its bytes, so fewer, larger
//     loads stream faster (when K is not a multiple of 256, two 2-D loads per
//     operand and slot).  Every load lands in the issuing CTA's own shared
//     memory and counts on the leader CTA's barrier (no multicast loads).  The
//     operand and scale loads carry an L2 evict-last policy: every A and B tile
//     is read by many clusters, while Y passes through L2 once;
//   * the block scales (E4M3, one per 16 elements; 512-byte "128 rows x 4 groups"
//     blocks) travel in a ring of their own whose slots also hold two main steps
//     (one SFA and one SFB load per slot), loaded two main steps ahead of the
//     operands.  Two copy warps move each step's blocks into one of four rotating
//     TMEM scale buffers with tcgen05.cp, two 64-element k-blocks per warp, so that
//     a step's scales are normally in TMEM before its operand tiles land: a CTA-pair
//     copy holds its issuing thread for about as long as an MMA runs, and neither one
//     thread issuing all twelve copies of a step nor copies waiting for their step's
//     operands keeps pace with the MMAs.  Each CTA holds its 128 rows of A-scales
//     and all 256 columns of B-scales;
//   * the leader's MMA warp waits only for a slot's operands (and, rarely, a
//     step's scales), issues kind::mxf4nvf4 block-scaled MMAs into an fp32 TMEM
//     accumulator and then ceil(r/64) extra ring slots in which the operand slots
//     hold Z (bf16) and L2s (bf16): kind::f16 MMAs add Z L2s^T into the *same*
//     accumulator.  L2s was divided by (g_x g_w) at pack time, so the epilogue's
//     single multiply by g_x g_w scales both terms and Y is written once;
//   * eight epilogue warps per CTA drain TMEM (tcgen05.ld) into registers and
//     release the accumulator at once, then apply g_x g_w and the bias and store
//     bf16 Y from registers while the next tile's MMAs run: each thread writes
//     256 contiguous bytes of its row with 32-byte (one sector) stores that do not
//     allocate in L1, which halves the write requests of 16-byte stores (32 rows
//     per warp instruction).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "svdq_device.cuh"

namespace svdq {
namespace {

constexpr int kBM = 256, kBN = 256;           // pair tile
constexpr int kRows = 128;                    // A rows (and B rows) per CTA
constexpr int kKTile = 256;                   // E2M1 elements per pipeline step
constexpr int kStages = 3;                    // operand ring of double steps (two K steps per slot)
constexpr int kSfStages = 2;                  // scale ring (slots of two main steps)
constexpr int kSfLead = 2;                    // scale loads run this many main steps ahead
constexpr int kCopyWarps = 2;                 // NVFP4: two k-blocks (64 elements each) of a step each
constexpr int kProdWarp = 0, kMmaWarp = 1, kCopyWarp0 = 2, kEpiWarp0 = 4;
constexpr int kEpiWarps = 8;
// 12 warps: three per SM sub-partition, whose 16K registers then allow 168 per thread
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);   // 384
constexpr uint32_t kABytes = kRows * 128;     // 16 KB
constexpr uint32_t kBBytes = kRows * 128;     // 16 KB
constexpr uint32_t kStageBytes = 2 * (kABytes + kBBytes);  // [A step 0][A step 1][B step 0][B step 1]
constexpr uint32_t kTxMain = 2 * kStageBytes;               // both CTAs
constexpr uint32_t kTxLowRank = 2 * (kABytes + kBBytes);

// Per-flavour sizes: scale blocks (512 bytes = 128 rows x 4 groups) per step and row block.
template <bool MX>
struct Fp4Cfg {
  static constexpr int kSfBlk = MX ? 2 : 4;                       // 4 groups of 32 or of 16
  static constexpr uint32_t kSfaBytes = kSfBlk * 512;            // 128 rows
  static constexpr uint32_t kSfbBytes = 2 * kSfBlk * 512;        // 256 rows (two row blocks)
  static constexpr uint32_t kSfStageBytes = 2 * (kSfaBytes + kSfbBytes);   // two steps: 12 KB (NVFP4), 6 KB (MXFP4)
  static constexpr uint32_t kTxSf = 2 * kSfStageBytes;           // both CTAs
  static constexpr uint32_t kTmemSfStride = 12 * kSfBlk;         // A-scales 4 cols, B-scales 8 per block
};
constexpr uint32_t kTmemCols = 512;
// TMEM columns: accumulator [0, 256); four scale buffers of 48 columns from 256 (A-scales 16,
// B-scales 32), used round-robin by the main steps.
constexpr int kSfBufs = 4;
constexpr uint32_t kTmemSf0 = 256;

// E2M1 x E2M1 with UE8M0 scales (bit 23); sf_id (bits 29-30 for A, 4-5 for B) selects the
// byte of the TMEM scale column where the MMA's scales start.
__host__ __device__ constexpr uint32_t idesc_mxf4(int m, int n, uint32_t sf_id) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(m >> 4) << 24) | (sf_id << 29) | (sf_id << 4);
}
__host__ __device__ constexpr uint32_t idesc_nvf4(int m, int n) {
  // E2M1 x E2M1, UE4M3 scales, K-major A and B, dense
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (0u << 23) |
         (static_cast<uint32_t>(m >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n) {
  // bf16 x bf16 -> fp32, K-major A and B
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

struct SharedTail {
  uint64_t full[kStages];       // operand slot s holds its step's tiles (TMA bytes, both CTAs)
  uint64_t empty[kStages];      // the MMAs that read operand slot s have completed
  uint64_t sf_full[kSfStages];  // scale slot holds its step's blocks
  uint64_t sf_empty[kSfStages]; // the copies that read scale slot have completed (one arrival per copy warp)
  uint64_t sf_ready[kSfBufs];   // TMEM scale buffer b holds its step's scales (one arrival per copy warp)
  uint64_t sf_free[kSfBufs];    // the MMAs that read TMEM scale buffer b have completed
  uint64_t acc_full;
  uint64_t acc_empty;
  uint32_t tmem_base;
  int abort_flag;
};

template <bool MX>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_fp4_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                      const __grid_constant__ CUtensorMap tmap_z, const __grid_constant__ CUtensorMap tmap_l2,
                      GemmParams p) {
  using C = Fp4Cfg<MX>;
  constexpr int kSfBlk = C::kSfBlk;
  constexpr uint32_t kSfaBytes = C::kSfaBytes, kSfStageBytes = C::kSfStageBytes;
  constexpr uint32_t kTxSf = C::kTxSf, kTmemSfStride = C::kTmemSfStride;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sf_smem = smem + kStages * kStageBytes;
  SharedTail* sh = reinterpret_cast<SharedTail*>(sf_smem + kSfStages * kSfStageBytes);
  volatile int* abort_flag = &sh->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();      // 0 = leader of the pair
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
  const int nk_main = (p.K + kKTile - 1) / kKTile;
  const int nk_lr = (p.rank + 63) / 64;
  const int ndbl = (nk_main + 1) / 2;                // operand slots of the 4-bit product per tile
  const int nstg = ndbl + nk_lr;                     // ... plus one per 64-column chunk of Z L2s
  const int kblk64 = p.K / 64;
  const TileSeq tiles(p.num_tiles, p.tiles_n, cluster, nclusters);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&sh->full[s], 1);
      ptx::mbar_init(&sh->empty[s], 1);
    }
    for (int s = 0; s < kSfStages; ++s) {
      ptx::mbar_init(&sh->sf_full[s], 1);
      ptx::mbar_init(&sh->sf_empty[s], kCopyWarps);
    }
    for (int b = 0; b < kSfBufs; ++b) {
      ptx::mbar_init(&sh->sf_ready[b], kCopyWarps);
      ptx::mbar_init(&sh->sf_free[b], 1);
    }
    ptx::mbar_init(&sh->acc_full, 1);
    ptx::mbar_init(&sh->acc_empty, 2 * kEpiWarps);
    sh->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc_pair(&sh->tmem_base, kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();
  ptx::tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  // the set-up above may overlap the end of the prologue kernel; its outputs (A codes and
  // scales, Z) are read only after it has completed
  ptx::griddep_wait();

  if (warp == kProdWarp) {
    // ------------------------------------------------------------ producer (both CTAs)
    // Operand slots of two steps; the scale slot holding main step mi + 1 + kSfLead is loaded
    // before the operand slot whose first step is mi.
    if (lane == 0) {
      ptx::prefetch_tmap(&tmap_a);
      ptx::prefetch_tmap(&tmap_b);
      ptx::prefetch_tmap(&tmap_sfa);
      ptx::prefetch_tmap(&tmap_sfb);
      if (nk_lr > 0) {
        ptx::prefetch_tmap(&tmap_z);
        ptx::prefetch_tmap(&tmap_l2);
      }
      int it = 0, mi = 0, si = 0;
      bool ok = true;
      // A, B and their scales are re-read by the other clusters' tiles: evict them from L2
      // after other lines (Y is written once and stored without allocating in L1)
      const uint64_t keep = ptx::l2_evict_last_policy();
      // scale slot q = (tile j, steps 2u and 2u + 1) holds both steps' blocks: SFA [2 kSfBlk][512 B],
      // then SFB [2 row blocks][2 kSfBlk][512 B]; one TMA load per tensor and slot
      const int npair = (nk_main + 1) / 2;
      const int total_slots = tiles.count * npair;
      auto load_scales = [&](int upto) {
        for (; si < upto && si < total_slots && ok; ++si) {
          const int ss = si % kSfStages;
          if (!wait_bounded(&sh->sf_empty[ss], ((si / kSfStages) & 1) ^ 1u, abort_flag, p.err, kErrSiteGemmEmpty)) {
            ok = false;
            break;
          }
          const int js = si / npair, ks = 2 * (si % npair);
          const int m0s = tiles.mb(js) * kBM + static_cast<int>(rank) * kRows;
          const int n0s = tiles.nb(js) * kBN;
          const uint32_t full_leader = ptx::mapa_shared(ptx::smem_u32(&sh->sf_full[ss]), 0);
          const uint32_t st = ptx::smem_u32(sf_smem + ss * kSfStageBytes);
          if (rank == 0) ptx::mbar_arrive_expect_tx(&sh->sf_full[ss], kTxSf);
          ptx::tma_load_3d_pair_hint(st, &tmap_sfa, full_leader, 0, ks * kSfBlk, m0s / 128, keep);
          ptx::tma_load_3d_pair_hint(st + 2 * kSfaBytes, &tmap_sfb, full_leader, 0, ks * kSfBlk, n0s / 128, keep);
        }
      };
      for (int j = 0; j < tiles.count && ok; ++j) {
        const int mb = tiles.mb(j), nb = tiles.nb(j);
        const int m0 = mb * kBM + static_cast<int>(rank) * kRows;     // this CTA's A rows
        const int nb0 = nb * kBN + static_cast<int>(rank) * kRows;    // this CTA's B rows
        for (int d = 0; d < nstg && ok; ++d, ++it) {
          const bool main_stage = d < ndbl;
          if (main_stage) {
            const int ml = mi + 1 + kSfLead;   // the last main step whose scales must be on their way
            load_scales((ml / nk_main) * npair + (ml % nk_main) / 2 + 1);
          }
          if (!ok) break;
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!wait_bounded(&sh->empty[s], ph ^ 1u, abort_flag, p.err, kErrSiteGemmEmpty)) { ok = false; break; }
          const uint32_t full_leader = ptx::mapa_shared(ptx::smem_u32(&sh->full[s]), 0);
          const uint32_t st = ptx::smem_u32(smem + s * kStageBytes);
          if (main_stage) {
            const int k = 2 * d;
            const bool two = k + 1 < nk_main;
            if (p.op_pair) {
              // one load per operand: K steps k and k + 1 (a missing second step reads as zeros)
              if (rank == 0) ptx::mbar_arrive_expect_tx(&sh->full[s], kTxMain);
              ptx::tma_load_3d_pair_hint(st, &tmap_a, full_leader, 0, m0, k, keep);
              ptx::tma_load_3d_pair_hint(st + 2 * kABytes, &tmap_b, full_leader, 0, nb0, k, keep);
            } else {
              if (rank == 0) ptx::mbar_arrive_expect_tx(&sh->full[s], two ? kTxMain : kTxMain / 2);
              ptx::tma_load_2d_pair_hint(st, &tmap_a, full_leader, k * (kKTile / 2), m0, keep);
              ptx::tma_load_2d_pair_hint(st + 2 * kABytes, &tmap_b, full_leader, k * (kKTile / 2), nb0, keep);
              if (two) {
                ptx::tma_load_2d_pair_hint(st + kABytes, &tmap_a, full_leader, (k + 1) * (kKTile / 2), m0, keep);
                ptx::tma_load_2d_pair_hint(st + 3 * kABytes, &tmap_b, full_leader, (k + 1) * (kKTile / 2), nb0, keep);
              }
            }
            mi += two ? 2 : 1;
          } else {
            const int c = d - ndbl;
            if (rank == 0) ptx::mbar_arrive_expect_tx(&sh->full[s], kTxLowRank);
            ptx::tma_load_2d_pair(st, &tmap_z, full_leader, c * 64, m0);
            ptx::tma_load_2d_pair(st + 2 * kABytes, &tmap_l2, full_leader, c * 64, nb0);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp >= kCopyWarp0 && warp < kCopyWarp0 + kCopyWarps) {
    // ------------------------------------------------------------ scale copiers (leader CTA only)
    // Copy warp w moves blocks [w * per, (w + 1) * per) of every main step (A rows, and both row
    // blocks of B) into the step's TMEM buffer, in both CTAs; a warp whose blocks a short last step
    // lacks still arrives on the step's barriers.
    const int w = warp - kCopyWarp0;
    constexpr int per = kSfBlk / kCopyWarps;
    if (rank == 0) {
      int mi = 0;
      bool ok = true;
      for (int j = 0; j < tiles.count && ok; ++j) {
        for (int k = 0; k < nk_main; ++k, ++mi) {
          const int slot = j * ((nk_main + 1) / 2) + k / 2;
          const int ss = slot % kSfStages;
          const int b = mi % kSfBufs;
          if (!wait_bounded(&sh->sf_full[ss], (slot / kSfStages) & 1, abort_flag, p.err, kErrSiteGemmFull) ||
              !wait_bounded(&sh->sf_free[b], ((mi / kSfBufs) & 1) ^ 1u, abort_flag, p.err, kErrSiteGemmSfFree)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          if (lane == 0) {
            const int nkb = min(kKTile / 64, kblk64 - k * (kKTile / 64));
            const int nblk = MX ? (nkb + 1) / 2 : nkb;            // scale blocks of this step
            const uint32_t st = ptx::smem_u32(sf_smem + ss * kSfStageBytes) + (k & 1) * kSfaBytes;
            const uint32_t sfa = tmem + kTmemSf0 + b * kTmemSfStride;
            const uint32_t sfb = sfa + 4 * kSfBlk;
#pragma unroll
            for (int u = 0; u < per; ++u) {
              const int blk = w * per + u;
              if (blk < nblk) {
                ptx::tmem_cp_32x128b_warpx4_pair(sfa + blk * 4, ptx::sdesc_sf(st + blk * 512));
                ptx::tmem_cp_32x128b_warpx4_pair(sfb + blk * 8, ptx::sdesc_sf(st + 2 * kSfaBytes + blk * 512));
                ptx::tmem_cp_32x128b_warpx4_pair(sfb + blk * 8 + 4,
                                                 ptx::sdesc_sf(st + 4 * kSfaBytes + blk * 512));
              }
            }
            ptx::tc_commit_pair_local(&sh->sf_ready[b]);
            // the slot is free once the copies of both its steps have completed
            if ((k & 1) == 1 || k == nk_main - 1) ptx::tc_commit_pair(&sh->sf_empty[ss], 0x3);
          }
          __syncwarp();
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer (leader CTA only)
    if (rank == 0) {
      int it = 0, mi = 0;
      uint32_t acc_ph = 0;
      bool ok = true;
      const uint32_t id4 = idesc_nvf4(kBM, kBN);
      const uint32_t id16 = idesc_bf16(kBM, kBN);
      for (int j = 0; j < tiles.count && ok; ++j) {
        if (!wait_bounded(&sh->acc_empty, acc_ph ^ 1u, abort_flag, p.err, kErrSiteGemmAccEmpty)) break;
        ptx::tc_fence_after();
        for (int d = 0; d < nstg && ok; ++d, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!wait_bounded(&sh->full[s], ph, abort_flag, p.err, kErrSiteGemmFull)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t st = ptx::smem_u32(smem + s * kStageBytes);
          if (d < ndbl) {
            for (int h2 = 0; h2 < 2; ++h2) {
              const int k = 2 * d + h2;
              if (k >= nk_main) break;
              const int b = mi % kSfBufs;
              if (!wait_bounded(&sh->sf_ready[b], (mi / kSfBufs) & 1, abort_flag, p.err, kErrSiteGemmSfReady)) {
                ok = false;
                break;
              }
              ptx::tc_fence_after();
              if (lane == 0) {
                const uint32_t sa_op = st + h2 * kABytes, sb_op = st + 2 * kABytes + h2 * kABytes;
                const int nkb = min(kKTile / 64, kblk64 - k * (kKTile / 64));
                const uint32_t sfa = tmem + kTmemSf0 + b * kTmemSfStride;
                const uint32_t sfb = sfa + 4 * kSfBlk;
                for (int kb = 0; kb < nkb; ++kb) {
                  const uint64_t adesc = ptx::sdesc_sw128(sa_op + kb * 32), bdesc = ptx::sdesc_sw128(sb_op + kb * 32);
                  const uint32_t acc = (k | kb) != 0 ? 1u : 0u;
                  if (MX) {
                    // block kb/2 of 4 scales per row; this MMA's two start at byte 2 (kb & 1)
                    const uint32_t id = (kb & 1) * 2u;
                    ptx::umma_mxf4_pair(tmem, adesc, bdesc, idesc_mxf4(kBM, kBN, id), (sfa + (kb >> 1) * 4) | (id << 30),
                                        (sfb + (kb >> 1) * 8) | (id << 30), acc);
                  } else {
                    ptx::umma_nvf4_pair(tmem, adesc, bdesc, id4, sfa + kb * 4, sfb + kb * 8, acc);
                  }
                }
                ptx::tc_commit_pair_local(&sh->sf_free[b]);
              }
              __syncwarp();
              ++mi;
            }
            if (!ok) break;
          } else if (lane == 0) {
            const int c = d - ndbl;
            const int nmma = min(64, p.rank - c * 64) / 16;
            for (int jj = 0; jj < nmma; ++jj)
              ptx::umma_f16_pair(tmem, ptx::sdesc_sw128(st + jj * 32), ptx::sdesc_sw128(st + 2 * kABytes + jj * 32),
                                 id16, 1u);
          }
          if (lane == 0) ptx::tc_commit_pair(&sh->empty[s], 0x3);
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) ptx::tc_commit_pair(&sh->acc_full, 0x3);
        __syncwarp();
        acc_ph ^= 1u;
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------ epilogue (8 warps, both CTAs)
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int h = (warp - kEpiWarp0) >> 2;  // column half of the 256-wide tile
    const uint32_t acc_empty_leader = ptx::mapa_shared(ptx::smem_u32(&sh->acc_empty), 0);
    const float sc = p.out_scale;
    uint32_t acc_ph = 0;
    for (int j = 0; j < tiles.count; ++j) {
      const int mb = tiles.mb(j), nb = tiles.nb(j);
      const int m0 = mb * kBM + static_cast<int>(rank) * kRows;
      const int col0 = nb * kBN + h * 128;
      const bool active = col0 < p.N;
      if (!wait_bounded(&sh->acc_full, acc_ph, abort_flag, p.err, kErrSiteGemmAccFull)) break;
      ptx::tc_fence_after();
      // the whole 128-column slice into registers, then the accumulator goes back to the MMA
      // warp at once: the next tile's MMAs run while this one is scaled and stored
      uint32_t v[4][32];
      if (active) {
        const uint32_t base = tmem + (static_cast<uint32_t>(q * 32) << 16) + h * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tmem_ld_32x32b_x32(base + c * 32, v[c]);
        ptx::tmem_wait_ld();
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_peer(acc_empty_leader);
      acc_ph ^= 1u;
      if (!active) continue;
      // Y = g_x g_w * acc + bias -> bf16, written straight from registers: each thread
      // stores its row's 128 columns (256 contiguous bytes), 32 bytes (one sector) per store
      // when Y is 32-byte aligned; rows past M are skipped.
      const int row = m0 + q * 32 + lane;
      if (row >= p.M) continue;
      __nv_bfloat16* yrow = p.Y + static_cast<size_t>(row) * p.N + col0;
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16) {
        const int cl = c16 * 16;                             // column within this warp's 128
        float bv[16];
        const bool in_n = SVDQ_IN_GLOBAL(col0 + cl + 16 <= p.N, p.err);
        if (p.bias && in_n) {
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            const uint4 braw = __ldg(reinterpret_cast<const uint4*>(p.bias + col0 + cl + 8 * hb));
            const uint32_t bw[4] = {braw.x, braw.y, braw.z, braw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              bv[8 * hb + 2 * e] = __uint_as_float(bw[e] << 16);
              bv[8 * hb + 2 * e + 1] = __uint_as_float(bw[e] & 0xFFFF0000u);
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) bv[e] = 0.f;
        }
        uint32_t o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float y0 = fmaf(__uint_as_float(v[cl / 32][cl % 32 + 2 * e]), sc, bv[2 * e]);
          const float y1 = fmaf(__uint_as_float(v[cl / 32][cl % 32 + 2 * e + 1]), sc, bv[2 * e + 1]);
          __nv_bfloat162 hv = __floats2bfloat162_rn(y0, y1);
          o[e] = *reinterpret_cast<uint32_t*>(&hv);
        }
        if (!in_n) {
        } else if (p.y_align32) {
          ptx::st_global_v8_na(yrow + cl, o);
        } else {
          *reinterpret_cast<uint4*>(yrow + cl) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(yrow + cl + 8) = make_uint4(o[4], o[5], o[6], o[7]);
        }
      }
    }
  }

  // Both CTAs finished: every MMA has completed (each epilogue saw its last
  // accumulator) and no remote arrive is still in flight.
  ptx::tc_fence_before();
  ptx::cluster_sync();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, kTmemCols);
  }
}

template <bool MX>
int max_active_clusters(size_t smem) {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_fp4_kernel<MX>, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 0;
  }
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

template <bool MX>
size_t smem_bytes() {
  return 1024 + kStages * kStageBytes + kSfStages * Fp4Cfg<MX>::kSfStageBytes +
         sizeof(SharedTail);
}
static_assert(1024 + kStages * kStageBytes + kSfStages * Fp4Cfg<false>::kSfStageBytes +
                      sizeof(SharedTail) <= 232448,
              "shared memory of one CTA");

template <bool MX>
cudaError_t launch(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsfa, const CUtensorMap& tsfb,
                   const CUtensorMap& tz, const CUtensorMap& tl2, const GemmParams& p,
                   int num_sms, cudaStream_t s) {
  const size_t smem = smem_bytes<MX>();
  cudaError_t e = set_smem_limit_once(reinterpret_cast<const void*>(gemm_fp4_kernel<MX>), smem);
  if (e != cudaSuccess) return e;
  int clusters = max_active_clusters<MX>(smem);
  if (clusters <= 0) clusters = num_sms / 2;
  if (clusters > p.num_tiles) clusters = p.num_tiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // may start under the prologue
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, gemm_fp4_kernel<MX>, ta, tb, tsfa, tsfb, tz, tl2, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_fp4(bool mx, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsfa,
                            const CUtensorMap& tsfb, const CUtensorMap& tz, const CUtensorMap& tl2,
                            const GemmParams& p, int num_sms, cudaStream_t s) {
  return mx ? launch<true>(ta, tb, tsfa, tsfb, tz, tl2, p, num_sms, s)
            : launch<false>(ta, tb, tsfa, tsfb, tz, tl2, p, num_sms, s);
}

}  // namespace svdq
