// W8A8 GEMM with the fused low-rank up projection (sm_100a, CTA pairs).
//
// The 8-bit setting of "SVDQuant 阅读笔记：用少量高精度计算保护 4-bit 扩散模型" §8
// (appendix D): activations quantized per token, weights per output channel, a rank-16
// branch.  With one scale per row and per column the 8-bit product needs no per-group
// rescaling: sum_k q_x q_w is exact in an s32 accumulator over all of K, and
//     Y = bf16( s_x[m] s_w[n] sum_k q_x q_w + Z L2^T + bias )
// keeps the data flow of §6.1 "算法 2" steps 4-8 (one read of the codes, the branch merged
// before the single write of Y).
//
// B200 design:
//   * CTA pairs compute 256 x 256 tiles with tcgen05 cta_group::2 kind::i8 MMAs (each CTA
//     holds 128 rows of A and 128 rows of B); persistent clusters take contiguous runs of
//     the N-fastest tile numbering; K is staged 128 bytes per row at a time through a
//     6-deep TMA ring (tile loads into each CTA's own shared memory, completion counted on
//     the leader's barrier; no multicast loads);
//   * two TMEM accumulators of 256 columns alternate between tiles, so the MMAs of tile t+1
//     run while the epilogue drains tile t;
//   * the branch cannot share the s32 accumulator, so the epilogue first converts it in
//     place: acc -> fp32(acc) * s_x s_w, written back with tcgen05.st.  The MMA warp then
//     adds Z L2^T onto the converted values with kind::f16 MMAs (accumulate on), issued
//     halfway through the next tile's main loop so that the conversion has finished by then
//     and the tensor pipe does not wait for it;
//   * eight epilogue warps per CTA read the final fp32 values, add the bias and store bf16
//     Y through 128B-swizzled staging and TMA stores.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "svdq_device.cuh"

namespace svdq {
namespace {

constexpr int kBM = 256, kBN = 256;           // pair tile
constexpr int kRows = 128;                    // A rows (and B rows) per CTA
constexpr int kKTile = 128;                   // int8 elements (bytes) per row per pipeline step
constexpr int kStages = 6;
constexpr int kThreads = 320;                 // producer, MMA, 8 epilogue warps
constexpr int kEpiWarp0 = 2;
constexpr int kEpiWarps = 8;
constexpr uint32_t kABytes = kRows * 128;     // 16 KB
constexpr uint32_t kBBytes = kRows * 128;     // 16 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kTx = 2 * kStageBytes;     // both CTAs (main and low-rank steps alike)
constexpr uint32_t kEpiBoxBytes = 32 * 128;   // 32 rows x 64 bf16 per epilogue warp
constexpr uint32_t kTmemCols = 512;           // two accumulators of 256 columns

__host__ __device__ constexpr uint32_t idesc_s8(int m, int n) {
  // s8 x s8 -> s32, K-major A and B
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n) {
  // bf16 x bf16 -> fp32, K-major A and B
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

struct SharedTail {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];    // main MMAs of the buffer's tile completed
  uint64_t conv_done[2];   // epilogue converted the buffer to fp32 (both CTAs)
  uint64_t acc_final[2];   // branch MMAs completed onto the converted buffer
  uint64_t acc_empty[2];   // epilogue read the buffer's final values (both CTAs)
  uint32_t tmem_base;
  int abort_flag;
};

// Position of the low-rank steps in the pipeline: those of tile t-1 come after the first
// `ins` main steps of tile t (half of them: by then the epilogue has long finished converting
// tile t-1, while the epilogue still has the other half to read tile t-1's final values before
// tile t+1 needs the buffer); those of the last tile come after its main steps.
__device__ __forceinline__ int lr_insert_at(int nk_main) { return nk_main > 1 ? nk_main / 2 : 1; }

__global__ void __launch_bounds__(kThreads, 1)
    gemm_w8a8_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                     const __grid_constant__ CUtensorMap tmap_z, const __grid_constant__ CUtensorMap tmap_l2,
                     const __grid_constant__ CUtensorMap tmap_y, GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi_smem = smem + kStages * kStageBytes;
  SharedTail* sh = reinterpret_cast<SharedTail*>(epi_smem + kEpiWarps * kEpiBoxBytes);
  volatile int* abort_flag = &sh->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int cluster = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;
  const int nk_main = p.K / kKTile;
  const int nk_lr = (p.rank + 63) / 64;
  const int ins = lr_insert_at(nk_main);
  const TileSeq tiles(p.num_tiles, p.tiles_n, cluster, nclusters);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&sh->full[s], 1);
      ptx::mbar_init(&sh->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&sh->acc_full[b], 1);
      ptx::mbar_init(&sh->conv_done[b], 2 * kEpiWarps);
      ptx::mbar_init(&sh->acc_final[b], 1);
      ptx::mbar_init(&sh->acc_empty[b], 2 * kEpiWarps);
    }
    sh->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(&sh->tmem_base, kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();
  ptx::tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  // the set-up above may overlap the end of the prologue kernel; its outputs are read only
  // after it has completed
  ptx::griddep_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      ptx::prefetch_tmap(&tmap_a);
      ptx::prefetch_tmap(&tmap_b);
      if (nk_lr > 0) {
        ptx::prefetch_tmap(&tmap_z);
        ptx::prefetch_tmap(&tmap_l2);
      }
      int it = 0;
      bool ok = true;
      // one pipeline step: main step k of tile j (k >= 0) or low-rank step c of tile j (k = -1 - c)
      auto step = [&](int j, int k) -> bool {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        ++it;
        if (!wait_bounded(&sh->empty[s], ph ^ 1u, abort_flag, p.err, kErrSiteGemmEmpty)) return false;
        const int m0 = tiles.mb(j) * kBM + static_cast<int>(rank) * kRows;
        const int nb0 = tiles.nb(j) * kBN + static_cast<int>(rank) * kRows;
        const uint32_t full_leader = ptx::mapa_shared(ptx::smem_u32(&sh->full[s]), 0);
        const uint32_t st = ptx::smem_u32(smem + s * kStageBytes);
        if (rank == 0) ptx::mbar_arrive_expect_tx(&sh->full[s], kTx);
        if (k >= 0) {
          ptx::tma_load_2d_pair(st, &tmap_a, full_leader, k * kKTile, m0);
          ptx::tma_load_2d_pair(st + kABytes, &tmap_b, full_leader, k * kKTile, nb0);
        } else {
          const int c = -1 - k;
          ptx::tma_load_2d_pair(st, &tmap_z, full_leader, c * 64, m0);
          ptx::tma_load_2d_pair(st + kABytes, &tmap_l2, full_leader, c * 64, nb0);
        }
        return true;
      };
      for (int j = 0; j < tiles.count && ok; ++j) {
        for (int k = 0; k < nk_main && ok; ++k) {
          ok = step(j, k);
          if (ok && k == ins - 1 && j > 0)
            for (int c = 0; c < nk_lr && ok; ++c) ok = step(j - 1, -1 - c);
        }
      }
      if (ok && tiles.count > 0)
        for (int c = 0; c < nk_lr && ok; ++c) ok = step(tiles.count - 1, -1 - c);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader CTA only)
    if (rank == 0) {
      int it = 0;
      bool ok = true;
      const uint32_t id8 = idesc_s8(kBM, kBN);
      const uint32_t id16 = idesc_bf16(kBM, kBN);
      auto ring_wait = [&]() -> uint32_t {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        ++it;
        if (!wait_bounded(&sh->full[s], ph, abort_flag, p.err, kErrSiteGemmFull)) return 0xFFFFFFFFu;
        ptx::tc_fence_after();
        return static_cast<uint32_t>(s);
      };
      // Z L2^T of tile j added onto its converted accumulator
      auto branch = [&](int j) -> bool {
        const int b = j & 1;
        if (!wait_bounded(&sh->conv_done[b], (j >> 1) & 1, abort_flag, p.err, kErrSiteGemmConvDone)) return false;
        ptx::tc_fence_after();
        for (int c = 0; c < nk_lr; ++c) {
          const uint32_t s = ring_wait();
          if (s == 0xFFFFFFFFu) return false;
          if (lane == 0) {
            const uint32_t st = ptx::smem_u32(smem + s * kStageBytes);
            const int nmma = min(64, p.rank - c * 64) / 16;
            for (int q = 0; q < nmma; ++q)
              ptx::umma_f16_pair(tmem + b * 256, ptx::sdesc_sw128(st + q * 32), ptx::sdesc_sw128(st + kABytes + q * 32),
                                 id16, 1u);
            ptx::tc_commit_pair(&sh->empty[s], 0x3);
          }
          __syncwarp();
        }
        if (lane == 0) ptx::tc_commit_pair(&sh->acc_final[b], 0x3);
        __syncwarp();
        return true;
      };
      for (int j = 0; j < tiles.count && ok; ++j) {
        const int b = j & 1;
        if (!wait_bounded(&sh->acc_empty[b], ((j >> 1) & 1) ^ 1u, abort_flag, p.err, kErrSiteGemmAccEmpty)) break;
        ptx::tc_fence_after();
        for (int k = 0; k < nk_main && ok; ++k) {
          const uint32_t s = ring_wait();
          if (s == 0xFFFFFFFFu) { ok = false; break; }
          if (lane == 0) {
            const uint32_t st = ptx::smem_u32(smem + s * kStageBytes);
#pragma unroll
            for (int kb = 0; kb < kKTile / 32; ++kb)
              ptx::umma_i8_pair(tmem + b * 256, ptx::sdesc_sw128(st + kb * 32), ptx::sdesc_sw128(st + kABytes + kb * 32),
                                id8, (k | kb) != 0 ? 1u : 0u);
            ptx::tc_commit_pair(&sh->empty[s], 0x3);
            if (k == nk_main - 1) ptx::tc_commit_pair(&sh->acc_full[b], 0x3);
          }
          __syncwarp();
          if (k == ins - 1 && j > 0 && nk_lr > 0) ok = branch(j - 1);
        }
      }
      if (ok && tiles.count > 0 && nk_lr > 0) branch(tiles.count - 1);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-9, both CTAs)
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int h = (warp - kEpiWarp0) >> 2;  // column half of the 256-wide tile
    const uint32_t conv_leader0 = ptx::mapa_shared(ptx::smem_u32(&sh->conv_done[0]), 0);
    const uint32_t conv_leader1 = ptx::mapa_shared(ptx::smem_u32(&sh->conv_done[1]), 0);
    const uint32_t empty_leader0 = ptx::mapa_shared(ptx::smem_u32(&sh->acc_empty[0]), 0);
    const uint32_t empty_leader1 = ptx::mapa_shared(ptx::smem_u32(&sh->acc_empty[1]), 0);
    const float* sw_all = reinterpret_cast<const float*>(p.w_scales);
    const float* sx_all = reinterpret_cast<const float*>(p.a_scales);
    uint8_t* buf = epi_smem + (warp - kEpiWarp0) * kEpiBoxBytes;
    const bool lowrank = nk_lr > 0;
    for (int j = 0; j < tiles.count; ++j) {
      const int b = j & 1;
      const uint32_t par = (j >> 1) & 1;
      const int m0 = tiles.mb(j) * kBM + static_cast<int>(rank) * kRows;
      const int col0 = tiles.nb(j) * kBN + h * 128;
      const int row = m0 + q * 32 + lane;
      const bool active = col0 < p.N &&        // the second half of a last tile may lie past N
                          SVDQ_IN_GLOBAL(col0 + 128 <= p.N, p.err);
      const float sx = row < p.Mpad ? __ldg(sx_all + row) : 0.f;
      const uint32_t base = tmem + (static_cast<uint32_t>(q * 32) << 16) + b * 256 + h * 128;
      if (!wait_bounded(&sh->acc_full[b], par, abort_flag, p.err, kErrSiteGemmAccFull)) break;
      ptx::tc_fence_after();
      if (lowrank) {
        // s32 -> fp32(acc) * (s_x s_w), in place, so that the branch MMAs can add onto it
#pragma unroll 1
        for (int c = 0; c < (active ? 4 : 0); ++c) {
          uint32_t v[32];
          ptx::tmem_ld_32x32b_x32(base + c * 32, v);
          ptx::tmem_wait_ld();
          const float4* swp = reinterpret_cast<const float4*>(sw_all + col0 + c * 32);
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 w = __ldg(swp + e4);
            v[4 * e4 + 0] = __float_as_uint(__int2float_rn(static_cast<int>(v[4 * e4 + 0])) * (sx * w.x));
            v[4 * e4 + 1] = __float_as_uint(__int2float_rn(static_cast<int>(v[4 * e4 + 1])) * (sx * w.y));
            v[4 * e4 + 2] = __float_as_uint(__int2float_rn(static_cast<int>(v[4 * e4 + 2])) * (sx * w.z));
            v[4 * e4 + 3] = __float_as_uint(__int2float_rn(static_cast<int>(v[4 * e4 + 3])) * (sx * w.w));
          }
          ptx::tmem_st_32x32b_x32(base + c * 32, v);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(b ? conv_leader1 : conv_leader0);
        if (!wait_bounded(&sh->acc_final[b], par, abort_flag, p.err, kErrSiteGemmAccFinal)) break;
        ptx::tc_fence_after();
      }
      if (!active) {
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(b ? empty_leader1 : empty_leader0);
        continue;
      }
      // final values (+ bias) -> bf16, two boxes of 64 columns per warp
#pragma unroll 1
      for (int box = 0; box < 2; ++box) {
        if (lane == 0) ptx::bulk_wait_group_read<0>();
        __syncwarp();
#pragma unroll 1
        for (int c2 = 0; c2 < 2; ++c2) {
          const int cc = box * 64 + c2 * 32;          // column within this warp's 128
          uint32_t v[32];
          ptx::tmem_ld_32x32b_x32(base + cc, v);
          ptx::tmem_wait_ld();
          if (box == 1 && c2 == 1) {
            // every column of this buffer has been read: hand it back to the MMA warp
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(b ? empty_leader1 : empty_leader0);
          }
          float y[32];
          if (lowrank) {
#pragma unroll
            for (int e = 0; e < 32; ++e) y[e] = __uint_as_float(v[e]);
          } else {
            const float4* swp = reinterpret_cast<const float4*>(sw_all + col0 + cc);
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
              const float4 w = __ldg(swp + e4);
              y[4 * e4 + 0] = __int2float_rn(static_cast<int>(v[4 * e4 + 0])) * (sx * w.x);
              y[4 * e4 + 1] = __int2float_rn(static_cast<int>(v[4 * e4 + 1])) * (sx * w.y);
              y[4 * e4 + 2] = __int2float_rn(static_cast<int>(v[4 * e4 + 2])) * (sx * w.z);
              y[4 * e4 + 3] = __int2float_rn(static_cast<int>(v[4 * e4 + 3])) * (sx * w.w);
            }
          }
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            const int cl = c2 * 32 + c8 * 8;          // column within the 64-column box
            float bv[8];
            if (p.bias && SVDQ_IN_GLOBAL(col0 + box * 64 + cl + 8 <= p.N, p.err)) {
              const uint4 braw = __ldg(reinterpret_cast<const uint4*>(p.bias + col0 + box * 64 + cl));
              const uint32_t bw[4] = {braw.x, braw.y, braw.z, braw.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                bv[2 * e] = __uint_as_float(bw[e] << 16);
                bv[2 * e + 1] = __uint_as_float(bw[e] & 0xFFFF0000u);
              }
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) bv[e] = 0.f;
            }
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 hv = __floats2bfloat162_rn(y[c8 * 8 + 2 * e] + bv[2 * e], y[c8 * 8 + 2 * e + 1] + bv[2 * e + 1]);
              o[e] = *reinterpret_cast<uint32_t*>(&hv);
            }
            const int chunk = cl / 8;                 // 16-byte chunk of the 128-byte row
            if (SVDQ_IN_SMEM(smem_raw, buf + lane * 128 + ((chunk ^ (lane & 7)) << 4), 16, p.err))
              *reinterpret_cast<uint4*>(buf + lane * 128 + ((chunk ^ (lane & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          ptx::tma_store_2d(&tmap_y, buf, col0 + box * 64, m0 + q * 32);
          ptx::bulk_commit_group();
        }
      }
    }
    if (lane == 0) ptx::bulk_wait_group<0>();
    __syncwarp();
  }

  // Both CTAs finished: every MMA has completed (each epilogue saw its last accumulator)
  // and no remote arrive is still in flight.
  ptx::tc_fence_before();
  ptx::cluster_sync();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, kTmemCols);
  }
}

size_t smem_bytes() { return 1024 + kStages * kStageBytes + kEpiWarps * kEpiBoxBytes + sizeof(SharedTail); }

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
  if (cudaOccupancyMaxActiveClusters(&n, gemm_w8a8_kernel, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 0;
  }
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

}  // namespace

cudaError_t launch_gemm_w8a8(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tz,
                             const CUtensorMap& tl2, const CUtensorMap& ty, const GemmParams& p, int num_sms,
                             cudaStream_t s) {
  const size_t smem = smem_bytes();
  cudaError_t e = set_smem_limit_once(reinterpret_cast<const void*>(gemm_w8a8_kernel), smem);
  if (e != cudaSuccess) return e;
  int clusters = max_active_clusters(smem);
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
  e = cudaLaunchKernelEx(&cfg, gemm_w8a8_kernel, ta, tb, tz, tl2, ty, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace svdq
