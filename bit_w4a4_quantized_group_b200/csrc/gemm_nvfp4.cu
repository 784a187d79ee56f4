// NVFP4 W4A4 GEMM with the fused low-rank up projection (sm_100a).
//
// "SVDQuant 阅读笔记：用少量高精度计算保护 4-bit 扩散模型", §6.1 "算法 2"
// steps 4-8 and eq.(7): the 4-bit product Q(X_hat) Q(R) and the 16-bit branch
// Z L2 are merged before the single write of Y.
//
// B200 design:
//   * persistent CTAs (one per SM), 128 x 256 output tiles, K staged 256
//     E2M1 elements (128 bytes per row) at a time through a 4-deep TMA ring;
//   * warp 0 issues TMA (codes as 128B-swizzled tiles, E4M3 scale blocks as
//     plain bulk copies), warp 1 issues tcgen05 block-scaled MMAs
//     (kind::mxf4nvf4, UE4M3 scales per 16 elements) into an fp32 TMEM
//     accumulator, after moving the scale blocks smem -> TMEM with tcgen05.cp;
//   * the low-rank branch is ceil(r/64) extra pipeline steps in which the ring
//     slots hold Z (bf16, [128 x 64]) and L2s (bf16, [256 x 64]); warp 1 adds
//     Z L2s^T into the *same* accumulator with kind::f16 MMAs.  L2s was divided
//     by (g_x g_w) at pack time, so one multiply by g_x g_w in the epilogue
//     scales both terms correctly and Y gets no extra pass;
//   * warps 2-9 drain TMEM (tcgen05.ld), free it for the next tile at once,
//     then apply g_x g_w and the bias and store bf16 Y.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "svdq_device.cuh"

namespace svdq {
namespace {

constexpr int kBM = 128, kBN = 256;
constexpr int kKTile = 256;                   // E2M1 elements per pipeline step
constexpr int kStages = 4;
constexpr int kThreads = 320;                 // producer, MMA, 8 epilogue warps
constexpr uint32_t kABytes = kBM * 128;       // 16 KB
constexpr uint32_t kBBytes = kBN * 128;       // 32 KB
constexpr uint32_t kSfaOff = kABytes + kBBytes;
constexpr uint32_t kSfbOff = kSfaOff + 2048;
constexpr uint32_t kStageBytes = kSfbOff + 4096;   // 54 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemSfa = 256, kTmemSfb = 272;

__host__ __device__ constexpr uint32_t idesc_nvf4(int n) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (0u << 23) |
         (static_cast<uint32_t>(kBM >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(kBM >> 4) << 24);
}

struct SharedTail {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(kThreads, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_z, const __grid_constant__ CUtensorMap tmap_l2,
                      GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SharedTail* sh = reinterpret_cast<SharedTail*>(smem + kStages * kStageBytes);
  volatile int* abort_flag = &sh->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nk_main = (p.K + kKTile - 1) / kKTile;
  const int nk_lr = (p.rank + 63) / 64;
  const int nk = nk_main + nk_lr;
  const int kblk64 = p.K / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&sh->full[s], 1);
      ptx::mbar_init(&sh->empty[s], 1);
    }
    ptx::mbar_init(&sh->acc_full, 1);
    ptx::mbar_init(&sh->acc_empty, 8);
    sh->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&sh->tmem_base, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tmap_a);
      ptx::prefetch_tmap(&tmap_b);
      if (nk_lr > 0) {
        ptx::prefetch_tmap(&tmap_z);
        ptx::prefetch_tmap(&tmap_l2);
      }
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        const int mb = t % p.tiles_m, nb = t / p.tiles_m;
        const int m0 = mb * kBM, n0 = nb * kBN;
        const bool full_n = (n0 + kBN) <= p.N;
        for (int k = 0; k < nk; ++k, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!wait_bounded(&sh->empty[s], ph ^ 1u, abort_flag, p.err, kErrSiteGemmEmpty)) { ok = false; break; }
          uint8_t* st = smem + s * kStageBytes;
          if (k < nk_main) {
            const int kb0 = k * (kKTile / 64);                 // first 64-element block
            const int nkb = min(kKTile / 64, kblk64 - kb0);
            const uint32_t sfbytes = nkb * 512u;
            const uint32_t bytes = kABytes + kBBytes + sfbytes * (full_n ? 3u : 2u);
            ptx::mbar_arrive_expect_tx(&sh->full[s], bytes);
            ptx::tma_load_2d(st, &tmap_a, &sh->full[s], k * (kKTile / 2), m0);
            ptx::tma_load_2d(st + kABytes, &tmap_b, &sh->full[s], k * (kKTile / 2), n0);
            ptx::bulk_load(st + kSfaOff, p.a_scales + (static_cast<size_t>(mb) * kblk64 + kb0) * 512, sfbytes,
                           &sh->full[s]);
            ptx::bulk_load(st + kSfbOff, p.w_scales + (static_cast<size_t>(n0 / 128) * kblk64 + kb0) * 512,
                           sfbytes, &sh->full[s]);
            if (full_n)
              ptx::bulk_load(st + kSfbOff + 2048,
                             p.w_scales + (static_cast<size_t>(n0 / 128 + 1) * kblk64 + kb0) * 512, sfbytes,
                             &sh->full[s]);
          } else {
            const int c = k - nk_main;
            ptx::mbar_arrive_expect_tx(&sh->full[s], kABytes + kBBytes);
            ptx::tma_load_2d(st, &tmap_z, &sh->full[s], c * 64, m0);
            ptx::tma_load_2d(st + kABytes, &tmap_l2, &sh->full[s], c * 64, n0);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    int it = 0;
    uint32_t acc_ph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
      const int n0 = (t / p.tiles_m) * kBN;
      const int ntile = min(kBN, p.N - n0);
      const uint32_t id4 = idesc_nvf4(ntile);
      const uint32_t id16 = idesc_bf16(ntile);
      if (!wait_bounded(&sh->acc_empty, acc_ph ^ 1u, abort_flag, p.err, kErrSiteGemmAccEmpty)) break;
      ptx::tc_fence_after();
      for (int k = 0; k < nk; ++k, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!wait_bounded(&sh->full[s], ph, abort_flag, p.err, kErrSiteGemmFull)) { ok = false; break; }
        ptx::tc_fence_after();
        if (lane == 0) {
          const uint32_t st = ptx::smem_u32(smem + s * kStageBytes);
          if (k < nk_main) {
            const int nkb = min(kKTile / 64, kblk64 - k * (kKTile / 64));
            for (int kb = 0; kb < nkb; ++kb) {
              ptx::tmem_cp_32x128b_warpx4(tmem + kTmemSfa + kb * 4, ptx::sdesc_sf(st + kSfaOff + kb * 512));
              ptx::tmem_cp_32x128b_warpx4(tmem + kTmemSfb + kb * 8, ptx::sdesc_sf(st + kSfbOff + kb * 512));
              if (ntile == kBN)
                ptx::tmem_cp_32x128b_warpx4(tmem + kTmemSfb + kb * 8 + 4,
                                            ptx::sdesc_sf(st + kSfbOff + 2048 + kb * 512));
            }
            for (int kb = 0; kb < nkb; ++kb) {
              ptx::umma_nvf4(tmem, ptx::sdesc_sw128(st + kb * 32), ptx::sdesc_sw128(st + kABytes + kb * 32), id4,
                             tmem + kTmemSfa + kb * 4, tmem + kTmemSfb + kb * 8, (k | kb) != 0 ? 1u : 0u);
            }
          } else {
            const int c = k - nk_main;
            const int nmma = min(64, p.rank - c * 64) / 16;
            for (int j = 0; j < nmma; ++j) {
              ptx::umma_f16(tmem, ptx::sdesc_sw128(st + j * 32), ptx::sdesc_sw128(st + kABytes + j * 32), id16,
                            1u);
            }
          }
          ptx::tc_commit(&sh->empty[s]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) ptx::tc_commit(&sh->acc_full);
      __syncwarp();
      acc_ph ^= 1u;
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-9)
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int h = (warp - 2) >> 2;          // column half of the 256-wide tile
    uint32_t acc_ph = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
      const int mb = t % p.tiles_m, nb = t / p.tiles_m;
      const int m0 = mb * kBM, n0 = nb * kBN;
      const int ntile = min(kBN, p.N - n0);
      const bool active = (h * 128) < ntile;
      if (!wait_bounded(&sh->acc_full, acc_ph, abort_flag, p.err, kErrSiteGemmAccFull)) break;
      ptx::tc_fence_after();
      uint32_t v[4][32];
      if (active) {
        const uint32_t base = tmem + (static_cast<uint32_t>(q * 32) << 16) + h * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tmem_ld_32x32b_x32(base + c * 32, v[c]);
        ptx::tmem_wait_ld();
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&sh->acc_empty);
      acc_ph ^= 1u;
      if (!active) continue;
      const int row = m0 + q * 32 + lane;
      if (row < p.M) {
        const int col0 = n0 + h * 128;
        __nv_bfloat16* yrow = p.Y + static_cast<size_t>(row) * p.N + col0;
        const float sc = p.out_scale;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            float bv[8];
            if (p.bias) {
              const uint4 braw = __ldg(reinterpret_cast<const uint4*>(p.bias + col0 + c * 32 + c8 * 8));
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
              const float y0 = fmaf(__uint_as_float(v[c][c8 * 8 + 2 * e]), sc, bv[2 * e]);
              const float y1 = fmaf(__uint_as_float(v[c][c8 * 8 + 2 * e + 1]), sc, bv[2 * e + 1]);
              __nv_bfloat162 hv = __floats2bfloat162_rn(y0, y1);
              o[e] = *reinterpret_cast<uint32_t*>(&hv);
            }
            *reinterpret_cast<uint4*>(yrow + c * 32 + c8 * 8) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm_nvfp4(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tz,
                              const CUtensorMap& tl2, const GemmParams& p, int num_sms, cudaStream_t s) {
  const size_t smem = 1024 + kStages * kStageBytes + sizeof(SharedTail);
  cudaError_t e = cudaFuncSetAttribute(gemm_nvfp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
  gemm_nvfp4_kernel<<<grid, kThreads, smem, s>>>(ta, tb, tz, tl2, p);
  return cudaGetLastError();
}

}  // namespace svdq
