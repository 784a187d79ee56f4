// INT4 (g64, fp16 scales) W4A4 GEMM with the fused low-rank up projection (sm_100a).
//
// "SVDQuant 阅读笔记：用少量高精度计算保护 4-bit 扩散模型", §2.2 eq.(1) and §8:
// symmetric INT4 codes in groups of 64 along K with one 16-bit scale per group;
// §6.1 "算法 2" steps 4-8 and eq.(7): the 4-bit product and the 16-bit branch
// Z L2 are merged before the single write of Y.
//
//   Y[m, n] = sum_g s_x[m, g] s_w[n, g] D_g[m, n] + (Z L2^T)[m, n] + bias[n],
//   D_g[m, n] = sum_{k in group g} q_x[m, k] q_w[n, k]   (an exact integer)
//
// B200 design (one CTA per SM, 128 x 128 output tiles, persistent):
//   * a producer warp streams the packed codes of 128-column K steps into a
//     3-deep ring with TMA (64B-swizzled, so the row reads below are free of
//     bank conflicts); four widening warps turn every code q into the int8 byte
//     16 q in the 128B-swizzled K-major layout of the MMA, in a second 3-deep
//     ring.  A nibble moved to the top of its byte *is* 16 q in two's complement,
//     so eight codes take two logic operations: the even nibbles of a 32-bit word
//     go to one word, the odd ones to the next.  That permutes K inside every
//     8-element chunk, identically for A and B, which leaves each group's dot
//     product unchanged;
//   * the MMA warp issues tcgen05 kind::i8 MMAs (s8 x s8 -> s32) per 64-element
//     group into one of four TMEM group buffers.  Each buffer is preset to the
//     bit pattern of the float 1.5 * 2^23, so after the MMAs it holds the fp32
//     number 1.5 * 2^23 + 256 D_g exactly (|256 D_g| <= 2^20): subtracting
//     1.5 * 2^23 recovers 256 D_g exactly without an int-to-float conversion;
//   * eight epilogue warps drain each group buffer, preset it again, release it,
//     and add 256 D_g * (s_x s_w / 256) in fp32 into register accumulators with
//     packed f32x2 operations (the products and sums are those of D_g * s_x s_w);
//     the low-rank branch is one more "group" (bf16 kind::f16 MMAs, scale 1)
//     whose Z and L2 tiles the producer loads with TMA into their own slot;
//   * Y leaves through 128B-swizzled shared-memory boxes and TMA stores.
// The per-group fp32 scaling is CUDA-core work of the same order as the MMAs;
// it is what the INT4 format costs next to NVFP4, whose group scales the
// tensor cores apply themselves.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"
#include "svdq_device.cuh"

namespace svdq {
namespace {

constexpr int kBM = 128, kBN = 128;
constexpr int kKStep = 128;                    // elements per pipeline step (two groups)
constexpr int kStages = 3;                     // widened (E4M3) ring
constexpr int kPkStages = 3;                   // packed-code ring
constexpr int kLoadWarps = 4, kMmaWarp = 4, kProdWarp = 5, kEpiWarp0 = 6, kEpiWarps = 8;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);   // 448
constexpr uint32_t kOpBytes = kBM * 128;       // 16 KB: 128 rows x 128 bytes
constexpr uint32_t kStageBytes = 2 * kOpBytes; // A then B
constexpr uint32_t kPkOpBytes = kBM * 64;      // 8 KB: 128 rows x 64 packed bytes
constexpr uint32_t kPkStageBytes = 2 * kPkOpBytes;
constexpr uint32_t kLrBytes = 2 * kOpBytes;    // Z tile + L2 tile (bf16, 64 columns)
constexpr int kScStages = 8;                   // group-scale ring, one slot per K step
constexpr uint32_t kScBytes = 1024;            // s_x: 2 groups x 128 rows, s_w: 2 groups x 128 columns (fp16)
constexpr uint32_t kEpiBoxBytes = 32 * 128;    // 32 rows x 64 bf16
constexpr int kGroupBufs = 4;                  // TMEM: 4 x 128 fp32 columns

__host__ __device__ constexpr uint32_t idesc_s8(int m, int n) {
  // s8 x s8 -> s32, K-major A and B
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}
constexpr uint32_t kAccBias = 0x4B400000u;    // bits of 1.5 * 2^23
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

struct SharedTail {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t pk_full[kPkStages];
  uint64_t pk_empty[kPkStages];
  uint64_t lr_full;
  uint64_t lr_empty;
  uint64_t sc_full[kScStages];
  uint64_t sc_empty[kScStages];
  uint64_t grp_full[kGroupBufs];
  uint64_t grp_empty[kGroupBufs];
  uint32_t tmem_base;
  int abort_flag;
};

// Eight 4-bit two's complement codes (low nibble first) -> eight int8 bytes 16 q:
// .x = codes 0, 2, 4, 6 and .y = codes 1, 3, 5, 7 (the K permutation described above).
__device__ __forceinline__ uint2 int4x8_to_s8x8_x16(uint32_t w) {
  return make_uint2((w << 4) & 0xF0F0F0F0u, w & 0xF0F0F0F0u);
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_int4_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                     const __grid_constant__ CUtensorMap tmap_z, const __grid_constant__ CUtensorMap tmap_l2,
                     const __grid_constant__ CUtensorMap tmap_y, const __grid_constant__ CUtensorMap tmap_sa,
                     const __grid_constant__ CUtensorMap tmap_sb, GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* pk_smem = smem + kStages * kStageBytes;
  uint8_t* lr_smem = pk_smem + kPkStages * kPkStageBytes;
  uint8_t* sc_smem = lr_smem + kLrBytes;
  uint8_t* epi_smem = sc_smem + kScStages * kScBytes;
  float* sbuf = reinterpret_cast<float*>(epi_smem + kEpiWarps * kEpiBoxBytes);   // 8 warps x 64 scales
  SharedTail* sh = reinterpret_cast<SharedTail*>(sbuf + kEpiWarps * 64);
  volatile int* abort_flag = &sh->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int K = p.K;
  const int G = K / 64;
  const int nk_main = (K + kKStep - 1) / kKStep;
  const int nk_lr = (p.rank + 63) / 64;
  const int nk = nk_main + nk_lr;
  const int K2 = K / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&sh->full[s], 32 * kLoadWarps);
      ptx::mbar_init(&sh->empty[s], 1);
    }
    for (int s = 0; s < kPkStages; ++s) {
      ptx::mbar_init(&sh->pk_full[s], 1);
      ptx::mbar_init(&sh->pk_empty[s], 32 * kLoadWarps);
    }
    ptx::mbar_init(&sh->lr_full, 1);
    ptx::mbar_init(&sh->lr_empty, 1);
    for (int s = 0; s < kScStages; ++s) {
      ptx::mbar_init(&sh->sc_full[s], 1);
      ptx::mbar_init(&sh->sc_empty[s], kEpiWarps);
    }
    for (int b = 0; b < kGroupBufs; ++b) {
      ptx::mbar_init(&sh->grp_full[b], 1);
      ptx::mbar_init(&sh->grp_empty[b], kEpiWarps);
    }
    sh->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(&sh->tmem_base, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  if (warp >= kEpiWarp0) {
    // preset every group buffer (this warp's 32 lanes x 64 columns of each) to the bias pattern
    const uint32_t base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + ((warp - kEpiWarp0) >> 2) * 64;
#pragma unroll
    for (int b = 0; b < kGroupBufs; ++b) {
      ptx::tmem_st_32x32b_x32_same(base + b * kBN, kAccBias);
      ptx::tmem_st_32x32b_x32_same(base + b * kBN + 32, kAccBias);
    }
    ptx::tmem_wait_st();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();

  if (warp == kProdWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tmap_a);
      ptx::prefetch_tmap(&tmap_b);
      int pi = 0, li = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        const int m0 = (t % p.tiles_m) * kBM, n0 = (t / p.tiles_m) * kBN;
        for (int k = 0; k < nk_main; ++k, ++pi) {
          const int s = pi % kPkStages;
          if (!wait_bounded(&sh->pk_empty[s], ((pi / kPkStages) & 1) ^ 1u, abort_flag, p.err, kErrSiteGemmEmpty)) {
            ok = false;
            break;
          }
          uint8_t* st = pk_smem + s * kPkStageBytes;
          ptx::mbar_arrive_expect_tx(&sh->pk_full[s], kPkStageBytes);
          ptx::tma_load_2d(st, &tmap_a, &sh->pk_full[s], k * (kKStep / 2), m0);
          ptx::tma_load_2d(st + kPkOpBytes, &tmap_b, &sh->pk_full[s], k * (kKStep / 2), n0);
          // the two groups' scales of this K step, for the epilogue
          const int ss = pi % kScStages;
          if (!wait_bounded(&sh->sc_empty[ss], ((pi / kScStages) & 1) ^ 1u, abort_flag, p.err, kErrSiteGemmEmpty)) {
            ok = false;
            break;
          }
          uint8_t* sc = sc_smem + ss * kScBytes;
          ptx::mbar_arrive_expect_tx(&sh->sc_full[ss], kScBytes);
          ptx::tma_load_2d(sc, &tmap_sa, &sh->sc_full[ss], m0, 2 * k);
          ptx::tma_load_2d(sc + 512, &tmap_sb, &sh->sc_full[ss], n0, 2 * k);
        }
        for (int c = 0; c < nk_lr && ok; ++c, ++li) {
          if (!wait_bounded(&sh->lr_empty, (li & 1) ^ 1u, abort_flag, p.err, kErrSiteGemmEmpty)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(&sh->lr_full, kLrBytes);
          ptx::tma_load_2d(lr_smem, &tmap_z, &sh->lr_full, c * 64, m0);
          ptx::tma_load_2d(lr_smem + kOpBytes, &tmap_l2, &sh->lr_full, c * 64, n0);
        }
      }
    }
    __syncwarp();
  } else if (warp < kLoadWarps) {
    // ------------------------------------------------------------ widening warps
    const int r = threadIdx.x;                  // tile row handled by this thread (A and B)
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
      for (int k = 0; k < nk_main; ++k, ++it) {
        const int ps = it % kPkStages;
        const int s = it % kStages;
        if (!wait_bounded(&sh->pk_full[ps], (it / kPkStages) & 1, abort_flag, p.err, kErrSiteGemmConvFull)) {
          ok = false;
          break;
        }
        // this row's 64 packed bytes of A and of B (64B-swizzled rows)
        const uint8_t* pa = pk_smem + ps * kPkStageBytes + r * 64;
        const uint8_t* pb = pa + kPkOpBytes;
        const int sw = (r >> 1) & 3;
        uint4 va[4], vb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          va[i] = *reinterpret_cast<const uint4*>(pa + ((i ^ sw) << 4));
          vb[i] = *reinterpret_cast<const uint4*>(pb + ((i ^ sw) << 4));
        }
        ptx::mbar_arrive(&sh->pk_empty[ps]);
        if (!wait_bounded(&sh->empty[s], ((it / kStages) & 1) ^ 1u, abort_flag, p.err, kErrSiteGemmConvEmpty)) {
          ok = false;
          break;
        }
        uint8_t* arow_s = smem + s * kStageBytes + r * 128;
        uint8_t* brow_s = arow_s + kOpBytes;
        // 64 packed bytes -> 128 E4M3 bytes = 8 chunks of 16 bytes, 128B-swizzled by row
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t wa[4] = {va[i].x, va[i].y, va[i].z, va[i].w};
          const uint32_t wb[4] = {vb[i].x, vb[i].y, vb[i].z, vb[i].w};
          uint2 ea[4], eb[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            ea[j] = int4x8_to_s8x8_x16(wa[j]);
            eb[j] = int4x8_to_s8x8_x16(wb[j]);
          }
          const int c0 = 2 * i, c1 = 2 * i + 1;
          *reinterpret_cast<uint4*>(arow_s + ((c0 ^ (r & 7)) << 4)) = make_uint4(ea[0].x, ea[0].y, ea[1].x, ea[1].y);
          *reinterpret_cast<uint4*>(arow_s + ((c1 ^ (r & 7)) << 4)) = make_uint4(ea[2].x, ea[2].y, ea[3].x, ea[3].y);
          *reinterpret_cast<uint4*>(brow_s + ((c0 ^ (r & 7)) << 4)) = make_uint4(eb[0].x, eb[0].y, eb[1].x, eb[1].y);
          *reinterpret_cast<uint4*>(brow_s + ((c1 ^ (r & 7)) << 4)) = make_uint4(eb[2].x, eb[2].y, eb[3].x, eb[3].y);
        }
        ptx::fence_proxy_async_smem();        // generic-proxy writes -> visible to the tensor cores
        ptx::mbar_arrive(&sh->full[s]);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    int it = 0, gi = 0, li = 0;
    bool ok = true;
    const uint32_t id8 = idesc_s8(kBM, kBN);
    const uint32_t id16 = idesc_bf16(kBM, kBN);
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
      for (int k = 0; k < nk_main && ok; ++k, ++it) {
        const int s = it % kStages;
        if (!wait_bounded(&sh->full[s], (it / kStages) & 1, abort_flag, p.err, kErrSiteGemmConvFull)) {
          ok = false;
          break;
        }
        const uint32_t st = ptx::smem_u32(smem + s * kStageBytes);
        for (int j = 0; j < 2; ++j, ++gi) {
          const int b = gi % kGroupBufs;
          if (!wait_bounded(&sh->grp_empty[b], ((gi / kGroupBufs) & 1) ^ 1u, abort_flag, p.err,
                            kErrSiteGemmAccEmpty)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          if (lane == 0) {
            const uint32_t d = tmem + b * kBN;
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              const uint32_t off = j * 64 + kk * 32;
              // accumulate onto the preset bias pattern (see the header)
              ptx::umma_i8(d, ptx::sdesc_sw128(st + off), ptx::sdesc_sw128(st + kOpBytes + off), id8, 1u);
            }
            ptx::tc_commit(&sh->grp_full[b]);
          }
          __syncwarp();
        }
        if (lane == 0) ptx::tc_commit(&sh->empty[s]);
        __syncwarp();
      }
      if (!ok || nk_lr == 0) continue;
      // low-rank branch: Z L2^T into one more group buffer
      const int b = gi % kGroupBufs;
      if (!wait_bounded(&sh->grp_empty[b], ((gi / kGroupBufs) & 1) ^ 1u, abort_flag, p.err, kErrSiteGemmAccEmpty)) {
        ok = false;
        break;
      }
      for (int c = 0; c < nk_lr; ++c, ++li) {
        if (!wait_bounded(&sh->lr_full, li & 1, abort_flag, p.err, kErrSiteGemmFull)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        if (lane == 0) {
          const uint32_t st = ptx::smem_u32(lr_smem);
          const uint32_t d = tmem + b * kBN;
          const int nmma = min(64, p.rank - c * 64) / 16;
          for (int j = 0; j < nmma; ++j)
            ptx::umma_f16(d, ptx::sdesc_sw128(st + j * 32), ptx::sdesc_sw128(st + kOpBytes + j * 32), id16,
                          (c > 0 || j > 0) ? 1u : 0u);
          ptx::tc_commit(&sh->lr_empty);
          if (c == nk_lr - 1) ptx::tc_commit(&sh->grp_full[b]);
        }
        __syncwarp();
      }
      ++gi;
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 6-13)
    const int e = warp - kEpiWarp0;
    const int q = warp & 3;                    // TMEM lane quarter
    const int h = e >> 2;                      // 64-column half of the tile
    float* sb_s = sbuf + e * 64;
    uint8_t* buf = epi_smem + e * kEpiBoxBytes;
    int gi = 0, sc_it = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
      const int m0 = (t % p.tiles_m) * kBM, n0 = (t / p.tiles_m) * kBN;
      const int col0 = n0 + h * 64;
      float2 acc[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) acc[c] = make_float2(0.f, 0.f);
      bool ok = true;
      const int ngroups = G + (p.rank > 0 ? 1 : 0);
      for (int g = 0; g < ngroups; ++g, ++gi) {
        const bool lowrank = g == G;
        float sa = 1.f;
        const int kstep = g >> 1;
        const int ss = (sc_it + kstep) % kScStages;
        if (!lowrank) {
          if ((g & 1) == 0 &&
              !wait_bounded(&sh->sc_full[ss], ((sc_it + kstep) / kScStages) & 1, abort_flag, p.err, kErrSiteGemmFull)) {
            ok = false;
            break;
          }
          // this warp's 64 column scales of group g divided by 256 (exact), as fp32 in shared memory
          const uint8_t* sc = sc_smem + ss * kScBytes + (g & 1) * 256;
          const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(sc + 512 + (h * 64 + 2 * lane) * 2));
          sa = __half2float(*reinterpret_cast<const __half*>(sc + (q * 32 + lane) * 2));
          __syncwarp();
          *reinterpret_cast<float2*>(sb_s + 2 * lane) = make_float2(fb.x * 0.00390625f, fb.y * 0.00390625f);
          __syncwarp();
        }
        const int b = gi % kGroupBufs;
        if (!wait_bounded(&sh->grp_full[b], (gi / kGroupBufs) & 1, abort_flag, p.err, kErrSiteGemmAccFull)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t base = tmem + (static_cast<uint32_t>(q * 32) << 16) + b * kBN + h * 64;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t v[32];
          ptx::tmem_ld_32x32b_x32(base + half * 32, v);
          ptx::tmem_wait_ld();
          if (lowrank) {
#pragma unroll
            for (int c = 0; c < 16; ++c)
              acc[half * 16 + c] = __fadd2_rn(acc[half * 16 + c],
                                              make_float2(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1])));
          } else {
            const float2 sa2 = make_float2(sa, sa);
            const float2 nb2 = make_float2(-12582912.f, -12582912.f);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float2 sb2 = *reinterpret_cast<const float2*>(sb_s + half * 32 + 2 * c);
              const float2 d = __fadd2_rn(make_float2(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1])), nb2);
              acc[half * 16 + c] = __ffma2_rn(d, __fmul2_rn(sa2, sb2), acc[half * 16 + c]);
            }
          }
          // this half is consumed: preset it again for the buffer's next use
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) ptx::tmem_st_32x32b_x8_same(base + half * 32 + c8 * 8, kAccBias);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          ptx::mbar_arrive(&sh->grp_empty[b]);
          if (!lowrank && (g & 1) == 1) ptx::mbar_arrive(&sh->sc_empty[ss]);
        }
      }
      sc_it += nk_main;
      if (!ok) break;
      // Y = acc + bias -> bf16, one 32-row x 64-column box through shared memory and a TMA store
      if (lane == 0) ptx::bulk_wait_group_read<0>();
      __syncwarp();
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        float bv[8];
        if (p.bias) {
          const uint4 braw = __ldg(reinterpret_cast<const uint4*>(p.bias + col0 + c8 * 8));
          const uint32_t bw[4] = {braw.x, braw.y, braw.z, braw.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            bv[2 * u] = __uint_as_float(bw[u] << 16);
            bv[2 * u + 1] = __uint_as_float(bw[u] & 0xFFFF0000u);
          }
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) bv[u] = 0.f;
        }
        uint32_t o[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 a2 = acc[c8 * 4 + u];
          __nv_bfloat162 hv = __floats2bfloat162_rn(a2.x + bv[2 * u], a2.y + bv[2 * u + 1]);
          o[u] = *reinterpret_cast<uint32_t*>(&hv);
        }
        *reinterpret_cast<uint4*>(buf + lane * 128 + ((c8 ^ (lane & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        ptx::tma_store_2d(&tmap_y, buf, col0, m0 + q * 32);
        ptx::bulk_commit_group();
      }
    }
    if (lane == 0) ptx::bulk_wait_group<0>();
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

}  // namespace

size_t gemm_int4_smem_bytes() {
  return 1024 + kStages * kStageBytes + kPkStages * kPkStageBytes + kLrBytes + kScStages * kScBytes +
         kEpiWarps * kEpiBoxBytes + kEpiWarps * 64 * 4 + sizeof(SharedTail);
}

cudaError_t launch_gemm_int4(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tz,
                             const CUtensorMap& tl2, const CUtensorMap& ty, const CUtensorMap& tsa,
                             const CUtensorMap& tsb, const GemmParams& p, int num_sms,
                             cudaStream_t s) {
  const size_t smem = gemm_int4_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(gemm_int4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
  gemm_int4_kernel<<<grid, kThreads, smem, s>>>(ta, tb, tz, tl2, ty, tsa, tsb, p);
  return cudaGetLastError();
}

}  // namespace svdq
