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
//     bank conflicts); two widening warps turn every code q into the int8 byte
//     16 q in the 128B-swizzled K-major layout of the MMA, in a second 3-deep
//     ring (two rows per thread).  A nibble moved to the top of its byte *is* 16 q in two's complement,
//     so eight codes take two logic operations: the even nibbles of a 32-bit word
//     go to one word, the odd ones to the next.  That permutes K inside every
//     8-element chunk, identically for A and B, which leaves each group's dot
//     product unchanged;
//   * the MMA warp issues tcgen05 kind::i8 MMAs (s8 x s8 -> s32) per 64-element
//     group into one of four TMEM group buffers (the group's first MMA overwrites
//     the buffer with 256 D_g);
//   * the widening warps also turn each K step's fp16 group scales into fp32 once,
//     s_w/256 per column and s_x per row for both groups, in a ring of their own, so
//     that no epilogue warp converts scales;
//   * eight epilogue warps (two per TMEM lane quarter, 64 columns each) read each
//     group buffer in the 16x256b shape (4 rows x 16 columns per thread) and hand
//     it back at once.  Adding the bits of B = 1.5 * 2^23 to the s32 value gives
//     the fp32 number v = B + 256 D_g exactly (|256 D_g| < 2^22).  The scaling then
//     takes two fp32 FMAs per element and group:
//        t = fma(v, s_w/256, -B s_w/256) = RN(D_g s_w)  (B s_w/256 is exact, and
//            the fma rounds v s_w/256 - B s_w/256 = D_g s_w once),
//        acc = fma(t, s_x, acc),
//     packed two columns at a time (f32x2);
//   * the low-rank branch is one more "group" (bf16 kind::f16 MMAs, added as is)
//     whose Z and L2 tiles the producer loads with TMA into their own slot;
//   * Y leaves through 128B-swizzled 32 x 64 shared-memory boxes and TMA stores.
// The per-group fp32 scaling is CUDA-core work larger than the MMAs (two FMAs per
// output element and group against the tensor core's 64 multiply-adds); it is what
// the INT4 format costs next to NVFP4, whose group scales the tensor cores apply.
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
constexpr int kStages = 3;                     // widened (int8) ring
constexpr int kPkStages = 3;                   // packed-code ring
// 12 warps (three per SM sub-partition, whose 16K registers then allow 168 per thread):
// two widening warps (two tile rows per thread), the MMA warp, the producer, 8 epilogue warps
constexpr int kLoadWarps = 2, kMmaWarp = 2, kProdWarp = 3, kEpiWarp0 = 4, kEpiWarps = 8;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);   // 384
constexpr uint32_t kOpBytes = kBM * 128;       // 16 KB: 128 rows x 128 bytes
constexpr uint32_t kStageBytes = 2 * kOpBytes; // A then B
constexpr uint32_t kPkOpBytes = kBM * 64;      // 8 KB: 128 rows x 64 packed bytes
constexpr uint32_t kPkStageBytes = 2 * kPkOpBytes;
constexpr uint32_t kLrBytes = 2 * kOpBytes;    // Z tile + L2 tile (bf16, 64 columns)
constexpr int kScStages = 3;                   // fp16 group-scale ring (TMA), one slot per K step
constexpr int kCvtStages = 6;                  // fp32 scale ring (widening warps -> epilogue), one slot per K step
constexpr uint32_t kCvtBytes = 2048;           // s_w / 256: 2 groups x 128 columns, s_x: 2 groups x 128 rows (fp32)
constexpr uint32_t kScBytes = 1024;            // s_x: 2 groups x 128 rows, s_w: 2 groups x 128 columns (fp16)
constexpr uint32_t kEpiBoxBytes = 32 * 128;    // 32 rows x 64 bf16
constexpr int kGroupBufs = 4;                  // TMEM: 4 x 128 fp32 columns

__host__ __device__ constexpr uint32_t idesc_s8(int m, int n) {
  // s8 x s8 -> s32, K-major A and B
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}
constexpr uint32_t kAccBias = 0x4B400000u;    // bits of B = 1.5 * 2^23
constexpr float kAccBiasF = 12582912.0f;
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
  uint64_t cvt_full[kCvtStages];
  uint64_t cvt_empty[kCvtStages];
  uint64_t grp_full[kGroupBufs];
  uint64_t grp_empty[kGroupBufs];
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kSmemBytes = 1024 + kStages * kStageBytes + kPkStages * kPkStageBytes + kLrBytes +
                              kScStages * kScBytes + kCvtStages * kCvtBytes + kEpiWarps * kEpiBoxBytes +
                              sizeof(SharedTail);
static_assert(kSmemBytes <= 232448, "shared memory of one CTA");

// Eight 4-bit two's complement codes (low nibble first) -> eight int8 bytes 16 q:
// .x = codes 0, 2, 4, 6 and .y = codes 1, 3, 5, 7 (the K permutation described above).
__device__ __forceinline__ uint2 int4x8_to_s8x8_x16(uint32_t w) {
  return make_uint2((w << 4) & 0xF0F0F0F0u, w & 0xF0F0F0F0u);
}

__device__ __forceinline__ float2 u2f2(uint32_t a, uint32_t b) { return make_float2(__uint_as_float(a), __uint_as_float(b)); }

template <bool SPLIT>
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
  float* cvt_smem = reinterpret_cast<float*>(sc_smem + kScStages * kScBytes);
  uint8_t* epi_smem = reinterpret_cast<uint8_t*>(cvt_smem) + kCvtStages * kCvtBytes;
  SharedTail* sh = reinterpret_cast<SharedTail*>(epi_smem + kEpiWarps * kEpiBoxBytes);
  volatile int* abort_flag = &sh->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int K = p.K;
  const int nk_main = (K + kKStep - 1) / kKStep;
  // K split (few tiles): the S CTAs of a cluster share one tile, CTA q taking the K steps
  // [kb, ke) and CTA 0 also the low-rank group; without the split a CTA runs whole tiles.
  const int S = SPLIT ? p.ksplit : 1;
  const int sq = SPLIT ? static_cast<int>(ptx::cluster_ctarank()) : 0;
  const int t_first = SPLIT ? static_cast<int>(blockIdx.x) / S : static_cast<int>(blockIdx.x);
  const int t_step = SPLIT ? static_cast<int>(gridDim.x) / S : static_cast<int>(gridDim.x);
  const int nks = (nk_main + S - 1) / S;
  const int kb = SPLIT ? min(nk_main, sq * nks) : 0;
  const int ke = SPLIT ? min(nk_main, kb + nks) : nk_main;
  const int nk_lr = sq == 0 ? (p.rank + 63) / 64 : 0;

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
      ptx::mbar_init(&sh->sc_empty[s], kLoadWarps);
    }
    for (int s = 0; s < kCvtStages; ++s) {
      ptx::mbar_init(&sh->cvt_full[s], kLoadWarps);
      ptx::mbar_init(&sh->cvt_empty[s], kEpiWarps);
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
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // the set-up above may overlap the end of the prologue kernel; its outputs (A codes and
  // scales, Z) are read only after it has completed
  ptx::griddep_wait();

  if (warp == kProdWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tmap_a);
      ptx::prefetch_tmap(&tmap_b);
      int pi = 0, li = 0;
      bool ok = true;
      for (int t = t_first; t < p.num_tiles && ok; t += t_step) {
        const int m0 = (t % p.tiles_m) * kBM, n0 = (t / p.tiles_m) * kBN;
        for (int k = kb; k < ke; ++k, ++pi) {
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
    int it = 0;
    bool ok = true;
    for (int t = t_first; t < p.num_tiles && ok; t += t_step) {
      for (int k = kb; k < ke; ++k, ++it) {
        const int ps = it % kPkStages;
        const int s = it % kStages;
        if (!wait_bounded(&sh->pk_full[ps], (it / kPkStages) & 1, abort_flag, p.err, kErrSiteGemmConvFull)) {
          ok = false;
          break;
        }
        // rows r and r + 64 of the tile (A and B): 64 packed bytes each, 64B-swizzled rows
        uint4 va[2][4], vb[2][4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int r = threadIdx.x + 64 * h;
          const uint8_t* pa = pk_smem + ps * kPkStageBytes + r * 64;
          const uint8_t* pb = pa + kPkOpBytes;
          const int sw = (r >> 1) & 3;
          const bool in_s = SVDQ_IN_SMEM(smem_raw, pa, 64, p.err) && SVDQ_IN_SMEM(smem_raw, pb, 64, p.err);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            va[h][i] = in_s ? *reinterpret_cast<const uint4*>(pa + ((i ^ sw) << 4)) : make_uint4(0, 0, 0, 0);
            vb[h][i] = in_s ? *reinterpret_cast<const uint4*>(pb + ((i ^ sw) << 4)) : make_uint4(0, 0, 0, 0);
          }
        }
        ptx::mbar_arrive(&sh->pk_empty[ps]);
        if (!wait_bounded(&sh->empty[s], ((it / kStages) & 1) ^ 1u, abort_flag, p.err, kErrSiteGemmConvEmpty)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int r = threadIdx.x + 64 * h;
          uint8_t* arow_s = smem + s * kStageBytes + r * 128;
          uint8_t* brow_s = arow_s + kOpBytes;
          if (!(SVDQ_IN_SMEM(smem_raw, arow_s, 128, p.err) && SVDQ_IN_SMEM(smem_raw, brow_s, 128, p.err))) continue;
          // 64 packed bytes -> 128 int8 bytes = 8 chunks of 16 bytes, 128B-swizzled by row
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t wa[4] = {va[h][i].x, va[h][i].y, va[h][i].z, va[h][i].w};
            const uint32_t wb[4] = {vb[h][i].x, vb[h][i].y, vb[h][i].z, vb[h][i].w};
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
        }
        ptx::fence_proxy_async_smem();        // generic-proxy writes -> visible to the tensor cores
        ptx::mbar_arrive(&sh->full[s]);
        // the step's group scales as fp32 for the epilogue, once for all its warps: s_w / 256 of
        // the 128 columns and s_x of the 128 rows, both groups (thread t: entries t + 64 u)
        {
          const int ss = it % kScStages, cs = it % kCvtStages;
          if (!wait_bounded(&sh->sc_full[ss], (it / kScStages) & 1, abort_flag, p.err, kErrSiteGemmFull) ||
              !wait_bounded(&sh->cvt_empty[cs], ((it / kCvtStages) & 1) ^ 1u, abort_flag, p.err, kErrSiteGemmEmpty)) {
            ok = false;
            break;
          }
          const __half* sch = reinterpret_cast<const __half*>(sc_smem + ss * kScBytes);   // s_x [2][128], s_w [2][128]
          float* cv = cvt_smem + cs * (kCvtBytes / 4);                                    // s_w/256 [2][128], s_x [2][128]
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = threadIdx.x + 64 * u;
            cv[e] = __half2float(sch[256 + e]) * 0.00390625f;
            cv[256 + e] = __half2float(sch[e]);
          }
          __syncwarp();
          if ((threadIdx.x & 31) == 0) {
            ptx::mbar_arrive(&sh->sc_empty[ss]);
            ptx::mbar_arrive(&sh->cvt_full[cs]);
          }
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    int it = 0, gi = 0, li = 0;
    bool ok = true;
    const uint32_t id8 = idesc_s8(kBM, kBN);
    const uint32_t id16 = idesc_bf16(kBM, kBN);
    for (int t = t_first; t < p.num_tiles && ok; t += t_step) {
      for (int k = kb; k < ke && ok; ++k, ++it) {
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
              // the group's first MMA overwrites the buffer (s32 256 D_g)
              ptx::umma_i8(d, ptx::sdesc_sw128(st + off), ptx::sdesc_sw128(st + kOpBytes + off), id8, kk ? 1u : 0u);
            }
            ptx::tc_commit(&sh->grp_full[b]);
          }
          __syncwarp();
        }
        if (lane == 0) ptx::tc_commit(&sh->empty[s]);
        __syncwarp();
      }
      if (!ok || nk_lr == 0) continue;
      // low-rank branch: Z L2^T into one more group buffer (its first MMA overwrites it)
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
    // ------------------------------------------------------------ epilogue (warps 4-11)
    // Each warp owns 32 rows (its TMEM lane quarter) x 64 columns and reads them in the
    // 16x256b shape: thread l holds rows {l/4, l/4 + 8} of each 16-row slab and the column
    // pairs 8i + 2(l%4) + {0, 1}, i = 0..7, i.e. 4 rows x 16 columns.  A thread then reads the
    // weight scales of 16 columns per group (8 shared loads) instead of 64.
    const int e = warp - kEpiWarp0;
    const int q = warp & 3;                    // TMEM lane quarter (rows q*32 .. q*32+31)
    const int h = e >> 2;                      // 64-column half of the tile
    const int lr = lane >> 2, lc = lane & 3;   // row within an 8-row group, column pair within a chunk
    uint8_t* buf = epi_smem + e * kEpiBoxBytes;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16) + h * 64;
    const int gm = 2 * (ke - kb);              // this CTA's groups of the 4-bit product
    const int ngroups = gm + (nk_lr > 0 ? 1 : 0);
    int gi = 0, sc_it = 0;
    bool ok = true;
    for (int t = t_first; t < p.num_tiles && ok; t += t_step) {
      const int m0 = (t % p.tiles_m) * kBM, n0 = (t / p.tiles_m) * kBN;
      const int col0 = n0 + h * 64;
      float2 acc[4][8];                        // [row j = 2 slab + half][chunk i]
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[j][i] = make_float2(0.f, 0.f);
      for (int g = 0; g < ngroups; ++g, ++gi) {
        const bool lowrank = g == gm;
        const int b = gi % kGroupBufs;
        const uint32_t base = lane_base + b * kBN;
        float sa[4] = {1.f, 1.f, 1.f, 1.f};
        const float* cva = cvt_smem + ((sc_it + (g >> 1)) % kCvtStages) * (kCvtBytes / 4) + (g & 1) * 128;
        if (!lowrank) {
          // this group's fp32 scales, converted once per K step by the widening warps
          const int cs = (sc_it + (g >> 1)) % kCvtStages;
          if ((g & 1) == 0 &&
              !wait_bounded(&sh->cvt_full[cs], ((sc_it + (g >> 1)) / kCvtStages) & 1, abort_flag, p.err,
                            kErrSiteGemmFull)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) sa[j] = cva[256 + q * 32 + 8 * j + lr];
        }
        if (!wait_bounded(&sh->grp_full[b], (gi / kGroupBufs) & 1, abort_flag, p.err, kErrSiteGemmAccFull)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        // both 16-row slabs into registers, then the buffer goes back to the MMA warp
        uint32_t v[2][32];
        ptx::tmem_ld_16x256b_x8(base, v[0]);
        ptx::tmem_ld_16x256b_x8(base + (16u << 16), v[1]);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh->grp_empty[b]);
        if (lowrank) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              acc[j][i] = __fadd2_rn(acc[j][i], u2f2(v[j >> 1][4 * i + 2 * (j & 1)], v[j >> 1][4 * i + 2 * (j & 1) + 1]));
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float* ap = cva + h * 64 + 8 * i + 2 * lc;
            const float2 a2 = SVDQ_IN_SMEM(smem_raw, ap, 8, p.err) ? *reinterpret_cast<const float2*>(ap)
                                                                   : make_float2(0.f, 0.f);
            const float2 b2 = __fmul2_rn(a2, make_float2(-kAccBiasF, -kAccBiasF));   // -B s_w / 256, exact
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              // s32 256 D + the bits of B is the float B + 256 D exactly (|256 D| < 2^22)
              const uint32_t* vv = &v[j >> 1][4 * i + 2 * (j & 1)];
              const float2 vf = u2f2(vv[0] + kAccBias, vv[1] + kAccBias);
              const float2 tt = __ffma2_rn(vf, a2, b2);
              acc[j][i] = __ffma2_rn(tt, make_float2(sa[j], sa[j]), acc[j][i]);
            }
          }
        }
        if (!lowrank && (g & 1) == 1) {
          // both groups of the K step have read their scales: the slot goes back
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&sh->cvt_empty[(sc_it + (g >> 1)) % kCvtStages]);
        }
      }
      sc_it += ke - kb;
      if (!ok) break;
      if (SPLIT) {
        // this CTA's fp32 partial of the tile to shared memory (the int8 ring is idle now: the
        // last group's MMAs have completed), float4 k of thread x at [k][thread]
        float4* part = reinterpret_cast<float4*>(smem);
        const int x = e * 32 + lane;
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            float4* dst = part + ((j * 4 + i / 2) * (kEpiWarps * 32) + x);
            if (SVDQ_IN_SMEM(smem_raw, dst, 16, p.err))
              *dst = make_float4(acc[j][i].x, acc[j][i].y, acc[j][i + 1].x, acc[j][i + 1].y);
          }
        continue;
      }
      // Y = acc + bias -> bf16, one 32-row x 64-column 128B-swizzled box and a TMA store
      if (lane == 0) ptx::bulk_wait_group_read<0>();
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float2 bv = make_float2(0.f, 0.f);
        if (p.bias && SVDQ_IN_GLOBAL(col0 + 8 * i + 2 * lc + 2 <= p.N, p.err)) {
          const uint32_t bw = __ldg(reinterpret_cast<const unsigned int*>(p.bias + col0 + 8 * i + 2 * lc));
          bv = make_float2(__uint_as_float(bw << 16), __uint_as_float(bw & 0xFFFF0000u));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int row = 8 * j + lr;
          __nv_bfloat162 hv = __floats2bfloat162_rn(acc[j][i].x + bv.x, acc[j][i].y + bv.y);
          if (SVDQ_IN_SMEM(smem_raw, buf + row * 128 + ((i ^ (row & 7)) << 4) + lc * 4, 4, p.err))
            *reinterpret_cast<__nv_bfloat162*>(buf + row * 128 + ((i ^ (row & 7)) << 4) + lc * 4) = hv;
        }
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

  if (SPLIT) {
    // CTA 0 adds the partials of the cluster's CTAs in CTA order (its own first), then the bias,
    // and writes Y.  Every thread of every CTA reaches both cluster barriers, also after a wait
    // that ran out above (the outputs are then undefined and the error word says so).
    ptx::cluster_sync();                                  // every partial is in shared memory
    if (sq == 0 && warp >= kEpiWarp0 && t_first < p.num_tiles) {
      const int e = warp - kEpiWarp0, q = warp & 3, h = e >> 2, lr = lane >> 2, lc = lane & 3;
      const int m0 = (t_first % p.tiles_m) * kBM, n0 = (t_first / p.tiles_m) * kBN;
      const int col0 = n0 + h * 64;
      const int x = e * 32 + lane;
      const float4* part = reinterpret_cast<const float4*>(smem);
      float4 sum[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) sum[k] = part[k * (kEpiWarps * 32) + x];
      const uint32_t pbase = ptx::smem_u32(smem);
      for (int r = 1; r < S; ++r) {
        float4 v[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)                      // all of a peer's values in flight at once
          v[k] = ptx::ld_shared_cluster_v4f32(
              ptx::mapa_shared(pbase + static_cast<uint32_t>((k * (kEpiWarps * 32) + x) * 16), static_cast<uint32_t>(r)));
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          sum[k].x += v[k].x;
          sum[k].y += v[k].y;
          sum[k].z += v[k].z;
          sum[k].w += v[k].w;
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float2 bv = make_float2(0.f, 0.f);
        const int c = col0 + 8 * i + 2 * lc;
        if (p.bias && SVDQ_IN_GLOBAL(c + 2 <= p.N, p.err)) {
          const uint32_t bw = __ldg(reinterpret_cast<const unsigned int*>(p.bias + c));
          bv = make_float2(__uint_as_float(bw << 16), __uint_as_float(bw & 0xFFFF0000u));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 f = sum[j * 4 + i / 2];
          const float2 a = (i & 1) ? make_float2(f.z, f.w) : make_float2(f.x, f.y);
          const int row = m0 + q * 32 + 8 * j + lr;
          if (row < p.M && SVDQ_IN_GLOBAL(c + 2 <= p.N, p.err))
            *reinterpret_cast<__nv_bfloat162*>(p.Y + static_cast<size_t>(row) * p.N + c) =
                __floats2bfloat162_rn(a.x + bv.x, a.y + bv.y);
        }
      }
    }
    ptx::cluster_sync();                                  // peers keep their partials until read
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

}  // namespace

size_t gemm_int4_smem_bytes() { return kSmemBytes; }

namespace {

// Largest number of clusters of `ks` CTAs of the split kernel that can be resident at once on
// the current device (0 if none or on error), queried once per device and split size.
int int4_resident_clusters(int ks, size_t smem) {
  constexpr int kDevs = 64;
  static int cached[kDevs][9];            // 0: not queried yet, else 1 + the figure
  int dev = 0;
  if (ks < 2 || ks > 8 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevs) return 0;
  if (cached[dev][ks] > 0) return cached[dev][ks] - 1;
  if (set_smem_limit_once(reinterpret_cast<const void*>(gemm_int4_kernel<true>), smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ks), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(ks);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_int4_kernel<true>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cached[dev][ks] = n + 1;
  return n;
}

}  // namespace

cudaError_t launch_gemm_int4(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tz,
                             const CUtensorMap& tl2, const CUtensorMap& ty, const CUtensorMap& tsa,
                             const CUtensorMap& tsb, const GemmParams& p, int num_sms,
                             cudaStream_t s) {
  const size_t smem = gemm_int4_smem_bytes();
  // Few tiles (small batches) leave most SMs idle, and each tile runs its K groups one after
  // another at the epilogue's pace: split each tile's K steps over a cluster of up to 8 CTAs
  // (the largest split that leaves every CTA a step and keeps all clusters resident at once).
  GemmParams q = p;
  q.ksplit = 1;
  const int nk_main = p.K / kKStep;
  if (p.num_tiles * 2 <= num_sms) {
    for (int ks = 8; ks >= 2; --ks) {
      const int nks = (nk_main + ks - 1) / ks;
      if (ks <= nk_main && nks * (ks - 1) < nk_main && p.num_tiles * ks <= num_sms &&
          int4_resident_clusters(ks, smem) >= p.num_tiles) {
        q.ksplit = ks;
        break;
      }
    }
  }
  const bool split = q.ksplit > 1;
  const void* kern = split ? reinterpret_cast<const void*>(gemm_int4_kernel<true>)
                           : reinterpret_cast<const void*>(gemm_int4_kernel<false>);
  cudaError_t e = set_smem_limit_once(kern, smem);
  if (e != cudaSuccess) return e;
  const int grid = split ? p.num_tiles * q.ksplit : (p.num_tiles < num_sms ? p.num_tiles : num_sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // may start under the prologue
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(q.ksplit);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = split ? 2 : 1;
  e = split ? cudaLaunchKernelEx(&cfg, gemm_int4_kernel<true>, ta, tb, tz, tl2, ty, tsa, tsb, q)
            : cudaLaunchKernelEx(&cfg, gemm_int4_kernel<false>, ta, tb, tz, tl2, ty, tsa, tsb, q);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace svdq
