// Device-side declarations shared by the kernels of libsvdq.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "ptx.cuh"

namespace svdq {

constexpr int kFmtNvfp4 = 1;
constexpr int kFmtInt4 = 2;
constexpr int kFmtMxfp4 = 3;
constexpr int kFmtW8a8 = 4;

// Codes recorded in the device error word when a bounded wait runs out.
enum : int {
  kErrSiteProEmpty = 1,
  kErrSiteProFull = 2,
  kErrSiteGemmEmpty = 11,
  kErrSiteGemmFull = 12,
  kErrSiteGemmAccEmpty = 13,
  kErrSiteGemmAccFull = 14,
  kErrSiteGemmConvEmpty = 15,
  kErrSiteGemmConvFull = 16,
  kErrSiteGemmSfFree = 17,
  kErrSiteGemmSfReady = 18,
  kErrSiteGemmConvDone = 19,
  kErrSiteGemmAccFinal = 20,
  kErrSiteSelftest = 90,
  // Debug builds (-DSVDQ_DEBUG) only: an access outside its buffer was found and skipped.
  kErrSiteBoundsGlobal = 201,   // a plain global load or store past its buffer
  kErrSiteBoundsShared = 202,   // a shared-memory access past the dynamic allocation
};

// Bounds checks of the debug build.  SVDQ_DEBUG_OK(cond, site, err) is true in a release build
// (the check compiles away); in a debug build a false condition records `site` in the device
// error word (first failure wins) and the caller skips the access, so a bad index never turns
// into an out-of-bounds access.
#ifdef SVDQ_DEBUG
__device__ __forceinline__ bool debug_in_bounds(bool ok, int site, int* err) {
  if (!ok) atomicCAS(err, 0, site);
  return ok;
}
__device__ __forceinline__ uint32_t dynamic_smem_bytes() {
  uint32_t v;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(v));
  return v;
}
// [p, p + bytes) lies inside this CTA's dynamic shared memory starting at base
__device__ __forceinline__ bool smem_in_bounds(const void* base, const void* p, uint32_t bytes) {
  const uintptr_t b = reinterpret_cast<uintptr_t>(base), a = reinterpret_cast<uintptr_t>(p);
  return a >= b && a + bytes <= b + dynamic_smem_bytes();
}
#define SVDQ_DEBUG_OK(cond, site, err) (::svdq::debug_in_bounds((cond), (site), (err)))
#else
#define SVDQ_DEBUG_OK(cond, site, err) (true)
#endif
// A plain global access whose index satisfies `cond`; a shared-memory access of `bytes` at
// `ptr` inside the dynamic allocation that starts at `base`.
#define SVDQ_IN_GLOBAL(cond, err) SVDQ_DEBUG_OK((cond), ::svdq::kErrSiteBoundsGlobal, (err))
#define SVDQ_IN_SMEM(base, ptr, bytes, err) \
  SVDQ_DEBUG_OK(::svdq::smem_in_bounds((base), (ptr), (bytes)), ::svdq::kErrSiteBoundsShared, (err))

// A wait gives up after this many nanoseconds (~1 s); legitimate waits here
// last microseconds.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// Parity wait on an mbarrier with a time limit.  On time-out the first waiter
// records its site in the device error word, raises the CTA's abort flag and
// returns false; waiters that see the abort flag return false as well.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                             int* err, int site, uint64_t limit_ns = kWaitLimitNs) {
  const uint32_t a = ptx::smem_u32(bar);
  if (ptx::mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  uint32_t spins = 0;
  while (true) {
    if (ptx::mbar_try_wait(a, parity)) return true;
    if ((++spins & 63u) == 0) {
      if (*abort_flag) return false;
      if (ptx::globaltimer() - t0 > limit_ns) {
        atomicCAS(err, 0, site);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Tile schedule of the persistent pair GEMMs: cluster c takes the contiguous run
// [begin, begin + count) of the N-fastest tile numbering, so consecutive tiles of a
// cluster share the M block.
struct TileSeq {
  int begin, count, tiles_n;
  __device__ TileSeq(int num_tiles, int tiles_n_, int cluster, int nclusters) : tiles_n(tiles_n_) {
    const int base = num_tiles / nclusters, extra = num_tiles % nclusters;
    begin = cluster * base + min(cluster, extra);
    count = base + (cluster < extra ? 1 : 0);
  }
  __device__ int mb(int j) const { return (begin + j) / tiles_n; }
  __device__ int nb(int j) const { return (begin + j) % tiles_n; }
};

// Named barrier `id` over `count` threads (a multiple of 32).
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

constexpr int kProBoxes = 4;   // 64-column boxes per prologue TMA load

// Self-test of the bounded wait: a wait on a barrier nothing arrives at.
cudaError_t launch_selftest_bounded_wait(int* err, uint64_t limit_ns, cudaStream_t s);
// Raises a kernel's dynamic shared-memory limit to `smem` bytes on the current device, once
// per (kernel, device, size): the attribute belongs to the function in the device's context,
// and setting it on every launch costs host time.
cudaError_t set_smem_limit_once(const void* kernel, size_t smem);

struct ProParams {
  int M, K, rank, Mpad, stages;
  int ksplit;                // CTAs of a cluster that split one row block's K stages (1: none)
  const float* lam;          // nullable
  float gscale;              // activation tensor scale (NVFP4), 1 for INT4
  uint8_t* codes;            // [M][K/2] (W8A8: [M][K])
  void* scales;              // format-specific layout (W8A8: fp32 [Mpad])
  __nv_bfloat16* Z;          // [M][rank]
  int* err;                  // device error word
};

struct GemmParams {
  int M, N, K, rank;
  int Mpad, Npad;
  float out_scale;           // act_gscale * w_gscale
  const uint8_t* a_scales;   // NVFP4: blocked E4M3; INT4: fp16 [K/64][Mpad]; W8A8: fp32 [Mpad]
  const uint8_t* w_scales;   // NVFP4: blocked E4M3; INT4: fp16 [K/64][Npad]; W8A8: fp32 [Npad]
  const uint8_t* a_codes;    // [M][K/2] (W8A8: s8 [M][K])
  const uint8_t* w_codes;    // [N][K/2] (W8A8: s8 [N][K])
  const __nv_bfloat16* bias; // nullable
  __nv_bfloat16* Y;          // [M][N]
  int* err;
  int num_tiles, tiles_m, tiles_n;
  int op_pair;               // FP4: A and B tensor maps are 3-D and load two K steps at once
  int y_align32;             // Y is 32-byte aligned (256-bit stores)
  int ksplit;                // INT4: CTAs of a cluster that split one tile's K steps (1: none)
};

cudaError_t launch_prologue(int fmt, const CUtensorMap& tx, const CUtensorMap& tl1, const ProParams& p,
                            cudaStream_t s);

// NVFP4 (mx = false) or MXFP4 (mx = true) GEMM with the fused low-rank up projection.
cudaError_t launch_gemm_fp4(bool mx, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsfa,
                            const CUtensorMap& tsfb, const CUtensorMap& tz, const CUtensorMap& tl2,
                            const GemmParams& p, int num_sms, cudaStream_t s);
size_t gemm_int4_smem_bytes();
// W8A8 GEMM: s32 accumulation of the 8-bit product, per-row / per-column fp32 scales in the
// epilogue, the low-rank product in a second (fp32) TMEM accumulator.
cudaError_t launch_gemm_w8a8(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tz,
                             const CUtensorMap& tl2, const CUtensorMap& ty, const GemmParams& p, int num_sms,
                             cudaStream_t s);
cudaError_t launch_gemm_int4(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tz,
                             const CUtensorMap& tl2, const CUtensorMap& ty, const CUtensorMap& tsa,
                             const CUtensorMap& tsb, const GemmParams& p, int num_sms, cudaStream_t s);

}  // namespace svdq
