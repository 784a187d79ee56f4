// C ABI of libsvdq: argument checks, TMA descriptor set-up and launches.
// The operations are specified in include/svdq.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "svdq.h"
#include "svdq_device.cuh"
#include "svdq_internal.h"

namespace svdq {

__device__ int g_device_error = 0;   // the library's one piece of device state (per device)

namespace {

thread_local int t_last_launch_count = 0;
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

svdq_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = e;
  return SVDQ_ERR_CUDA;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D row-major tensor [outer][inner] of `elem` bytes per element, tiled with a
// box of box_inner x box_outer elements (128-byte swizzle unless stated).
bool make_tmap(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem, uint64_t inner,
               uint64_t outer, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * static_cast<uint64_t>(elem)};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D tensor [d2][d1][d0] (d0 innermost) with byte strides s1, s2, no swizzle.
bool make_tmap_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2,
                  CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_NONE) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The 128x4 blocked scale layout (groups of g) seen as [rows/128][K/(4g)][64 x 8-byte words]:
// one TMA box = `blocks` row blocks x the scale blocks of 256 columns (4 for g = 16, 2 for g = 32).
bool make_tmap_sf(CUtensorMap* m, const void* base, int64_t rows_pad, int64_t K, int g, uint32_t blocks) {
  const uint64_t kblocks = static_cast<uint64_t>(K / (4 * g));
  return make_tmap_3d(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT64, 64, kblocks, static_cast<uint64_t>(rows_pad / 128), 512,
                      kblocks * 512, 64, static_cast<uint32_t>(2 * 256 / (4 * g)), blocks);
}

}  // namespace

cudaError_t set_smem_limit_once(const void* kernel, size_t smem) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  struct Seen {
    const void* kernel;
    int dev;
    size_t smem;
  };
  static Seen seen[512];
  static int n = 0;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
      if (seen[i].kernel == kernel && seen[i].dev == dev && seen[i].smem == smem) return cudaSuccess;
  }
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (n < 512) seen[n++] = Seen{kernel, dev, smem};
  return cudaSuccess;
}

namespace {

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  static int cache[64] = {0};
  if (dev < 0 || dev >= 64) return 0;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

int* device_error_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

size_t scale_bytes(svdq_format fmt, int64_t rows, int64_t K) {
  const int64_t rp = (rows + 127) / 128 * 128;
  if (fmt == SVDQ_FMT_INT4_G64) return static_cast<size_t>(rp * (K / 64) * 2);
  if (fmt == SVDQ_FMT_W8A8) return static_cast<size_t>(rp * 4);
  return static_cast<size_t>(rp * (K / fp4_group(fmt)));
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" const char* svdq_status_string(svdq_status s) {
  switch (s) {
    case SVDQ_OK: return "ok";
    case SVDQ_ERR_INVALID_ARG: return "invalid argument";
    case SVDQ_ERR_UNSUPPORTED: return "unsupported";
    case SVDQ_ERR_CUDA: return "CUDA error";
    case SVDQ_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

extern "C" svdq_status svdq_buffer_sizes(svdq_format fmt, int64_t M, int64_t N, int64_t K, int rank,
                                         svdq_sizes* out) {
  svdq_status st = check_dims(fmt, M, N, K, rank);
  if (st != SVDQ_OK) return st;
  if (!out) return SVDQ_ERR_INVALID_ARG;
  out->x = static_cast<size_t>(M * K * 2);
  out->a_codes = code_bytes(fmt, M, K);
  out->a_scales = scale_bytes(fmt, M, K);
  out->z = static_cast<size_t>(M * rank * 2);
  out->w_codes = code_bytes(fmt, N, K);
  out->w_scales = scale_bytes(fmt, N, K);
  out->l1 = static_cast<size_t>(int64_t(rank) * K * 2);
  out->l2 = static_cast<size_t>(N * rank * 2);
  out->bias = static_cast<size_t>(N * 2);
  out->y = static_cast<size_t>(M * N * 2);
  return SVDQ_OK;
}

extern "C" int svdq_last_launch_count(void) { return t_last_launch_count; }

extern "C" const char* svdq_last_cuda_error(void) { return cudaGetErrorName(t_last_cuda_error); }

extern "C" svdq_status svdq_get_last_device_error(void* cuda_stream, int* site) {
  if (site) *site = 0;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess) return SVDQ_ERR_CUDA;
  int* w = device_error_word();
  if (!w) return SVDQ_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return SVDQ_ERR_CUDA;
    if (site) *site = v;
    return SVDQ_ERR_TIMEOUT;
  }
  return SVDQ_OK;
}

extern "C" svdq_status svdq_selftest_bounded_wait(int64_t limit_ns, void* cuda_stream) {
  t_last_launch_count = 0;
  if (limit_ns < 1000 || limit_ns > 5000000000ll) return SVDQ_ERR_INVALID_ARG;
  int* err = device_error_word();
  if (!err) return SVDQ_ERR_CUDA;
  cudaError_t e = launch_selftest_bounded_wait(err, static_cast<uint64_t>(limit_ns),
                                               static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) return cuda_fail(e);
  t_last_launch_count = 1;
  return SVDQ_OK;
}

extern "C" svdq_status svdq_quantize_act_lowrank_down(svdq_format fmt, int64_t M, int64_t K, int rank,
                                                      const void* X_bf16, const float* lambda, float act_gscale,
                                                      const void* L1_bf16, void* a_codes, void* a_scales,
                                                      void* Z_bf16, void* cuda_stream) {
  t_last_launch_count = 0;
  svdq_status st = check_dims(fmt, M, 128, K, rank);
  if (st != SVDQ_OK) return st;
  if (!X_bf16 || !a_codes || !a_scales) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X_bf16) || !aligned16(a_codes) || !aligned16(a_scales)) return SVDQ_ERR_INVALID_ARG;
  if (lambda && !aligned16(lambda)) return SVDQ_ERR_INVALID_ARG;
  if (rank > 0 && (!L1_bf16 || !Z_bf16 || !aligned16(L1_bf16) || !aligned16(Z_bf16))) return SVDQ_ERR_INVALID_ARG;
  if (!is_pow2_positive(act_gscale)) return SVDQ_ERR_INVALID_ARG;
  if (fmt != SVDQ_FMT_NVFP4_G16 && act_gscale != 1.0f) return SVDQ_ERR_INVALID_ARG;

  // X and L1 seen as [K/64 column blocks][rows][64 columns]: one load brings kProBoxes
  // 64-column boxes (128B-swizzled) of 32 X rows or of all L1 rows
  CUtensorMap tx, tl1;
  const uint64_t rs = static_cast<uint64_t>(K) * 2;
  if (!make_tmap_3d(&tx, X_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64, M, K / 64, rs, 128, 64, 32, kProBoxes,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return SVDQ_ERR_CUDA;
  if (rank > 0) {
    if (!make_tmap_3d(&tl1, L1_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64, rank, K / 64, rs, 128, 64, rank,
                      kProBoxes, CU_TENSOR_MAP_SWIZZLE_128B))
      return SVDQ_ERR_CUDA;
  } else {
    tl1 = tx;
  }
  ProParams p{};
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(K);
  p.rank = rank;
  p.Mpad = static_cast<int>((M + 127) / 128 * 128);
  p.lam = lambda;
  p.gscale = act_gscale;
  p.codes = static_cast<uint8_t*>(a_codes);
  p.scales = a_scales;
  p.Z = static_cast<__nv_bfloat16*>(Z_bf16);
  p.err = device_error_word();
  if (!p.err) return SVDQ_ERR_CUDA;
  const int kf = fmt == SVDQ_FMT_NVFP4_G16   ? kFmtNvfp4
                 : fmt == SVDQ_FMT_MXFP4_G32 ? kFmtMxfp4
                 : fmt == SVDQ_FMT_W8A8      ? kFmtW8a8
                                             : kFmtInt4;
  cudaError_t e = launch_prologue(kf, tx, tl1, p,
                                  static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) return cuda_fail(e);
  t_last_launch_count = 1;
  return SVDQ_OK;
}

extern "C" svdq_status svdq_w4a4_gemm_lowrank_up(svdq_format fmt, int64_t M, int64_t N, int64_t K, int rank,
                                                 const void* a_codes, const void* a_scales, float act_gscale,
                                                 const void* w_codes, const void* w_scales, float w_gscale,
                                                 const void* Z_bf16, const void* L2_bf16, const void* bias_bf16,
                                                 void* Y_bf16, void* cuda_stream) {
  t_last_launch_count = 0;
  svdq_status st = check_dims(fmt, M, N, K, rank);
  if (st != SVDQ_OK) return st;
  if (!a_codes || !a_scales || !w_codes || !w_scales || !Y_bf16) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(Y_bf16))
    return SVDQ_ERR_INVALID_ARG;
  if (bias_bf16 && !aligned16(bias_bf16)) return SVDQ_ERR_INVALID_ARG;
  if (rank > 0 && (!Z_bf16 || !L2_bf16 || !aligned16(Z_bf16) || !aligned16(L2_bf16))) return SVDQ_ERR_INVALID_ARG;
  if (!is_pow2_positive(act_gscale) || !is_pow2_positive(w_gscale)) return SVDQ_ERR_INVALID_ARG;
  if (fmt != SVDQ_FMT_NVFP4_G16 && (act_gscale != 1.0f || w_gscale != 1.0f)) return SVDQ_ERR_INVALID_ARG;

  const int sms = device_sm_count();
  if (sms <= 0) return SVDQ_ERR_CUDA;
  GemmParams p{};
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.rank = rank;
  p.Mpad = static_cast<int>((M + 127) / 128 * 128);
  p.Npad = static_cast<int>((N + 127) / 128 * 128);
  p.out_scale = act_gscale * w_gscale;
  p.a_codes = static_cast<const uint8_t*>(a_codes);
  p.w_codes = static_cast<const uint8_t*>(w_codes);
  p.a_scales = static_cast<const uint8_t*>(a_scales);
  p.w_scales = static_cast<const uint8_t*>(w_scales);
  p.bias = static_cast<const __nv_bfloat16*>(bias_bf16);
  p.Y = static_cast<__nv_bfloat16*>(Y_bf16);
  p.y_align32 = (reinterpret_cast<uintptr_t>(Y_bf16) & 31u) == 0 ? 1 : 0;
  p.err = device_error_word();
  if (!p.err) return SVDQ_ERR_CUDA;

  CUtensorMap tz, tl2;
  cudaError_t e;
  if (fmt == SVDQ_FMT_NVFP4_G16 || fmt == SVDQ_FMT_MXFP4_G32) {
    const int g = fp4_group(fmt);
    p.tiles_m = static_cast<int>((M + 255) / 256);
    p.tiles_n = static_cast<int>((N + 255) / 256);
    p.num_tiles = p.tiles_m * p.tiles_n;
    CUtensorMap ta, tb, tsfa, tsfb;
    // K a multiple of 256: each operand load covers two K steps (a 3-D view of the rows as
    // [K/256 chunks][rows][128 bytes]); otherwise two 2-D loads per slot
    p.op_pair = (K % 256) == 0 ? 1 : 0;
    if (p.op_pair) {
      if (!make_tmap_3d(&ta, a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, M, K / 256, K / 2, 128, 128, 128, 2,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return SVDQ_ERR_CUDA;
      if (!make_tmap_3d(&tb, w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, N, K / 256, K / 2, 128, 128, 128, 2,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return SVDQ_ERR_CUDA;
    } else {
      if (!make_tmap(&ta, a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, M, 128, 128)) return SVDQ_ERR_CUDA;
      if (!make_tmap(&tb, w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, 128, 128)) return SVDQ_ERR_CUDA;
    }
    if (!make_tmap_sf(&tsfa, a_scales, p.Mpad, K, g, 1)) return SVDQ_ERR_CUDA;
    if (!make_tmap_sf(&tsfb, w_scales, p.Npad, K, g, 2)) return SVDQ_ERR_CUDA;
    if (rank > 0) {
      if (!make_tmap(&tz, Z_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rank, M, 64, 128)) return SVDQ_ERR_CUDA;
      if (!make_tmap(&tl2, L2_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rank, N, 64, 128)) return SVDQ_ERR_CUDA;
    } else {
      tz = ta;
      tl2 = tb;
    }
    e = launch_gemm_fp4(fmt == SVDQ_FMT_MXFP4_G32, ta, tb, tsfa, tsfb, tz, tl2, p, sms,
                        static_cast<cudaStream_t>(cuda_stream));
  } else if (fmt == SVDQ_FMT_W8A8) {
    p.tiles_m = static_cast<int>((M + 255) / 256);
    p.tiles_n = static_cast<int>((N + 255) / 256);
    p.num_tiles = p.tiles_m * p.tiles_n;
    CUtensorMap ta, tb, ty;
    if (!make_tmap(&ta, a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M, 128, 128)) return SVDQ_ERR_CUDA;
    if (!make_tmap(&tb, w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N, 128, 128)) return SVDQ_ERR_CUDA;
    if (rank > 0) {
      if (!make_tmap(&tz, Z_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rank, M, 64, 128)) return SVDQ_ERR_CUDA;
      if (!make_tmap(&tl2, L2_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rank, N, 64, 128)) return SVDQ_ERR_CUDA;
    } else {
      tz = ta;
      tl2 = tb;
    }
    if (!make_tmap(&ty, Y_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, M, 64, 32)) return SVDQ_ERR_CUDA;
    e = launch_gemm_w8a8(ta, tb, tz, tl2, ty, p, sms, static_cast<cudaStream_t>(cuda_stream));
  } else {
    p.tiles_m = static_cast<int>((M + 127) / 128);
    p.tiles_n = static_cast<int>(N / 128);
    p.num_tiles = p.tiles_m * p.tiles_n;
    CUtensorMap ty, ta, tb;
    if (!make_tmap(&ty, Y_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, M, 64, 32)) return SVDQ_ERR_CUDA;
    if (!make_tmap(&ta, a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, M, 64, 128, CU_TENSOR_MAP_SWIZZLE_64B))
      return SVDQ_ERR_CUDA;
    if (!make_tmap(&tb, w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, 64, 128, CU_TENSOR_MAP_SWIZZLE_64B))
      return SVDQ_ERR_CUDA;
    if (rank > 0) {
      if (!make_tmap(&tz, Z_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rank, M, 64, 128)) return SVDQ_ERR_CUDA;
      if (!make_tmap(&tl2, L2_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rank, N, 64, 128)) return SVDQ_ERR_CUDA;
    } else {
      tz = ta;
      tl2 = tb;
    }
    // group scales: fp16 [K/64][rows_pad] tensors, boxes of 128 rows x 2 groups
    CUtensorMap tsa, tsb;
    if (!make_tmap(&tsa, a_scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, p.Mpad, K / 64, 128, 2,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
      return SVDQ_ERR_CUDA;
    if (!make_tmap(&tsb, w_scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, p.Npad, K / 64, 128, 2,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
      return SVDQ_ERR_CUDA;
    e = launch_gemm_int4(ta, tb, tz, tl2, ty, tsa, tsb, p, sms, static_cast<cudaStream_t>(cuda_stream));
  }
  if (e != cudaSuccess) return cuda_fail(e);
  t_last_launch_count = 1;
  return SVDQ_OK;
}
