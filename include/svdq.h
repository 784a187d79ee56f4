/*
 * svdq.h -- C ABI of the B200 (sm_100a) SVDQuant W4A4 + low-rank linear layer.
 *
 * The layer computes, for smoothed activations X_hat = X diag(lambda)^-1,
 *
 *     Y = Q(X_hat) Q(R) + (X_hat L1) L2 + bias
 *
 * ("SVDQuant 阅读笔记：用少量高精度计算保护 4-bit 扩散模型", §4.2 eq.(7); the
 * smoothing of §3.1 eq.(3); the forward identity of the msModelSlim page
 * "SVDQuant：基于低秩残差重构的扩散模型后训练量化算法说明", "前向等价关系").
 * It runs as two device calls that follow the fused data flow of §6.1
 * ("算法 2"): a prologue that reads X once to smooth, quantize and
 * down-project it, and a W4A4 GEMM whose epilogue adds the up-projection,
 * the bias and writes Y once.  A third, host-only call packs an
 * already-decomposed layer.
 *
 * Notation: M = tokens (b), K = input features (m), N = output features (n),
 * r = rank of the low-rank branch.  g = 16 (NVFP4), 32 (MXFP4) or 64 (INT4), G = K / g.
 * The W8A8 format (8-bit codes, one scale per row) runs through the same two calls.
 *
 * Conventions for every call
 *   - Ownership: the caller owns every buffer.  The library never allocates
 *     or frees memory; its only state is one static device error word per
 *     device (see svdq_get_last_device_error).
 *   - Device calls are asynchronous on the given CUDA stream (a cudaStream_t
 *     passed as void*; NULL = the legacy default stream).  They return after
 *     launching.  Pointers of device calls are device pointers.
 *   - Arguments are checked before any launch; a bad argument returns a
 *     status and launches nothing.  Limits: M >= 1, K % 128 == 0, N % 128 == 0,
 *     0 <= r <= 128 with r % 16 == 0, 16-byte aligned pointers, tensor scales
 *     that are positive powers of two.
 *   - Errors: launch failures map to SVDQ_ERR_CUDA.  Every wait inside the
 *     kernels is bounded; a wait that runs out records SVDQ_ERR_TIMEOUT in the
 *     device error word and the kernel returns early (read it with
 *     svdq_get_last_device_error).  After SVDQ_ERR_TIMEOUT the outputs of the
 *     calls that ran since the error word was last cleared are undefined: the
 *     kernel stopped before writing all of them.  NaN / Inf inputs are outside
 *     the contract.
 *
 * Buffer layouts (all row-major, little-endian)
 *   X        bf16 [M][K]
 *   lambda   fp32 [K]                    (NULL means lambda = 1); every entry finite,
 *                                        normal and > 0 (the divide assumes a normal
 *                                        positive divisor; other values are outside
 *                                        the contract)
 *   L1       bf16 [r][K]                 (the "l1 = V^T" [rank, in] shape)
 *   Z        bf16 [M][r]                 Z = bf16(X_hat L1^T), fp32 accumulation
 *   L2s      bf16 [N][r]                 (the "l2 = U S" [out, rank] shape), stored
 *                                        divided by (act_gscale * w_gscale)
 *   bias     bf16 [N]                    (nullable)
 *   Y        bf16 [M][N]
 *   codes    u8   [rows][K/2]            element k of a row in the low nibble of
 *                                        byte k/2 when k is even, high nibble when odd.
 *                                        NVFP4, MXFP4: E2M1 code (bit 3 = sign);
 *                                        INT4: 4-bit two's complement in -7..7.
 *            W8A8: s8 [rows][K]          one byte per element, two's complement in -127..127.
 *   NVFP4 scales  u8 (E4M3), MXFP4 scales u8 (E8M0: the scale is 2^(byte - 127)), both in the
 *       "128x4 blocked" layout, rows padded to Rp = ceil(rows/128)*128:
 *       byte offset of (row, grp) = ((row/128)*(K/(4g)) + grp/4)*512
 *                                   + (row%32)*16 + ((row%128)/32)*4 + grp%4
 *       size = Rp * K / g bytes.  Padding rows hold 0.
 *   INT4 scales   fp16, group-major, rows padded to Rp = ceil(rows/128)*128:
 *       element offset of (row, grp) = grp*Rp + row;  size = Rp * (K/64) * 2 bytes.
 *   W8A8 scales   fp32 [Rp], one per row (per token for activations, per output
 *       channel for weights); size = Rp * 4 bytes.  Padding rows hold 0.
 *   ("rows" is M for activations, N for weights.)
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,  /* bad size, NULL or misaligned pointer, bad scale */
  SVDQ_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement    */
  SVDQ_ERR_CUDA = 3,         /* a CUDA runtime / launch error                    */
  SVDQ_ERR_TIMEOUT = 4       /* a bounded wait inside a kernel ran out           */
} svdq_status;

typedef enum {
  /* E2M1 codes, groups of 16 along K, E4M3 group scales, power-of-two tensor
   * scales ("SVDQuant 阅读笔记" §2.2 and §8: NVFP4 g16 with FP8 scale). */
  SVDQ_FMT_NVFP4_G16 = 1,
  /* symmetric INT4 codes -7..7, groups of 64 along K, fp16 group scales
   * ("SVDQuant 阅读笔记" §2.2 eq.(1) and §8: INT4 g64 with 16-bit scale). */
  SVDQ_FMT_INT4_G64 = 2,
  /* E2M1 codes, groups of 32 along K, one shared power-of-two scale per group stored
   * as its E8M0 byte: X = 2^(floor(log2 a) - 2), clamped to [2^-127, 2^127], the MX
   * shared scale of the OCP Microscaling format for E2M1 (largest value 6 = 1.5 * 2^2);
   * q = e2m1_satfinite(x / X).  No tensor scale: act_gscale and w_gscale are 1.
   * ("SVDQuant（实验性功能）": its Nunchaku export needs E2M1 weights and activations in
   * 32-element groups, quantized symmetrically.) */
  SVDQ_FMT_MXFP4_G32 = 3,
  /* symmetric INT8 codes -127..127 with one fp32 scale per row spanning all of K:
   * s = fp32(a/127) with a = max|x| over the row, q = clamp(rint(fp32(x/s)), -127, 127)
   * (a zero row gives s = 0 and zero codes).  Activations are quantized per token by
   * the prologue, weights per output channel by the pack.  No tensor scale.
   * ("SVDQuant 阅读笔记" §8, appendix D: the 8-bit setting uses rank 16, per-token
   * dynamic activation quantization and per-channel weight quantization.) */
  SVDQ_FMT_W8A8 = 4
} svdq_format;

/* Byte sizes of every buffer of one layer call (no allocation happens). */
typedef struct {
  size_t x;          /* X      M*K*2                */
  size_t a_codes;    /* M*K/2 (W8A8: M*K)           */
  size_t a_scales;   /* per the scale layout above  */
  size_t z;          /* M*r*2                       */
  size_t w_codes;    /* N*K/2 (W8A8: N*K)           */
  size_t w_scales;   /* per the scale layout above  */
  size_t l1;         /* r*K*2                       */
  size_t l2;         /* N*r*2                       */
  size_t bias;       /* N*2                         */
  size_t y;          /* M*N*2                       */
} svdq_sizes;

/* Fills *out for (fmt, M, N, K, rank).  Same argument checks as the calls. */
svdq_status svdq_buffer_sizes(svdq_format fmt, int64_t M, int64_t N, int64_t K, int rank,
                              svdq_sizes* out);

/*
 * Host-only pack of an already-decomposed layer ("SVDQuant 阅读笔记" §5
 * "算法 1" steps 5 and 9: quantize the residual, save factors, codes and
 * scales).  Inputs are host fp32 arrays:
 *   R  [N][K]   residual of the smoothed weight, one row per output channel
 *   L1 [rank][K], L2 [N][rank]   (NULL when rank == 0)
 * Outputs are host buffers of the sizes given by svdq_buffer_sizes:
 *   w_codes, w_scales   quantized R in the layouts above; each group of g
 *                       elements of a row along K gets
 *                       INT4:  s = fp16(fp32(a/7)), q = clamp(rint(fp32(x/s)), -7, 7)
 *                       NVFP4: s = e4m3_satfinite(fp32(fp32(a/6)/g_w)),
 *                              q = e2m1_satfinite(fp32(x/(s*g_w)))
 *                       with a = max|x| over the group (a zero scale gives zero codes)
 *                       MXFP4: the rule of SVDQ_FMT_MXFP4_G32 (a zero group gets byte 0)
 *                       W8A8: the rule of SVDQ_FMT_W8A8, one scale per row of R
 *   *w_gscale           NVFP4: g_w = 2^ceil(log2(max|R| / (6*448))) (1 if R == 0);
 *                       INT4, MXFP4, W8A8: 1
 *   L1_bf16             bf16 of L1 (round to nearest even)
 *   L2_bf16             bf16 of bf16(L2) / (act_gscale * g_w); must be exact
 * act_gscale is the activation tensor scale later given to the device calls
 * (a positive power of two; 1 for INT4, MXFP4 and W8A8).  Returns SVDQ_ERR_INVALID_ARG for
 * bad sizes / NULL pointers / a non power-of-two act_gscale, and
 * SVDQ_ERR_UNSUPPORTED if pre-dividing L2 would not be exact in bf16.
 */
svdq_status svdq_pack_weight(svdq_format fmt, int64_t N, int64_t K, int rank, float act_gscale,
                             const float* R, const float* L1, const float* L2,
                             void* w_codes, void* w_scales, float* w_gscale,
                             uint16_t* L1_bf16, uint16_t* L2_bf16);

/*
 * Device prologue ("算法 2" steps 1-3 of "SVDQuant 阅读笔记" §6.1): one read of X.
 *   X_hat = bf16(fp32(X) / lambda)            (IEEE fp32 divide, one bf16 rounding)
 *   a_codes, a_scales = group quantization of X_hat along K (rules of svdq_pack_weight,
 *                       with act_gscale in place of g_w; INT4, MXFP4 and W8A8 require
 *                       act_gscale == 1).  W8A8 quantizes each token row with its own
 *                       scale, so its prologue reads X twice: once for the row maxima
 *                       (and Z), once to write the codes (the second read is served
 *                       mostly from L2).
 *   Z = bf16(X_hat L1^T)                      (fp32 accumulation; skipped when rank == 0)
 * X, lambda, L1 are inputs; a_codes, a_scales, Z outputs (Z may be NULL when rank == 0).
 */
svdq_status svdq_quantize_act_lowrank_down(svdq_format fmt, int64_t M, int64_t K, int rank,
                                           const void* X_bf16, const float* lambda,
                                           float act_gscale, const void* L1_bf16,
                                           void* a_codes, void* a_scales, void* Z_bf16,
                                           void* cuda_stream);

/*
 * Device W4A4 GEMM with the fused up-projection ("算法 2" steps 4-8):
 *   Y = bf16( act_gscale * w_gscale * ( sum_G s_x s_w sum_{k in G} q_x q_w + Z L2s^T ) + bias )
 * which equals Q(X_hat) Q(R) + Z L2 + bias because L2s = L2 / (act_gscale * w_gscale).
 * The low-rank product is accumulated on the tensor cores into the same fp32
 * accumulator as the 4-bit product, so Y is written exactly once.
 * W8A8: Y = bf16( s_x[m] s_w[n] sum_k q_x q_w + Z L2^T + bias ), the 8-bit sum exact in
 * an s32 accumulator and the low-rank product in a second, fp32 accumulator, both on
 * the tensor cores and combined in the epilogue (act_gscale = w_gscale = 1, L2s = L2).
 * Z and L2s may be NULL when rank == 0; bias may be NULL.
 * Stream order is kept: the GEMM is launched so that it may start its set-up while the
 * kernel before it on the stream (normally this library's prologue) finishes, but it reads
 * its inputs only after that kernel has completed (programmatic dependent launch).
 */
svdq_status svdq_w4a4_gemm_lowrank_up(svdq_format fmt, int64_t M, int64_t N, int64_t K, int rank,
                                      const void* a_codes, const void* a_scales, float act_gscale,
                                      const void* w_codes, const void* w_scales, float w_gscale,
                                      const void* Z_bf16, const void* L2_bf16,
                                      const void* bias_bf16, void* Y_bf16, void* cuda_stream);

/* Human-readable name of a status. */
const char* svdq_status_string(svdq_status s);

/*
 * Synchronizes the stream, then reads and clears the device error word of the
 * current device.  Returns SVDQ_OK, SVDQ_ERR_TIMEOUT (a bounded wait ran out;
 * *site, if not NULL, receives the code of the wait that ran out) or
 * SVDQ_ERR_CUDA (a sticky CUDA error).
 */
svdq_status svdq_get_last_device_error(void* cuda_stream, int* site);

/*
 * Failure-path self-test: launches one warp that waits on a barrier nothing arrives
 * at, with the same bounded wait the kernels use but a limit of limit_ns
 * nanoseconds (1e3 <= limit_ns <= 5e9).  The wait runs out, the kernel records
 * site 90 in the device error word and returns, leaving the context usable; a
 * following svdq_get_last_device_error returns SVDQ_ERR_TIMEOUT with *site == 90.
 * Returns SVDQ_ERR_INVALID_ARG for a limit out of range, SVDQ_ERR_CUDA if the
 * launch fails.
 */
svdq_status svdq_selftest_bounded_wait(int64_t limit_ns, void* cuda_stream);

/* Number of kernels the last successful device call launched (for launch accounting). */
int svdq_last_launch_count(void);

/* Name of the CUDA runtime error behind the last SVDQ_ERR_CUDA returned on this
 * host thread ("cudaSuccess" if none). */
const char* svdq_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H_ */
