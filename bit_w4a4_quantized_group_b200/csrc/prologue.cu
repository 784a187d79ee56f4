// Prologue kernel: smoothing divide, group quantization and low-rank down
// projection in one read of X.
//
// "SVDQuant 阅读笔记：用少量高精度计算保护 4-bit 扩散模型", §6.1 "算法 2"
// steps 1-3: read a tile of the high-precision activations once, reuse it for
// Z = X_hat L1 and for the 4-bit quantization (codes + scales).  The smoothing
// divide is X D^-1 of §3.1 eq.(3); the quantizers are eq.(1) (INT4 g64,
// 16-bit scale) and NVFP4 g16 with E4M3 scales (§2.2, §8).
//
// Design (B200, HBM-bound): a producer warp streams 32-row tiles of X (and the
// matching columns of L1) into a shared-memory ring with TMA, and writes
// lambda and RN(1/lambda) for the tile's columns next to them.  NW compute
// warps each own a 16-row x 64-column box of every tile.  X_hat is formed in
// registers in the m16n8k16 fragment layout, so the same registers feed the
// bf16 tensor-core MMA for Z and the quantizer; codes are staged per warp in
// shared memory and written back as 16-byte row segments.  Z partials of the
// warps that share a row strip are summed in a fixed order (deterministic).
//
// Few rows (small batches) leave most SMs idle, since a CTA owns 32 rows over all of K.  The
// 4-bit formats then split each row block's K stages over a cluster of up to 8 CTAs: codes
// and scales are local to their groups, and the Z partials of the CTAs are added by CTA 0
// of the cluster through distributed shared memory, in CTA order (deterministic).
//
// W8A8 (the 8-bit setting: one scale per token row over all of K) needs each row's
// maximum before any code can be formed, so the kernel makes two passes over its rows:
// the first forms X_hat, the Z products and the row maxima; the compute warps then
// combine their maxima and write the fp32 row scales; the second pass re-reads X (the
// CTAs' rows were just read, so the L2 serves most of it), re-forms X_hat and writes
// one-byte codes with an IEEE-exact divide by the row scale.  Under the K split each CTA
// publishes its rows' maxima after the first pass and signals every peer of the cluster
// (a remote mbarrier arrive with release at cluster scope); once all peers have signalled,
// it takes the maximum over the cluster (exact, order-independent) before the second pass.
//
// Divisions are IEEE-exact without the divide instruction sequence:
//  * X / lambda uses Markstein's correction (P. Markstein, "Computation of
//    elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
//    Dev. 34(1), 1990): with y = RN(1/b) and an approximation q of a/b, the
//    remainder r = a - b q is exact under FMA and RN(q + r y) = RN(a/b) once q
//    is within one ulp.  Two correction steps from q0 = RN(a y) are used: the
//    first brings q within one ulp, the second rounds correctly.
//  * x_hat / (s g) only decides a 4-bit code: x_hat has 8 significant bits and
//    (s g) at most 11, so the exact quotient is either exactly a rounding
//    midpoint of the code grid or at least 2^-16 (relative) away from every
//    midpoint.  One correction step from an approximate reciprocal recovers
//    exact midpoints exactly and leaves every other quotient within 2^-20 of
//    its value, so the code equals the code of the correctly rounded quotient.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"
#include "svdq_device.cuh"

namespace svdq {

namespace {

constexpr int kProRows = 32;                      // rows per CTA (two 16-row strips)
constexpr uint32_t kXBoxBytes = kProRows * 128;   // 32 rows x 64 bf16

__host__ __device__ constexpr int compute_warps(int rank) { return rank <= 64 ? 16 : 8; }

struct ProSmemLayout {
  uint32_t x_off, l1_off, lam_off, rlam_off, stage_bytes;
};

__host__ __device__ inline ProSmemLayout pro_layout(int rank, int boxes) {
  ProSmemLayout L;
  L.x_off = 0;
  L.l1_off = boxes * kXBoxBytes;
  L.lam_off = L.l1_off + boxes * 128u * rank;
  L.rlam_off = L.lam_off + boxes * 64u * 4u;
  uint32_t sz = L.rlam_off + boxes * 64u * 4u;
  L.stage_bytes = (sz + 1023u) & ~1023u;
  return L;
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Packed form of the divides below, two lanes at once: the inputs are the negated
// dividends na = -a and the negated reciprocals ny = -y.  RN(na ny) = RN(a y),
// fma(b, q, na) = RN(b q - a) and fma(r, ny, q) = RN(q - r y), so every step equals
// the scalar step bit for bit, signed zeros included, with no negations in the chain.
__device__ __forceinline__ float2 div_rn2(float2 na, float2 b, float2 ny) {
  float2 q = __fmul2_rn(na, ny);
  float2 r = __ffma2_rn(b, q, na);
  q = __ffma2_rn(r, ny, q);
  r = __ffma2_rn(b, q, na);
  return __ffma2_rn(r, ny, q);
}
__device__ __forceinline__ float2 div_code2(float2 na, float2 b, float2 ny) {
  const float2 q = __fmul2_rn(na, ny);
  return __ffma2_rn(__ffma2_rn(b, q, na), ny, q);
}
// -lo and -hi of a bf16 pair as floats
__device__ __forceinline__ float2 neg_bf16x2(uint32_t v) {
  return make_float2(__uint_as_float((v << 16) ^ 0x80000000u), __uint_as_float((v & 0xFFFF0000u) ^ 0x80000000u));
}

// RN(a / b) given y = RN(1 / b), b > 0 (two Markstein corrections).
// The remainder is formed as (b q - a) and subtracted, which keeps the sign of a
// zero quotient: for a = -0 every step stays -0.
__device__ __forceinline__ float div_rn(float a, float b, float y) {
  const float q0 = a * y;
  const float q1 = fmaf(-fmaf(b, q0, -a), y, q0);
  return fmaf(-fmaf(b, q1, -a), y, q1);
}
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
// a / b accurate enough to decide a 4-bit code (see the header), exact on midpoints.
__device__ __forceinline__ float div_code(float a, float b, float y) {
  const float q0 = a * y;
  return fmaf(-fmaf(b, q0, -a), y, q0);
}

// Bytes of code staging per compute warp: 16 rows x 64 columns of 4-bit or 8-bit codes.
__host__ __device__ constexpr int code_stage_bytes(int fmt) { return fmt == kFmtW8a8 ? 1024 : 512; }
__host__ __device__ constexpr int passes(int fmt) { return fmt == kFmtW8a8 ? 2 : 1; }

template <int FMT, int RANK, bool SPLIT>
__global__ void __launch_bounds__(32 * (compute_warps(RANK) + 1), 1)
    prologue_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_l1,
                    ProParams p) {
  constexpr int NW = compute_warps(RANK);      // compute warps
  constexpr int BOXES = NW / 2;                 // 64-column boxes per stage
  static_assert(BOXES % kProBoxes == 0, "a stage holds whole TMA loads");
  constexpr int BK = 64 * BOXES;                // columns per stage
  constexpr int NT = RANK / 8;                  // n8 tiles of Z
  const ProSmemLayout L = pro_layout(RANK, BOXES);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * L.stage_bytes);
  uint64_t* empty = full + S;
  constexpr int CSTB = code_stage_bytes(FMT);
  constexpr int NPASS = passes(FMT);
  uint8_t* cstage = reinterpret_cast<uint8_t*>(empty + S);          // NW warps x CSTB code staging
  float* rmax_s = reinterpret_cast<float*>(cstage + NW * CSTB);     // W8A8: [BOXES][2 strips][16 rows]
  float* rmax_cta = rmax_s + BOXES * 32;                              // W8A8 K split: this CTA's 32 row maxima
  uint64_t* rm_bar = reinterpret_cast<uint64_t*>(rmax_cta + 32);      // ... published by every peer
  volatile int* abort_flag = reinterpret_cast<volatile int*>(rm_bar + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = SPLIT ? static_cast<int>(blockIdx.x) % p.ksplit : 0;   // rank in the K-split cluster
  const int rb = SPLIT ? static_cast<int>(blockIdx.x) / p.ksplit : static_cast<int>(blockIdx.x);  // row block
  const int m0 = rb * kProRows;
  const int nkt_all = (p.K + BK - 1) / BK;
  const int nks = SPLIT ? (nkt_all + p.ksplit - 1) / p.ksplit : nkt_all;
  const int kbeg = split * nks;                                   // this CTA's stages [kbeg, kbeg + nkt)
  const int nkt = SPLIT ? max(0, min(nkt_all, kbeg + nks) - kbeg) : nkt_all;
  // Every CTA reads all of its L1 columns; starting the K loop at a different stage per CTA
  // spreads those reads over the L2 instead of sending every SM to the same lines at once.
  const int kt0 = nkt > 0 ? rb % nkt : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full[s], 32);     // every producer lane arrives (its lambda stores) + TMA bytes
      ptx::mbar_init(&empty[s], NW);
    }
    if (SPLIT && FMT == kFmtW8a8) ptx::mbar_init(rm_bar, static_cast<uint32_t>(p.ksplit - 1));
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  // W8A8 K split: every CTA's barriers are initialised before any peer can arrive on them
  if (SPLIT && FMT == kFmtW8a8) ptx::cluster_sync();
  // the GEMM launched after this kernel may start its own set-up now (on SMs this grid leaves
  // free); it reads this kernel's outputs only after the whole grid has completed
  ptx::griddep_launch_dependents();

  if (warp == NW) {
    // ---------------------------------------------------------------- producer warp
    if (lane == 0) {
      ptx::prefetch_tmap(&tmap_x);
      if (RANK > 0) ptx::prefetch_tmap(&tmap_l1);
    }
    // lambda of the next stage is loaded into registers one stage ahead, so that its latency
    // overlaps the current stage instead of holding back the stage's release
    float lv[BK / 32];
    auto load_lambda = [&](int kt) {
#pragma unroll
      for (int i = 0; i < BK / 32; ++i) {           // independent loads, all in flight together
        const int c = kt * BK + i * 32 + lane;
        lv[i] = (p.lam != nullptr && c < p.K) ? __ldg(p.lam + c) : 1.f;
      }
    };
    if (nkt > 0) load_lambda(kbeg + kt0 % nkt);
    const int nit = NPASS * nkt;
    for (int it = 0; it < nit; ++it) {
      const int s = it % S;
      const uint32_t ph = (it / S) & 1;
      if (!wait_bounded(&empty[s], ph ^ 1u, abort_flag, p.err, kErrSiteProEmpty)) break;
      const int ki = it % nkt;
      const bool with_l1 = RANK > 0 && it < nkt;      // L1 is only needed by the first pass
      const int kt = kbeg + (kt0 + ki) % nkt;
      const int col0 = kt * BK;
      const int nbox = min(BK, p.K - col0) / 64;
      uint8_t* st = smem + s * L.stage_bytes;
      float* lam_s = reinterpret_cast<float*>(st + L.lam_off);
      float* rlam_s = reinterpret_cast<float*>(st + L.rlam_off);
      if (lane == 0) {
        // kProBoxes boxes per load; boxes past K are zero-filled and counted like the others
        const int nload = (nbox + kProBoxes - 1) / kProBoxes;
        ptx::mbar_expect_tx(&full[s], nload * kProBoxes * (kXBoxBytes + (with_l1 ? 128u * RANK : 0u)));
        for (int b = 0; b < nload * kProBoxes; b += kProBoxes) {
          ptx::tma_load_3d(st + L.x_off + b * kXBoxBytes, &tmap_x, &full[s], 0, m0, col0 / 64 + b);
          if (with_l1) ptx::tma_load_3d(st + L.l1_off + b * 128 * RANK, &tmap_l1, &full[s], 0, 0, col0 / 64 + b);
        }
      }
      float cur[BK / 32];
#pragma unroll
      for (int i = 0; i < BK / 32; ++i) cur[i] = lv[i];
      if (it + 1 < nit) load_lambda(kbeg + (kt0 + (it + 1) % nkt) % nkt);
      if (!(SVDQ_IN_SMEM(smem_raw, lam_s, BK * 4, p.err) && SVDQ_IN_SMEM(smem_raw, rlam_s, BK * 4, p.err))) {
        ptx::mbar_arrive(&full[s]);
        continue;
      }
#pragma unroll
      for (int i = 0; i < BK / 32; ++i) {
        lam_s[i * 32 + lane] = cur[i];
        rlam_s[i * 32 + lane] = -__frcp_rn(cur[i]);   // negated, for the packed divides
      }
      ptx::mbar_arrive(&full[s]);   // each lane releases its own lambda stores
    }
  } else {
    // ---------------------------------------------------------------- compute warps
    const int strip = warp & 1;         // rows 16*strip .. 16*strip+15 of the CTA tile
    const int phase = warp >> 1;        // 64-column box of every stage
    const int g = lane >> 2, tig = lane & 3;
    const int row_a = m0 + strip * 16 + g;   // rows of this thread's fragments
    const int row_b = row_a + 8;
    float acc[NT > 0 ? NT : 1][4];
#pragma unroll
    for (int i = 0; i < (NT > 0 ? NT : 1); ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    uint8_t* cst = cstage + warp * CSTB;
    const int K2 = p.K / 2;
    const float gs = p.gscale;
    const float inv_gs = 1.0f / gs;     // exact: gs is a power of two
    constexpr float kRcp6 = 1.0f / 6.0f, kRcp7 = 1.0f / 7.0f;
    bool ok = true;
    // W8A8: running max |x_hat| of rows row_a / row_b over this warp's boxes (first pass), then
    // the row scales as divisors for the second pass: x_hat / s is formed as (x_hat f) / (s f)
    // with f = 2^64 for scales below 2^-64 (exact), so that RN(1 / (s f)) stays finite
    float rmax_a = 0.f, rmax_b = 0.f;
    float w8_fa = 1.f, w8_fb = 1.f, w8_ba = 0.f, w8_bb = 0.f, w8_nya = 0.f, w8_nyb = 0.f;  // b = 0: zero codes

    for (int pass = 0; pass < NPASS; ++pass) {
    for (int ki = 0; ki < nkt && ok; ++ki) {
      const int it = pass * nkt + ki;
      const int s = it % S;
      const uint32_t ph = (it / S) & 1;
      if (!wait_bounded(&full[s], ph, abort_flag, p.err, kErrSiteProFull)) { ok = false; break; }
      const int kt = kbeg + (kt0 + ki) % nkt;
      const int col0 = kt * BK + phase * 64;
      if (col0 < p.K &&
          SVDQ_IN_SMEM(smem_raw, smem + s * L.stage_bytes + L.x_off + phase * kXBoxBytes, kXBoxBytes, p.err) &&
          (RANK == 0 || SVDQ_IN_SMEM(smem_raw, smem + s * L.stage_bytes + L.l1_off + phase * 128 * RANK, 128 * RANK, p.err)) &&
          SVDQ_IN_SMEM(smem_raw, smem + s * L.stage_bytes + L.lam_off + phase * 256, 256, p.err) &&
          SVDQ_IN_SMEM(smem_raw, smem + s * L.stage_bytes + L.rlam_off + phase * 256, 256, p.err) &&
          SVDQ_IN_SMEM(smem_raw, cst, CSTB, p.err)) {
        const uint8_t* st = smem + s * L.stage_bytes;
        const uint32_t xbox = ptx::smem_u32(st + L.x_off + phase * kXBoxBytes);
        const uint32_t l1box = ptx::smem_u32(st + L.l1_off + phase * 128 * RANK);
        const float* lam_s = reinterpret_cast<const float*>(st + L.lam_off) + phase * 64;
        const float* rlam_s = reinterpret_cast<const float*>(st + L.rlam_off) + phase * 64;
        // -X_hat as float pairs: [k16 tile][row g: pairs 0, 1; row g+8: pairs 2, 3]
        float2 nx[4][4];
        uint32_t sc_pack_a = 0, sc_pack_b = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t a[4];
          {
            const int r = strip * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int ch = 2 * j + (lane >> 4);
            ptx::ldmatrix_x4(xbox + r * 128 + ((ch ^ (r & 7)) << 4), a[0], a[1], a[2], a[3]);
          }
          const int c0 = j * 16 + tig * 2;
          // smoothing divide X / lambda (IEEE-exact), one rounding to bf16
          const float2 l01 = *reinterpret_cast<const float2*>(lam_s + c0);
          const float2 l89 = *reinterpret_cast<const float2*>(lam_s + c0 + 8);
          const float2 n01 = *reinterpret_cast<const float2*>(rlam_s + c0);
          const float2 n89 = *reinterpret_cast<const float2*>(rlam_s + c0 + 8);
          uint32_t ah[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 qq = div_rn2(neg_bf16x2(a[i]), i < 2 ? l01 : l89, i < 2 ? n01 : n89);
            ah[i] = pack_bf16x2(qq.x, qq.y);
          }
          nx[j][0] = neg_bf16x2(ah[0]);
          nx[j][1] = neg_bf16x2(ah[2]);
          nx[j][2] = neg_bf16x2(ah[1]);
          nx[j][3] = neg_bf16x2(ah[3]);
          // low-rank down projection on the tensor cores (first pass only)
#pragma unroll
          for (int nt2 = 0; nt2 < (pass == 0 ? NT / 2 : 0); ++nt2) {
            uint32_t b[4];
            const int n = nt2 * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
            const int ch = 2 * j + ((lane >> 3) & 1);
            ptx::ldmatrix_x4(l1box + n * 128 + ((ch ^ (n & 7)) << 4), b[0], b[1], b[2], b[3]);
            ptx::mma_bf16_16816(acc[2 * nt2], ah, b[0], b[1]);
            ptx::mma_bf16_16816(acc[2 * nt2 + 1], ah, b[2], b[3]);
          }
          if (FMT == kFmtNvfp4) {
            // one 16-element group per row per k16 tile
            float ma = fmaxf(fmaxf(fabsf(nx[j][0].x), fabsf(nx[j][0].y)), fmaxf(fabsf(nx[j][1].x), fabsf(nx[j][1].y)));
            float mb = fmaxf(fmaxf(fabsf(nx[j][2].x), fabsf(nx[j][2].y)), fmaxf(fabsf(nx[j][3].x), fabsf(nx[j][3].y)));
            ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, 1));
            mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
            ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, 2));
            mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
            // s = e4m3(RN(a / 6) / g) for both rows at once (the divide by g is exact)
            const float2 s6 = div_rn2(make_float2(-ma, -mb), make_float2(6.0f, 6.0f), make_float2(-kRcp6, -kRcp6));
            const uint32_t sab = ptx::cvt_e4m3x2(s6.x * inv_gs, s6.y * inv_gs);
            const float2 dab = ptx::e4m3x2_to_f32x2(sab);
            const float da = dab.x * gs, db = dab.y * gs;
            uint32_t qa0 = 0, qa1 = 0, qb0 = 0, qb1 = 0;
            if (da > 0.f) {
              const float2 dd = make_float2(da, da);
              const float ny = -rcp_approx(da);
              const float2 nyy = make_float2(ny, ny);
              const float2 q0 = div_code2(nx[j][0], dd, nyy), q1 = div_code2(nx[j][1], dd, nyy);
              qa0 = ptx::cvt_e2m1x2(q0.x, q0.y);
              qa1 = ptx::cvt_e2m1x2(q1.x, q1.y);
            }
            if (db > 0.f) {
              const float2 dd = make_float2(db, db);
              const float ny = -rcp_approx(db);
              const float2 nyy = make_float2(ny, ny);
              const float2 q2 = div_code2(nx[j][2], dd, nyy), q3 = div_code2(nx[j][3], dd, nyy);
              qb0 = ptx::cvt_e2m1x2(q2.x, q2.y);
              qb1 = ptx::cvt_e2m1x2(q3.x, q3.y);
            }
            cst[g * 32 + j * 8 + tig] = static_cast<uint8_t>(qa0);
            cst[g * 32 + j * 8 + 4 + tig] = static_cast<uint8_t>(qa1);
            cst[(g + 8) * 32 + j * 8 + tig] = static_cast<uint8_t>(qb0);
            cst[(g + 8) * 32 + j * 8 + 4 + tig] = static_cast<uint8_t>(qb1);
            sc_pack_a |= (sab & 0xFFu) << (8 * j);
            sc_pack_b |= (sab >> 8) << (8 * j);
          }
        }
        if (FMT == kFmtMxfp4) {
          // two 32-element groups per row per box (k16 tiles 0-1 and 2-3).  X = 2^s with
          // s = clamp(floor(log2 a) - 2, -127, 127): for a normal absmax a the exponent field f
          // gives the E8M0 byte max(f - 2, 0); zero and subnormal a give byte 0 (s = -127).
          uint32_t sb_a = 0, sb_b = 0;
#pragma unroll
          for (int gi = 0; gi < 2; ++gi) {
            const int j0 = 2 * gi;
            float ma = fmaxf(fmaxf(fmaxf(fabsf(nx[j0][0].x), fabsf(nx[j0][0].y)), fmaxf(fabsf(nx[j0][1].x), fabsf(nx[j0][1].y))),
                             fmaxf(fmaxf(fabsf(nx[j0 + 1][0].x), fabsf(nx[j0 + 1][0].y)), fmaxf(fabsf(nx[j0 + 1][1].x), fabsf(nx[j0 + 1][1].y))));
            float mb = fmaxf(fmaxf(fmaxf(fabsf(nx[j0][2].x), fabsf(nx[j0][2].y)), fmaxf(fabsf(nx[j0][3].x), fabsf(nx[j0][3].y))),
                             fmaxf(fmaxf(fabsf(nx[j0 + 1][2].x), fabsf(nx[j0 + 1][2].y)), fmaxf(fabsf(nx[j0 + 1][3].x), fabsf(nx[j0 + 1][3].y))));
            ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, 1));
            mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
            ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, 2));
            mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
            const int fa = static_cast<int>(__float_as_uint(ma) >> 23);    // |a|: sign bit is 0
            const int fb = static_cast<int>(__float_as_uint(mb) >> 23);
            const uint32_t ba = static_cast<uint32_t>(max(fa - 2, 0)), bb = static_cast<uint32_t>(max(fb - 2, 0));
            sb_a |= ba << (8 * gi);
            sb_b |= bb << (8 * gi);
            // -1/X = -2^(127 - byte): exponent field 254 - byte (2..254, always normal); the
            // product with -x_hat is x_hat / X exactly
            const float na = -__uint_as_float((254u - ba) << 23), nb = -__uint_as_float((254u - bb) << 23);
            const float2 naa = make_float2(na, na), nbb = make_float2(nb, nb);
#pragma unroll
            for (int jj = j0; jj < j0 + 2; ++jj) {
              const float2 q0 = __fmul2_rn(nx[jj][0], naa), q1 = __fmul2_rn(nx[jj][1], naa);
              const float2 q2 = __fmul2_rn(nx[jj][2], nbb), q3 = __fmul2_rn(nx[jj][3], nbb);
              cst[g * 32 + jj * 8 + tig] = static_cast<uint8_t>(ptx::cvt_e2m1x2(q0.x, q0.y));
              cst[g * 32 + jj * 8 + 4 + tig] = static_cast<uint8_t>(ptx::cvt_e2m1x2(q1.x, q1.y));
              cst[(g + 8) * 32 + jj * 8 + tig] = static_cast<uint8_t>(ptx::cvt_e2m1x2(q2.x, q2.y));
              cst[(g + 8) * 32 + jj * 8 + 4 + tig] = static_cast<uint8_t>(ptx::cvt_e2m1x2(q3.x, q3.y));
            }
          }
          if (tig == 0) {
            // two consecutive E8M0 bytes of the 128x4 blocked layout (groups of 32) per row
            const int grp = col0 / 32;               // first of the box's two groups
            uint8_t* sc = reinterpret_cast<uint8_t*>(p.scales);
            const size_t ba = (static_cast<size_t>(row_a / 128) * (p.K / 128) + grp / 4) * 512 +
                              (row_a % 32) * 16 + ((row_a % 128) / 32) * 4 + grp % 4;
            const size_t bb = (static_cast<size_t>(row_b / 128) * (p.K / 128) + grp / 4) * 512 +
                              (row_b % 32) * 16 + ((row_b % 128) / 32) * 4 + grp % 4;
            const size_t nsc = static_cast<size_t>(p.Mpad) * (p.K / 32);
            if (SVDQ_IN_GLOBAL(ba + 2 <= nsc && bb + 2 <= nsc, p.err)) {
              *reinterpret_cast<uint16_t*>(sc + ba) = static_cast<uint16_t>(sb_a);
              *reinterpret_cast<uint16_t*>(sc + bb) = static_cast<uint16_t>(sb_b);
            }
          }
        } else if (FMT == kFmtInt4) {
          // one 64-element group per row per box
          float ma = 0.f, mb = 0.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            ma = fmaxf(ma, fmaxf(fmaxf(fabsf(nx[j][0].x), fabsf(nx[j][0].y)), fmaxf(fabsf(nx[j][1].x), fabsf(nx[j][1].y))));
            mb = fmaxf(mb, fmaxf(fmaxf(fabsf(nx[j][2].x), fabsf(nx[j][2].y)), fmaxf(fabsf(nx[j][3].x), fabsf(nx[j][3].y))));
          }
          ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, 1));
          mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
          ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, 2));
          mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
          // s = fp16(RN(a / 7)) for both rows at once
          const float2 s7 = div_rn2(make_float2(-ma, -mb), make_float2(7.0f, 7.0f), make_float2(-kRcp7, -kRcp7));
          const __half ha = __float2half_rn(fminf(s7.x, 65504.0f));
          const __half hb = __float2half_rn(fminf(s7.y, 65504.0f));
          const float fa = __half2float(ha), fb = __half2float(hb);
          const float2 nya = make_float2(fa > 0.f ? -rcp_approx(fa) : 0.f, fa > 0.f ? -rcp_approx(fa) : 0.f);
          const float2 nyb = make_float2(fb > 0.f ? -rcp_approx(fb) : 0.f, fb > 0.f ? -rcp_approx(fb) : 0.f);
          const float2 faa = make_float2(fa, fa), fbb = make_float2(fb, fb);
          // q = clamp(rint(x / s), -7, 7): clamp first (rint is monotonic and +-7 are integers),
          // then round by adding 1.5 * 2^23, whose low mantissa bits are then q in two's complement
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t q[8];
#pragma unroll
            for (int pi = 0; pi < 4; ++pi) {
              const bool rb = pi >= 2;
              float2 qq = make_float2(0.f, 0.f);
              if (rb ? fb > 0.f : fa > 0.f) qq = div_code2(nx[j][pi], rb ? fbb : faa, rb ? nyb : nya);
              qq.x = fminf(fmaxf(qq.x, -7.0f), 7.0f);
              qq.y = fminf(fmaxf(qq.y, -7.0f), 7.0f);
              qq = __fadd2_rn(qq, make_float2(12582912.0f, 12582912.0f));
              q[2 * pi] = __float_as_uint(qq.x) & 0xFu;
              q[2 * pi + 1] = __float_as_uint(qq.y) & 0xFu;
            }
            cst[g * 32 + j * 8 + tig] = static_cast<uint8_t>(q[0] | (q[1] << 4));
            cst[g * 32 + j * 8 + 4 + tig] = static_cast<uint8_t>(q[2] | (q[3] << 4));
            cst[(g + 8) * 32 + j * 8 + tig] = static_cast<uint8_t>(q[4] | (q[5] << 4));
            cst[(g + 8) * 32 + j * 8 + 4 + tig] = static_cast<uint8_t>(q[6] | (q[7] << 4));
          }
          if (tig == 0) {
            const int grp = col0 / 64;
            __half* sc = reinterpret_cast<__half*>(p.scales);
            if (SVDQ_IN_GLOBAL(grp < p.K / 64 && row_b < p.Mpad, p.err)) {
              sc[static_cast<size_t>(grp) * p.Mpad + row_a] = ha;
              sc[static_cast<size_t>(grp) * p.Mpad + row_b] = hb;
            }
          }
        } else if (FMT == kFmtW8a8) {
          if (pass == 0) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              rmax_a = fmaxf(rmax_a, fmaxf(fmaxf(fabsf(nx[j][0].x), fabsf(nx[j][0].y)), fmaxf(fabsf(nx[j][1].x), fabsf(nx[j][1].y))));
              rmax_b = fmaxf(rmax_b, fmaxf(fmaxf(fabsf(nx[j][2].x), fabsf(nx[j][2].y)), fmaxf(fabsf(nx[j][3].x), fabsf(nx[j][3].y))));
            }
          } else {
            // q = clamp(rint(RN(x_hat / s)), -127, 127); the clamp comes first (rint is monotonic
            // and +-127 are integers), then adding 1.5 * 2^23 rounds to the nearest even integer
            // and leaves q in the low byte as two's complement
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
              for (int pi = 0; pi < 4; ++pi) {
                const bool rb = pi >= 2;
                float2 qq = make_float2(0.f, 0.f);
                const float bdiv = rb ? w8_bb : w8_ba;
                if (bdiv > 0.f) {
                  const float f = rb ? w8_fb : w8_fa, ny = rb ? w8_nyb : w8_nya;
                  qq = div_rn2(__fmul2_rn(nx[j][pi], make_float2(f, f)), make_float2(bdiv, bdiv), make_float2(ny, ny));
                }
                qq.x = fminf(fmaxf(qq.x, -127.0f), 127.0f);
                qq.y = fminf(fmaxf(qq.y, -127.0f), 127.0f);
                qq = __fadd2_rn(qq, make_float2(12582912.0f, 12582912.0f));
                const uint32_t b2 = (__float_as_uint(qq.x) & 0xFFu) | ((__float_as_uint(qq.y) & 0xFFu) << 8);
                const int r = rb ? g + 8 : g;
                const int c = j * 16 + (pi & 1) * 8 + 2 * tig;
                *reinterpret_cast<uint16_t*>(cst + r * 64 + c) = static_cast<uint16_t>(b2);
              }
            }
          }
        } else {
          if (tig == 0) {
            // 4 consecutive E4M3 bytes of the 128x4 blocked layout per row
            const int grp4 = col0 / 64;              // index of the 4-group block along K
            uint8_t* sc = reinterpret_cast<uint8_t*>(p.scales);
            const size_t ba = (static_cast<size_t>(row_a / 128) * (p.K / 64) + grp4) * 512 +
                              (row_a % 32) * 16 + ((row_a % 128) / 32) * 4;
            const size_t bb = (static_cast<size_t>(row_b / 128) * (p.K / 64) + grp4) * 512 +
                              (row_b % 32) * 16 + ((row_b % 128) / 32) * 4;
            const size_t nsc = static_cast<size_t>(p.Mpad) * (p.K / 16);
            if (SVDQ_IN_GLOBAL(ba + 4 <= nsc && bb + 4 <= nsc, p.err)) {
              *reinterpret_cast<uint32_t*>(sc + ba) = sc_pack_a;
              *reinterpret_cast<uint32_t*>(sc + bb) = sc_pack_b;
            }
          }
        }
        __syncwarp();
        if (FMT != kFmtW8a8) {
          // 16 rows x 32 bytes of codes -> global, one 16-byte segment per lane
          const int r = lane >> 1, h = lane & 1;
          const int row = m0 + strip * 16 + r;
          const uint4 v = *reinterpret_cast<const uint4*>(cst + r * 32 + h * 16);
          if (row < p.M && SVDQ_IN_GLOBAL(col0 / 2 + h * 16 + 16 <= K2, p.err))
            *reinterpret_cast<uint4*>(p.codes + static_cast<size_t>(row) * K2 + col0 / 2 + h * 16) = v;
        } else if (pass == 1) {
          // 16 rows x 64 bytes of 8-bit codes -> global, two 16-byte segments per lane
          const int r = lane >> 1, h = lane & 1;
          const int row = m0 + strip * 16 + r;
          const uint4 v0 = *reinterpret_cast<const uint4*>(cst + r * 64 + h * 32);
          const uint4 v1 = *reinterpret_cast<const uint4*>(cst + r * 64 + h * 32 + 16);
          if (row < p.M && SVDQ_IN_GLOBAL(col0 + h * 32 + 32 <= p.K, p.err)) {
            uint8_t* dst = p.codes + static_cast<size_t>(row) * p.K + col0 + h * 32;
            *reinterpret_cast<uint4*>(dst) = v0;
            *reinterpret_cast<uint4*>(dst + 16) = v1;
          }
        }
        __syncwarp();
      }
      if (lane == 0) ptx::mbar_arrive(&empty[s]);
    }
    if (FMT == kFmtW8a8 && pass == 0) {
      // Row maxima of the whole K: quad lanes, then the BOXES warps of each row strip.  Every
      // compute warp reaches this barrier (a wait that ran out only ends the loop above).
      rmax_a = fmaxf(rmax_a, __shfl_xor_sync(0xffffffffu, rmax_a, 1));
      rmax_b = fmaxf(rmax_b, __shfl_xor_sync(0xffffffffu, rmax_b, 1));
      rmax_a = fmaxf(rmax_a, __shfl_xor_sync(0xffffffffu, rmax_a, 2));
      rmax_b = fmaxf(rmax_b, __shfl_xor_sync(0xffffffffu, rmax_b, 2));
      if (tig == 0 && SVDQ_IN_SMEM(smem_raw, rmax_s + (phase * 2 + strip) * 16, 64, p.err)) {
        rmax_s[(phase * 2 + strip) * 16 + g] = rmax_a;
        rmax_s[(phase * 2 + strip) * 16 + g + 8] = rmax_b;
      }
      named_barrier_sync(2, 32 * NW);
      float amax_a = 0.f, amax_b = 0.f;
#pragma unroll
      for (int ph2 = 0; ph2 < BOXES; ++ph2) {
        amax_a = fmaxf(amax_a, rmax_s[(ph2 * 2 + strip) * 16 + g]);
        amax_b = fmaxf(amax_b, rmax_s[(ph2 * 2 + strip) * 16 + g + 8]);
      }
      // s = RN_f32(a / 127): the fp64 quotient rounded to fp32 is the correctly rounded fp32
      // quotient (53 >= 2 * 24 + 2 bits, so the double rounding is innocuous)
      if (SPLIT) {
        // K split: the scale needs the row maximum over all of K, i.e. over the cluster.  Every
        // CTA publishes its 32 rows' maxima and signals every peer (release at cluster scope);
        // after all peers have signalled, it takes the maximum of all CTAs' values (exact and
        // order-independent: every CTA derives the same scales)
        if (phase == 0 && tig == 0) {
          rmax_cta[strip * 16 + g] = amax_a;
          rmax_cta[strip * 16 + g + 8] = amax_b;
        }
        named_barrier_sync(2, 32 * NW);
        if (warp == 0 && lane == 0) {
          for (int q = 0; q < p.ksplit; ++q)
            if (q != split) ptx::mbar_arrive_cluster(ptx::mapa_shared(ptx::smem_u32(rm_bar), static_cast<uint32_t>(q)));
        }
        if (!wait_bounded(rm_bar, 0u, abort_flag, p.err, kErrSiteProFull)) ok = false;
        ptx::fence_acq_rel_cluster();
        if (ok) {
          const uint32_t ra = ptx::smem_u32(rmax_cta + strip * 16 + g), rb2 = ptx::smem_u32(rmax_cta + strip * 16 + g + 8);
          for (int q = 0; q < p.ksplit; ++q) {
            if (q == split) continue;
            amax_a = fmaxf(amax_a, ptx::ld_shared_cluster_f32(ptx::mapa_shared(ra, static_cast<uint32_t>(q))));
            amax_b = fmaxf(amax_b, ptx::ld_shared_cluster_f32(ptx::mapa_shared(rb2, static_cast<uint32_t>(q))));
          }
        }
      }
      const float sa = __double2float_rn(__ddiv_rn(static_cast<double>(amax_a), 127.0));
      const float sb = __double2float_rn(__ddiv_rn(static_cast<double>(amax_b), 127.0));
      if (phase == 0 && tig == 0 && split == 0) {
        float* sc = reinterpret_cast<float*>(p.scales);
        if (SVDQ_IN_GLOBAL(row_b < p.Mpad, p.err)) {
          sc[row_a] = sa;             // rows up to Mpad; rows past M read zeros and get 0
          sc[row_b] = sb;
        }
      }
      w8_fa = sa < 0x1p-64f ? 0x1p64f : 1.f;
      w8_fb = sb < 0x1p-64f ? 0x1p64f : 1.f;
      w8_ba = sa * w8_fa;            // exact: a power-of-two factor on a tiny scale
      w8_bb = sb * w8_fb;
      w8_nya = w8_ba > 0.f ? -__frcp_rn(w8_ba) : 0.f;
      w8_nyb = w8_bb > 0.f ? -__frcp_rn(w8_bb) : 0.f;
    }
    }

    // ---------------------------------------------------------------- Z = X_hat L1^T
    if (NT > 0) {
      named_barrier_sync(1, 32 * NW);
      float* zbuf = reinterpret_cast<float*>(smem);       // [phase][strip][16][RANK]
      float* zb = zbuf + ((phase * 2 + strip) * 16) * RANK;
      const bool zb_ok = SVDQ_IN_SMEM(smem_raw, zb, 16 * RANK * 4, p.err);
#pragma unroll
      for (int nt = 0; nt < (zb_ok ? NT : 0); ++nt) {
        const int c = nt * 8 + tig * 2;
        zb[g * RANK + c] = acc[nt][0];
        zb[g * RANK + c + 1] = acc[nt][1];
        zb[(g + 8) * RANK + c] = acc[nt][2];
        zb[(g + 8) * RANK + c + 1] = acc[nt][3];
      }
      named_barrier_sync(1, 32 * NW);
      // all compute warps sum the partials of the CTA's 32 x RANK outputs, two columns per
      // thread, each in phase order, and store bf16 (or this CTA's partial for the K split)
      {
        constexpr int R1 = RANK > 0 ? RANK : 1;
        for (int idx = warp * 32 + lane; idx < 16 * R1; idx += 32 * NW) {
          const int sr = (idx * 2) / R1, c = (idx * 2) % R1;   // row of the 32-row block, column
          const int st = sr >> 4, r = sr & 15;
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int ph = 0; ph < BOXES; ++ph) {
            const float* src = zbuf + ((ph * 2 + st) * 16 + r) * R1 + c;
            s0 += src[0];
            s1 += src[1];
          }
          const int row = m0 + sr;
          if (SPLIT) {
            float* zsum = zbuf + BOXES * 2 * 16 * R1;         // this CTA's partial [32][RANK]
            zsum[sr * R1 + c] = s0;
            zsum[sr * R1 + c + 1] = s1;
          } else if (row < p.M) {
            __nv_bfloat162 v = __floats2bfloat162_rn(s0, s1);
            *reinterpret_cast<__nv_bfloat162*>(p.Z + static_cast<size_t>(row) * R1 + c) = v;
          }
        }
      }
    }
  }

  // K split over a cluster: CTA 0 adds the other CTAs' Z partials (read through distributed
  // shared memory, in CTA order) and writes Z.  Every thread of every CTA reaches both
  // cluster barriers; a wait that ran out above only ends its loop early.
  if (SPLIT && (RANK > 0 || FMT == kFmtW8a8)) {
    constexpr int R1 = RANK > 0 ? RANK : 1;
    ptx::cluster_sync();                                      // every partial is in shared memory
    if (RANK > 0 && split == 0) {
      // every thread of CTA 0 takes two columns of the 32 x RANK block: the peers' partials
      // are all requested before any is added (remote reads overlap), then added in CTA order
      constexpr int kMaxSplit = 8;
      const float* zsum = reinterpret_cast<const float*>(smem) + BOXES * 2 * 16 * R1;
      const uint32_t zaddr = ptx::smem_u32(zsum);
      for (int idx = threadIdx.x; idx < 16 * R1; idx += blockDim.x) {
        const int sr = (idx * 2) / R1, c = (idx * 2) % R1;
        const int o = sr * R1 + c;
        float v0[kMaxSplit - 1], v1[kMaxSplit - 1];
#pragma unroll
        for (int q = 1; q < kMaxSplit; ++q) {
          v0[q - 1] = 0.f;
          v1[q - 1] = 0.f;
          if (q < p.ksplit) {
            const uint32_t a = ptx::mapa_shared(zaddr + static_cast<uint32_t>(o) * 4u, static_cast<uint32_t>(q));
            v0[q - 1] = ptx::ld_shared_cluster_f32(a);
            v1[q - 1] = ptx::ld_shared_cluster_f32(a + 4u);
          }
        }
        float s0 = zsum[o], s1 = zsum[o + 1];
#pragma unroll
        for (int q = 1; q < kMaxSplit; ++q) {
          if (q < p.ksplit) {
            s0 += v0[q - 1];
            s1 += v1[q - 1];
          }
        }
        const int row = m0 + sr;
        if (row < p.M) {
          __nv_bfloat162 v = __floats2bfloat162_rn(s0, s1);
          *reinterpret_cast<__nv_bfloat162*>(p.Z + static_cast<size_t>(row) * R1 + c) = v;
        }
      }
    }
    ptx::cluster_sync();                                      // peers keep their partials until read
  }
}

template <int FMT, int RANK>
size_t smem_bytes_for(int stages) {
  constexpr int NW = compute_warps(RANK);
  const ProSmemLayout L = pro_layout(RANK, NW / 2);
  return 1024 + static_cast<size_t>(stages) * L.stage_bytes + 2 * stages * 8 + NW * code_stage_bytes(FMT) +
         (NW / 2) * 32 * 4 + 32 * 4 + 8 + 16;
}

template <int FMT, int RANK>
int stages_for() {
  constexpr int NW = compute_warps(RANK);
  const ProSmemLayout L = pro_layout(RANK, NW / 2);
  const size_t budget = 220 * 1024 - 1024 - NW * code_stage_bytes(FMT) - (NW / 2) * 32 * 4 - 32 * 4 - 8 - 64;
  int s = static_cast<int>(budget / L.stage_bytes);
  if (s > 4) s = 4;
  return s;
}

// Largest number of clusters of `ks` split CTAs that can be resident at once on the current
// device (0 if none or on error), queried once per device, template instance, split size and
// shared-memory size.
template <int FMT, int RANK>
static int resident_clusters(int ks, size_t smem) {
  constexpr int kDevs = 64;
  static int cached[kDevs][9];            // 0: not queried yet, else 1 + the figure
  static size_t cached_smem[kDevs][9];
  int dev = 0;
  if (ks < 2 || ks > 8 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevs) return 0;
  if (cached[dev][ks] > 0 && cached_smem[dev][ks] == smem) return cached[dev][ks] - 1;
  auto kern = prologue_kernel<FMT, RANK, true>;
  if (set_smem_limit_once(reinterpret_cast<const void*>(kern), smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ks), 1, 1);
  cfg.blockDim = dim3(32 * (compute_warps(RANK) + 1), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(ks);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cached_smem[dev][ks] = smem;
  cached[dev][ks] = n + 1;
  return n;
}

template <int FMT, int RANK>
static cudaError_t launch_pro(const CUtensorMap& tx, const CUtensorMap& tl1, ProParams p, cudaStream_t stream) {
  p.stages = stages_for<FMT, RANK>();
  if (p.stages < 2) return cudaErrorInvalidConfiguration;
  const size_t smem = smem_bytes_for<FMT, RANK>(p.stages);
  const int blocks = p.Mpad / kProRows;
  // K split for small batches (4-bit formats): the largest cluster of up to 8 CTAs per row
  // block that keeps one wave on the SMs (every cluster resident at once) and leaves no CTA
  // without a stage.
  constexpr int BK = 64 * (compute_warps(RANK) / 2);
  const int nkt_all = (p.K + BK - 1) / BK;
  int sms = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cudaErrorInvalidDevice;
  p.ksplit = 1;
  {
    for (int ks = 8; ks >= 2; --ks) {
      const int nks = (nkt_all + ks - 1) / ks;
      if (ks <= nkt_all && nks * (ks - 1) < nkt_all && blocks * ks <= sms &&
          resident_clusters<FMT, RANK>(ks, smem) >= blocks) {
        p.ksplit = ks;
        break;
      }
    }
  }
  if (p.ksplit == 1) {
    auto kern = prologue_kernel<FMT, RANK, false>;
    cudaError_t e = set_smem_limit_once(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    kern<<<blocks, 32 * (compute_warps(RANK) + 1), smem, stream>>>(tx, tl1, p);
    return cudaGetLastError();
  }
  auto kern = prologue_kernel<FMT, RANK, true>;
  cudaError_t e = set_smem_limit_once(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks * p.ksplit, 1, 1);
  cfg.blockDim = dim3(32 * (compute_warps(RANK) + 1), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(p.ksplit);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tx, tl1, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int FMT>
static cudaError_t launch_pro_rank(const CUtensorMap& tx, const CUtensorMap& tl1, const ProParams& p,
                                   cudaStream_t s) {
  switch (p.rank) {
    case 0: return launch_pro<FMT, 0>(tx, tl1, p, s);
    case 16: return launch_pro<FMT, 16>(tx, tl1, p, s);
    case 32: return launch_pro<FMT, 32>(tx, tl1, p, s);
    case 48: return launch_pro<FMT, 48>(tx, tl1, p, s);
    case 64: return launch_pro<FMT, 64>(tx, tl1, p, s);
    case 80: return launch_pro<FMT, 80>(tx, tl1, p, s);
    case 96: return launch_pro<FMT, 96>(tx, tl1, p, s);
    case 112: return launch_pro<FMT, 112>(tx, tl1, p, s);
    case 128: return launch_pro<FMT, 128>(tx, tl1, p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_prologue(int fmt, const CUtensorMap& tx, const CUtensorMap& tl1, const ProParams& p,
                            cudaStream_t s) {
  if (fmt == kFmtNvfp4) return launch_pro_rank<kFmtNvfp4>(tx, tl1, p, s);
  if (fmt == kFmtMxfp4) return launch_pro_rank<kFmtMxfp4>(tx, tl1, p, s);
  if (fmt == kFmtW8a8) return launch_pro_rank<kFmtW8a8>(tx, tl1, p, s);
  return launch_pro_rank<kFmtInt4>(tx, tl1, p, s);
}

}  // namespace svdq
