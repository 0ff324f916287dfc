// K1b: chunkwise KDA prefill on tcgen05 tensor cores (bf16 q/k/v, fp32 gates and state).
//
// Math (Kimi Linear summary, section 3.1 "Hardware-Efficient Chunkwise Algorithm";
// the per-chunk equations are derived from the recurrence of section 3). For a chunk
// of <= 64 rows entering with state S, with G_r = sum_{j<=r} log alpha_j per channel:
//
//   A_ri = beta_r sum_c k_rc k_ic e^{G_rc - G_ic}  (i < r),  P_ri = sum_c q_rc k_ic e^{G_rc - G_ic}  (i <= r)
//   T = (I + A)^{-1}  (UT transform, forward substitution)
//   Delta = T diag(beta) V - T diag(beta) (K * e^G) S
//   O = (Q * e^G) S + P Delta,     S <- Diag(e^{G_C}) S + (K * e^{G_C - G})^T Delta
//
// Decay factors. One reference row m (the chunk's middle row) splits every pairwise
// factor as e^{G_r - G_i} = E_r * F_i with E = e^{G - G_m}, F = e^{G_m - G} = 1/E, so
// the two Gram matrices A and P are one tensor-core product [K*E ; Q*E] (K*F)^T.
// The remaining factors fold into the operands:
//   K * e^G = (K * E) Diag(e^{G_m}),  Q * e^G = (Q * E) Diag(e^{G_m}),
//   K * e^{G_C - G} = (K * F) Diag(e^{G_C - G_m}),
// so only three bf16 tiles per chunk are built: Rk = K*E, Rq = Q*E, Ck = K*F, and
//   S' = Diag(e^{G_m}) S          (the bf16 state operand)
//   W' = T diag(beta) Rk,  U = T diag(beta) V
//   Delta = U - W' S',  O = Rq S' + P Delta
//   S <- Diag(e^{G_C}) S + Diag(e^{G_C - G_m}) Ck^T Delta
// This is exact in real arithmetic. It needs E and F inside the floating-point
// range, so a chunk whose decay range max_c (G_0c - G_63c) exceeds 60 nats takes an
// exact path instead (the pages' reason for secondary chunking): pairwise factors
// evaluated element by element for A and P, and tiles built with reference row
// "before the chunk" (E = e^G, Ck = K * e^{G_C - G}, all factors <= 1).
//
// Partition. Columns of S evolve independently, so a CTA owns one (sequence, head)
// and DV = 32 value columns: 4 CTAs per head. Per CTA (448 threads):
//   warps 0-7   prep: cumsum, factor tiles, Gram readout, UT solve, W' readout
//   warps 8-11  state: Delta, state update, S' tile, output epilogue (fp32 state in registers)
//   warp 12     TMA producer (k, q, v tiles; L2 prefetch of the log-decay)
//   warp 13     tcgen05.mma issuer (one thread) and TMEM owner
// The prep of chunk c+1 overlaps the sequential state pass of chunk c; TMA runs
// a further chunk ahead (3-slot ring). Every wait is bounded; a timeout flags
// KDA_ERR_TIMEOUT and all roles leave their loops.
#pragma once

#include "kda_common.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace tc {

using namespace sm100;

constexpr int DV = 32;
constexpr int NSPLIT = D / DV;
constexpr int PREP_WARPS = 8;
constexpr int ST_WARP0 = 8;
constexpr int LD_WARP = 12;
constexpr int MM_WARP = 13;
constexpr int THREADS = 14 * 32;
constexpr int PREP_THREADS = PREP_WARPS * 32;
constexpr int ST_THREADS = 128;
constexpr uint32_t BAR_PREP = 1, BAR_ST = 2;   // named barriers (0 is __syncthreads)
constexpr float LOG2E = 1.4426950408889634f;
constexpr float GUARD_LOG2 = 60.0f * 1.4426950408889634f;
constexpr uint64_t WAIT_NS = 2000000000ull;

// ---- shared memory layout (offsets from a 1024-byte aligned base) ----
constexpr uint32_t QR_BYTES = 32768;     // [Rk/W' rows 0-63 ; Rq rows 64-127], 2 kblocks x 16 KB
constexpr uint32_t CKPT_BYTES = 32768;   // Ck (16 KB) | P (8 KB) | T*beta (8 KB)
constexpr uint32_t V_BYTES = 4096;       // [64][32] bf16, 64B swizzle
constexpr uint32_t OFF_QR = 0;
constexpr uint32_t OFF_CKPT = OFF_QR + 3 * QR_BYTES;
constexpr uint32_t OFF_V = OFF_CKPT + 2 * CKPT_BYTES;
constexpr uint32_t OFF_SP = OFF_V + 3 * V_BYTES;      // S' [128][32] bf16, 64B swizzle
constexpr uint32_t OFF_DL = OFF_SP + 8192;            // Delta [64][32] bf16, 64B swizzle
constexpr int AW = 68;                                // fp32 pitch of the A / T workspace
constexpr uint32_t OFF_AW = OFF_DL + 4096;
constexpr uint32_t OFF_TX = OFF_AW + 64 * AW * 4;     // T blocks (2,1), (3,2), (3,1)
constexpr uint32_t OFF_SCR = OFF_TX + 3 * 1024;       // 4 per-warp 16x16 scratch blocks
constexpr uint32_t OFF_BETA = OFF_SCR + 4 * 1024;     // [3][64]
constexpr uint32_t OFF_SCAL = OFF_BETA + 3 * 64 * 4;  // [3 slots][3][128]: e^{G_m}, e^{G_C}, e^{G_C-G_m}
constexpr uint32_t OFF_WSUM = OFF_SCAL + 9 * 128 * 4; // [8][128] cumsum warp totals
constexpr uint32_t OFF_GROW = OFF_WSUM + 8 * 128 * 4; // [3][128] G2 of rows 0, 31, 63
constexpr uint32_t OFF_BAR = OFF_GROW + 3 * 128 * 4;
constexpr int NBARS = 32;
constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
constexpr uint32_t SMEM_USED = OFF_MISC + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// ---- TMEM columns (512 allocated) ----
constexpr uint32_t TM_AP = 0;     // 2 x 64 cols, M=128: rows 0-63 A, rows 64-127 P
constexpr uint32_t TM_W = 128;    // 128 cols, M=64: W'
constexpr uint32_t TM_U = 256;    // 2 x 32 cols, M=64: U, then Delta = U - W'S'
constexpr uint32_t TM_O = 320;    // 2 x 32 cols, M=64: O
constexpr uint32_t TM_Z = 384;    // 32 cols, M=128: Ck^T Delta
constexpr uint32_t TM_COLS = 512;

// ---- mbarriers ----
enum : int {
  B_FULL = 0,       // [3] TMA of k, q, v landed
  B_QRFREE = 3,     // [3] slot's k/q tiles no longer needed
  B_TILES = 6,      // [2] Rk, Rq, Ck and scalars written
  B_GRAM = 8,       // [2] Gram MMA done
  B_TB = 10,        // [2] P and T*beta tiles written
  B_WDONE = 12,     // [2] W' and U MMAs done
  B_READY = 14,     // [3] W' tile written
  B_CKFREE = 17,    // [2] Ck/P/Tb slot no longer needed
  B_DUFREE = 19,    // [2] Delta accumulator read
  B_ADONE = 21,     // Delta and Rq S' MMAs done
  B_DREADY = 22,    // Delta tile written
  B_BDONE = 23,     // P Delta and Ck^T Delta MMAs done
  B_SREADY = 24,    // S' tile written
  B_FINAL = 25,     // drain
  NUM_BARS = 26
};

struct Args {
  const float* log_alpha;
  const float* beta;
  const float* h0;
  const int32_t* cu_seqlens;
  __nv_bfloat16* o;
  float* hT;
  int n_seqs;
  int n_heads;
  int64_t t_total;
};

struct Ctx {
  uint8_t* sm;
  uint64_t* bars;
  volatile int* abort_flag;
  uint32_t tmem;
  int n, h, j0, n_chunks;
  int64_t bos, eos;
  size_t rs;   // elements between consecutive tokens of q/k/v/o/log_alpha
};

__device__ __forceinline__ void raise_abort(const Ctx& x) {
  *x.abort_flag = 1;
  flag_error(DEVERR_TIMEOUT);
}

// Bounded per-thread wait that also gives up when another role aborted.
__device__ __forceinline__ bool wait_b(const Ctx& x, int b, uint32_t parity) {
  uint64_t* bar = &x.bars[b];
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*x.abort_flag) return false;
      if (globaltimer_ns() - t0 > WAIT_NS) {
        raise_abort(x);
        return false;
      }
    }
  }
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcpf(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&a),
                             *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// ============================================================================
// TMA producer (one thread)
// ============================================================================
__device__ void load_role(const Ctx& x, const CUtensorMap* map_k, const CUtensorMap* map_q,
                          const CUtensorMap* map_v, const CUtensorMap* map_la) {
  const int xk = x.h * D;
  for (int c = 0; c < 2 && c < x.n_chunks; ++c)
    tma_prefetch_2d(map_la, xk, (int)(x.bos + (int64_t)c * CHUNK));
  int issued = 0;
  for (int c = 0; c < x.n_chunks; ++c) {
    const int s3 = c % 3;
    if (c >= 3 && !wait_b(x, B_QRFREE + s3, ((c - 3) / 3) & 1)) break;
    const int y = (int)(x.bos + (int64_t)c * CHUNK);
    uint8_t* qr = x.sm + OFF_QR + s3 * QR_BYTES;
    uint64_t* full = &x.bars[B_FULL + s3];
    mbar_arrive_expect_tx(full, 4 * 8192 + V_BYTES);
    tma_load_2d(qr, map_k, xk, y, full);
    tma_load_2d(qr + 16384, map_k, xk + 64, y, full);
    tma_load_2d(qr + 8192, map_q, xk, y, full);
    tma_load_2d(qr + 16384 + 8192, map_q, xk + 64, y, full);
    tma_load_2d(x.sm + OFF_V + s3 * V_BYTES, map_v, xk + x.j0, y, full);
    if (c + 2 < x.n_chunks) tma_prefetch_2d(map_la, xk, y + 2 * CHUNK);
    issued = c + 1;
  }
  // never leave with copies in flight: wait (bounded) for the last load of each slot
  for (int c = issued - 3 < 0 ? 0 : issued - 3; c < issued; ++c) {
    uint64_t* full = &x.bars[B_FULL + c % 3];
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(full, (c / 3) & 1))
      if (globaltimer_ns() - t0 > 100000000ull) break;
  }
}

// ============================================================================
// MMA issuer (one thread)
// ============================================================================
__device__ __forceinline__ uint64_t kdesc128(uint32_t addr) {
  return make_sdesc(addr, 16, 1024, SWZ_128B);
}

__device__ void mma_role(const Ctx& x) {
  const uint32_t sbase = smem_u32(x.sm);
  int g = 0, w = 0, a = 0, b = 0;
  uint64_t last = globaltimer_ns();
  const int n = x.n_chunks;
  while (b < n) {
    bool did = false;
    if (b < a && mbar_test_wait(&x.bars[B_DREADY], b & 1)) {
      tc_fence_after();
      const uint32_t ck = sbase + OFF_CKPT + (b & 1) * CKPT_BYTES;
      const uint32_t dl = sbase + OFF_DL;
      const uint32_t d_o = x.tmem + TM_O + (b & 1) * 32;
      // O += P Delta   (M=64, N=32, K=64)
      for (int kk = 0; kk < 4; ++kk)
        umma_bf16(d_o, kdesc128(ck + 16384 + kk * 32), make_sdesc(dl + kk * 1024, 4096, 512, SWZ_64B),
                  idesc_bf16(64, 32, 0, 1), 1u);
      // Z = Ck^T Delta (M=128 channels, N=32, K=64); Ck read as an MN-major A operand
      for (int kk = 0; kk < 4; ++kk)
        umma_bf16(x.tmem + TM_Z, make_sdesc(ck + kk * 2048, 8192, 1024, SWZ_128B),
                  make_sdesc(dl + kk * 1024, 4096, 512, SWZ_64B), idesc_bf16(128, 32, 1, 1),
                  kk > 0 ? 1u : 0u);
      umma_commit(&x.bars[B_BDONE]);
      umma_commit(&x.bars[B_CKFREE + (b & 1)]);
      ++b;
      did = true;
    } else if (a < w && mbar_test_wait(&x.bars[B_READY + a % 3], (a / 3) & 1) &&
               mbar_test_wait(&x.bars[B_SREADY], a & 1)) {
      tc_fence_after();
      const uint32_t qr = sbase + OFF_QR + (a % 3) * QR_BYTES;
      const uint32_t sp = sbase + OFF_SP;
      const uint32_t d_u = x.tmem + TM_U + (a & 1) * 32;
      const uint32_t d_o = x.tmem + TM_O + (a & 1) * 32;
      // Delta = U - W' S'   (M=64, N=32, K=128; negate A)
      for (int kk = 0; kk < 8; ++kk)
        umma_bf16(d_u, kdesc128(qr + (kk >> 2) * 16384 + (kk & 3) * 32),
                  make_sdesc(sp + kk * 1024, 4096, 512, SWZ_64B), idesc_bf16(64, 32, 0, 1, 1), 1u);
      // O = Rq S'
      for (int kk = 0; kk < 8; ++kk)
        umma_bf16(d_o, kdesc128(qr + 8192 + (kk >> 2) * 16384 + (kk & 3) * 32),
                  make_sdesc(sp + kk * 1024, 4096, 512, SWZ_64B), idesc_bf16(64, 32, 0, 1),
                  kk > 0 ? 1u : 0u);
      umma_commit(&x.bars[B_ADONE]);
      ++a;
      did = true;
    } else if (w < g && mbar_test_wait(&x.bars[B_TB + (w & 1)], (w >> 1) & 1) &&
               (w < 2 || mbar_test_wait(&x.bars[B_DUFREE + (w & 1)], ((w - 2) >> 1) & 1))) {
      tc_fence_after();
      const uint32_t qr = sbase + OFF_QR + (w % 3) * QR_BYTES;
      const uint32_t tb = sbase + OFF_CKPT + (w & 1) * CKPT_BYTES + 24576;
      const uint32_t vv = sbase + OFF_V + (w % 3) * V_BYTES;
      // W' = (T beta) Rk   (M=64, N=128, K=64); Rk read as an MN-major B operand
      for (int kk = 0; kk < 4; ++kk)
        umma_bf16(x.tmem + TM_W, kdesc128(tb + kk * 32),
                  make_sdesc(qr + kk * 2048, 16384, 1024, SWZ_128B), idesc_bf16(64, 128, 0, 1),
                  kk > 0 ? 1u : 0u);
      // U = (T beta) V     (M=64, N=32, K=64)
      for (int kk = 0; kk < 4; ++kk)
        umma_bf16(x.tmem + TM_U + (w & 1) * 32, kdesc128(tb + kk * 32),
                  make_sdesc(vv + kk * 1024, 4096, 512, SWZ_64B), idesc_bf16(64, 32, 0, 1),
                  kk > 0 ? 1u : 0u);
      umma_commit(&x.bars[B_WDONE + (w & 1)]);
      ++w;
      did = true;
    } else if (g < n && mbar_test_wait(&x.bars[B_TILES + (g & 1)], (g >> 1) & 1)) {
      tc_fence_after();
      const uint32_t qr = sbase + OFF_QR + (g % 3) * QR_BYTES;
      const uint32_t ck = sbase + OFF_CKPT + (g & 1) * CKPT_BYTES;
      // [A ; P] = [Rk ; Rq] Ck^T   (M=128, N=64, K=128)
      for (int kk = 0; kk < 8; ++kk)
        umma_bf16(x.tmem + TM_AP + (g & 1) * 64, kdesc128(qr + (kk >> 2) * 16384 + (kk & 3) * 32),
                  kdesc128(ck + (kk >> 2) * 8192 + (kk & 3) * 32), idesc_bf16(128, 64, 0, 0),
                  kk > 0 ? 1u : 0u);
      umma_commit(&x.bars[B_GRAM + (g & 1)]);
      ++g;
      did = true;
    }
    if (did) {
      last = globaltimer_ns();
    } else if (*x.abort_flag) {
      break;
    } else if (globaltimer_ns() - last > WAIT_NS) {
      raise_abort(x);
      break;
    }
  }
  // drain: every issued MMA completes before TMEM is released
  umma_commit(&x.bars[B_FINAL]);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(&x.bars[B_FINAL], 0))
    if (globaltimer_ns() - t0 > 100000000ull) break;
}

// ============================================================================
// prep warps (256 threads)
// ============================================================================

// acc (two n-halves of a 16x16 C fragment) += X(16x16) * Y(16x16), fp32 blocks in smem
__device__ __forceinline__ void blk_mma(float (&acc)[2][4], const float* X, int ldx, const float* Y,
                                        int ldy, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    uint32_t af[4] = {f2tf32(X[g * ldx + 8 * ks + t]), f2tf32(X[(g + 8) * ldx + 8 * ks + t]),
                      f2tf32(X[g * ldx + 8 * ks + t + 4]), f2tf32(X[(g + 8) * ldx + 8 * ks + t + 4])};
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
      uint32_t bfr[2] = {f2tf32(Y[(8 * ks + t) * ldy + 8 * nh + g]),
                         f2tf32(Y[(8 * ks + t + 4) * ldy + 8 * nh + g])};
      mma_tf32_16x8x8(acc[nh], af, bfr);
    }
  }
}
__device__ __forceinline__ void blk_store(float* C, int ldc, const float (&acc)[2][4], float scale,
                                          int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nh = 0; nh < 2; ++nh) {
    C[g * ldc + 8 * nh + 2 * t] = scale * acc[nh][0];
    C[g * ldc + 8 * nh + 2 * t + 1] = scale * acc[nh][1];
    C[(g + 8) * ldc + 8 * nh + 2 * t] = scale * acc[nh][2];
    C[(g + 8) * ldc + 8 * nh + 2 * t + 1] = scale * acc[nh][3];
  }
}

// Location of block (a, b), a >= b, of T = (I + A)^{-1} once the solve has run.
__device__ __forceinline__ const float* tblock(const uint8_t* sm, int a, int b, int& ld) {
  const float* aw = reinterpret_cast<const float*>(sm + OFF_AW);
  const float* tx = reinterpret_cast<const float*>(sm + OFF_TX);
  if (a == 2 && b == 1) { ld = 16; return tx; }
  if (a == 3 && b == 2) { ld = 16; return tx + 256; }
  if (a == 3 && b == 1) { ld = 16; return tx + 512; }
  ld = AW;
  return aw + (16 * a) * AW + 16 * b;
}

__device__ void prep_role(const Ctx& x, const Args& p) {
  const int tid = threadIdx.x;
  const int w = tid >> 5, lane = tid & 31;
  const int kb = lane >> 4;              // kblock of this thread's 4 channels
  const uint32_t cbyte = (lane & 15) * 8; // byte offset of the channels within the kblock row
  const int c0 = 4 * lane;
  float* wsum = reinterpret_cast<float*>(x.sm + OFF_WSUM);
  float* grow = reinterpret_cast<float*>(x.sm + OFF_GROW);
  float* aw = reinterpret_cast<float*>(x.sm + OFF_AW);

  float lam_next[8][4];
  auto load_lam = [&](int c, float (&dst)[8][4]) {
    const int64_t t0 = x.bos + (int64_t)c * CHUNK;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t t = t0 + 8 * w + j;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c < x.n_chunks && t < x.eos)
        v = __ldg(reinterpret_cast<const float4*>(p.log_alpha + (size_t)t * x.rs + x.h * D + c0));
      dst[j][0] = v.x; dst[j][1] = v.y; dst[j][2] = v.z; dst[j][3] = v.w;
    }
  };
  load_lam(0, lam_next);

  for (int c = 0; c < x.n_chunks; ++c) {
    const int s3 = c % 3, s2 = c & 1;
    const int64_t t0 = x.bos + (int64_t)c * CHUNK;
    const int L = (x.eos - t0) < CHUNK ? (int)(x.eos - t0) : CHUNK;
    uint8_t* qr = x.sm + OFF_QR + s3 * QR_BYTES;
    uint8_t* ck = x.sm + OFF_CKPT + s2 * CKPT_BYTES;
    float* betas = reinterpret_cast<float*>(x.sm + OFF_BETA) + s3 * 64;
    float* scal = reinterpret_cast<float*>(x.sm + OFF_SCAL) + s3 * 384;

    float g2[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) g2[j][k] = lam_next[j][k];
    load_lam(c + 1, lam_next);   // next chunk's log-decay, in flight during this one

    if (tid < 64) betas[tid] = tid < L ? __ldg(p.beta + (size_t)(t0 + tid) * p.n_heads + x.h) : 0.f;

    // ---- inclusive cumsum over rows, in log2 units
    {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          acc[k] = fmaf(g2[j][k], LOG2E, acc[k]);
          g2[j][k] = acc[k];
        }
      *reinterpret_cast<float4*>(&wsum[w * 128 + c0]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    }
    named_bar_sync(BAR_PREP, PREP_THREADS);
    {
      float pre[4] = {0.f, 0.f, 0.f, 0.f};
      for (int ww = 0; ww < w; ++ww) {
        const float4 v = *reinterpret_cast<const float4*>(&wsum[ww * 128 + c0]);
        pre[0] += v.x; pre[1] += v.y; pre[2] += v.z; pre[3] += v.w;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int k = 0; k < 4; ++k) g2[j][k] += pre[k];
      if (w == 0) *reinterpret_cast<float4*>(&grow[c0]) = make_float4(g2[0][0], g2[0][1], g2[0][2], g2[0][3]);
      if (w == 3) *reinterpret_cast<float4*>(&grow[128 + c0]) = make_float4(g2[7][0], g2[7][1], g2[7][2], g2[7][3]);
      if (w == 7) *reinterpret_cast<float4*>(&grow[256 + c0]) = make_float4(g2[7][0], g2[7][1], g2[7][2], g2[7][3]);
    }
    // raw k/q/v in smem, and this Ck/P/Tb slot free again
    bool ok = wait_b(x, B_FULL + s3, (c / 3) & 1);
    if (ok && c >= 2) ok = wait_b(x, B_CKFREE + s2, ((c - 2) >> 1) & 1);
    if (named_bar_or(BAR_PREP, PREP_THREADS, !ok)) break;

    // ---- range guard: max over channels of G_0 - G_63
    bool bad = false;
#pragma unroll
    for (int k = 0; k < 4; ++k) bad |= (grow[c0 + k] - grow[256 + c0 + k]) > GUARD_LOG2;
    const bool exact = named_bar_or(BAR_PREP, PREP_THREADS, bad);

    float gm[4], gc[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      gm[k] = exact ? 0.f : grow[128 + c0 + k];
      gc[k] = grow[256 + c0 + k];
    }

    if (!exact) {
      // ---- factored tiles: Rk = K E, Rq = Q E (in place), Ck = K F
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int r = 8 * w + j;
        const bool valid = r < L;
        uint2* kp = reinterpret_cast<uint2*>(qr + kb * 16384 + swz128(r * 128 + cbyte));
        uint2* qp = reinterpret_cast<uint2*>(qr + kb * 16384 + swz128((r + 64) * 128 + cbyte));
        uint2* cp = reinterpret_cast<uint2*>(ck + kb * 8192 + swz128(r * 128 + cbyte));
        uint2 kr = valid ? *kp : make_uint2(0u, 0u);
        uint2 qv = valid ? *qp : make_uint2(0u, 0u);
        float e[4], f[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          e[k] = ex2f(g2[j][k] - gm[k]);
          f[k] = rcpf(e[k]);
        }
        const uint32_t e01 = pack_bf16(e[0], e[1]), e23 = pack_bf16(e[2], e[3]);
        const uint32_t f01 = pack_bf16(f[0], f[1]), f23 = pack_bf16(f[2], f[3]);
        *kp = make_uint2(mul_bf16x2(kr.x, e01), mul_bf16x2(kr.y, e23));
        *qp = make_uint2(mul_bf16x2(qv.x, e01), mul_bf16x2(qv.y, e23));
        *cp = make_uint2(mul_bf16x2(kr.x, f01), mul_bf16x2(kr.y, f23));
      }
    } else {
      // ---- exact path: G (log2 units) into the Ck/P/Tb slot, pairwise factors one by one
      float* gsm = reinterpret_cast<float*>(ck);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<float4*>(&gsm[(8 * w + j) * 128 + c0]) =
            make_float4(g2[j][0], g2[j][1], g2[j][2], g2[j][3]);
      named_bar_sync(BAR_PREP, PREP_THREADS);
      // warp w takes lower-triangle pairs p = w, w+8, ... (row-major r(r+1)/2 + i)
      float pval[9];
      int pidx[9];
#pragma unroll
      for (int bt = 0; bt < 9; ++bt) {
        pval[bt] = 0.f;
        pidx[bt] = -1;
#pragma unroll 1
        for (int qq = 0; qq < 32; ++qq) {
          const int m = bt * 32 + qq;
          const int pp = w + 8 * m;
          if (pp >= 2080) break;
          int r = (int)((sqrtf(8.f * pp + 1.f) - 1.f) * 0.5f);
          while ((r + 1) * (r + 2) / 2 <= pp) ++r;
          while (r * (r + 1) / 2 > pp) --r;
          const int i = pp - r * (r + 1) / 2;
          float sa = 0.f, sp = 0.f;
          if (r < L && i < L) {
            const uint2 kr = *reinterpret_cast<const uint2*>(qr + kb * 16384 + swz128(r * 128 + cbyte));
            const uint2 ki = *reinterpret_cast<const uint2*>(qr + kb * 16384 + swz128(i * 128 + cbyte));
            const uint2 qv = *reinterpret_cast<const uint2*>(qr + kb * 16384 + swz128((r + 64) * 128 + cbyte));
            const float4 gr = *reinterpret_cast<const float4*>(&gsm[r * 128 + c0]);
            const float4 gi = *reinterpret_cast<const float4*>(&gsm[i * 128 + c0]);
            const float ee[4] = {ex2f(gr.x - gi.x), ex2f(gr.y - gi.y), ex2f(gr.z - gi.z), ex2f(gr.w - gi.w)};
            const float krf[4] = {bf_lo(kr.x), bf_hi(kr.x), bf_lo(kr.y), bf_hi(kr.y)};
            const float kif[4] = {bf_lo(ki.x), bf_hi(ki.x), bf_lo(ki.y), bf_hi(ki.y)};
            const float qf[4] = {bf_lo(qv.x), bf_hi(qv.x), bf_lo(qv.y), bf_hi(qv.y)};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float ke = kif[k] * ee[k];
              sa = fmaf(krf[k], ke, sa);
              sp = fmaf(qf[k], ke, sp);
            }
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            sa += __shfl_xor_sync(0xffffffffu, sa, off);
            sp += __shfl_xor_sync(0xffffffffu, sp, off);
          }
          if (lane == 0 && i < r) aw[r * AW + i] = betas[r] * sa;
          if (lane == qq) {
            pval[bt] = sp;
            pidx[bt] = r * 64 + i;
          }
        }
      }
      named_bar_sync(BAR_PREP, PREP_THREADS);
      // P tile: zero, then scatter the lower triangle
      uint8_t* pt = ck + 16384;
      for (int idx = tid; idx < 512; idx += PREP_THREADS)
        *reinterpret_cast<uint4*>(pt + idx * 16) = make_uint4(0u, 0u, 0u, 0u);
      named_bar_sync(BAR_PREP, PREP_THREADS);
#pragma unroll
      for (int bt = 0; bt < 9; ++bt)
        if (pidx[bt] >= 0) {
          const int r = pidx[bt] >> 6, i = pidx[bt] & 63;
          *reinterpret_cast<__nv_bfloat16*>(pt + swz128(r * 128 + i * 2)) = __float2bfloat16_rn(pval[bt]);
        }
      // tiles with the reference before the chunk: Rk = K e^G, Rq = Q e^G, Ck = K e^{G_C - G}
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int r = 8 * w + j;
        const bool valid = r < L;
        uint2* kp = reinterpret_cast<uint2*>(qr + kb * 16384 + swz128(r * 128 + cbyte));
        uint2* qp = reinterpret_cast<uint2*>(qr + kb * 16384 + swz128((r + 64) * 128 + cbyte));
        uint2* cp = reinterpret_cast<uint2*>(ck + kb * 8192 + swz128(r * 128 + cbyte));
        const uint2 kr = valid ? *kp : make_uint2(0u, 0u);
        const uint2 qv = valid ? *qp : make_uint2(0u, 0u);
        const float krf[4] = {bf_lo(kr.x), bf_hi(kr.x), bf_lo(kr.y), bf_hi(kr.y)};
        const float qf[4] = {bf_lo(qv.x), bf_hi(qv.x), bf_lo(qv.y), bf_hi(qv.y)};
        float e[4], f[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          e[k] = ex2f(g2[j][k]);
          f[k] = ex2f(gc[k] - g2[j][k]);
        }
        *kp = make_uint2(pack_bf16(krf[0] * e[0], krf[1] * e[1]), pack_bf16(krf[2] * e[2], krf[3] * e[3]));
        *qp = make_uint2(pack_bf16(qf[0] * e[0], qf[1] * e[1]), pack_bf16(qf[2] * e[2], qf[3] * e[3]));
        *cp = make_uint2(pack_bf16(krf[0] * f[0], krf[1] * f[1]), pack_bf16(krf[2] * f[2], krf[3] * f[3]));
      }
    }
    // per-channel scalars of this chunk
    if (w == 0) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        scal[c0 + k] = exact ? 1.f : ex2f(gm[k]);           // e^{G_m}
        scal[128 + c0 + k] = ex2f(gc[k]);                    // e^{G_C}
        scal[256 + c0 + k] = exact ? 1.f : ex2f(gc[k] - gm[k]);  // e^{G_C - G_m}
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(BAR_PREP, PREP_THREADS);
    if (tid == 0) mbar_arrive(&x.bars[B_TILES + s2]);

    // ---- Gram readout: A rows (beta-scaled, strictly lower) -> fp32 workspace; P -> bf16 tile
    if (!exact) {
      ok = wait_b(x, B_GRAM + s2, (c >> 1) & 1);
      tc_fence_after();
      const int q = w & 3;
      const int col0 = (w >= 4) ? 32 : 0;
      float v[32];
      tmem_ld32(x.tmem + TM_AP + s2 * 64 + ((uint32_t)(32 * q) << 16) + col0, v);
      tmem_ld_wait();
      if (q < 2) {
        const int r = 32 * q + lane;
        const float br = betas[r];
#pragma unroll
        for (int m = 0; m < 32; m += 4) {
          float4 o4;
          o4.x = (col0 + m + 0 < r) ? br * v[m + 0] : 0.f;
          o4.y = (col0 + m + 1 < r) ? br * v[m + 1] : 0.f;
          o4.z = (col0 + m + 2 < r) ? br * v[m + 2] : 0.f;
          o4.w = (col0 + m + 3 < r) ? br * v[m + 3] : 0.f;
          *reinterpret_cast<float4*>(&aw[r * AW + col0 + m]) = o4;
        }
      } else {
        const int r = 32 * (q - 2) + lane;
        uint8_t* pt = ck + 16384;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t u[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i0 = col0 + ch * 8 + 2 * e;
            u[e] = pack_bf16(i0 <= r ? v[ch * 8 + 2 * e] : 0.f, i0 + 1 <= r ? v[ch * 8 + 2 * e + 1] : 0.f);
          }
          *reinterpret_cast<uint4*>(pt + swz128(r * 128 + col0 * 2 + ch * 16)) = make_uint4(u[0], u[1], u[2], u[3]);
        }
      }
      tc_fence_before();
    }
    if (named_bar_or(BAR_PREP, PREP_THREADS, !ok)) break;

    // ---- UT transform: T = (I + A)^{-1}, 16x16 diagonal blocks by forward substitution
    if (w < 4 && lane < 16) {
      const int a = w, j = lane;
      const float* Ab = aw + (16 * a) * AW + 16 * a;
      float t[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int i = 0; i + 1 < r; i += 2) {
          s0 = fmaf(Ab[r * AW + i], t[i], s0);
          s1 = fmaf(Ab[r * AW + i + 1], t[i + 1], s1);
        }
        if (r & 1) s0 = fmaf(Ab[r * AW + r - 1], t[r - 1], s0);
        t[r] = (r == j ? 1.f : 0.f) - (s0 + s1);
      }
      __syncwarp(0x0000ffffu);
      float* Tb = aw + (16 * a) * AW + 16 * a;
#pragma unroll
      for (int r = 0; r < 16; ++r) Tb[r * AW + j] = t[r];
    }
    named_bar_sync(BAR_PREP, PREP_THREADS);
    // off-diagonal blocks with warp-level tf32 MMAs:
    //   T_ab = -T_aa * sum_{b<=m<a} A_am T_mb
    {
      float* scr = reinterpret_cast<float*>(x.sm + OFF_SCR) + (w & 3) * 256;
      // level 1: (1,0), (2,1), (3,2)
      if (w < 3) {
        const int a = w + 1, b = w;
        float acc[2][4] = {};
        int ld1, ld2;
        const float* Tbb = tblock(x.sm, b, b, ld1);
        blk_mma(acc, aw + (16 * a) * AW + 16 * b, AW, Tbb, ld1, lane);
        blk_store(scr, 16, acc, 1.f, lane);
        __syncwarp();
        float acc2[2][4] = {};
        const float* Taa = tblock(x.sm, a, a, ld2);
        blk_mma(acc2, Taa, ld2, scr, 16, lane);
        int ldo;
        float* dst = const_cast<float*>(tblock(x.sm, a, b, ldo));
        blk_store(dst, ldo, acc2, -1.f, lane);
      }
      named_bar_sync(BAR_PREP, PREP_THREADS);
      // level 2: (2,0), (3,1)
      if (w < 2) {
        const int a = w + 2, b = w;
        float acc[2][4] = {};
        int l1, l2;
        const float* T1 = tblock(x.sm, b, b, l1);
        blk_mma(acc, aw + (16 * a) * AW + 16 * b, AW, T1, l1, lane);
        const float* T2 = tblock(x.sm, b + 1, b, l2);
        blk_mma(acc, aw + (16 * a) * AW + 16 * (b + 1), AW, T2, l2, lane);
        blk_store(scr, 16, acc, 1.f, lane);
        __syncwarp();
        float acc2[2][4] = {};
        int l3;
        const float* Taa = tblock(x.sm, a, a, l3);
        blk_mma(acc2, Taa, l3, scr, 16, lane);
        int ldo;
        float* dst = const_cast<float*>(tblock(x.sm, a, b, ldo));
        blk_store(dst, ldo, acc2, -1.f, lane);
      }
      named_bar_sync(BAR_PREP, PREP_THREADS);
      // level 3: (3,0)
      if (w == 0) {
        float acc[2][4] = {};
#pragma unroll
        for (int m = 0; m < 3; ++m) {
          int l1;
          const float* Tm = tblock(x.sm, m, 0, l1);
          blk_mma(acc, aw + 48 * AW + 16 * m, AW, Tm, l1, lane);
        }
        blk_store(scr, 16, acc, 1.f, lane);
        __syncwarp();
        float acc2[2][4] = {};
        int l3;
        const float* Taa = tblock(x.sm, 3, 3, l3);
        blk_mma(acc2, Taa, l3, scr, 16, lane);
        int ldo;
        float* dst = const_cast<float*>(tblock(x.sm, 3, 0, ldo));
        blk_store(dst, ldo, acc2, -1.f, lane);
      }
      named_bar_sync(BAR_PREP, PREP_THREADS);
    }
    // ---- T*beta tile (bf16, K-major [64 r][64 i], 128B swizzle)
    {
      const int r = tid >> 2, qb = tid & 3;   // row, 16-column block
      uint8_t* tt = ck + 24576;
      const int a = r >> 4, rr = r & 15;
      uint32_t u[8];
      if (qb <= a) {
        int ld;
        const float* Tb = tblock(x.sm, a, qb, ld);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int i0 = 16 * qb + 2 * e;
          const float v0 = (i0 <= r) ? Tb[rr * ld + 2 * e] * betas[i0] : 0.f;
          const float v1 = (i0 + 1 <= r) ? Tb[rr * ld + 2 * e + 1] * betas[i0 + 1] : 0.f;
          u[e] = pack_bf16(v0, v1);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) u[e] = 0u;
      }
      *reinterpret_cast<uint4*>(tt + swz128(r * 128 + qb * 32)) = make_uint4(u[0], u[1], u[2], u[3]);
      *reinterpret_cast<uint4*>(tt + swz128(r * 128 + qb * 32 + 16)) = make_uint4(u[4], u[5], u[6], u[7]);
    }
    fence_proxy_async_smem();
    named_bar_sync(BAR_PREP, PREP_THREADS);
    if (tid == 0) mbar_arrive(&x.bars[B_TB + s2]);

    // ---- W' readout (M=64 layout: rows 16q..16q+15 in lanes 32q..32q+15) -> bf16 over Rk
    ok = wait_b(x, B_WDONE + s2, (c >> 1) & 1);
    tc_fence_after();
    {
      const int q = w & 3;
      const int colh = (w >= 4) ? 64 : 0;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float v[32];
        tmem_ld32(x.tmem + TM_W + ((uint32_t)(32 * q) << 16) + colh + 32 * half, v);
        tmem_ld_wait();
        if (lane < 16) {
          const int r = 16 * q + lane;
          uint8_t* rowp = qr + (colh >> 6) * 16384;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint4 u;
            u.x = pack_bf16(v[ch * 8 + 0], v[ch * 8 + 1]);
            u.y = pack_bf16(v[ch * 8 + 2], v[ch * 8 + 3]);
            u.z = pack_bf16(v[ch * 8 + 4], v[ch * 8 + 5]);
            u.w = pack_bf16(v[ch * 8 + 6], v[ch * 8 + 7]);
            *reinterpret_cast<uint4*>(rowp + swz128(r * 128 + half * 64 + ch * 16)) = u;
          }
        }
      }
    }
    tc_fence_before();
    fence_proxy_async_smem();
    if (named_bar_or(BAR_PREP, PREP_THREADS, !ok)) break;
    if (tid == 0) mbar_arrive(&x.bars[B_READY + s3]);
  }
}

// ============================================================================
// state warps (128 threads): the sequential pass over chunks
// ============================================================================
__device__ void state_role(const Ctx& x, const Args& p) {
  const int tid = threadIdx.x - ST_WARP0 * 32;
  const int q = tid >> 5, lane = tid & 31;
  const int crow = tid;                                   // key channel owned by this thread
  const uint32_t lane_base = (uint32_t)(32 * q) << 16;
  uint8_t* sp = x.sm + OFF_SP;
  uint8_t* dl = x.sm + OFF_DL;
  const size_t sbase = (((size_t)x.n * p.n_heads + x.h) * D + crow) * D + x.j0;

  float S[DV];
  if (p.h0) {
#pragma unroll
    for (int m = 0; m < DV; m += 4) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(p.h0 + sbase + m));
      S[m] = v.x; S[m + 1] = v.y; S[m + 2] = v.z; S[m + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int m = 0; m < DV; ++m) S[m] = 0.f;
  }

  auto write_sprime = [&](const float* scal_next) {
    const float eg = scal_next[crow];
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      uint4 u;
      u.x = pack_bf16(eg * S[ch * 8 + 0], eg * S[ch * 8 + 1]);
      u.y = pack_bf16(eg * S[ch * 8 + 2], eg * S[ch * 8 + 3]);
      u.z = pack_bf16(eg * S[ch * 8 + 4], eg * S[ch * 8 + 5]);
      u.w = pack_bf16(eg * S[ch * 8 + 6], eg * S[ch * 8 + 7]);
      *reinterpret_cast<uint4*>(sp + swz64(crow * 64 + ch * 16)) = u;
    }
  };
  const float* scal_all = reinterpret_cast<const float*>(x.sm + OFF_SCAL);

  bool ok = true;
  if (x.n_chunks > 0) {
    ok = wait_b(x, B_TILES + 0, 0);
    write_sprime(scal_all);
    fence_proxy_async_smem();
    if (named_bar_or(BAR_ST, ST_THREADS, !ok)) ok = false;
    else if (tid == 0) mbar_arrive(&x.bars[B_SREADY]);
  }
  for (int c = 0; ok && c < x.n_chunks; ++c) {
    const int s2 = c & 1, s3 = c % 3;
    const int64_t t0 = x.bos + (int64_t)c * CHUNK;
    const int L = (x.eos - t0) < CHUNK ? (int)(x.eos - t0) : CHUNK;
    // ---- Delta (fp32 in TMEM) -> bf16 tile
    bool okw = wait_b(x, B_ADONE, c & 1);
    tc_fence_after();
    {
      float v[32];
      tmem_ld32(x.tmem + TM_U + s2 * 32 + lane_base, v);
      tmem_ld_wait();
      if (lane < 16) {
        const int r = 16 * q + lane;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint4 u;
          u.x = pack_bf16(v[ch * 8 + 0], v[ch * 8 + 1]);
          u.y = pack_bf16(v[ch * 8 + 2], v[ch * 8 + 3]);
          u.z = pack_bf16(v[ch * 8 + 4], v[ch * 8 + 5]);
          u.w = pack_bf16(v[ch * 8 + 6], v[ch * 8 + 7]);
          *reinterpret_cast<uint4*>(dl + swz64(r * 64 + ch * 16)) = u;
        }
      }
    }
    tc_fence_before();
    fence_proxy_async_smem();
    if (named_bar_or(BAR_ST, ST_THREADS, !okw)) break;
    if (tid == 0) {
      mbar_arrive(&x.bars[B_DREADY]);
      mbar_arrive(&x.bars[B_DUFREE + s2]);
    }
    // ---- state update: S <- e^{G_C} S + e^{G_C - G_m} (Ck^T Delta)
    okw = wait_b(x, B_BDONE, c & 1);
    tc_fence_after();
    {
      float z[32];
      tmem_ld32(x.tmem + TM_Z + lane_base, z);
      tmem_ld_wait();
      const float* scal = scal_all + s3 * 384;
      const float egc = scal[128 + crow], ecm = scal[256 + crow];
#pragma unroll
      for (int m = 0; m < DV; ++m) S[m] = fmaf(egc, S[m], ecm * z[m]);
    }
    if (c + 1 < x.n_chunks) {
      okw = okw && wait_b(x, B_TILES + ((c + 1) & 1), ((c + 1) >> 1) & 1);
      write_sprime(scal_all + ((c + 1) % 3) * 384);
      fence_proxy_async_smem();
    }
    tc_fence_before();
    if (named_bar_or(BAR_ST, ST_THREADS, !okw)) break;
    if (tid == 0) {
      if (c + 1 < x.n_chunks) mbar_arrive(&x.bars[B_SREADY]);
      mbar_arrive(&x.bars[B_QRFREE + s3]);
    }
    // ---- output epilogue (off the sequential path)
    {
      float v[32];
      tmem_ld32(x.tmem + TM_O + s2 * 32 + lane_base, v);
      tmem_ld_wait();
      const int r = 16 * q + lane;
      if (lane < 16 && r < L) {
        __nv_bfloat16* orow = p.o + (size_t)(t0 + r) * x.rs + x.h * D + x.j0;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint4 u;
          u.x = pack_bf16(v[ch * 8 + 0], v[ch * 8 + 1]);
          u.y = pack_bf16(v[ch * 8 + 2], v[ch * 8 + 3]);
          u.z = pack_bf16(v[ch * 8 + 4], v[ch * 8 + 5]);
          u.w = pack_bf16(v[ch * 8 + 6], v[ch * 8 + 7]);
          *reinterpret_cast<uint4*>(orow + ch * 8) = u;
        }
      }
    }
  }
  if (p.hT && !*x.abort_flag) {
#pragma unroll
    for (int m = 0; m < DV; m += 4)
      *reinterpret_cast<float4*>(p.hT + sbase + m) = make_float4(S[m], S[m + 1], S[m + 2], S[m + 3]);
  }
}

// ============================================================================
// kernel
// ============================================================================
__global__ void __launch_bounds__(THREADS, 1)
kda_chunk_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_la,
                    const Args args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Ctx x;
  x.sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  x.bars = reinterpret_cast<uint64_t*>(x.sm + OFF_BAR);
  x.abort_flag = reinterpret_cast<volatile int*>(x.sm + OFF_MISC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(x.sm + OFF_MISC + 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chain = blockIdx.x / NSPLIT;
  x.n = chain / args.n_heads;
  x.h = chain % args.n_heads;
  x.j0 = (blockIdx.x % NSPLIT) * DV;
  seq_bounds(args.cu_seqlens, x.n, args.n_seqs, args.t_total, x.bos, x.eos);
  x.n_chunks = (int)((x.eos - x.bos + CHUNK - 1) / CHUNK);
  x.rs = (size_t)args.n_heads * D;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NUM_BARS; ++i) mbar_init(&x.bars[i], 1);
    *x.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == LD_WARP && lane == 0) {
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_q);
    prefetch_tensormap(&map_v);
    prefetch_tensormap(&map_la);
  }
  if (warp == MM_WARP) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  x.tmem = *tmem_slot;

  if (warp < PREP_WARPS) {
    prep_role(x, args);
  } else if (warp < ST_WARP0 + 4) {
    state_role(x, args);
  } else if (warp == LD_WARP) {
    if (lane == 0) load_role(x, &map_k, &map_q, &map_v, &map_la);
  } else if (warp == MM_WARP) {
    if (lane == 0) mma_role(x);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == MM_WARP) {
    tc_fence_after();
    tmem_dealloc(x.tmem, TM_COLS);
  }
}

}  // namespace tc
}  // namespace kda
