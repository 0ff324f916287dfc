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
// Delta and Rq S' come out of ONE 128-row MMA: A = [-W' ; Rq] accumulating onto
// [U ; 0]; O += P Delta then accumulates onto the Rq S' rows. (The tensor pipe
// costs about the same per instruction for any N <= 128, so stacking saves time.)
// This is exact in real arithmetic. It needs E and F inside the floating-point
// range, so a chunk whose decay range max_c (G_0c - G_63c) exceeds 60 nats takes an
// exact path instead (the pages' reason for secondary chunking): pairwise factors
// evaluated element by element for A and P, and tiles built with reference row
// "before the chunk" (E = e^G, Ck = K * e^{G_C - G}, all factors <= 1).
//
// Partition. Columns of S evolve independently, so a CTA owns one (sequence, head)
// and DV = 32 value columns: 4 CTAs per head. Per CTA (608 threads), a pipeline
// three chunks deep:
//   warps 0-7   prep A (chunk c+2): cumsum, range guard, Rk/Rq/Ck tiles, scalars
//   warps 8-11  prep B (chunk c+1): Gram readout, UT solve, T*beta tile, W' tile
//   warps 12-15 state  (chunk c):   Delta tile, fp32 state update, S' tile, output
//   warp 16     TMA producer (k, q, v tiles; L2 prefetch of the log-decay)
//   warp 17     tcgen05.mma issuer for the sequential state pass; TMEM owner
//   warp 18     tcgen05.mma issuer for prep (Gram, W', U)
// Every wait is bounded; a timeout flags KDA_ERR_TIMEOUT and all roles leave
// their loops.
#pragma once

#include "kda_common.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace tc {

using namespace sm100;

constexpr int DV = 32;
constexpr int NSPLIT = D / DV;
constexpr int PA_WARPS = 8;
constexpr int PB_WARP0 = 8;
constexpr int ST_WARP0 = 12;
constexpr int LD_WARP = 16;
constexpr int MC_WARP = 17;
constexpr int MP_WARP = 18;
constexpr int THREADS = 19 * 32;
constexpr int PA_THREADS = PA_WARPS * 32;
constexpr int PB_THREADS = 128;
constexpr int ST_THREADS = 128;
constexpr uint32_t BAR_PA = 1, BAR_PB = 2, BAR_ST = 3;   // named barriers (0 is __syncthreads)
constexpr float LOG2E = 1.4426950408889634f;
constexpr float GUARD_LOG2 = 60.0f * 1.4426950408889634f;
constexpr uint64_t WAIT_NS = 2000000000ull;

// ---- shared memory layout (offsets from a 1024-byte aligned base) ----
constexpr uint32_t QR_BYTES = 32768;     // [Rk/W' rows 0-63 ; Rq rows 64-127], 2 kblocks x 16 KB
constexpr uint32_t CKP_BYTES = 24576;    // Ck [64][128] (16 KB) | P [64][64] (8 KB)
constexpr uint32_t V_BYTES = 4096;       // [64][32] bf16, 64B swizzle
constexpr uint32_t OFF_QR = 0;
constexpr uint32_t OFF_CKP = OFF_QR + 3 * QR_BYTES;
constexpr uint32_t OFF_V = OFF_CKP + 2 * CKP_BYTES;
constexpr uint32_t OFF_SP = OFF_V + 3 * V_BYTES;      // S' [128][32] bf16, 64B swizzle
constexpr uint32_t OFF_DL = OFF_SP + 8192;            // Delta [64][32] bf16, 64B swizzle
// prep B workspace (also the staging area of the exact path, >= 32 KB contiguous)
constexpr uint32_t OFF_TB = OFF_DL + 4096;            // [T*beta ; 0] [128][64] bf16, 128B swizzle
constexpr int AW = 68;                                // fp32 pitch of the A / T workspace
constexpr uint32_t OFF_AW = OFF_TB + 16384;
constexpr uint32_t OFF_XS = OFF_AW + 64 * AW * 4;     // 6 extra 16x16 fp32 blocks
constexpr uint32_t OFF_SCR = OFF_XS + 6 * 1024;       // 4 per-warp 16x16 scratch blocks
constexpr uint32_t OFF_BETA = OFF_SCR + 4 * 1024;     // [3][64]
constexpr uint32_t OFF_SCAL = OFF_BETA + 3 * 64 * 4;  // [3 slots][3][128]: e^{G_m}, e^{G_C}, e^{G_C-G_m}
constexpr uint32_t OFF_WSUM = OFF_SCAL + 9 * 128 * 4; // [8][128] cumsum warp totals
constexpr uint32_t OFF_GROW = OFF_WSUM + 8 * 128 * 4; // [3][128] G2 of rows 0, 31, 63
constexpr uint32_t OFF_XFLAG = OFF_GROW + 3 * 128 * 4; // [3] exact-path flag per slot
constexpr uint32_t OFF_BAR = OFF_XFLAG + 16;
constexpr int NBARS = 40;
constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
constexpr uint32_t SMEM_USED = OFF_MISC + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(OFF_SCR + 4 * 1024 - OFF_TB >= 32768, "exact-path staging needs 32 KB");

// ---- TMEM columns (512 allocated) ----
constexpr uint32_t TM_AP = 0;     // 2 x 64 cols, M=128: rows 0-63 A, rows 64-127 P
constexpr uint32_t TM_W = 128;    // 128 cols, M=64: W'
constexpr uint32_t TM_C = 256;    // 2 x 32 cols, M=128: rows 0-63 U then Delta, rows 64-127 Rq S' then O
constexpr uint32_t TM_Z = 320;    // 32 cols, M=128: Ck^T Delta
constexpr uint32_t TM_COLS = 512;

// ---- mbarriers ----
enum : int {
  B_FULL = 0,       // [3] TMA of k, q, v landed
  B_QRFREE = 3,     // [3] slot's k/q tiles no longer needed
  B_TILES = 6,      // [2] Rk, Rq, Ck, scalars and exact flag written
  B_GRAM = 8,       // [2] Gram MMA done
  B_TB = 10,        // [2] P and T*beta tiles written
  B_WDONE = 12,     // [2] W' and U MMAs done
  B_READY = 14,     // [3] W' tile written
  B_CKFREE = 17,    // [2] Ck/P slot no longer needed
  B_DCFREE = 19,    // [2] Delta/O accumulator read
  B_ADONE = 21,     // [-W' ; Rq] S' MMA done
  B_DREADY = 22,    // Delta tile written
  B_BDONE = 23,     // Ck^T Delta MMA done
  B_ODONE = 24,     // P Delta MMA done (O complete)
  B_SREADY = 25,    // S' tile written
  B_PBIDLE = 26,    // prep B finished a chunk (workspace free)
  B_FIN_C = 27,     // drains
  B_FIN_P = 28,
  NUM_BARS = 29
};
static_assert(NUM_BARS <= NBARS, "barrier slots");

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

// Bounded per-thread wait that also gives up when another role aborted. The
// thread sleeps in the barrier (suspend hint) instead of spinning.
__device__ __noinline__ bool wait_b_slow(const Ctx& x, uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, 200000u)) return true;
    if (*x.abort_flag) return false;
    if (globaltimer_ns() - t0 > WAIT_NS) {
      raise_abort(x);
      return false;
    }
  }
}
// Fast path inline (phase already complete), the sleeping loop out of line.
__device__ __forceinline__ bool wait_b(const Ctx& x, int b, uint32_t parity) {
  uint64_t* bar = &x.bars[b];
  if (mbar_try_wait(bar, parity)) return true;
  return wait_b_slow(x, bar, parity);
}

// Global loads issued exactly where written (volatile): used to prefetch the next
// chunk's log-decay a whole chunk ahead of its use.
__device__ __forceinline__ float4 ldg_nc_v4(const float* p) {
  float4 v;
  asm volatile("ld.global.nc.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ float ldg_nc_f32(const float* p) {
  float v;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 1/x for normal positive x on the FMA pipe: integer-subtraction seed (relative
// error < 1/8 over a binade) refined by two Newton-Raphson steps y <- y (2 - x y),
// which square the relative error each time (< 2.5e-4 after two steps).
__device__ __forceinline__ float rcp_nr(float x) {
  float y = __int_as_float(0x7EF311C3 - __float_as_int(x));
  y = y * fmaf(-x, y, 2.f);
  y = y * fmaf(-x, y, 2.f);
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
__device__ __forceinline__ uint4 pack8(const float* v) {
  return make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                    pack_bf16(v[6], v[7]));
}
__device__ __forceinline__ uint64_t kdesc128(uint32_t addr) {
  return make_sdesc(addr, 16, 1024, SWZ_128B);
}

// ============================================================================
// TMA producer (one thread)
// ============================================================================
__device__ void load_role(const Ctx& x, const CUtensorMap* map_k, const CUtensorMap* map_q,
                          const CUtensorMap* map_v, const CUtensorMap* map_la) {
  const int xk = x.h * D;
  for (int c = 0; c < 3 && c < x.n_chunks; ++c)
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
    if (c + 3 < x.n_chunks) tma_prefetch_2d(map_la, xk, y + 3 * CHUNK);
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
// MMA issuers (one thread each)
// ============================================================================
__device__ void drain(const Ctx& x, int bar) {
  umma_commit(&x.bars[bar]);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(&x.bars[bar], 0))
    if (globaltimer_ns() - t0 > 100000000ull) break;
}

// Sequential state pass: per chunk one stacked MMA gives Delta and Rq S', then
// Ck^T Delta (the next state) and only then P Delta (the output).
__device__ void mma_state_role(const Ctx& x) {
  const uint32_t sbase = smem_u32(x.sm);
  const uint32_t sp = sbase + OFF_SP, dl = sbase + OFF_DL;
  for (int c = 0; c < x.n_chunks; ++c) {
    if (!wait_b(x, B_READY + c % 3, (c / 3) & 1) || !wait_b(x, B_SREADY, c & 1)) break;
    tc_fence_after();
    const uint32_t qr = sbase + OFF_QR + (c % 3) * QR_BYTES;
    const uint32_t d_c = x.tmem + TM_C + (c & 1) * 32;
    // [U ; 0] += [-W' ; Rq] S'   (M=128, N=32, K=128)
    for (int kk = 0; kk < 8; ++kk)
      umma_bf16(d_c, kdesc128(qr + (kk >> 2) * 16384 + (kk & 3) * 32),
                make_sdesc(sp + kk * 1024, 4096, 512, SWZ_64B), idesc_bf16(128, 32, 0, 1), 1u);
    umma_commit(&x.bars[B_ADONE]);
    if (!wait_b(x, B_DREADY, c & 1)) break;
    tc_fence_after();
    const uint32_t ck = sbase + OFF_CKP + (c & 1) * CKP_BYTES;
    // Z = Ck^T Delta (M=128 channels, N=32, K=64); Ck read as an MN-major A operand
    for (int kk = 0; kk < 4; ++kk)
      umma_bf16(x.tmem + TM_Z, make_sdesc(ck + kk * 2048, 8192, 1024, SWZ_128B),
                make_sdesc(dl + kk * 1024, 4096, 512, SWZ_64B), idesc_bf16(128, 32, 1, 1),
                kk > 0 ? 1u : 0u);
    umma_commit(&x.bars[B_BDONE]);
    // O += P Delta: a 128-row A operand whose rows 64-127 are P (rows 0-63 are Ck's
    // second kblock, which only touches the already-consumed Delta rows)
    for (int kk = 0; kk < 4; ++kk)
      umma_bf16(d_c, kdesc128(ck + 8192 + kk * 32), make_sdesc(dl + kk * 1024, 4096, 512, SWZ_64B),
                idesc_bf16(128, 32, 0, 1), 1u);
    umma_commit(&x.bars[B_ODONE]);
    umma_commit(&x.bars[B_CKFREE + (c & 1)]);
  }
  drain(x, B_FIN_C);
}

// Prep products in chunk order: Gram(0), W(0), Gram(1), W(1), ... The Gram of
// chunk c+1 is queued right behind W(c), so it is done before prep B turns to
// chunk c+1. (Queuing Gram(c+1) before W(c) could deadlock: on the exact path the
// tiles of chunk c+1 wait for prep B to finish chunk c, which needs W(c).)
__device__ void mma_prep_role(const Ctx& x) {
  const uint32_t sbase = smem_u32(x.sm);
  const int n = x.n_chunks;
  auto gram = [&](int g) -> bool {
    if (!wait_b(x, B_TILES + (g & 1), (g >> 1) & 1)) return false;
    tc_fence_after();
    const uint32_t qr = sbase + OFF_QR + (g % 3) * QR_BYTES;
    const uint32_t ck = sbase + OFF_CKP + (g & 1) * CKP_BYTES;
    // [A ; P] = [Rk ; Rq] Ck^T   (M=128, N=64, K=128)
    for (int kk = 0; kk < 8; ++kk)
      umma_bf16(x.tmem + TM_AP + (g & 1) * 64, kdesc128(qr + (kk >> 2) * 16384 + (kk & 3) * 32),
                kdesc128(ck + (kk >> 2) * 8192 + (kk & 3) * 32), idesc_bf16(128, 64, 0, 0),
                kk > 0 ? 1u : 0u);
    umma_commit(&x.bars[B_GRAM + (g & 1)]);
    return true;
  };
  for (int w = 0; w < n; ++w) {
    if (!gram(w)) break;
    if (!wait_b(x, B_TB + (w & 1), (w >> 1) & 1)) break;
    if (w >= 2 && !wait_b(x, B_DCFREE + (w & 1), ((w - 2) >> 1) & 1)) break;
    tc_fence_after();
    const uint32_t qr = sbase + OFF_QR + (w % 3) * QR_BYTES;
    const uint32_t tb = sbase + OFF_TB;
    const uint32_t vv = sbase + OFF_V + (w % 3) * V_BYTES;
    // -W' = -(T beta) Rk   (M=64, N=128, K=64; negate A); Rk read as an MN-major B operand
    for (int kk = 0; kk < 4; ++kk)
      umma_bf16(x.tmem + TM_W, kdesc128(tb + kk * 32),
                make_sdesc(qr + kk * 2048, 16384, 1024, SWZ_128B), idesc_bf16(64, 128, 0, 1, 1),
                kk > 0 ? 1u : 0u);
    // [U ; 0] = [T beta ; 0] V   (M=128, N=32, K=64): initialises the Delta/O accumulator
    for (int kk = 0; kk < 4; ++kk)
      umma_bf16(x.tmem + TM_C + (w & 1) * 32, kdesc128(tb + kk * 32),
                make_sdesc(vv + kk * 1024, 4096, 512, SWZ_64B), idesc_bf16(128, 32, 0, 1),
                kk > 0 ? 1u : 0u);
    umma_commit(&x.bars[B_WDONE + (w & 1)]);
  }
  drain(x, B_FIN_P);
}

// Exact path of prep A for a chunk whose decay range is too wide for the factored
// Gram (kept out of line: it is rare and large). Pairwise factors are evaluated
// one by one; A goes to prep B's workspace, P to its tile, and the operand tiles are
// built with the reference before the chunk (all factors <= 1).
__device__ __noinline__ bool prep_a_exact(const Ctx& x, int c, int L, uint8_t* qr, uint8_t* ck,
                                          const float* betas, const float (&g2)[8][4],
                                          const float (&gc)[4]) {
  const int tid = threadIdx.x;
  const int w = tid >> 5, lane = tid & 31;
  const int kb = lane >> 4;
  const uint32_t cbyte = (lane & 15) * 8;
  const int c0 = 4 * lane;
  const int s2 = c & 1;
  float* aw = reinterpret_cast<float*>(x.sm + OFF_AW);
  bool ok = true;
  // ---- exact path. Needs prep B's workspace (idle after chunk c-1) and this Ck/P slot.
  ok = (c < 1) || wait_b(x, B_PBIDLE, (c - 1) & 1);
  ok = ok && ((c < 2) || wait_b(x, B_CKFREE + s2, ((c - 2) >> 1) & 1));
  if (named_bar_or(BAR_PA, PA_THREADS, !ok)) return false;
  float* gsm = reinterpret_cast<float*>(x.sm + OFF_TB);   // G (log2 units), [64][128] fp32
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<float4*>(&gsm[(8 * w + j) * 128 + c0]) =
        make_float4(g2[j][0], g2[j][1], g2[j][2], g2[j][3]);
  named_bar_sync(BAR_PA, PA_THREADS);
  // warp w takes lower-triangle pairs p = w, w+8, ... (row-major r(r+1)/2 + i)
  float pval[9], aval[9];
  int pidx[9];
#pragma unroll
  for (int bt = 0; bt < 9; ++bt) {
    pval[bt] = 0.f;
    aval[bt] = 0.f;
    pidx[bt] = -1;
#pragma unroll 1
    for (int qq = 0; qq < 32; ++qq) {
      const int pp = w + 8 * (bt * 32 + qq);
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
      if (lane == qq) {
        pval[bt] = sp;
        aval[bt] = sa;
        pidx[bt] = r * 64 + i;
      }
    }
  }
  named_bar_sync(BAR_PA, PA_THREADS);
  // A (beta-scaled, strictly lower) into prep B's workspace; P tile zeroed then filled
  uint8_t* pt = ck + 16384;
  for (int idx = tid; idx < 512; idx += PA_THREADS)
    *reinterpret_cast<uint4*>(pt + idx * 16) = make_uint4(0u, 0u, 0u, 0u);
  named_bar_sync(BAR_PA, PA_THREADS);
#pragma unroll
  for (int bt = 0; bt < 9; ++bt)
    if (pidx[bt] >= 0) {
      const int r = pidx[bt] >> 6, i = pidx[bt] & 63;
      *reinterpret_cast<__nv_bfloat16*>(pt + swz128(r * 128 + i * 2)) = __float2bfloat16_rn(pval[bt]);
      if (i < r) aw[r * AW + i] = betas[r] * aval[bt];
    }
  // the staging area covered the zero rows of prep B's [T*beta ; 0] operand: restore them
  for (int idx = tid; idx < 512; idx += PA_THREADS)
    *reinterpret_cast<uint4*>(x.sm + OFF_TB + 8192 + idx * 16) = make_uint4(0u, 0u, 0u, 0u);
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
  return ok;
}

// ============================================================================
// prep A (warps 0-7): decay factors and the three bf16 tiles of a chunk
// ============================================================================
__device__ void prep_a_role(const Ctx& x, const Args& p) {
  const int tid = threadIdx.x;
  const int w = tid >> 5, lane = tid & 31;
  const int kb = lane >> 4;                // kblock of this thread's 4 channels
  const uint32_t cbyte = (lane & 15) * 8;  // byte offset of the channels in the kblock row
  const int c0 = 4 * lane;
  float* wsum = reinterpret_cast<float*>(x.sm + OFF_WSUM);
  float* grow = reinterpret_cast<float*>(x.sm + OFF_GROW);
  int* xflag = reinterpret_cast<int*>(x.sm + OFF_XFLAG);

  float lam_next[8][4];
  float beta_next = 0.f;
  auto load_next = [&](int c) {
    const int64_t t0 = x.bos + (int64_t)c * CHUNK;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t t = t0 + 8 * w + j;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c < x.n_chunks && t < x.eos)
        v = ldg_nc_v4(p.log_alpha + (size_t)t * x.rs + x.h * D + c0);
      lam_next[j][0] = v.x; lam_next[j][1] = v.y; lam_next[j][2] = v.z; lam_next[j][3] = v.w;
    }
    beta_next = 0.f;
    if (tid < 64 && c < x.n_chunks && t0 + tid < x.eos)
      beta_next = ldg_nc_f32(p.beta + (size_t)(t0 + tid) * p.n_heads + x.h);
  };
  load_next(0);

  for (int c = 0; c < x.n_chunks; ++c) {
    const int s3 = c % 3, s2 = c & 1;
    const int64_t t0 = x.bos + (int64_t)c * CHUNK;
    const int L = (x.eos - t0) < CHUNK ? (int)(x.eos - t0) : CHUNK;
    uint8_t* qr = x.sm + OFF_QR + s3 * QR_BYTES;
    uint8_t* ck = x.sm + OFF_CKP + s2 * CKP_BYTES;
    float* betas = reinterpret_cast<float*>(x.sm + OFF_BETA) + s3 * 64;
    float* scal = reinterpret_cast<float*>(x.sm + OFF_SCAL) + s3 * 384;

    float g2[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) g2[j][k] = lam_next[j][k];
    if (tid < 64) betas[tid] = beta_next;
    load_next(c + 1);   // next chunk's log-decay and beta, in flight during this one

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
    named_bar_sync(BAR_PA, PA_THREADS);
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
    bool ok = wait_b(x, B_FULL + s3, (c / 3) & 1);
    if (named_bar_or(BAR_PA, PA_THREADS, !ok)) break;

    // ---- range guard: max over channels of G_0 - G_63
    bool bad = false;
#pragma unroll
    for (int k = 0; k < 4; ++k) bad |= (grow[c0 + k] - grow[256 + c0 + k]) > GUARD_LOG2;
    const bool exact = named_bar_or(BAR_PA, PA_THREADS, bad);

    float gm[4], gc[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      gm[k] = exact ? 0.f : grow[128 + c0 + k];
      gc[k] = grow[256 + c0 + k];
    }

    if (!exact) {
      // ---- factored tiles: Rk = K E, Rq = Q E in place; Ck = K F once the slot is free
      uint32_t kf[8][2];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int r = 8 * w + j;
        const bool valid = r < L;
        uint2* kp = reinterpret_cast<uint2*>(qr + kb * 16384 + swz128(r * 128 + cbyte));
        uint2* qp = reinterpret_cast<uint2*>(qr + kb * 16384 + swz128((r + 64) * 128 + cbyte));
        const uint2 kr = valid ? *kp : make_uint2(0u, 0u);
        const uint2 qv = valid ? *qp : make_uint2(0u, 0u);
        float e[4], f[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          e[k] = ex2f(g2[j][k] - gm[k]);
          f[k] = rcpf(e[k]);
        }
        const uint32_t e01 = pack_bf16(e[0], e[1]), e23 = pack_bf16(e[2], e[3]);
        *kp = make_uint2(mul_bf16x2(kr.x, e01), mul_bf16x2(kr.y, e23));
        *qp = make_uint2(mul_bf16x2(qv.x, e01), mul_bf16x2(qv.y, e23));
        kf[j][0] = mul_bf16x2(kr.x, pack_bf16(f[0], f[1]));
        kf[j][1] = mul_bf16x2(kr.y, pack_bf16(f[2], f[3]));
      }
      ok = (c < 2) || wait_b(x, B_CKFREE + s2, ((c - 2) >> 1) & 1);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint2*>(ck + kb * 8192 + swz128((8 * w + j) * 128 + cbyte)) =
            make_uint2(kf[j][0], kf[j][1]);
    } else {
      ok = prep_a_exact(x, c, L, qr, ck, betas, g2, gc);
      if (!ok) break;
    }
    // per-channel scalars and the path flag of this chunk
    if (w == 0) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        scal[c0 + k] = exact ? 1.f : ex2f(gm[k]);               // e^{G_m}
        scal[128 + c0 + k] = ex2f(gc[k]);                        // e^{G_C}
        scal[256 + c0 + k] = exact ? 1.f : ex2f(gc[k] - gm[k]);  // e^{G_C - G_m}
      }
      if (lane == 0) xflag[s3] = exact ? 1 : 0;
    }
    fence_proxy_async_smem();
    if (named_bar_or(BAR_PA, PA_THREADS, !ok)) break;
    if (tid == 0) mbar_arrive(&x.bars[B_TILES + s2]);
  }
}

// ============================================================================
// prep B (warps 8-11): Gram readout, UT solve, T*beta tile, W' tile
// ============================================================================

// acc (two n-halves of a 16x16 C fragment) += X(16x16) * Y(16x16), fp32 blocks in smem.
// The fp32 bit patterns are used as tf32 operands directly (the MMA reads the top 19
// bits, i.e. truncates), which saves the conversions.
__device__ __forceinline__ void blk_mma(float (&acc)[2][4], const float* X, int ldx, const float* Y,
                                        int ldy, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    uint32_t af[4] = {__float_as_uint(X[g * ldx + 8 * ks + t]), __float_as_uint(X[(g + 8) * ldx + 8 * ks + t]),
                      __float_as_uint(X[g * ldx + 8 * ks + t + 4]),
                      __float_as_uint(X[(g + 8) * ldx + 8 * ks + t + 4])};
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
      uint32_t bfr[2] = {__float_as_uint(Y[(8 * ks + t) * ldy + 8 * nh + g]),
                         __float_as_uint(Y[(8 * ks + t + 4) * ldy + 8 * nh + g])};
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

// Block (a, b), a >= b, of T = (I + A)^{-1} after the solve (fp32, 16x16).
// Diagonal and (1,0), (2,0), (3,0), (3,1), (3,2) overwrite the matching A block;
// (2,1) lives in the extra-block area.
__device__ __forceinline__ const float* tblk(const uint8_t* sm, int a, int b, int& ld) {
  if (a == 2 && b == 1) {
    ld = 16;
    return reinterpret_cast<const float*>(sm + OFF_XS) + 4 * 256;
  }
  ld = AW;
  return reinterpret_cast<const float*>(sm + OFF_AW) + (16 * a) * AW + 16 * b;
}

__device__ void prep_b_role(const Ctx& x) {
  const int tid = threadIdx.x - PB_WARP0 * 32;
  const int q = tid >> 5, lane = tid & 31;   // q = warp within the group = TMEM lane quarter
  const uint32_t lane_base = (uint32_t)(32 * q) << 16;
  float* aw = reinterpret_cast<float*>(x.sm + OFF_AW);
  float* scr = reinterpret_cast<float*>(x.sm + OFF_SCR) + q * 256;
  const int* xflag = reinterpret_cast<const int*>(x.sm + OFF_XFLAG);
  auto A = [&](int a, int b) { return aw + (16 * a) * AW + 16 * b; };
  // rows 64-127 of the [T*beta ; 0] operand stay zero for the whole kernel
  for (int i = tid; i < 512; i += PB_THREADS)
    *reinterpret_cast<uint4*>(x.sm + OFF_TB + 8192 + i * 16) = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();

  for (int c = 0; c < x.n_chunks; ++c) {
    const int s3 = c % 3, s2 = c & 1;
    uint8_t* qr = x.sm + OFF_QR + s3 * QR_BYTES;
    uint8_t* ck = x.sm + OFF_CKP + s2 * CKP_BYTES;
    const float* betas = reinterpret_cast<const float*>(x.sm + OFF_BETA) + s3 * 64;

    bool ok = wait_b(x, B_TILES + s2, (c >> 1) & 1);
    const bool exact = ok && xflag[s3] != 0;
    // ---- Gram readout: A rows (beta-scaled, strictly lower) -> fp32 workspace; P -> bf16 tile
    if (ok && !exact) {
      ok = wait_b(x, B_GRAM + s2, (c >> 1) & 1);
      tc_fence_after();
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int col0 = 32 * half;
        float v[32];
        tmem_ld32(x.tmem + TM_AP + s2 * 64 + lane_base + col0, v);
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
            float pv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) pv[e] = (col0 + ch * 8 + e <= r) ? v[ch * 8 + e] : 0.f;
            *reinterpret_cast<uint4*>(pt + swz128(r * 128 + col0 * 2 + ch * 16)) = pack8(pv);
          }
        }
      }
      tc_fence_before();
    }
    if (named_bar_or(BAR_PB, PB_THREADS, !ok)) break;

    // ---- UT transform: T = (I + A)^{-1}. 16x16 diagonal blocks by forward substitution:
    //      lane j of warp a keeps column j of T_aa in registers (the A values are
    //      independent of it, so their loads pipeline), then the block replaces A_aa.
    if (lane < 16) {
      const int j = lane;
      float* Ab = A(q, q);
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
#pragma unroll
      for (int r = 0; r < 16; ++r) Ab[r * AW + j] = t[r];
    }
    named_bar_sync(BAR_PB, PB_THREADS);
    // Off-diagonal blocks by 2x2 block doubling (tf32 warp MMAs), three levels:
    //   T_10 = -T_11 A_10 T_00, T_32 = -T_33 A_32 T_22,
    //   X = A[2:4, 0:2] T[0:2, 0:2],  T[2:4, 0:2] = -T[2:4, 2:4] X.
    {
      float* xs = reinterpret_cast<float*>(x.sm + OFF_XS);
      float* X20 = xs;
      float* X21 = xs + 256;
      float* X30 = xs + 512;
      float* X31 = xs + 768;
      float* T21 = xs + 1024;
      float* T31p = xs + 1280;
      if (q == 0) {        // T_10
        float acc[2][4] = {};
        blk_mma(acc, A(1, 0), AW, A(0, 0), AW, lane);
        blk_store(scr, 16, acc, 1.f, lane);
        __syncwarp();
        float acc2[2][4] = {};
        blk_mma(acc2, A(1, 1), AW, scr, 16, lane);
        blk_store(A(1, 0), AW, acc2, -1.f, lane);
      } else if (q == 1) { // T_32
        float acc[2][4] = {};
        blk_mma(acc, A(3, 2), AW, A(2, 2), AW, lane);
        blk_store(scr, 16, acc, 1.f, lane);
        __syncwarp();
        float acc2[2][4] = {};
        blk_mma(acc2, A(3, 3), AW, scr, 16, lane);
        blk_store(A(3, 2), AW, acc2, -1.f, lane);
      } else if (q == 2) { // X21 = A_21 T_11
        float acc[2][4] = {};
        blk_mma(acc, A(2, 1), AW, A(1, 1), AW, lane);
        blk_store(X21, 16, acc, 1.f, lane);
      } else {             // X31 = A_31 T_11
        float acc[2][4] = {};
        blk_mma(acc, A(3, 1), AW, A(1, 1), AW, lane);
        blk_store(X31, 16, acc, 1.f, lane);
      }
      named_bar_sync(BAR_PB, PB_THREADS);
      if (q == 0) {        // X20 = A_20 T_00 + A_21 T_10
        float acc[2][4] = {};
        blk_mma(acc, A(2, 0), AW, A(0, 0), AW, lane);
        blk_mma(acc, A(2, 1), AW, A(1, 0), AW, lane);
        blk_store(X20, 16, acc, 1.f, lane);
      } else if (q == 1) { // X30 = A_30 T_00 + A_31 T_10
        float acc[2][4] = {};
        blk_mma(acc, A(3, 0), AW, A(0, 0), AW, lane);
        blk_mma(acc, A(3, 1), AW, A(1, 0), AW, lane);
        blk_store(X30, 16, acc, 1.f, lane);
      } else if (q == 2) { // T_21 = -T_22 X21
        float acc[2][4] = {};
        blk_mma(acc, A(2, 2), AW, X21, 16, lane);
        blk_store(T21, 16, acc, -1.f, lane);
      } else {             // partial of T_31: T_33 X31
        float acc[2][4] = {};
        blk_mma(acc, A(3, 3), AW, X31, 16, lane);
        blk_store(T31p, 16, acc, 1.f, lane);
      }
      named_bar_sync(BAR_PB, PB_THREADS);
      if (q == 0) {        // T_20 = -T_22 X20
        float acc[2][4] = {};
        blk_mma(acc, A(2, 2), AW, X20, 16, lane);
        blk_store(A(2, 0), AW, acc, -1.f, lane);
      } else if (q == 1) { // T_30 = -(T_32 X20 + T_33 X30)
        float acc[2][4] = {};
        blk_mma(acc, A(3, 2), AW, X20, 16, lane);
        blk_mma(acc, A(3, 3), AW, X30, 16, lane);
        blk_store(A(3, 0), AW, acc, -1.f, lane);
      } else if (q == 2) { // T_31 = -(T_32 X21 + T_33 X31)
        float acc[2][4] = {};
        blk_mma(acc, A(3, 2), AW, X21, 16, lane);
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int nh = 0; nh < 2; ++nh) {
          acc[nh][0] += T31p[g * 16 + 8 * nh + 2 * t];
          acc[nh][1] += T31p[g * 16 + 8 * nh + 2 * t + 1];
          acc[nh][2] += T31p[(g + 8) * 16 + 8 * nh + 2 * t];
          acc[nh][3] += T31p[(g + 8) * 16 + 8 * nh + 2 * t + 1];
        }
        blk_store(A(3, 1), AW, acc, -1.f, lane);
      }
      named_bar_sync(BAR_PB, PB_THREADS);
    }
    // ---- T*beta tile (bf16, K-major [64 r][64 i], 128B swizzle): thread = (row, 32-col half)
    {
      const int r = tid >> 1, hh = tid & 1;
      uint8_t* tt = x.sm + OFF_TB;
      const int a = r >> 4, rr = r & 15;
#pragma unroll
      for (int bb = 0; bb < 2; ++bb) {
        const int b = 2 * hh + bb;   // 16-column block
        float tv[16];
        if (b <= a) {
          int ld;
          const float* Tb = tblk(x.sm, a, b, ld);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int i = 16 * b + e;
            tv[e] = (i <= r) ? Tb[rr * ld + e] * betas[i] : 0.f;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) tv[e] = 0.f;
        }
        *reinterpret_cast<uint4*>(tt + swz128(r * 128 + b * 32)) = pack8(tv);
        *reinterpret_cast<uint4*>(tt + swz128(r * 128 + b * 32 + 16)) = pack8(tv + 8);
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(BAR_PB, PB_THREADS);
    if (tid == 0) mbar_arrive(&x.bars[B_TB + s2]);

    // ---- -W' readout (M=64 layout: rows 16q..16q+15 in lanes 32q..32q+15) -> bf16 over Rk
    ok = wait_b(x, B_WDONE + s2, (c >> 1) & 1);
    tc_fence_after();
#pragma unroll 1
    for (int part = 0; part < 4; ++part) {
      float v[32];
      tmem_ld32(x.tmem + TM_W + lane_base + 32 * part, v);
      tmem_ld_wait();
      if (lane < 16) {
        const int r = 16 * q + lane;
        uint8_t* rowp = qr + (part >> 1) * 16384;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
          *reinterpret_cast<uint4*>(rowp + swz128(r * 128 + (part & 1) * 64 + ch * 16)) =
              pack8(v + ch * 8);
      }
    }
    tc_fence_before();
    fence_proxy_async_smem();
    if (named_bar_or(BAR_PB, PB_THREADS, !ok)) break;
    if (tid == 0) {
      mbar_arrive(&x.bars[B_READY + s3]);
      mbar_arrive(&x.bars[B_PBIDLE]);
    }
  }
}

// ============================================================================
// state warps (12-15): the sequential pass over chunks
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

  const float* scal_all = reinterpret_cast<const float*>(x.sm + OFF_SCAL);
  auto write_sprime = [&](const float* scal_next) {
    const float eg = scal_next[crow];
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      float t[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) t[e] = eg * S[ch * 8 + e];
      *reinterpret_cast<uint4*>(sp + swz64(crow * 64 + ch * 16)) = pack8(t);
    }
  };

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
    // ---- Delta (fp32, accumulator rows 0-63 = lanes 0-63) -> bf16 tile (warps 0-1)
    bool okw = wait_b(x, B_ADONE, c & 1);
    tc_fence_after();
    if (q < 2) {
      float v[32];
      tmem_ld32(x.tmem + TM_C + s2 * 32 + lane_base, v);
      tmem_ld_wait();
      const int r = 32 * q + lane;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch)
        *reinterpret_cast<uint4*>(dl + swz64(r * 64 + ch * 16)) = pack8(v + ch * 8);
    }
    tc_fence_before();
    fence_proxy_async_smem();
    if (named_bar_or(BAR_ST, ST_THREADS, !okw)) break;
    if (tid == 0) mbar_arrive(&x.bars[B_DREADY]);
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
    // ---- output epilogue (off the sequential path): accumulator rows 64-127 (warps 2-3)
    okw = wait_b(x, B_ODONE, c & 1);
    tc_fence_after();
    if (q >= 2) {
      float v[32];
      tmem_ld32(x.tmem + TM_C + s2 * 32 + lane_base, v);
      tmem_ld_wait();
      const int r = 32 * (q - 2) + lane;
      if (okw && r < L) {
        __nv_bfloat16* orow = p.o + (size_t)(t0 + r) * x.rs + x.h * D + x.j0;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) *reinterpret_cast<uint4*>(orow + ch * 8) = pack8(v + ch * 8);
      }
    }
    tc_fence_before();
    named_bar_sync(BAR_ST, ST_THREADS);
    if (tid == 0) mbar_arrive(&x.bars[B_DCFREE + s2]);
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
  if (warp == MC_WARP) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  x.tmem = *tmem_slot;

  if (warp < PA_WARPS) {
    prep_a_role(x, args);
  } else if (warp < ST_WARP0) {
    prep_b_role(x);
  } else if (warp < LD_WARP) {
    state_role(x, args);
  } else if (warp == LD_WARP) {
    if (lane == 0) load_role(x, &map_k, &map_q, &map_v, &map_la);
  } else if (warp == MC_WARP) {
    if (lane == 0) mma_state_role(x);
  } else if (warp == MP_WARP) {
    if (lane == 0) mma_prep_role(x);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == MC_WARP) {
    tc_fence_after();
    tmem_dealloc(x.tmem, TM_COLS);
  }
}

}  // namespace tc
}  // namespace kda
