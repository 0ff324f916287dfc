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
// Decay factors. The chunk's last row is the reference: with E = e^{G - G_C} (>= 1)
// and its reciprocal F = e^{G_C - G} (<= 1), every pairwise factor is
// e^{G_r - G_i} = E_r F_i, so A and P come out of one tensor-core product
// [K*E ; Q*E] (K*F)^T, and the remaining factors fold into the state operand:
//   Rk = K*E, Rq = Q*E, Ck = K*F           (three bf16 tiles per chunk)
//   S'' = Diag(e^{G_C}) S                  (the decayed state, the bf16 MMA operand)
//   W' = T diag(beta) Rk,  U = T diag(beta) V
//   Delta = U - W' S'',  O = Rq S'' + P Delta,  S <- S'' + Ck^T Delta
// so the state update is a plain accumulate onto the decayed fp32 state. This is
// exact in real arithmetic. E must stay in range: a chunk whose decay range
// max_c (G_0c - G_63c) exceeds 60 nats takes an exact path instead (the pages'
// reason for secondary chunking): A and P from pairwise factors evaluated element
// by element, Rk and Rq built about the point before the chunk (K e^G, Q e^G, all
// factors <= 1) and the undecayed state as the operand.
//
// Layout. One CTA owns one (sequence, head) and all 128 value columns. The state
// lives in tensor memory for the whole sequence, transposed (lane = value column,
// column = key channel), so every state product has the state as its A operand:
//   [O | Delta]^T = S''^T [Rq ; -W']^T   (A = S''^T read from TMEM, M=128, N=128)
//   S^T += Delta^T Ck,  O^T += Delta^T P^T,  U^T = V^T (T beta)^T
//   W'^T = -Rk^T (T beta)^T               (the -W' tile is written from it)
// TMEM (512 columns):   0 S^T fp32 | 128 S''^T bf16 pairs | 192 O (odd chunks) |
//   256 U then Delta | 320 O (even chunks) | 384 Gram [A;P] | 448 -W'^T
//   (Delta^T is read out of 256-319 and written back there as bf16 pairs)
// The stacked B operand alternates [-W' ; Rq] (even chunks) and [Rq ; -W'] (odd)
// so that Delta always lands in columns 256-319 while the output alternates
// between the two regions around it: the output of chunk c is read while chunk
// c+1 is already accumulating.
//
// Roles (640 threads), a pipeline three chunks deep:
//   warps 0-7   prep A (chunk c+2): cumsum, range guard, Rk/Rq/Ck tiles, scalars;
//               its first thread issues the Gram product once prep B has read out
//               the previous one
//   warps 8-11  prep B (chunk c+1): Gram readout, UT solve, T*beta tile; its first
//               thread issues the k/q TMA loads and the L2 prefetch of the log-decay
//   warps 12-19 state  (chunk c):   decay S in TMEM and write S'', the -W' tile, Delta
//               as bf16 pairs back into TMEM (the A operand of the update), the
//               output tile; its first thread issues the state products, W', U, the
//               v TMA loads and the output's TMA store
// Every mbarrier wait is bounded; a timeout flags KDA_ERR_TIMEOUT and every role
// leaves (a group keeps meeting at its own named barriers, doing no work).
#pragma once

#include "kda_common.cuh"
#include "kda_segment.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace tc {

using namespace sm100;

constexpr int PA_WARPS = 8;
constexpr int PB_WARP0 = 8;
constexpr int ST_WARP0 = 12;
constexpr int ST_WARPS = 8;
constexpr int THREADS = 20 * 32;
constexpr int PA_THREADS = PA_WARPS * 32;
constexpr int PB_THREADS = 128;
constexpr int ST_THREADS = ST_WARPS * 32;
static_assert(PB_WARP0 % 4 == 0 && ST_WARP0 % 4 == 0, "TMEM lane quarters follow warp % 4");
constexpr uint32_t BAR_PA = 1, BAR_PB = 2, BAR_ST = 3;   // named barriers (0 is __syncthreads)
constexpr uint32_t BAR_OUT = 4;   // state warps: output tile staged (arrive), then stored
constexpr float LOG2E = 1.4426950408889634f;
constexpr float GUARD_LOG2 = 60.0f * 1.4426950408889634f;
constexpr uint64_t WAIT_NS = 2000000000ull;   // bound of every wait (unless a test sets its own)

// What the kernel reads and writes around the recurrence:
//   MODE_KDA    q, k (unit length), v, log_alpha [T, H, 128] fp32, beta [T, H] fp32 -> o
//   MODE_GDN    the same with one log-gate per token and head, log_alpha [T, H]
//   MODE_FUSED  the producing layer's activations and the output's post-processing
//               fused in: q and k are L2-normalised in the loader, the decay arrives
//               as a bf16 pre-activation x (log alpha = logsigmoid(x)), beta as a
//               pre-activation (sigmoid), and the output leaves as head-wise RMSNorm
//               times a weight times sigmoid(gate pre-activation)
enum : int { MODE_KDA = 0, MODE_GDN = 1, MODE_FUSED = 2 };
constexpr float L2_EPS = 1e-12f;   // guards the L2 normalisation of an all-zero row
constexpr float RMS_EPS = 1e-6f;   // RMSNorm epsilon

// ---- shared memory layout (offsets from a 1024-byte aligned base) ----
// Stage tile: 2 kblocks (channels 0-63, 64-127) x [128 rows][128 B], 128B swizzle.
// Rows 0-63 / 64-127 hold k (then Rk, then -W') and q (then Rq): k on top for even
// chunks, q on top for odd chunks.
constexpr uint32_t KQ_BYTES = 32768;
constexpr uint32_t CKP_BYTES = 24576;    // Ck [2 kblocks][64][128 B] (16 KB) | P [64][128 B] (8 KB)
constexpr uint32_t OFF_KQ = 0;
constexpr uint32_t OFF_CKP = OFF_KQ + 3 * KQ_BYTES;
constexpr uint32_t OFF_V = OFF_CKP + 2 * CKP_BYTES;   // v [2 column blocks][64][128 B]
constexpr uint32_t OFF_TB = OFF_V + 16384;            // T*beta [64 r][64 i] bf16, K-major
constexpr uint32_t OFF_DT = OFF_TB + 8192;            // output staging [64 rows][128 cols] bf16
constexpr int AW = 68;                                // fp32 pitch of the A / T workspace
constexpr uint32_t OFF_AW = OFF_DT + 16384;           // also the exact path's staging area
constexpr uint32_t OFF_XS = OFF_AW + 64 * AW * 4;     // 6 extra 16x16 fp32 blocks
constexpr uint32_t OFF_SCR = OFF_XS + 6 * 1024;       // 4 per-warp 16x16 scratch blocks
constexpr uint32_t OFF_BETA = OFF_SCR + 4 * 1024;     // [3][64]
constexpr uint32_t OFF_SCAL = OFF_BETA + 3 * 64 * 4;  // [3 slots][2][128]: state decay, operand scale
constexpr uint32_t OFF_WSUM = OFF_SCAL + 6 * 128 * 4; // [8][128] cumsum warp totals
constexpr uint32_t OFF_GROW = OFF_WSUM + 8 * 128 * 4; // [2][128] G of rows 0 and 63 (log2 units)
constexpr uint32_t OFF_XFLAG = OFF_GROW + 2 * 128 * 4; // [3] exact-path flag per slot
constexpr uint32_t OFF_BAR = OFF_XFLAG + 16;
constexpr int NBARS = 32;
constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;   // abort word, TMEM address, wait bound, test hook
constexpr uint32_t MISC_TMEM = 8, MISC_WAIT_NS = 16, MISC_SKIP_TB = 24;   // byte offsets in MISC
constexpr uint32_t OFF_ROWSQ = OFF_MISC + 64;         // fused output: [64 rows][4] partial sums of squares
constexpr uint32_t OFF_NORMW = OFF_ROWSQ + 64 * 4 * 4;  // fused output: RMSNorm weight [128]
constexpr uint32_t SMEM_USED = OFF_NORMW + 128 * 4;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(64 * 64 * 4 <= 64 * AW * 4, "exact-path staging of one channel half fits the workspace");

// ---- TMEM columns (512 allocated) ----
constexpr uint32_t TM_S = 0;      // S^T fp32 master: lane = value column, column = key channel
constexpr uint32_t TM_SB = 128;   // S''^T bf16, two channels per column (the A operand)
constexpr uint32_t TM_OA = 192;   // O^T of odd chunks
constexpr uint32_t TM_D = 256;    // U^T, then Delta^T fp32, then its bf16 pairs (see dpair_col)
constexpr uint32_t TM_OB = 320;   // O^T of even chunks
constexpr uint32_t TM_G = 384;    // Gram [A;P] or [P;A] (M=128, N=64)
constexpr uint32_t TM_W = 448;    // -W'^T (M=128 channels, N=64 rows)
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t IDESC_CRIT = idesc_bf16(128, 128, 0, 0);    // S''^T (TMEM) x stage tile
constexpr uint32_t IDESC_DELTA = idesc_bf16(128, 64, 0, 0);    // S''^T (TMEM) x -W' (no output)
constexpr uint32_t IDESC_Z = idesc_bf16(128, 128, 0, 1);       // Delta^T x Ck (MN-major)
constexpr uint32_t IDESC_PD = idesc_bf16(128, 64, 0, 0);       // Delta^T x P
constexpr uint32_t IDESC_GRAM = idesc_bf16(128, 64, 0, 0);     // stage tile x Ck
constexpr uint32_t IDESC_W = idesc_bf16(128, 64, 1, 0, 1);     // -Rk^T (MN-major) x (T beta)^T
constexpr uint32_t IDESC_U = idesc_bf16(128, 64, 1, 0);        // V^T (MN-major) x (T beta)

// ---- mbarriers ----
enum : int {
  B_FULL = 0,       // [3] TMA of k, q landed in a stage slot
  B_KQFREE = 3,     // [3] stage slot no longer needed (state product done)
  B_VFULL = 6,      // TMA of v landed
  B_TILES = 7,      // [2] Rk, Rq, Ck, scalars and exact flag written
  B_GRAM = 9,       // Gram MMA done
  B_TB = 10,        // P and T*beta tiles written
  B_WDONE = 11,     // W' MMA done
  B_UDONE = 12,     // U MMA done (v and T*beta free)
  B_GFREE = 13,     // Gram columns read out (by prep B): the next Gram may go out
  B_FIN_A = 14,     // drain of prep A's first thread (it issues the Gram)
  B_CRIT = 15,      // [O | Delta] product done
  B_ZDONE = 16,     // state update product done
  B_PD = 17,        // P Delta product done (output complete)
  B_CKFREE = 18,    // [2] Ck/P slot no longer needed
  B_WFREE = 20,     // prep B done with a chunk (workspace free)
  B_FIN_C = 21,     // drains
  B_FIN_P = 22,
  NUM_BARS = 23
};
static_assert(NUM_BARS <= NBARS, "barrier slots");

// Work plans. PLAN_SEQ: one CTA per (sequence of cu_seqlens, head). The time split
// of one long sequence cuts it into n_seg >= 2 segments of whole chunks, balanced to
// within one chunk (segment j starts at chunk j*seg_base + min(j, seg_rem); the last
// one ends at t_total). Every step of the recurrence is affine in the state, so a
// segment maps its entering state S to M S + R (M the product of its transitions, R
// its final state from a zero start), and its output is its output from a zero
// start plus the output of the same segment run from S with v = 0 (the correction).
// Slots of seg_states [2 n_seg - 2][H][128][128]. The split runs
//   PLAN_ZERO (grid H x (2 n_seg - 2)), in block order:
//     Z_0 .. Z_{n-1}   every segment from a zero state (segment 0 from the caller's
//                      h0), storing its output; final states: segment 0's to slot
//                      0, R_j to slot j (j = 1 .. n-2), R_{n-1} to slot 2 n_seg - 3
//     M_1 .. M_{n-2}   segment j from the identity with v = 0, output discarded: its
//                      final state is M_j (slot n_seg - 2 + j). Once the state is
//                      exactly zero it stays zero, so the CTA stops there. These
//                      take the SMs the Z CTAs leave free, or follow them.
//   the segment scan (slot j <- S_{j+1} = M_j S_j + R_j), then
//   PLAN_CORR (grid H x (n_seg - 1)): segment j = 1 .. n_seg-1 from slot j-1 with
//     v = 0, adding its output onto o and stopping once its state is exactly zero
//     (every later correction is zero); for the last segment the caller's hT =
//     R_{n-1} + the chain's final state (zero after a stop).
// With typical decay the corrections die out within some tens of chunks, so a call
// costs about one pass over 1/n_seg of the sequence; without decay or erase they run
// to the ends of their segments (two such passes). The fused variant's output is not
// linear in o (its RMSNorm): in the split only segment 0's CTAs apply the norm and
// the gate, the other Z CTAs and the corrections work on the raw output, and a last
// pass (kda_norm_gate_kernel) normalises and gates segments 1 .. n-1.
// The kernel's SPLIT instance serves PLAN_ZERO and PLAN_CORR and reads the per-CTA
// flags below; the PLAN_SEQ instance has them all off at compile time.
enum : int { PLAN_SEQ = 0, PLAN_ZERO = 1, PLAN_CORR = 2 };
// What a CTA does with its output: store it, discard it (a transition chain), or
// add it onto o (a correction)
enum : int { OUT_STORE = 0, OUT_NONE = 1, OUT_ADD = 2 };

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
  int plan;
  int n_seg;
  int seg_base, seg_rem;   // chunks per segment: seg_base, plus one for the first seg_rem
  float* seg_states;   // [2 n_seg - 2][H][128][128]
  const int32_t* seq_order;   // PLAN_SEQ: sequences longest first (or null: index order)
  // MODE_FUSED: log_alpha and beta are unused; these take their place
  const __nv_bfloat16* decay_pre;   // [T, H, 128], log alpha = logsigmoid(decay_pre)
  const float* beta_pre;            // [T, H], beta = sigmoid(beta_pre)
  const __nv_bfloat16* gate_pre;    // [T, H, 128], output gate = sigmoid(gate_pre)
  const float* norm_w;              // [128] RMSNorm weight
  // testing only (kda_testing_chunk_fwd_stall): the bound of every wait, and one chunk
  // whose "T*beta ready" arrive prep B leaves out (-1: none)
  uint64_t wait_ns;
  int debug_skip_tb;
};

struct Ctx {
  uint8_t* sm;
  uint64_t* bars;
  volatile int* abort_flag;
  uint32_t tmem;
  int h, n_chunks;
  int64_t bos, eos;
  size_t rs;          // elements between consecutive tokens of q/k/v/o/log_alpha
  const float* h0;    // this CTA's entering state [channel][value], or null (zeros)
  float* hT;          // where its final state goes, or null
  const float* hT_base;   // if not null: hT = hT_base + the final state
  bool h0_identity;   // entering state = I (transition of a segment)
  bool v_zero;        // v taken as zero (no loads)
  int out_mode;       // OUT_STORE, OUT_NONE or OUT_ADD
  bool stop_on_zero;  // stop once the state is exactly zero (v = 0 chains)
  bool gated;         // MODE_FUSED: the output is final (RMSNorm and gate applied)
};


// Values of the shared abort word: a role that gives up a wait raises ABORT_TIMEOUT
// (and flags the device error); the state warps of a transition chain raise
// ABORT_DONE when the state has become exactly zero. Either way every role leaves
// its loop at its next wait.
constexpr int ABORT_TIMEOUT = 1, ABORT_DONE = 2;

// Bounded per-thread wait that also gives up when another role aborted. The
// thread sleeps in the barrier (suspend hint) instead of spinning, and looks at the
// abort word at least every WAKE_NS: a chain that stops early (ABORT_DONE) leaves its
// other roles blocked on barriers that will not complete, and the CTA holds its SM
// until they notice (with a 200 us hint, a correction pass of 2 segments took 0.51
// ms where its CTAs' work took 0.30). (Out of line, with scalar arguments only, so
// that callers keep their context in registers. The bound lives in shared memory
// beside the abort word: MISC_WAIT_NS.)
constexpr uint32_t WAKE_NS = 2000;
__device__ __noinline__ bool wait_b_slow(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const uint64_t t0 = globaltimer_ns();
  const uint64_t limit = *reinterpret_cast<const volatile uint64_t*>(
      reinterpret_cast<volatile uint8_t*>(abort_flag) + MISC_WAIT_NS);
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, WAKE_NS)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit) {
      *abort_flag = ABORT_TIMEOUT;
      flag_error(DEVERR_TIMEOUT);
      return false;
    }
  }
}
// Fast path inline (the first try blocks until the phase completes or a short
// hardware limit passes), the sleeping loop out of line.
__device__ __forceinline__ bool wait_b(const Ctx& x, int b, uint32_t parity) {
  uint64_t* bar = &x.bars[b];
  if (mbar_try_wait(bar, parity)) return true;
  return wait_b_slow(bar, parity, x.abort_flag);
}

// Global loads issued exactly where written (volatile), ahead of the barrier waits.
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
__device__ __forceinline__ float rcpf(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// logsigmoid(x) = min(x, 0) - log(1 + e^{-|x|}), sigmoid(x) = 1 / (1 + e^{-x}), both on
// the fast exp2/log2 units
__device__ __forceinline__ float logsigmoidf_fast(float x) {
  float l;
  const float e = ex2f(-fabsf(x) * LOG2E);
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(l) : "f"(1.f + e));
  return fminf(x, 0.f) - l * 0.6931471805599453f;
}
__device__ __forceinline__ float sigmoidf_fast(float x) { return rcpf(1.f + ex2f(-x * LOG2E)); }
__device__ __forceinline__ uint4 ldg_nc_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ldg_nc_u2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
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
// A 32 x 32 block of an fp32 TMEM region whose lanes index the columns of a bf16 tile
// and whose TMEM columns index its rows: TMEM lanes lane0 .. lane0+31 (the calling
// warp's quarter) x TMEM columns from taddr, written transposed into rows row0 ..
// row0+31 of a K-major tile with 128-byte swizzle (64 columns per block of
// kb_stride bytes), rounded to nearest even. Two fragment loads and four
// transposing matrix stores of 16-byte rows per warp.
__device__ __forceinline__ void tmem_block_to_tile_t(uint32_t taddr, int lane0, int row0,
                                                     uint8_t* tile, uint32_t kb_stride, int lane) {
  uint32_t v[2][16];
  tmem_ld16x256b_x4(taddr, v[0]);
  tmem_ld16x256b_x4(taddr + (16u << 16), v[1]);
  tmem_ld_wait();
  const int mi = lane >> 3;   // the matrix whose row address this thread gives
#pragma unroll
  for (int hf = 0; hf < 2; ++hf)
#pragma unroll
    for (int rp = 0; rp < 2; ++rp) {
      const uint32_t* w = v[hf] + 8 * rp;
      const int col = lane0 + 16 * hf + 8 * (mi & 1);       // first tile column of matrix mi
      const int row = row0 + 8 * (2 * rp + (mi >> 1)) + (lane & 7);
      const uint32_t addr =
          smem_u32(tile + (col >> 6) * kb_stride) + swz128((uint32_t)row * 128u + (uint32_t)(col & 63) * 2u);
      stmatrix_x4_trans(addr, pack_bf16(__uint_as_float(w[0]), __uint_as_float(w[1])),
                        pack_bf16(__uint_as_float(w[2]), __uint_as_float(w[3])),
                        pack_bf16(__uint_as_float(w[4]), __uint_as_float(w[5])),
                        pack_bf16(__uint_as_float(w[6]), __uint_as_float(w[7])));
    }
}

// tmem_block_to_tile_t that also sums the squares of each of the block's 32 tile rows
// over its 32 tile columns (from the fp32 values, before rounding) and leaves the sums
// in rowsq[row * 4 + quarter] (quarter: which 32 of the tile's 128 columns).
__device__ __forceinline__ void tmem_block_to_tile_t_rowsq(uint32_t taddr, int lane0, int row0,
                                                           uint8_t* tile, uint32_t kb_stride,
                                                           int lane, float* rowsq, int quarter) {
  uint32_t v[2][16];
  tmem_ld16x256b_x4(taddr, v[0]);
  tmem_ld16x256b_x4(taddr + (16u << 16), v[1]);
  tmem_ld_wait();
  // thread t holds columns 2(t%4), 2(t%4)+1 of every 8-row group: sum its 4 values per
  // row, then over the 8 threads with the same t%4
#pragma unroll
  for (int rep = 0; rep < 4; ++rep)
#pragma unroll
    for (int col = 0; col < 2; ++col) {
      float ss = 0.f;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const float a = __uint_as_float(v[hf][4 * rep + col]);
        const float b = __uint_as_float(v[hf][4 * rep + 2 + col]);
        ss = fmaf(a, a, fmaf(b, b, ss));
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 4);
      ss += __shfl_xor_sync(0xffffffffu, ss, 8);
      ss += __shfl_xor_sync(0xffffffffu, ss, 16);
      if (lane < 4) rowsq[(row0 + 8 * rep + 2 * lane + col) * 4 + quarter] = ss;
    }
  const int mi = lane >> 3;
#pragma unroll
  for (int hf = 0; hf < 2; ++hf)
#pragma unroll
    for (int rp = 0; rp < 2; ++rp) {
      const uint32_t* w = v[hf] + 8 * rp;
      const int col = lane0 + 16 * hf + 8 * (mi & 1);
      const int row = row0 + 8 * (2 * rp + (mi >> 1)) + (lane & 7);
      const uint32_t addr =
          smem_u32(tile + (col >> 6) * kb_stride) + swz128((uint32_t)row * 128u + (uint32_t)(col & 63) * 2u);
      stmatrix_x4_trans(addr, pack_bf16(__uint_as_float(w[0]), __uint_as_float(w[1])),
                        pack_bf16(__uint_as_float(w[2]), __uint_as_float(w[3])),
                        pack_bf16(__uint_as_float(w[4]), __uint_as_float(w[5])),
                        pack_bf16(__uint_as_float(w[6]), __uint_as_float(w[7])));
    }
}

__device__ __forceinline__ uint64_t kdesc128(uint32_t addr) {
  return make_sdesc(addr, 16, 1024, SWZ_128B);
}
// A descriptor moved on by a byte offset (a multiple of 16). Shared-memory addresses
// stay below 2^18, so the start-address field (bits 0-13, the address >> 4) takes the
// sum without a carry into the fields above it.
__device__ __forceinline__ uint64_t desc_at(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

// ============================================================================
// TMA and MMA issue (each by the first thread of the role that consumes the result)
//
// Code size. With a CTA on every SM, this kernel is bound by instruction fetch: the
// SMs of a GPC share one instruction cache level above their own (the GPC's L1.5),
// which serves about 300 requests per chunk and CTA and is busy 85 % of the time,
// and per-chunk times then differ by a third between GPCs holding fewer or more busy
// SMs. A chunk executes some 40 KB of distinct code, which does not stay in the SM's
// own cache from one chunk to the next. So the MMA issue loops below stay rolled
// (a few instructions more per product, a quarter of the code), and prep B's UT
// merges share their code between warps. Each measured alone on a full GPU: rolled
// issue loops 5.79 -> 5.38 us per chunk, rolled Gram readout -> 5.13, shared
// merges -> 4.80.
// ============================================================================
__device__ __forceinline__ void issue_kq(const Ctx& x, const CUtensorMap* map_k,
                                         const CUtensorMap* map_q, int c) {
  const int xk = x.h * D;
  const int y = (int)(x.bos + (int64_t)c * CHUNK);
  uint8_t* st = x.sm + OFF_KQ + (c % 3) * KQ_BYTES;
  const uint32_t koff = (c & 1) ? 8192u : 0u, qoff = 8192u - koff;
  uint64_t* full = &x.bars[B_FULL + c % 3];
  mbar_arrive_expect_tx(full, 4 * 8192);
  tma_load_2d(st + koff, map_k, xk, y, full);
  tma_load_2d(st + 16384 + koff, map_k, xk + 64, y, full);
  tma_load_2d(st + qoff, map_q, xk, y, full);
  tma_load_2d(st + 16384 + qoff, map_q, xk + 64, y, full);
}
template <bool SPLIT>
__device__ __forceinline__ void issue_v(const Ctx& x, const CUtensorMap* map_v, int c) {
  const int xk = x.h * D;
  const int y = (int)(x.bos + (int64_t)c * CHUNK);
  uint64_t* full = &x.bars[B_VFULL];
  if (SPLIT && x.v_zero) {   // the v tile stays zero: complete the phase without a copy
    mbar_arrive(full);
    return;
  }
  mbar_arrive_expect_tx(full, 2 * 8192);
  tma_load_2d(x.sm + OFF_V, map_v, xk, y, full);
  tma_load_2d(x.sm + OFF_V + 8192, map_v, xk + 64, y, full);
}
// On the way out: wait (bounded, ignoring the abort flag) for a copy still in flight.
__device__ void settle(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > 100000000ull) break;
}
// On the way out: wait (bounded) until this thread's tensor-core work is done.
__device__ void drain(const Ctx& x, int bar) {
  umma_commit(&x.bars[bar]);
  settle(&x.bars[bar], 0);
}

// [O | Delta]^T (or [Delta | O]^T) += S''^T [stage tile]^T   (M=128, N=128, K=128);
// the state operand comes from TMEM
__device__ __forceinline__ void issue_crit(const Ctx& x, int c) {
  tc_fence_after();
  const uint64_t b0 = kdesc128(smem_u32(x.sm) + OFF_KQ + (c % 3) * KQ_BYTES);
  const uint32_t d = x.tmem + ((c & 1) ? TM_OA : TM_D);
#pragma unroll 1
  for (int kk = 0; kk < 8; ++kk)
    umma_bf16_tmem_a(d, x.tmem + TM_SB + kk * 8, desc_at(b0, (kk >> 2) * 16384 + (kk & 3) * 32),
                     IDESC_CRIT, 1u);
  umma_commit(&x.bars[B_CRIT]);
  umma_commit(&x.bars[B_KQFREE + c % 3]);
}
// TMEM column of the bf16 Delta^T pairs of K step kk (chunk rows 16kk..16kk+15): the
// state warps write rows 0-31 into the first 16 columns of the Delta region and rows
// 32-63 into its last 16, each warp inside the columns it has just read
__device__ __forceinline__ uint32_t dpair_col(int kk) { return TM_D + (kk < 2 ? 8 * kk : 48 + 8 * (kk - 2)); }

// S^T += Delta^T Ck (the state update), then O^T += Delta^T P^T; Delta^T is the A
// operand, read from TMEM
__device__ __forceinline__ void issue_update(const Ctx& x, int c) {
  tc_fence_after();
  const uint32_t ck = smem_u32(x.sm) + OFF_CKP + (c & 1) * CKP_BYTES;
  // (M=128, N=128, K=64); Ck read as an MN-major B operand
  const uint64_t z0 = make_sdesc(ck, 8192, 1024, SWZ_128B);
#pragma unroll 1
  for (int kk = 0; kk < 4; ++kk)
    umma_bf16_tmem_a(x.tmem + TM_S, x.tmem + dpair_col(kk), desc_at(z0, kk * 2048), IDESC_Z, 1u);
  umma_commit(&x.bars[B_ZDONE]);
  // (M=128, N=64, K=64)
  const uint32_t o = x.tmem + ((c & 1) ? TM_OA : TM_OB);
  const uint64_t p0 = kdesc128(ck + 16384);
#pragma unroll 1
  for (int kk = 0; kk < 4; ++kk)
    umma_bf16_tmem_a(o, x.tmem + dpair_col(kk), desc_at(p0, kk * 32), IDESC_PD, 1u);
  umma_commit(&x.bars[B_PD]);
  umma_commit(&x.bars[B_CKFREE + (c & 1)]);
}
// U^T = V^T (T beta)^T   (M=128 value columns, N=64, K=64); v read as MN-major A (a
// zero tile for a v = 0 chain: U = 0, which the [O | Delta] product accumulates onto)
__device__ __forceinline__ void issue_u(const Ctx& x) {
  tc_fence_after();
  const uint32_t sbase = smem_u32(x.sm);
  const uint64_t a0 = make_sdesc(sbase + OFF_V, 8192, 1024, SWZ_128B), b0 = kdesc128(sbase + OFF_TB);
#pragma unroll 1
  for (int kk = 0; kk < 4; ++kk)
    umma_bf16(x.tmem + TM_D, desc_at(a0, kk * 2048), desc_at(b0, kk * 32), IDESC_U, kk > 0 ? 1u : 0u);
  umma_commit(&x.bars[B_UDONE]);
}
// -W'^T = -Rk^T (T beta)^T   (M=128 channels, N=64, K=64); Rk (the k half of the
// stage tile) read as an MN-major A operand
__device__ __forceinline__ void issue_w(const Ctx& x, int c) {
  tc_fence_after();
  const uint32_t sbase = smem_u32(x.sm);
  const uint64_t a0 = make_sdesc(sbase + OFF_KQ + (c % 3) * KQ_BYTES + ((c & 1) ? 8192u : 0u), 16384,
                                 1024, SWZ_128B);
  const uint64_t b0 = kdesc128(sbase + OFF_TB);
#pragma unroll 1
  for (int kk = 0; kk < 4; ++kk)
    umma_bf16(x.tmem + TM_W, desc_at(a0, kk * 2048), desc_at(b0, kk * 32), IDESC_W, kk > 0 ? 1u : 0u);
  umma_commit(&x.bars[B_WDONE]);
}

// Gram product of chunk g (issued by prep A's first thread once its tiles are written): [A ; P] or [P ; A] =
// stage tile x Ck^T (M=128, N=64, K=128). For an exact-path chunk only the commit
// goes out, so the barrier completes one phase per chunk either way.
__device__ __forceinline__ void issue_gram(const Ctx& x, int g) {
  const int* xflag = reinterpret_cast<const int*>(x.sm + OFF_XFLAG);
  if (xflag[g % 3]) {
    umma_commit(&x.bars[B_GRAM]);
    return;
  }
  tc_fence_after();
  const uint32_t sbase = smem_u32(x.sm);
  const uint64_t a0 = kdesc128(sbase + OFF_KQ + (g % 3) * KQ_BYTES);
  const uint64_t b0 = kdesc128(sbase + OFF_CKP + (g & 1) * CKP_BYTES);
#pragma unroll 1
  for (int kk = 0; kk < 8; ++kk)
    umma_bf16(x.tmem + TM_G, desc_at(a0, (kk >> 2) * 16384 + (kk & 3) * 32),
              desc_at(b0, (kk >> 2) * 8192 + (kk & 3) * 32), IDESC_GRAM, kk > 0 ? 1u : 0u);
  umma_commit(&x.bars[B_GRAM]);
}

// ============================================================================
// prep A (warps 0-7): decay factors and the three bf16 tiles of a chunk
// ============================================================================

// Exact path for a chunk whose decay range is too wide for the factored Gram (kept
// out of line, with arguments passed by value: it is rare and large). G of this
// thread's rows is recomputed from the (L2-resident) log-decay and the warp totals
// still in shared memory. Pairwise factors are evaluated one by one, one channel
// half at a time with G staged in prep B's workspace; A goes to that workspace, P
// to its tile, and Rk / Rq are built about the point before the chunk.
__device__ __noinline__ bool prep_a_exact(const Ctx x, const float* log_alpha,
                                          const __nv_bfloat16* decay_pre, int mode, int c, int L,
                                          uint8_t* kq, uint32_t koff, uint32_t qoff, uint8_t* ck,
                                          const float* betas) {
  const int tid = threadIdx.x;
  const int w = tid >> 5, lane = tid & 31;
  const int kb = lane >> 4;
  const uint32_t cbyte = (lane & 15) * 8;
  const int c0 = 4 * lane;
  float* aw = reinterpret_cast<float*>(x.sm + OFF_AW);
  const float* wsum = reinterpret_cast<const float*>(x.sm + OFF_WSUM);
  const float* grow = reinterpret_cast<const float*>(x.sm + OFF_GROW);
  float g2[8][4], gc[4];
  {
    const int64_t t0 = x.bos + (int64_t)c * CHUNK;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int ww = 0; ww < w; ++ww)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k] += wsum[ww * 128 + c0 + k];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t t = t0 + 8 * w + j;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t < x.eos) {
        if (mode == MODE_GDN) {   // one gate per token and head
          const float a = ldg_nc_f32(log_alpha + (size_t)t * (x.rs / D) + x.h);
          v = make_float4(a, a, a, a);
        } else if (mode == MODE_FUSED) {   // logsigmoid of the bf16 pre-activation
          const uint2 r = ldg_nc_u2(decay_pre + (size_t)t * x.rs + x.h * D + c0);
          v = make_float4(logsigmoidf_fast(bf_lo(r.x)), logsigmoidf_fast(bf_hi(r.x)),
                          logsigmoidf_fast(bf_lo(r.y)), logsigmoidf_fast(bf_hi(r.y)));
        } else {
          v = ldg_nc_v4(log_alpha + (size_t)t * x.rs + x.h * D + c0);
        }
      }
      const float lv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc[k] = fmaf(lv[k], LOG2E, acc[k]);
        g2[j][k] = acc[k];
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) gc[k] = grow[128 + c0 + k];
  }
  // prep B must be done with chunk c-1 (its workspace) and this Ck/P slot free
  bool ok = (c < 1) || wait_b(x, B_WFREE, (c - 1) & 1);
  ok = ok && ((c < 2) || wait_b(x, B_CKFREE + (c & 1), ((c - 2) >> 1) & 1));
  if (named_bar_or(BAR_PA, PA_THREADS, !ok)) return false;
  // warp w takes lower-triangle pairs p = w, w+8, ... (row-major r(r+1)/2 + i); the
  // lane that finishes a pair's reduction keeps it (the same lane in both halves)
  float pval[9], aval[9];
  int pidx[9];
#pragma unroll
  for (int bt = 0; bt < 9; ++bt) {
    pval[bt] = 0.f;
    aval[bt] = 0.f;
    pidx[bt] = -1;
  }
  float* gsm = aw;   // G (log2 units) of one channel half: [64 rows][64] fp32
  for (int hf = 0; hf < 2; ++hf) {
    if (kb == hf) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<float4*>(&gsm[(8 * w + j) * 64 + (c0 - 64 * hf)]) =
            make_float4(g2[j][0], g2[j][1], g2[j][2], g2[j][3]);
    }
    named_bar_sync(BAR_PA, PA_THREADS);
    const int ch = 2 * lane;                  // channel pair within the half
    const uint32_t cb = (uint32_t)ch * 2u;    // its byte offset in the kblock row
    const uint8_t* kt = kq + koff + hf * 16384;
    const uint8_t* qt = kq + qoff + hf * 16384;
#pragma unroll
    for (int bt = 0; bt < 9; ++bt) {
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
          const uint32_t kr = *reinterpret_cast<const uint32_t*>(kt + swz128(r * 128 + cb));
          const uint32_t ki = *reinterpret_cast<const uint32_t*>(kt + swz128(i * 128 + cb));
          const uint32_t qv = *reinterpret_cast<const uint32_t*>(qt + swz128(r * 128 + cb));
          const float2 gr = *reinterpret_cast<const float2*>(&gsm[r * 64 + ch]);
          const float2 gi = *reinterpret_cast<const float2*>(&gsm[i * 64 + ch]);
          const float ke0 = bf_lo(ki) * ex2f(gr.x - gi.x);
          const float ke1 = bf_hi(ki) * ex2f(gr.y - gi.y);
          sa = fmaf(bf_lo(kr), ke0, bf_hi(kr) * ke1);
          sp = fmaf(bf_lo(qv), ke0, bf_hi(qv) * ke1);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          sa += __shfl_xor_sync(0xffffffffu, sa, off);
          sp += __shfl_xor_sync(0xffffffffu, sp, off);
        }
        if (lane == qq) {
          pval[bt] += sp;
          aval[bt] += sa;
          pidx[bt] = r * 64 + i;
        }
      }
    }
    named_bar_sync(BAR_PA, PA_THREADS);   // the staging area is rewritten next
  }
  // P tile cleared, then A (beta-scaled, strictly lower) and P filled in
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
  // tiles about the point before the chunk: Rk = K e^G, Rq = Q e^G; Ck = K e^{G_C - G}
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int r = 8 * w + j;
    const bool valid = r < L;
    uint2* kp = reinterpret_cast<uint2*>(kq + koff + kb * 16384 + swz128(r * 128 + cbyte));
    uint2* qp = reinterpret_cast<uint2*>(kq + qoff + kb * 16384 + swz128(r * 128 + cbyte));
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
  return true;
}

template <bool SPLIT, int MODE>
__device__ void prep_a_role(const Ctx& x, const Args& p) {
  constexpr bool SG = MODE == MODE_GDN, FU = MODE == MODE_FUSED;
  const int tid = threadIdx.x;
  const int w = tid >> 5, lane = tid & 31;
  const int kb = lane >> 4;                // kblock of this thread's 4 channels
  const uint32_t cbyte = (lane & 15) * 8;  // byte offset of the channels in the kblock row
  const int c0 = 4 * lane;
  float* wsum = reinterpret_cast<float*>(x.sm + OFF_WSUM);
  float* grow = reinterpret_cast<float*>(x.sm + OFF_GROW);
  int* xflag = reinterpret_cast<int*>(x.sm + OFF_XFLAG);
  // beta of row tid of chunk cn (zero past the end of the sequence), loaded one chunk
  // early so that its latency hides behind a whole chunk of work
  auto load_beta = [&](int cn) -> float {
    const int64_t t = x.bos + (int64_t)cn * CHUNK + tid;
    if (FU)   // (the sigmoid is applied where the value is stored, a chunk later)
      return (tid < 64 && t < x.eos) ? ldg_nc_f32(p.beta_pre + (size_t)t * p.n_heads + x.h) : -1e30f;
    return (tid < 64 && t < x.eos) ? ldg_nc_f32(p.beta + (size_t)t * p.n_heads + x.h) : 0.f;
  };
  float beta_next = load_beta(0);

  for (int c = 0; c < x.n_chunks; ++c) {
    const int s3 = c % 3;
    const int64_t t0 = x.bos + (int64_t)c * CHUNK;
    const int L = (x.eos - t0) < CHUNK ? (int)(x.eos - t0) : CHUNK;
    uint8_t* kq = x.sm + OFF_KQ + s3 * KQ_BYTES;
    uint8_t* ck = x.sm + OFF_CKP + (c & 1) * CKP_BYTES;
    const uint32_t koff = (c & 1) ? 8192u : 0u, qoff = 8192u - koff;
    float* betas = reinterpret_cast<float*>(x.sm + OFF_BETA) + s3 * 64;
    float* scal = reinterpret_cast<float*>(x.sm + OFF_SCAL) + s3 * 256;

    // log-decay rows 8w..8w+7 of this chunk, channels c0..c0+3 (L2-prefetched three
    // chunks ahead by the thread that loads k/q); zero past the end of the sequence
    float g2[8][4];
    if (SG) {
      // one gate per row (the same address for the whole warp); the rows of the chunk
      // two ahead go to L2 now
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t t = t0 + 8 * w + j;
        const float a = t < x.eos ? ldg_nc_f32(p.log_alpha + (size_t)t * p.n_heads + x.h) : 0.f;
        g2[j][0] = a; g2[j][1] = a; g2[j][2] = a; g2[j][3] = a;
      }
      const int64_t tp = t0 + 2 * CHUNK + tid;
      if (tid < CHUNK && tp < x.eos) prefetch_l2(p.log_alpha + (size_t)tp * p.n_heads + x.h);
    } else if (FU) {
      // the bf16 decay pre-activation (L2-prefetched three chunks ahead), logsigmoid here
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t t = t0 + 8 * w + j;
        uint2 r = make_uint2(0u, 0u);
        if (t < x.eos) r = ldg_nc_u2(p.decay_pre + (size_t)t * x.rs + x.h * D + c0);
        g2[j][0] = bf_lo(r.x); g2[j][1] = bf_hi(r.x); g2[j][2] = bf_lo(r.y); g2[j][3] = bf_hi(r.y);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const bool valid = t0 + 8 * w + j < x.eos;
#pragma unroll
        for (int k = 0; k < 4; ++k) g2[j][k] = valid ? logsigmoidf_fast(g2[j][k]) : 0.f;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t t = t0 + 8 * w + j;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (t < x.eos) v = ldg_nc_v4(p.log_alpha + (size_t)t * x.rs + x.h * D + c0);
        g2[j][0] = v.x; g2[j][1] = v.y; g2[j][2] = v.z; g2[j][3] = v.w;
      }
    }
    // (the reader of this beta slot, prep B three chunks back, finished before this
    // role got the Ck slot of chunk c-1)
    if (tid < 64) betas[tid] = FU ? sigmoidf_fast(beta_next) : beta_next;
    beta_next = load_beta(c + 1);

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
      if (w == 7) *reinterpret_cast<float4*>(&grow[128 + c0]) = make_float4(g2[7][0], g2[7][1], g2[7][2], g2[7][3]);
    }
    bool ok = wait_b(x, B_FULL + s3, (c / 3) & 1);
    if (named_bar_or(BAR_PA, PA_THREADS, !ok)) break;
    if (FU) {
      // L2-normalise this warp's 8 rows of k and q in place: the 32 lanes hold the
      // 128 channels of a row, 4 each. All 16 row sums first, then their butterflies
      // side by side (independent shuffle chains), then the rescaled rows written back;
      // everything downstream reads the unit rows.
      float ss[2][8];
#pragma unroll
      for (int half = 0; half < 2; ++half)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint2 v = *reinterpret_cast<const uint2*>(kq + (half ? qoff : koff) + kb * 16384 +
                                                          swz128((8 * w + j) * 128 + cbyte));
          const float f0 = bf_lo(v.x), f1 = bf_hi(v.x), f2 = bf_lo(v.y), f3 = bf_hi(v.y);
          ss[half][j] = f0 * f0 + f1 * f1 + f2 * f2 + f3 * f3;
        }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int half = 0; half < 2; ++half)
#pragma unroll
          for (int j = 0; j < 8; ++j) ss[half][j] += __shfl_xor_sync(0xffffffffu, ss[half][j], off);
#pragma unroll
      for (int half = 0; half < 2; ++half)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint2* pp = reinterpret_cast<uint2*>(kq + (half ? qoff : koff) + kb * 16384 +
                                               swz128((8 * w + j) * 128 + cbyte));
          const uint2 v = *pp;
          const float inv = rsqrtf(ss[half][j] + L2_EPS);
          *pp = make_uint2(pack_bf16(bf_lo(v.x) * inv, bf_hi(v.x) * inv),
                           pack_bf16(bf_lo(v.y) * inv, bf_hi(v.y) * inv));
        }
      __syncwarp();
    }

    // ---- range guard: max over channels of G_0 - G_63
    bool bad = false;
#pragma unroll
    for (int k = 0; k < 4; ++k) bad |= (grow[c0 + k] - grow[128 + c0 + k]) > GUARD_LOG2;
    const bool exact = named_bar_or(BAR_PA, PA_THREADS, bad);

    float gc[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) gc[k] = grow[128 + c0 + k];

    if (!exact) {
      ok = (c < 2) || wait_b(x, B_CKFREE + (c & 1), ((c - 2) >> 1) & 1);
      // ---- factored tiles: Rk = K E, Rq = Q E in place, Ck = K F
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int r = 8 * w + j;
        const bool valid = r < L;
        uint2* kp = reinterpret_cast<uint2*>(kq + koff + kb * 16384 + swz128(r * 128 + cbyte));
        uint2* qp = reinterpret_cast<uint2*>(kq + qoff + kb * 16384 + swz128(r * 128 + cbyte));
        const uint2 kr = valid ? *kp : make_uint2(0u, 0u);
        const uint2 qv = valid ? *qp : make_uint2(0u, 0u);
        float e[4], f[4];
        if (SG) {   // one factor per row
          e[0] = ex2f(g2[j][0] - gc[0]);
          f[0] = rcpf(e[0]);
#pragma unroll
          for (int k = 1; k < 4; ++k) {
            e[k] = e[0];
            f[k] = f[0];
          }
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            e[k] = ex2f(g2[j][k] - gc[k]);
            f[k] = rcpf(e[k]);
          }
        }
        const uint32_t e01 = pack_bf16(e[0], e[1]), e23 = pack_bf16(e[2], e[3]);
        *kp = make_uint2(mul_bf16x2(kr.x, e01), mul_bf16x2(kr.y, e23));
        *qp = make_uint2(mul_bf16x2(qv.x, e01), mul_bf16x2(qv.y, e23));
        if (ok)
          *reinterpret_cast<uint2*>(ck + kb * 8192 + swz128(r * 128 + cbyte)) =
              make_uint2(mul_bf16x2(kr.x, pack_bf16(f[0], f[1])),
                         mul_bf16x2(kr.y, pack_bf16(f[2], f[3])));
      }
    } else {
      ok = prep_a_exact(x, p.log_alpha, p.decay_pre, MODE, c, L, kq, koff, qoff, ck, betas);
      if (!ok) break;
    }
    // per-channel scalars and the path flag of this chunk
    if (w == 0) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float egc = ex2f(gc[k]);
        scal[c0 + k] = egc;                        // decay of the state over the chunk
        scal[128 + c0 + k] = exact ? 1.f : egc;    // scale of the state operand
      }
      if (lane == 0) xflag[s3] = exact ? 1 : 0;
    }
    fence_proxy_async_smem();
    if (named_bar_or(BAR_PA, PA_THREADS, !ok)) break;
    if (tid == 0) {
      mbar_arrive(&x.bars[B_TILES + (c & 1)]);
      // the Gram product of this chunk, once prep B has read out the previous one. An
      // MMA issue holds the issuing thread until the product starts; prep A, ahead of
      // prep B, has the slack for that, prep B does not.
      if (c == 0 || wait_b(x, B_GFREE, (c - 1) & 1)) issue_gram(x, c);
    }
  }
  if (tid == 0) drain(x, B_FIN_A);
}

// ============================================================================
// prep B (warps 8-11): Gram readout, UT solve, T*beta tile (prep B issues no tensor-core
// product: an MMA issue holds the issuing thread until the product starts, and prep B's
// chain is the one that sets the pace)
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
// A finished block (a, b) of T, scaled by `scale`, into the bf16 T*beta tile (column i
// of T times beta_i), two columns per 32-bit store.
__device__ __forceinline__ void blk_store_tb(uint8_t* tt, int a, int b, const float (&acc)[2][4],
                                             float scale, const float* betas, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nh = 0; nh < 2; ++nh) {
    const int i = 16 * b + 8 * nh + 2 * t;
    const float b0 = scale * betas[i], b1 = scale * betas[i + 1];
    *reinterpret_cast<uint32_t*>(tt + swz128((16 * a + g) * 128 + i * 2)) =
        pack_bf16(acc[nh][0] * b0, acc[nh][1] * b1);
    *reinterpret_cast<uint32_t*>(tt + swz128((16 * a + g + 8) * 128 + i * 2)) =
        pack_bf16(acc[nh][2] * b0, acc[nh][3] * b1);
  }
}

template <bool SPLIT, int MODE>
__device__ void prep_b_role(const Ctx& x, const CUtensorMap* map_k, const CUtensorMap* map_q,
                            const CUtensorMap* map_la) {
  constexpr bool SG = MODE == MODE_GDN;
  const int tid = threadIdx.x - PB_WARP0 * 32;
  const int q = tid >> 5, lane = tid & 31;   // q = warp within the group = TMEM lane quarter
  const uint32_t lane_base = (uint32_t)(32 * q) << 16;
  float* aw = reinterpret_cast<float*>(x.sm + OFF_AW);
  float* scr = reinterpret_cast<float*>(x.sm + OFF_SCR) + q * 256;
  const int* xflag = reinterpret_cast<const int*>(x.sm + OFF_XFLAG);
  auto A = [&](int a, int b) { return aw + (16 * a) * AW + 16 * b; };
  uint8_t* tt = x.sm + OFF_TB;
  // (thread 0) the k/q loads of the CTA: each goes out once its stage slot is free
  // (the [O | Delta] product of the chunk three back done), and prefetches the
  // log-decay of the chunk three later into L2. At the start of chunk c, the loads up
  // to chunk c+1 are waited for (prep A needs them next) and chunk c+2's goes out if
  // its slot is already free (one call site per chunk: see the code-size note).
  const int xk = x.h * D;
  int kq_issued = 0;
  auto push_kq = [&](int upto, int block_upto) {
    while (kq_issued < x.n_chunks && kq_issued <= upto) {
      const int cn = kq_issued;
      if (cn >= 3) {
        uint64_t* fb = &x.bars[B_KQFREE + cn % 3];
        const uint32_t par = ((cn - 3) / 3) & 1;
        if (cn <= block_upto ? !wait_b(x, B_KQFREE + cn % 3, par) : !mbar_test_wait(fb, par)) return;
      }
      issue_kq(x, map_k, map_q, cn);
      // (a scalar gate is prefetched by prep A itself)
      if (!SG && cn + 3 < x.n_chunks)
        tma_prefetch_2d(map_la, xk, (int)(x.bos + (int64_t)(cn + 3) * CHUNK));
      ++kq_issued;
    }
  };
  if (tid == 0) {
    for (int c = 0; c < 3 && c < x.n_chunks && !SG; ++c)
      tma_prefetch_2d(map_la, xk, (int)(x.bos + (int64_t)c * CHUNK));
    push_kq(2, -1);
  }
  // blocks above the diagonal of the T*beta tile stay zero for the whole kernel
  for (int i = tid; i < 512; i += PB_THREADS)
    *reinterpret_cast<uint4*>(tt + i * 16) = make_uint4(0u, 0u, 0u, 0u);

  for (int c = 0; c < x.n_chunks; ++c) {
    const int s3 = c % 3;
    uint8_t* ck = x.sm + OFF_CKP + (c & 1) * CKP_BYTES;
    const float* betas = reinterpret_cast<const float*>(x.sm + OFF_BETA) + s3 * 64;

    if (tid == 0) push_kq(c + 2, c + 1);
    bool ok = wait_b(x, B_TILES + (c & 1), (c >> 1) & 1);
    const bool exact = ok && xflag[s3] != 0;
    // ---- Gram readout: A rows (beta-scaled, strictly lower) -> fp32 workspace; P -> bf16 tile.
    //      Lanes of the k half hold A, lanes of the q half hold P.
    ok = ok && wait_b(x, B_GRAM, c & 1);
    if (ok && !exact) {
      tc_fence_after();
      const bool a_rows = (q < 2) == ((c & 1) == 0);
      const int r = 32 * (q & 1) + lane;
      // A strictly below the diagonal and scaled by beta_r, P with its diagonal
      const float sc = a_rows ? betas[r] : 1.f;
      const int lim = a_rows ? r : r + 1;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        const int col0 = 32 * half;
        float v[32];
        tmem_ld32(x.tmem + TM_G + lane_base + col0, v);
        tmem_ld_wait();
#pragma unroll
        for (int m = 0; m < 32; ++m) v[m] = (col0 + m < lim) ? sc * v[m] : 0.f;
        if (a_rows) {
#pragma unroll
          for (int m = 0; m < 32; m += 4)
            *reinterpret_cast<float4*>(&aw[r * AW + col0 + m]) = make_float4(v[m], v[m + 1], v[m + 2], v[m + 3]);
        } else {
          uint8_t* pt = ck + 16384;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch)
            *reinterpret_cast<uint4*>(pt + swz128(r * 128 + col0 * 2 + ch * 16)) = pack8(&v[8 * ch]);
        }
      }
      tc_fence_before();
    }
    // the previous chunk's U and W' products must be done reading the T*beta tile (each
    // has its own commit)
    ok = ok && ((c < 1) || (wait_b(x, B_UDONE, (c - 1) & 1) && wait_b(x, B_WDONE, (c - 1) & 1)));
    if (named_bar_or(BAR_PB, PB_THREADS, !ok)) break;
    // the Gram columns are free again: prep A's thread may issue the next Gram
    if (tid == 0) mbar_arrive(&x.bars[B_GFREE]);

    // ---- UT transform: T = (I + A)^{-1}. 16x16 diagonal blocks by forward substitution:
    //      lane j of warp a keeps column j of T_aa in registers (the A values are
    //      independent of it, so their loads pipeline), then the block replaces A_aa
    //      and its T*beta entries go to the tile.
    if (lane < 16) {
      const int j = lane;
      float* Ab = A(q, q);
      float t[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float a[16];
#pragma unroll
        for (int i4 = 0; i4 < r; i4 += 4) {   // row r of A_qq (the pitch keeps rows 16-byte aligned)
          const float4 a4 = *reinterpret_cast<const float4*>(&Ab[r * AW + i4]);
          a[i4] = a4.x; a[i4 + 1] = a4.y; a[i4 + 2] = a4.z; a[i4 + 3] = a4.w;
        }
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int i = 0; i + 1 < r; i += 2) {
          s0 = fmaf(a[i], t[i], s0);
          s1 = fmaf(a[i + 1], t[i + 1], s1);
        }
        if (r & 1) s0 = fmaf(a[r - 1], t[r - 1], s0);
        t[r] = (r == j ? 1.f : 0.f) - (s0 + s1);
      }
      __syncwarp(0x0000ffffu);
      const float bj = betas[16 * q + j];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        Ab[r * AW + j] = t[r];
        *reinterpret_cast<__nv_bfloat16*>(tt + swz128((16 * q + r) * 128 + (16 * q + j) * 2)) =
            __float2bfloat16_rn(t[r] * bj);
      }
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
      float* T31p = xs + 1280;
      // (warp-uniform branches on q; blocks addressed at run time, strides fixed, so
      //  that the four warps share code instead of running four copies of it)
      {                    // T_10 = -T_11 (A_10 T_00), T_32 = -T_33 (A_32 T_22); X21, X31
        const int r1 = q == 0 ? 1 : (q == 2 ? 2 : 3), s1 = q == 0 ? 0 : (q == 1 ? 2 : 1);
        float acc[2][4] = {};
        blk_mma(acc, A(r1, s1), AW, A(s1, s1), AW, lane);
        blk_store(q < 2 ? scr : (q == 2 ? X21 : X31), 16, acc, 1.f, lane);
        if (q < 2) {
          __syncwarp();
          const int rr = q == 0 ? 1 : 3, ss = rr - 1;
          float acc2[2][4] = {};
          blk_mma(acc2, A(rr, rr), AW, scr, 16, lane);
          blk_store(A(rr, ss), AW, acc2, -1.f, lane);
          blk_store_tb(tt, rr, ss, acc2, -1.f, betas, lane);
        }
      }
      named_bar_sync(BAR_PB, PB_THREADS);
      if (q < 2) {         // X20 = A_20 T_00 + A_21 T_10, X30 = A_30 T_00 + A_31 T_10
        const int r = q + 2;
        float acc[2][4] = {};
        blk_mma(acc, A(r, 0), AW, A(0, 0), AW, lane);
        blk_mma(acc, A(r, 1), AW, A(1, 0), AW, lane);
        blk_store(q == 0 ? X20 : X30, 16, acc, 1.f, lane);
      } else {             // T_21 = -T_22 X21; the partial T_33 X31 of T_31
        const int r = q;
        float acc[2][4] = {};
        blk_mma(acc, A(r, r), AW, q == 2 ? X21 : X31, 16, lane);
        if (q == 2)
          blk_store_tb(tt, 2, 1, acc, -1.f, betas, lane);
        else
          blk_store(T31p, 16, acc, 1.f, lane);
      }
      named_bar_sync(BAR_PB, PB_THREADS);
      if (q < 3) {         // T_20 = -T_22 X20, T_30 = -(T_32 X20 + T_33 X30), T_31 = -(T_32 X21 + T_33 X31)
        const int r = q == 0 ? 2 : 3;
        float acc[2][4] = {};
        blk_mma(acc, A(r, 2), AW, q == 2 ? X21 : X20, 16, lane);
        if (q == 1) blk_mma(acc, A(3, 3), AW, X30, 16, lane);
        if (q == 2) {
          const int g = lane >> 2, t = lane & 3;
#pragma unroll
          for (int nh = 0; nh < 2; ++nh) {
            acc[nh][0] += T31p[g * 16 + 8 * nh + 2 * t];
            acc[nh][1] += T31p[g * 16 + 8 * nh + 2 * t + 1];
            acc[nh][2] += T31p[(g + 8) * 16 + 8 * nh + 2 * t];
            acc[nh][3] += T31p[(g + 8) * 16 + 8 * nh + 2 * t + 1];
          }
        }
        blk_store_tb(tt, r, q == 2 ? 1 : 0, acc, -1.f, betas, lane);
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(BAR_PB, PB_THREADS);
    if (tid == 0) {
      // (a test may leave one arrive out: the state warps' wait for it then runs out)
      if (c != *reinterpret_cast<const int*>(x.sm + OFF_MISC + MISC_SKIP_TB)) mbar_arrive(&x.bars[B_TB]);
      mbar_arrive(&x.bars[B_WFREE]);   // done with this chunk: the workspace is free
    }
  }
  if (tid == 0) {
    drain(x, B_FIN_P);
    // never leave with copies in flight: the last load into each slot has landed (an
    // earlier one into the same slot was consumed before that load went out)
    for (int cn = (kq_issued > 3 ? kq_issued - 3 : 0); cn < kq_issued; ++cn)
      settle(&x.bars[B_FULL + cn % 3], (cn / 3) & 1);
  }
}

// ---- the state warps' entering and final state, once per CTA. Thread = TMEM lane j of
//      its warp's quarter (lane_addr), 64 channels starting at cb. (Inline: a call out of
//      the state warps' code costs more code around it, saving and restoring registers,
//      than the helper itself.)

// the entering state (h0, the identity, or zeros) into the fp32 master, [channel][value]
__device__ __forceinline__ void st_load_state(uint32_t lane_addr, const float* h0, bool identity, int j,
                                           int cb) {
#pragma unroll 1
  for (int part = 0; part < 2; ++part) {
    const int cb0 = cb + 32 * part;
    uint32_t r[32];
#pragma unroll
    for (int i = 0; i < 32; ++i)
      r[i] = h0 ? __float_as_uint(__ldg(h0 + (size_t)(cb0 + i) * D + j))
                : (identity && cb0 + i == j ? 0x3F800000u : 0u);
    tmem_st32(lane_addr + cb0, r);
  }
  tmem_st_wait();
}
// the final state out of the fp32 master (plus base, if not null)
__device__ __forceinline__ void st_store_state(uint32_t lane_addr, float* hT, const float* base, int j,
                                            int cb) {
#pragma unroll 1
  for (int part = 0; part < 2; ++part) {
    const int cb0 = cb + 32 * part;
    float v[32];
    tmem_ld32(lane_addr + cb0, v);
    tmem_ld_wait();
    if (base) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] += __ldg(base + (size_t)(cb0 + i) * D + j);
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) hT[(size_t)(cb0 + i) * D + j] = v[i];
  }
}
// The valid rows (< L) of the staged output tile ([64 rows][128 columns] bf16 in two
// 64-column halves of 8 KB, 128B-swizzled rows) to o at orow (the chunk's first row,
// the head's first column). 16 bytes (8 columns) per step, all state threads.
__device__ __forceinline__ void tile_rows_out(const uint8_t* dt, __nv_bfloat16* orow, size_t rs, int L,
                                              int tid) {
#pragma unroll 1
  for (int i = tid; i < L * 16; i += ST_THREADS) {
    const int r = i >> 4, seg = i & 15;
    *reinterpret_cast<uint4*>(orow + (size_t)r * rs + 8 * seg) =
        *reinterpret_cast<const uint4*>(dt + (seg >> 3) * 8192 + swz128(r * 128 + (seg & 7) * 16));
  }
}

// ============================================================================
// state warps (12-19): the sequential pass over chunks. Thread = (TMEM lane j =
// value column, half hh of the key channels / of the chunk rows).
// ============================================================================
// (fused output) 8 bf16 outputs of one row times the row's inverse RMS, the norm
// weight and the sigmoid of the gate pre-activation
__device__ __forceinline__ uint4 gate_row8(uint4 o8, uint4 g8, const float* w8, float inv) {
  const uint32_t ov[4] = {o8.x, o8.y, o8.z, o8.w}, gv[4] = {g8.x, g8.y, g8.z, g8.w};
  uint32_t r[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = bf_lo(ov[i]) * inv * w8[2 * i] * sigmoidf_fast(bf_lo(gv[i]));
    const float b = bf_hi(ov[i]) * inv * w8[2 * i + 1] * sigmoidf_fast(bf_hi(gv[i]));
    r[i] = pack_bf16(a, b);
  }
  return make_uint4(r[0], r[1], r[2], r[3]);
}

template <bool SPLIT, int MODE>
__device__ void state_role(const Ctx& x, const Args& p, const CUtensorMap* map_v,
                           const CUtensorMap* map_o) {
  constexpr bool FU = MODE == MODE_FUSED;
  const int tid = threadIdx.x - ST_WARP0 * 32;
  const int sw = tid >> 5, lane = tid & 31;
  const int qd = sw & 3, hh = sw >> 2;
  const int j = 32 * qd + lane;
  const uint32_t lb = (uint32_t)(32 * qd) << 16;
  const float* scal_all = reinterpret_cast<const float*>(x.sm + OFF_SCAL);
  const int* xflag = reinterpret_cast<const int*>(x.sm + OFF_XFLAG);
  uint8_t* dt = x.sm + OFF_DT;
  const int n = x.n_chunks;

  // ---- prologue: the fp32 state (h0, identity or zeros) and cleared output accumulators
  float* rowsq = reinterpret_cast<float*>(x.sm + OFF_ROWSQ);
  float* normw = reinterpret_cast<float*>(x.sm + OFF_NORMW);
  if (FU && tid < D) normw[tid] = __ldg(p.norm_w + tid);
  st_load_state(x.tmem + TM_S + lb, x.h0, SPLIT && x.h0_identity, j, 64 * hh);
  tmem_st32_zero(x.tmem + TM_OA + lb + 32 * hh);
  tmem_st32_zero(x.tmem + TM_OB + lb + 32 * hh);
  tmem_st_wait();
  if (SPLIT && x.v_zero) {   // a zero v tile for every chunk (U = 0)
    for (int i = tid; i < 1024; i += ST_THREADS)
      *reinterpret_cast<uint4*>(x.sm + OFF_V + i * 16) = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }

  // decay the state over chunk cc in place and write the bf16 operand S''; returns
  // whether any of this thread's state entries was nonzero (only computed for a
  // transition chain, which stops once its state is exactly zero)
  auto s_pass = [&](int cc) -> bool {
    const float* ms = scal_all + (cc % 3) * 256;
    const bool ex = xflag[cc % 3] != 0;
    uint32_t nz = 0u;
#pragma unroll 1
    for (int part = 0; part < 2; ++part) {
      const int cb0 = 64 * hh + 32 * part;
      float v[32];
      tmem_ld32(x.tmem + TM_S + lb + cb0, v);
      tmem_ld_wait();
      if (SPLIT && x.stop_on_zero) {
#pragma unroll
        for (int i = 0; i < 32; ++i) nz |= __float_as_uint(v[i]) & 0x7FFFFFFFu;
      }
      uint32_t pk[16];
      if (ex) {   // exact path: the operand is the undecayed state
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(v[2 * i], v[2 * i + 1]);
      }
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const float4 m4 = *reinterpret_cast<const float4*>(ms + cb0 + i);
        v[i] *= m4.x; v[i + 1] *= m4.y; v[i + 2] *= m4.z; v[i + 3] *= m4.w;
      }
      if (!ex) {
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(v[2 * i], v[2 * i + 1]);
      }
      tmem_st32(x.tmem + TM_S + lb + cb0, reinterpret_cast<const uint32_t(&)[32]>(v));
      tmem_st16(x.tmem + TM_SB + lb + cb0 / 2, pk);
    }
    tmem_st_wait();
    tc_fence_before();
    return nz != 0u;
  };

  // Thread 0 issues this group's tensor-core products and the v loads. Per chunk:
  // W' (as soon as T*beta is there, at the latest right before its readout), U (once
  // v is there too), the [O | Delta] product, then the state update and P Delta once
  // Delta is back in TMEM; the next chunk's v load goes out once the current U
  // product is done (it precedes [O | Delta] in the pipe). W' used to be issued by
  // prep B: an MMA issue holds the issuing thread until the product starts, and
  // prep B's chain is the one that sets the pace.
  const bool issuer = tid == 0;
  int u_issued = 0, v_issued = 0, v_landed = 0;
  // W' of chunk cw (from T*beta; the previous W' was read out before the previous
  // [O | Delta] product, by these warps)
  int w_issued = 0;
  auto issue_w_of = [&](int cw, bool block) -> bool {
    if (block) {
      if (!wait_b(x, B_TB, cw & 1)) return false;
    } else if (!mbar_test_wait(&x.bars[B_TB], cw & 1)) {
      return true;   // not ready yet: issued later, before its readout
    }
    issue_w(x, cw);
    w_issued = cw + 1;
    return true;
  };
  auto issue_u_of = [&](int cu, bool block) -> bool {
    if (block) {
      if (!wait_b(x, B_TB, cu & 1) || !wait_b(x, B_VFULL, cu & 1)) return false;
    } else if (!mbar_test_wait(&x.bars[B_TB], cu & 1) || !mbar_test_wait(&x.bars[B_VFULL], cu & 1)) {
      return true;   // not ready yet: issued later, before the chunk's [O | Delta] product
    }
    v_landed = cu + 1;
    issue_u(x);
    u_issued = cu + 1;
    return true;
  };

  // -W' of chunk cc (TMEM, lane j = key channel, columns = rows) -> the k half of the
  // chunk's stage tile, rows 32hh..32hh+31: the B operand of the [O | Delta] product
  auto w_readout = [&](int cc) -> bool {
    if (!wait_b(x, B_WDONE, cc & 1)) return false;
    tc_fence_after();
    tmem_block_to_tile_t(x.tmem + TM_W + lb + 32 * hh, 32 * qd, 32 * hh,
                         x.sm + OFF_KQ + (cc % 3) * KQ_BYTES + ((cc & 1) ? 8192 : 0), 16384u, lane);
    fence_proxy_async_smem();
    tc_fence_before();
    return true;
  };

  // output: the fused epilogue (RMSNorm and gate) where the output is final, else the
  // plain one in the CTA's mode
  const bool fu_out = FU && (!SPLIT || x.gated);
  const int omode = SPLIT ? x.out_mode : OUT_STORE;
  bool alive = true;
  bool stopped = false;   // a v = 0 chain that stopped early (state exactly zero)
  if (issuer && n > 0) {
    issue_v<SPLIT>(x, map_v, 0);
    v_issued = 1;
  }
  // One pass of the loop per chunk c, plus one to finish the last output. Each step
  // appears once in the code: the roles' code shares the SM's instruction caches.
  //   (a) chunk c's decayed state S'' (once the update of chunk c-1 has landed), its
  //       -W' tile and the [O | Delta] product;
  //   (b) the output of chunk c-1, off the sequential path;
  //   (c) Delta of chunk c back into TMEM as bf16 pairs, then the state update.
  for (int c = 0; c <= n; ++c) {
    bool stop_now = false;
    if (c == n && c > 1) {
      // the last output reuses the output tile: the previous chunk's store must have
      // read it (for earlier chunks the wait in (a) covers this)
      if (issuer) bulk_wait_read_all();
      named_bar_sync(BAR_ST, ST_THREADS);
    }
    if (c < n) {
      alive = alive && (c == 0 || wait_b(x, B_ZDONE, (c - 1) & 1)) &&
              wait_b(x, B_TILES + (c & 1), (c >> 1) & 1);
      bool nonzero = true;
      if (alive) {
        tc_fence_after();
        nonzero = s_pass(c);
      }
      if (issuer && alive && w_issued < c + 1) alive = issue_w_of(c, true);
      alive = alive && w_readout(c);
      // (the output tile's last store must have read it before (b) stages the next)
      if (issuer && c > 1) bulk_wait_read_all();
      if (SPLIT && x.stop_on_zero && c > 0) {
        // A v = 0 chain whose state is exactly zero after chunk c-1 stays zero (every
        // later Delta, update and output is zero too): its final state is known, and
        // the CTA stops once the output of chunk c-1 is out. The other roles then
        // see ABORT_DONE at their next wait and leave; the update of chunk c-1 has
        // landed.
        if (!named_bar_or(BAR_ST, ST_THREADS, nonzero || !alive)) {
          stopped = true;
          stop_now = true;
        }
      } else {
        named_bar_sync(BAR_ST, ST_THREADS);
      }
      if (issuer && alive && !stop_now) {
        if (u_issued < c + 1) alive = issue_u_of(c, true);
        if (alive) issue_crit(x, c);
      }
    }
    if (fu_out && c > 0) {
      // ---- fused output of chunk c-1: RMSNorm over each row's 128 values, times the
      //      weight and the sigmoid gate. (i) every warp stages its 32 x 32 block as
      //      bf16 and leaves the fp32 row sums of squares; (ii) after the group's
      //      barrier each thread finishes 32 values of one row from the staged tile.
      const int co = c - 1;
      const int64_t t0 = x.bos + (int64_t)co * CHUNK;
      const int L = (x.eos - t0) < CHUNK ? (int)(x.eos - t0) : CHUNK;
      {   // the gate rows of the next chunk into L2
        const int64_t tn = t0 + CHUNK + (tid >> 2);
        if (tn < x.eos) prefetch_l2(p.gate_pre + (size_t)tn * x.rs + x.h * D + 32 * (tid & 3));
      }
      // this thread's 32 gate values of the chunk (row rr, channels 32 cq ..), in flight
      // while the block is staged
      const int rr = tid >> 2, cq = tid & 3;
      uint4 g8[4];
      {
        const __nv_bfloat16* gp = p.gate_pre + (size_t)(t0 + rr) * x.rs + x.h * D + 32 * cq;
#pragma unroll
        for (int sg = 0; sg < 4; ++sg)
          g8[sg] = rr < L ? ldg_nc_u4(gp + 8 * sg) : make_uint4(0u, 0u, 0u, 0u);
      }
      alive = alive && wait_b(x, B_PD, co & 1);
      if (alive) {
        tc_fence_after();
        const uint32_t ro = (co & 1) ? TM_OA : TM_OB;
        tmem_block_to_tile_t_rowsq(x.tmem + ro + lb + 32 * hh, 32 * qd, 32 * hh, dt, 8192u, lane,
                                   rowsq, qd);
        tmem_st32_zero(x.tmem + ro + lb + 32 * hh);
        tmem_st_wait();
        tc_fence_before();
      }
      named_bar_sync(BAR_OUT, ST_THREADS);
      if (alive && rr < L) {
        const float4 sq = *reinterpret_cast<const float4*>(rowsq + rr * 4);
        const float inv = rsqrtf((sq.x + sq.y + sq.z + sq.w) * (1.f / D) + RMS_EPS);
#pragma unroll
        for (int sg = 0; sg < 4; ++sg) {
          const int c8 = 32 * cq + 8 * sg;
          uint4* tp = reinterpret_cast<uint4*>(dt + (c8 >> 6) * 8192 +
                                               swz128((uint32_t)rr * 128u + (uint32_t)(c8 & 63) * 2u));
          const uint4 r8 = gate_row8(*tp, g8[sg], normw + c8, inv);
          if (L == CHUNK)
            *tp = r8;
          else   // ragged last chunk of a sequence: the valid rows go straight out
            *reinterpret_cast<uint4*>(p.o + (size_t)(t0 + rr) * x.rs + x.h * D + c8) = r8;
        }
        fence_proxy_async_smem();
      }
      named_bar_sync(BAR_OUT, ST_THREADS);
      if (issuer && alive && L == CHUNK) {
        tma_store_2d(map_o, dt, x.h * D, (int)t0);
        tma_store_2d(map_o, dt + 8192, x.h * D + 64, (int)t0);
        bulk_commit_group();
      }
    }
    if (!fu_out && c > 0) {
      const int co = c - 1;
      const int64_t t0 = x.bos + (int64_t)co * CHUNK;
      const int L = (x.eos - t0) < CHUNK ? (int)(x.eos - t0) : CHUNK;
      // The output goes through the output tile (its previous store has read it): a full
      // chunk to be stored leaves by one TMA store of [64 rows][128 columns], a correction
      // by one TMA reduce-add (its chunks are whole but for the very last of the tensor,
      // whose rows past the end the copy clips), and a ragged last chunk of a sequence by a
      // short loop over its valid rows.
      const bool staged = omode != OUT_NONE;
      const bool tile_out = (omode == OUT_STORE && L == CHUNK) || omode == OUT_ADD;
      alive = alive && wait_b(x, B_PD, co & 1);
      if (alive) {
        tc_fence_after();
        const uint32_t ro = (co & 1) ? TM_OA : TM_OB;
        if (staged) {
          tmem_block_to_tile_t(x.tmem + ro + lb + 32 * hh, 32 * qd, 32 * hh, dt, 8192u, lane);
          if (tile_out) fence_proxy_async_smem();
        }
        tmem_st32_zero(x.tmem + ro + lb + 32 * hh);
        tmem_st_wait();
        tc_fence_before();
      }
      if (staged && !tile_out) {
        named_bar_sync(BAR_OUT, ST_THREADS);
        if (alive) tile_rows_out(dt, p.o + (size_t)t0 * x.rs + x.h * D, x.rs, L, tid);
        named_bar_sync(BAR_OUT, ST_THREADS);   // (before the tile is staged again)
      }
      if (tile_out) {
        // the warps that do not issue only report their part staged and go on; the
        // issuing warp waits for all parts and sends the tile
        if (sw != 0) {
          named_bar_arrive(BAR_OUT, ST_THREADS);
        } else {
          named_bar_sync(BAR_OUT, ST_THREADS);
          if (issuer && alive) {
            if (omode == OUT_ADD) {
              tma_reduce_add_2d(map_o, dt, x.h * D, (int)t0);
              tma_reduce_add_2d(map_o, dt + 8192, x.h * D + 64, (int)t0);
            } else {
              tma_store_2d(map_o, dt, x.h * D, (int)t0);
              tma_store_2d(map_o, dt + 8192, x.h * D + 64, (int)t0);
            }
            bulk_commit_group();
          }
        }
      }
    }
    if (stop_now) {
      if (tid == 0) *x.abort_flag = ABORT_DONE;
      break;
    }
    if (c < n) {
      // ---- Delta^T fp32 (TMEM, chunk rows 32hh..32hh+31 of lane j) -> bf16 pairs in the
      //      same lanes, inside the columns just read: the A operand of the update
      alive = alive && wait_b(x, B_CRIT, c & 1);
      if (alive) {
        tc_fence_after();
        float v[32];
        tmem_ld32(x.tmem + TM_D + lb + 32 * hh, v);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(v[2 * i], v[2 * i + 1]);
        tmem_st16(x.tmem + TM_D + lb + 48 * hh, pk);
        tmem_st_wait();
        tc_fence_before();
        if (issuer && c + 1 < n) {   // U(c) is done: v of the next chunk may land
          issue_v<SPLIT>(x, map_v, c + 1);
          v_issued = c + 2;
        }
      }
      named_bar_sync(BAR_ST, ST_THREADS);
      if (issuer && alive) {
        issue_update(x, c);
        if (c + 1 < n) {
          alive = issue_w_of(c + 1, false);
          if (alive && w_issued == c + 2) alive = issue_u_of(c + 1, false);
        }
      }
    }
  }
  // ---- final state (after an early stop: the zero state, whose last update has landed)
  if (n > 0 && !stopped) alive = alive && wait_b(x, B_ZDONE, (n - 1) & 1);
  tc_fence_after();
  if (x.hT && alive && *x.abort_flag != ABORT_TIMEOUT)
    st_store_state(x.tmem + TM_S + lb, x.hT, SPLIT ? x.hT_base : nullptr, j, 64 * hh);
  if (issuer) {
    bulk_wait_all();
    drain(x, B_FIN_C);
    for (int c = v_landed; c < v_issued; ++c) settle(&x.bars[B_VFULL], c & 1);
  }
}

// ============================================================================
// kernel: one CTA per (sequence, head), or per (segment, head) of a time split.
// MODE (see the MODE_ constants): MODE_GDN reads one scalar gate per token and head and
// prep A evaluates each row's factor once; MODE_FUSED applies the producing layer's
// activations in prep A and the output's RMSNorm and gate in the state warps'
// epilogue. The chunk algebra in between is the same for all three.
// ============================================================================
template <bool SPLIT, int MODE>
__global__ void __launch_bounds__(THREADS, 1)
kda_chunk_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_la,
                    const __grid_constant__ CUtensorMap map_o, const Args args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Ctx x;
  x.sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  x.bars = reinterpret_cast<uint64_t*>(x.sm + OFF_BAR);
  x.abort_flag = reinterpret_cast<volatile int*>(x.sm + OFF_MISC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(x.sm + OFF_MISC + MISC_TMEM);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = args.n_heads;
  const int slot = blockIdx.x / H;
  x.h = blockIdx.x % H;
  x.rs = (size_t)H * D;
  x.h0_identity = false;
  x.hT_base = nullptr;
  x.v_zero = false;
  x.out_mode = OUT_STORE;
  x.stop_on_zero = false;
  x.gated = true;
  const size_t state_elems = (size_t)D * D;
  if (args.plan == PLAN_SEQ) {
    // CTAs start in index order; with seq_order the longest sequences go first, so
    // the last wave holds short ones
    int n = slot;
    if (args.seq_order) {
      const int o = args.seq_order[slot];
      n = (o >= 0 && o < args.n_seqs) ? o : slot;
    }
    seq_bounds(args.cu_seqlens, n, args.n_seqs, args.t_total, x.bos, x.eos);
    const size_t sidx = ((size_t)n * H + x.h) * state_elems;
    x.h0 = args.h0 ? args.h0 + sidx : nullptr;
    x.hT = args.hT ? args.hT + sidx : nullptr;
  } else {
    const int ns = args.n_seg;
    auto state_slot = [&](int s) { return args.seg_states + ((size_t)s * H + x.h) * state_elems; };
    int seg;
    if (args.plan == PLAN_ZERO) {
      if (slot < ns) {                  // Z_j, j = slot
        seg = slot;
        x.h0 = (seg == 0 && args.h0) ? args.h0 + (size_t)x.h * state_elems : nullptr;
        x.hT = state_slot(seg == ns - 1 ? 2 * ns - 3 : seg);
        x.gated = seg == 0;   // (the others' outputs take their corrections first)
      } else {                          // M_j, j = slot - n + 1
        seg = slot - ns + 1;
        x.gated = false;
        x.out_mode = OUT_NONE;
        x.h0 = nullptr;
        x.h0_identity = true;
        x.v_zero = true;
        x.stop_on_zero = true;
        x.hT = state_slot(ns - 2 + seg);
      }
    } else {                            // PLAN_CORR
      seg = slot + 1;
      x.h0 = state_slot(seg - 1);
      x.gated = false;
      x.v_zero = true;
      x.stop_on_zero = true;
      x.out_mode = OUT_ADD;
      if (seg == ns - 1 && args.hT) {
        x.hT = args.hT + (size_t)x.h * state_elems;
        x.hT_base = state_slot(2 * ns - 3);
      } else {
        x.hT = nullptr;
      }
    }
    auto seg_start = [&](int j) { return seg::seg_first_chunk(j, args.seg_base, args.seg_rem) * CHUNK; };
    x.bos = seg_start(seg);
    x.eos = (seg == ns - 1) ? args.t_total : seg_start(seg + 1);
    if (x.bos > args.t_total) x.bos = args.t_total;
    if (x.eos > args.t_total) x.eos = args.t_total;
    if (x.eos < x.bos) x.eos = x.bos;
  }
  x.n_chunks = (int)((x.eos - x.bos + CHUNK - 1) / CHUNK);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NUM_BARS; ++i) mbar_init(&x.bars[i], 1);
    *x.abort_flag = 0;
    *reinterpret_cast<uint64_t*>(x.sm + OFF_MISC + MISC_WAIT_NS) = args.wait_ns ? args.wait_ns : WAIT_NS;
    *reinterpret_cast<int*>(x.sm + OFF_MISC + MISC_SKIP_TB) = args.debug_skip_tb;
    fence_mbar_init();
  }
  if (threadIdx.x == 0) {
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_q);
    if (MODE != MODE_GDN) prefetch_tensormap(&map_la);
  }
  if (warp == ST_WARP0) {
    if (lane == 0) {
      prefetch_tensormap(&map_v);
      prefetch_tensormap(&map_o);
    }
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  x.tmem = *tmem_slot;

  if (warp < PA_WARPS) {
    prep_a_role<SPLIT, MODE>(x, args);
  } else if (warp < ST_WARP0) {
    prep_b_role<SPLIT, MODE>(x, &map_k, &map_q, &map_la);
  } else {
    state_role<SPLIT, MODE>(x, args, &map_v, &map_o);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == ST_WARP0) {
    tc_fence_after();
    tmem_dealloc(x.tmem, TM_COLS);
  }
}

// ============================================================================
// The fused variant's output of tokens [t0, t1) in a time split (segments 1 .. n-1,
// whose raw outputs take their corrections first), in place, per (token, head) row of
// 128 values: o <- o / sqrt(mean(o^2) + RMS_EPS) * norm_w * sigmoid(gate_pre), the
// epilogue of the chunk kernel's gated CTAs. 16 threads per row, 16 bytes each; rows
// are [row0, row0 + rows) of the [T*H][128] view.
// ============================================================================
constexpr int NG_THREADS = 256;
constexpr int NG_ROWS = NG_THREADS / 16;   // rows per block and pass

__global__ void __launch_bounds__(NG_THREADS)
kda_norm_gate_kernel(__nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ gate_pre,
                     const float* __restrict__ norm_w, int64_t row0, int64_t rows) {
  const int sub = threadIdx.x & 15;
  const unsigned mask = 0xFFFFu << (threadIdx.x & 16);   // this row's 16 lanes
  float w8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) w8[i] = __ldg(norm_w + 8 * sub + i);
  const int64_t stride = (int64_t)gridDim.x * NG_ROWS;
  for (int64_t r = (int64_t)blockIdx.x * NG_ROWS + (threadIdx.x >> 4); r < rows; r += stride) {
    const size_t e = (size_t)(row0 + r) * D + 8 * sub;
    const uint4 o8 = *reinterpret_cast<const uint4*>(o + e);
    const uint4 g8 = ldg_nc_u4(gate_pre + e);
    const uint32_t ov[4] = {o8.x, o8.y, o8.z, o8.w};
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) ss += bf_lo(ov[i]) * bf_lo(ov[i]) + bf_hi(ov[i]) * bf_hi(ov[i]);
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) ss += __shfl_xor_sync(mask, ss, off);
    const float inv = rsqrtf(ss * (1.f / D) + RMS_EPS);
    *reinterpret_cast<uint4*>(o + e) = gate_row8(o8, g8, w8, inv);
  }
}

}  // namespace tc
}  // namespace kda
