// General DPLR chunkwise prefill on CUDA cores, fp32: the comparison point the pages
// hold KDA against (Rationalist Deep-Dive, section 3.2 "DPLR Structure"; Kimi Linear
// summary, section 3.2 "Efficiency Analysis" and section 6.2 "Relation to DPLR":
// KDA's tied factors reduce four secondary-chunk matrices to two).
//
//     S_t = (Diag(alpha_t) - a_t b_t^T) S_{t-1} + k_t v_t^T,   o_t = S_t^T q_t
//
// with free low-rank factors a, b. For a chunk of <= 64 rows entering with state S
// (G inclusive cumulative log decay per channel, G_{-1} = 0, correction rows
// u_r = b_r^T S_{r-1}), derived from the recurrence:
//   Mbk_ri = sum_c b_rc e^{G_{r-1,c} - G_ic} k_ic,  Mba_ri = ... a_ic      (i < r)
//   Mqk_ri = sum_c q_rc e^{G_rc - G_ic} k_ic,       Mqa_ri = ... a_ic      (i <= r)
//   (I + Mba) U = (B * e^{G_prev}) S + Mbk V
//   O = (Q * e^G) S + Mqk V - Mqa U
//   S <- Diag(e^{G_C}) S + (K * e^{G_C - G})^T V - (A * e^{G_C - G})^T U
// Four decayed Grams and three more products than the KDA kernel's chunk form.
//
// Written in the style of the exact KDA CUDA-core kernel (kda_chunk_simt.cuh), so the
// two time the two algorithms on the same footing: one CTA per (sequence, head,
// 32 value columns), exact pairwise decay factors, forward substitution for the
// triangular inverse, fp32 throughout. The 64 x 128 operand tiles do not all fit
// in shared memory at once here, so the Grams accumulate over two 64-channel halves
// and the state update reloads k, a and the decay (from L2).
#pragma once

#include "kda_common.cuh"

namespace kda {

constexpr int DPLR_THREADS = 256;
constexpr int DPLR_DV = 32;          // value columns per CTA
constexpr int DPLR_HC = 64;          // channels per half
constexpr int DPLR_LDH = DPLR_HC + 1;
constexpr int DPLR_LDA = CHUNK + 1;
constexpr int DPLR_LDV = DPLR_DV + 1;

struct DplrSmem {
  float K[CHUNK * DPLR_LDH];   // one channel half of k (then k e^{G_C - G} in the update)
  float Q[CHUNK * DPLR_LDH];   // q, then q e^G
  float A[CHUNK * DPLR_LDH];   // a (then a e^{G_C - G})
  float B[CHUNK * DPLR_LDH];   // b, then b e^{G_prev}
  float G[CHUNK * DPLR_LDH];   // log alpha, then G (inclusive cumsum)
  float Al[CHUNK * DPLR_LDH];  // alpha = e^{log alpha}
  float Mbk[CHUNK * DPLR_LDA];
  float Mba[CHUNK * DPLR_LDA];   // then T = (I + Mba)^{-1}
  float Mqk[CHUNK * DPLR_LDA];
  float Mqa[CHUNK * DPLR_LDA];
  float S[D * DPLR_LDV];
  float V[CHUNK * DPLR_LDV];
  float U[CHUNK * DPLR_LDV];
  float Xb[CHUNK * DPLR_LDV];   // (B e^{G_prev}) S, then + Mbk V
  float Xq[CHUNK * DPLR_LDV];   // (Q e^G) S
  float gC[DPLR_HC];
};

template <typename TQ>
__global__ void __launch_bounds__(DPLR_THREADS, 1)
kda_dplr_simt_kernel(const TQ* __restrict__ q, const TQ* __restrict__ k, const TQ* __restrict__ v,
                     const TQ* __restrict__ a, const TQ* __restrict__ b,
                     const float* __restrict__ log_alpha, const float* __restrict__ h0,
                     const int32_t* __restrict__ cu_seqlens, int n_seqs, int64_t t_total,
                     int n_heads, TQ* __restrict__ o, float* __restrict__ hT) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  DplrSmem& sm = *reinterpret_cast<DplrSmem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = blockIdx.x / n_heads, h = blockIdx.x % n_heads;
  const int j0 = blockIdx.y * DPLR_DV;
  int64_t bos, eos;
  seq_bounds(cu_seqlens, n, n_seqs, t_total, bos, eos);
  const size_t rs = (size_t)n_heads * D;
  const size_t sbase = ((size_t)n * n_heads + h) * D * D;
  for (int idx = tid; idx < D * DPLR_DV; idx += DPLR_THREADS) {
    const int c = idx / DPLR_DV, j = idx % DPLR_DV;
    sm.S[c * DPLR_LDV + j] = h0 ? h0[sbase + (size_t)c * D + j0 + j] : 0.f;
  }
  const int jj = tid % DPLR_DV, rb = tid / DPLR_DV;
  constexpr int STRIDE = DPLR_THREADS / DPLR_DV;   // 8 rows (or channels) apart

  for (int64_t t0 = bos; t0 < eos; t0 += CHUNK) {
    const int L = (eos - t0) < CHUNK ? (int)(eos - t0) : CHUNK;
    __syncthreads();
    for (int idx = tid; idx < CHUNK * DPLR_LDA; idx += DPLR_THREADS) {
      sm.Mbk[idx] = 0.f; sm.Mba[idx] = 0.f; sm.Mqk[idx] = 0.f; sm.Mqa[idx] = 0.f;
    }
    for (int idx = tid; idx < CHUNK * DPLR_DV; idx += DPLR_THREADS) {
      const int r = idx / DPLR_DV, j = idx % DPLR_DV;
      sm.V[r * DPLR_LDV + j] = r < L ? to_f32(v[(size_t)(t0 + r) * rs + (size_t)h * D + j0 + j]) : 0.f;
      sm.Xb[r * DPLR_LDV + j] = 0.f;
      sm.Xq[r * DPLR_LDV + j] = 0.f;
    }
    // ---- the Grams and the incoming-state terms, one channel half at a time
    for (int hc = 0; hc < 2; ++hc) {
      __syncthreads();
      for (int idx = tid; idx < CHUNK * DPLR_HC; idx += DPLR_THREADS) {
        const int r = idx / DPLR_HC, c = idx % DPLR_HC;
        float kv = 0.f, qv = 0.f, av = 0.f, bv = 0.f, lv = 0.f;
        if (r < L) {
          const size_t g = (size_t)(t0 + r) * rs + (size_t)h * D + DPLR_HC * hc + c;
          kv = to_f32(k[g]); qv = to_f32(q[g]); av = to_f32(a[g]); bv = to_f32(b[g]);
          lv = log_alpha[g];
        }
        const int e = r * DPLR_LDH + c;
        sm.K[e] = kv; sm.Q[e] = qv; sm.A[e] = av; sm.B[e] = bv; sm.G[e] = lv;
        sm.Al[e] = expf(lv);
      }
      __syncthreads();
      if (tid < DPLR_HC) {
        float acc = 0.f;
        for (int r = 0; r < CHUNK; ++r) {
          acc += sm.G[r * DPLR_LDH + tid];
          sm.G[r * DPLR_LDH + tid] = acc;
        }
      }
      __syncthreads();
      // warp w takes rows w, w+8, ...; lane i the columns i and 32+i
      for (int r = warp; r < CHUNK; r += STRIDE) {
        const float* Br = &sm.B[r * DPLR_LDH];
        const float* Qr = &sm.Q[r * DPLR_LDH];
        const float* Ar = &sm.Al[r * DPLR_LDH];
        const float* Gp = r > 0 ? &sm.G[(r - 1) * DPLR_LDH] : nullptr;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int i = 32 * half + lane;
          if (i > r) continue;
          const float* Ki = &sm.K[i * DPLR_LDH];
          const float* Ai = &sm.A[i * DPLR_LDH];
          const float* Gi = &sm.G[i * DPLR_LDH];
          float bk = 0.f, ba = 0.f, qk = 0.f, qa = 0.f;
          if (i < r) {
            for (int c = 0; c < DPLR_HC; ++c) {
              const float ep = expf(Gp[c] - Gi[c]);   // e^{G_{r-1} - G_i}
              const float ec = ep * Ar[c];            // e^{G_r - G_i}
              const float be = Br[c] * ep, qe = Qr[c] * ec;
              bk = fmaf(be, Ki[c], bk);
              ba = fmaf(be, Ai[c], ba);
              qk = fmaf(qe, Ki[c], qk);
              qa = fmaf(qe, Ai[c], qa);
            }
          } else {   // i == r: no decay between a row and itself
            for (int c = 0; c < DPLR_HC; ++c) {
              qk = fmaf(Qr[c], Ki[c], qk);
              qa = fmaf(Qr[c], Ai[c], qa);
            }
          }
          const int e = r * DPLR_LDA + i;
          sm.Mbk[e] += bk; sm.Mba[e] += ba; sm.Mqk[e] += qk; sm.Mqa[e] += qa;
        }
      }
      __syncthreads();
      // B <- B e^{G_prev}, Q <- Q e^G (G_prev of row 0 is 0)
      for (int idx = tid; idx < CHUNK * DPLR_HC; idx += DPLR_THREADS) {
        const int r = idx / DPLR_HC, c = idx % DPLR_HC;
        const int e = r * DPLR_LDH + c;
        sm.Q[e] *= expf(sm.G[e]);
        if (r > 0) sm.B[e] *= expf(sm.G[e - DPLR_LDH]);
      }
      __syncthreads();
      for (int m = 0; m < CHUNK / STRIDE; ++m) {
        const int r = rb + m * STRIDE;
        float xb = 0.f, xq = 0.f;
        for (int c = 0; c < DPLR_HC; ++c) {
          const float s = sm.S[(DPLR_HC * hc + c) * DPLR_LDV + jj];
          xb = fmaf(sm.B[r * DPLR_LDH + c], s, xb);
          xq = fmaf(sm.Q[r * DPLR_LDH + c], s, xq);
        }
        sm.Xb[r * DPLR_LDV + jj] += xb;
        sm.Xq[r * DPLR_LDV + jj] += xq;
      }
    }
    __syncthreads();
    // ---- T = (I + Mba)^{-1} in place, row by row (forward substitution)
    if (tid == 0) sm.Mba[0] = 1.f;
    __syncthreads();
    {
      const int j = tid >> 2, part = tid & 3;
      for (int r = 1; r < CHUNK; ++r) {
        float acc = 0.f;
        if (j < r)
          for (int i = j + part; i < r; i += 4)
            acc = fmaf(sm.Mba[r * DPLR_LDA + i], sm.Mba[i * DPLR_LDA + j], acc);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        __syncthreads();
        if (part == 0) sm.Mba[r * DPLR_LDA + j] = (j < r) ? -acc : (j == r ? 1.f : 0.f);
        __syncthreads();
      }
    }
    // ---- R = Xb + Mbk V (in Xb), U = T R
    for (int m = 0; m < CHUNK / STRIDE; ++m) {
      const int r = rb + m * STRIDE;
      float acc = sm.Xb[r * DPLR_LDV + jj];
      for (int i = 0; i < r; ++i) acc = fmaf(sm.Mbk[r * DPLR_LDA + i], sm.V[i * DPLR_LDV + jj], acc);
      sm.Xb[r * DPLR_LDV + jj] = acc;
    }
    __syncthreads();
    for (int m = 0; m < CHUNK / STRIDE; ++m) {
      const int r = rb + m * STRIDE;
      float acc = 0.f;
      for (int i = 0; i <= r; ++i) acc = fmaf(sm.Mba[r * DPLR_LDA + i], sm.Xb[i * DPLR_LDV + jj], acc);
      sm.U[r * DPLR_LDV + jj] = acc;
    }
    __syncthreads();
    // ---- O = Xq + Mqk V - Mqa U
    for (int m = 0; m < CHUNK / STRIDE; ++m) {
      const int r = rb + m * STRIDE;
      float acc = sm.Xq[r * DPLR_LDV + jj];
      for (int i = 0; i <= r; ++i) {
        acc = fmaf(sm.Mqk[r * DPLR_LDA + i], sm.V[i * DPLR_LDV + jj], acc);
        acc = fmaf(-sm.Mqa[r * DPLR_LDA + i], sm.U[i * DPLR_LDV + jj], acc);
      }
      if (r < L) o[(size_t)(t0 + r) * rs + (size_t)h * D + j0 + jj] = from_f32<TQ>(acc);
    }
    // ---- S <- Diag(e^{G_C}) S + (K e^{G_C - G})^T V - (A e^{G_C - G})^T U, per half
    for (int hc = 0; hc < 2; ++hc) {
      __syncthreads();
      for (int idx = tid; idx < CHUNK * DPLR_HC; idx += DPLR_THREADS) {
        const int r = idx / DPLR_HC, c = idx % DPLR_HC;
        float kv = 0.f, av = 0.f, lv = 0.f;
        if (r < L) {
          const size_t g = (size_t)(t0 + r) * rs + (size_t)h * D + DPLR_HC * hc + c;
          kv = to_f32(k[g]); av = to_f32(a[g]); lv = log_alpha[g];
        }
        const int e = r * DPLR_LDH + c;
        sm.K[e] = kv; sm.A[e] = av; sm.G[e] = lv;
      }
      __syncthreads();
      if (tid < DPLR_HC) {
        float acc = 0.f;
        for (int r = 0; r < CHUNK; ++r) {
          acc += sm.G[r * DPLR_LDH + tid];
          sm.G[r * DPLR_LDH + tid] = acc;
        }
        sm.gC[tid] = acc;
      }
      __syncthreads();
      for (int idx = tid; idx < CHUNK * DPLR_HC; idx += DPLR_THREADS) {
        const int r = idx / DPLR_HC, c = idx % DPLR_HC;
        const int e = r * DPLR_LDH + c;
        const float f = expf(sm.gC[c] - sm.G[e]);
        sm.K[e] *= f;
        sm.A[e] *= f;
      }
      __syncthreads();
      for (int c = rb; c < DPLR_HC; c += STRIDE) {
        float acc = expf(sm.gC[c]) * sm.S[(DPLR_HC * hc + c) * DPLR_LDV + jj];
        for (int r = 0; r < CHUNK; ++r) {
          acc = fmaf(sm.K[r * DPLR_LDH + c], sm.V[r * DPLR_LDV + jj], acc);
          acc = fmaf(-sm.A[r * DPLR_LDH + c], sm.U[r * DPLR_LDV + jj], acc);
        }
        sm.S[(DPLR_HC * hc + c) * DPLR_LDV + jj] = acc;
      }
    }
  }
  __syncthreads();
  if (hT) {
    for (int idx = tid; idx < D * DPLR_DV; idx += DPLR_THREADS) {
      const int c = idx / DPLR_DV, j = idx % DPLR_DV;
      hT[sbase + (size_t)c * D + j0 + j] = sm.S[c * DPLR_LDV + j];
    }
  }
}

}  // namespace kda
