// K1a: chunkwise KDA prefill on CUDA cores, fp32 throughout.
//
// The chunk form (Kimi Linear summary, section 3.1 "Hardware-Efficient Chunkwise
// Algorithm": WY representation with auxiliary vectors, UT transform with a
// lower-triangular inverse by forward substitution, recurrent between chunks and
// parallel within a chunk). For one chunk of C <= 64 rows entering with state S
// (per channel c, G_rc = sum_{j<=r} log alpha_jc inside the chunk):
//
//     A_ri = beta_r sum_c k_rc k_ic exp(G_rc - G_ic)   (i < r)
//     P_ri =        sum_c q_rc k_ic exp(G_rc - G_ic)   (i <= r)
//     T    = (I + A)^{-1}                              (forward substitution, row by row)
//     R    = diag(beta) (V - (K * e^G) S)
//     Delta = T R                                      (= U - W S of the WY form)
//     O    = (Q * e^G) S + P Delta
//     S   <- Diag(e^{G_C}) S + (K * e^{G_C - G})^T Delta
//
// This kernel evaluates every pairwise decay factor exp(G_rc - G_ic) exactly
// (no factorisation), so it is stable for any log alpha <= 0 and accurate to fp32
// rounding. It is the precision path for fp32 inputs and an independent second
// GPU implementation for bf16 inputs.
//
// Grid: (n_seqs * n_heads, 128 / SIMT_DV). A CTA owns one (sequence, head) and a
// slice of SIMT_DV value columns (columns of S evolve independently), loops over
// the sequence's chunks in order and keeps its slice of S in shared memory.
#pragma once

#include "kda_common.cuh"

namespace kda {

constexpr int SIMT_THREADS = 256;
constexpr int SIMT_DV = 32;            // value columns per CTA
constexpr int SIMT_LDK = D + 1;        // padded row pitch for 64 x 128 tiles
constexpr int SIMT_LDA = CHUNK + 1;    // padded row pitch for 64 x 64 tiles
constexpr int SIMT_LDV = SIMT_DV + 1;

struct SimtSmem {
  float K[CHUNK * SIMT_LDK];   // k, then k * e^G
  float Q[CHUNK * SIMT_LDK];   // q, then q * e^G
  float G[CHUNK * SIMT_LDK];   // log alpha, then G (cumsum), then k * e^{G_C - G}
  float A[CHUNK * SIMT_LDA];   // A, then T = (I + A)^{-1}
  float P[CHUNK * SIMT_LDA];
  float S[D * SIMT_LDV];       // state slice [128 channels][SIMT_DV]
  float V[CHUNK * SIMT_LDV];   // v slice, then R
  float Dl[CHUNK * SIMT_LDV];  // Delta
  float beta[CHUNK];
  float gC[D];                 // G of the chunk's last row
};

// SG = true: Gated DeltaNet, one scalar gate per token and head (log_alpha [T, H]),
// read here as the same log-decay on every channel (the scalar commutes with the
// erase, so the chunk algebra is unchanged).
template <typename TQ, bool SG>
__global__ void __launch_bounds__(SIMT_THREADS, 1)
kda_chunk_simt_kernel(const TQ* __restrict__ q, const TQ* __restrict__ k, const TQ* __restrict__ v,
                  const float* __restrict__ log_alpha, const float* __restrict__ beta,
                  const float* __restrict__ h0, const int32_t* __restrict__ cu_seqlens,
                  int n_seqs, int64_t t_total, int n_heads, TQ* __restrict__ o,
                  float* __restrict__ hT) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SimtSmem& sm = *reinterpret_cast<SimtSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int n = blockIdx.x / n_heads;
  const int h = blockIdx.x % n_heads;
  const int j0 = blockIdx.y * SIMT_DV;
  int64_t bos, eos;
  seq_bounds(cu_seqlens, n, n_seqs, t_total, bos, eos);
  const size_t row_stride = (size_t)n_heads * D;   // elements between tokens in q/k/v/o

  // initial state slice
  const size_t sbase = ((size_t)n * n_heads + h) * D * D;
  for (int idx = tid; idx < D * SIMT_DV; idx += SIMT_THREADS) {
    const int c = idx / SIMT_DV, j = idx % SIMT_DV;
    sm.S[c * SIMT_LDV + j] = h0 ? h0[sbase + (size_t)c * D + j0 + j] : 0.f;
  }

  for (int64_t t0 = bos; t0 < eos; t0 += CHUNK) {
    const int L = (eos - t0) < CHUNK ? (int)(eos - t0) : CHUNK;
    __syncthreads();   // previous chunk fully consumed
    // ---- load the chunk (rows >= L are zero; zero log-decay keeps G constant there)
    for (int idx = tid; idx < CHUNK * D; idx += SIMT_THREADS) {
      const int r = idx / D, c = idx % D;
      float kv = 0.f, qv = 0.f, lv = 0.f;
      if (r < L) {
        const size_t g = (size_t)(t0 + r) * row_stride + (size_t)h * D + c;
        kv = to_f32(k[g]);
        qv = to_f32(q[g]);
        lv = SG ? log_alpha[(size_t)(t0 + r) * n_heads + h] : log_alpha[g];
      }
      sm.K[r * SIMT_LDK + c] = kv;
      sm.Q[r * SIMT_LDK + c] = qv;
      sm.G[r * SIMT_LDK + c] = lv;
    }
    for (int idx = tid; idx < CHUNK * SIMT_DV; idx += SIMT_THREADS) {
      const int r = idx / SIMT_DV, j = idx % SIMT_DV;
      sm.V[r * SIMT_LDV + j] =
          r < L ? to_f32(v[(size_t)(t0 + r) * row_stride + (size_t)h * D + j0 + j]) : 0.f;
    }
    if (tid < CHUNK) sm.beta[tid] = tid < L ? beta[(size_t)(t0 + tid) * n_heads + h] : 0.f;
    __syncthreads();

    // ---- G = inclusive cumsum of log alpha over the chunk's rows, per channel
    if (tid < D) {
      float acc = 0.f;
      for (int r = 0; r < CHUNK; ++r) {
        acc += sm.G[r * SIMT_LDK + tid];
        sm.G[r * SIMT_LDK + tid] = acc;
      }
      sm.gC[tid] = acc;
    }
    __syncthreads();

    // ---- A (strict lower, scaled by beta_r) and P (lower incl. diagonal), exact factors
    for (int r = warp; r < CHUNK; r += SIMT_THREADS / 32) {
      const float* Kr = &sm.K[r * SIMT_LDK];
      const float* Qr = &sm.Q[r * SIMT_LDK];
      const float* Gr = &sm.G[r * SIMT_LDK];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int i = half * 32 + lane;
        float a = 0.f, p = 0.f;
        if (i <= r) {
          const float* Ki = &sm.K[i * SIMT_LDK];
          const float* Gi = &sm.G[i * SIMT_LDK];
          for (int c = 0; c < D; ++c) {
            const float e = expf(Gr[c] - Gi[c]);
            const float ke = Ki[c] * e;
            a = fmaf(Kr[c], ke, a);
            p = fmaf(Qr[c], ke, p);
          }
        }
        sm.A[r * SIMT_LDA + i] = (i < r) ? sm.beta[r] * a : 0.f;
        sm.P[r * SIMT_LDA + i] = (i <= r) ? p : 0.f;
      }
    }
    __syncthreads();

    // ---- scale operands: Q <- Q e^G, K <- K e^G, G <- K e^{G_C - G}
    for (int idx = tid; idx < CHUNK * D; idx += SIMT_THREADS) {
      const int r = idx / D, c = idx % D;
      const float g = sm.G[r * SIMT_LDK + c];
      const float eg = expf(g);
      const float kk = sm.K[r * SIMT_LDK + c];
      sm.Q[r * SIMT_LDK + c] *= eg;
      sm.K[r * SIMT_LDK + c] = kk * eg;
      sm.G[r * SIMT_LDK + c] = kk * expf(sm.gC[c] - g);
    }
    // ---- T = (I + A)^{-1} in place, row by row (forward substitution)
    //      T[r][j] = -sum_{i=j}^{r-1} A[r][i] T[i][j]  (j < r),  T[r][r] = 1
    if (tid == 0) sm.A[0] = 1.f;
    __syncthreads();
    {
      const int j = tid >> 2, part = tid & 3;   // 64 columns x 4 partial sums
      for (int r = 1; r < CHUNK; ++r) {
        float acc = 0.f;
        if (j < r)
          for (int i = j + part; i < r; i += 4) acc = fmaf(sm.A[r * SIMT_LDA + i], sm.A[i * SIMT_LDA + j], acc);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        __syncthreads();
        if (part == 0) sm.A[r * SIMT_LDA + j] = (j < r) ? -acc : (j == r ? 1.f : 0.f);
        __syncthreads();
      }
    }

    // ---- R = diag(beta)(V - (K e^G) S) in place of V;  Y = (Q e^G) S kept in registers
    const int jj = tid % SIMT_DV;
    const int rb = tid / SIMT_DV;                     // 0..7
    constexpr int RPT = CHUNK / (SIMT_THREADS / SIMT_DV);  // 8 rows per thread
    float y[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
      const int r = rb + m * (SIMT_THREADS / SIMT_DV);
      float x = 0.f, yy = 0.f;
      for (int c = 0; c < D; ++c) {
        const float s = sm.S[c * SIMT_LDV + jj];
        x = fmaf(sm.K[r * SIMT_LDK + c], s, x);
        yy = fmaf(sm.Q[r * SIMT_LDK + c], s, yy);
      }
      y[m] = yy;
      sm.V[r * SIMT_LDV + jj] = sm.beta[r] * (sm.V[r * SIMT_LDV + jj] - x);
    }
    __syncthreads();
    // ---- Delta = T R
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
      const int r = rb + m * (SIMT_THREADS / SIMT_DV);
      float d = 0.f;
      for (int i = 0; i <= r; ++i) d = fmaf(sm.A[r * SIMT_LDA + i], sm.V[i * SIMT_LDV + jj], d);
      sm.Dl[r * SIMT_LDV + jj] = d;
    }
    __syncthreads();
    // ---- O = Y + P Delta (store valid rows)
#pragma unroll
    for (int m = 0; m < RPT; ++m) {
      const int r = rb + m * (SIMT_THREADS / SIMT_DV);
      float acc = y[m];
      for (int i = 0; i <= r; ++i) acc = fmaf(sm.P[r * SIMT_LDA + i], sm.Dl[i * SIMT_LDV + jj], acc);
      if (r < L) o[(size_t)(t0 + r) * row_stride + (size_t)h * D + j0 + jj] = from_f32<TQ>(acc);
    }
    // ---- S <- Diag(e^{G_C}) S + (K e^{G_C - G})^T Delta
    for (int c = rb; c < D; c += SIMT_THREADS / SIMT_DV) {
      float acc = expf(sm.gC[c]) * sm.S[c * SIMT_LDV + jj];
      for (int r = 0; r < CHUNK; ++r) acc = fmaf(sm.G[r * SIMT_LDK + c], sm.Dl[r * SIMT_LDV + jj], acc);
      sm.S[c * SIMT_LDV + jj] = acc;
    }
  }
  __syncthreads();
  if (hT) {
    for (int idx = tid; idx < D * SIMT_DV; idx += SIMT_THREADS) {
      const int c = idx / SIMT_DV, j = idx % SIMT_DV;
      hT[sbase + (size_t)c * D + j0 + j] = sm.S[c * SIMT_LDV + j];
    }
  }
}

}  // namespace kda
