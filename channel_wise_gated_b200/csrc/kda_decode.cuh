// K2: fused single-token KDA decode step (recurrent form, in-place fp32 state).
//
// Kimi Linear summary, section 6.3 "Complexity Analysis": autoregressive
// generation uses recurrent updates on a fixed 128 x 128 state per head. One step
// of the recurrence of section 3, rewritten so the state is read once and
// written once:
//     S' = Diag(alpha) S                 (decay first)
//     u  = S'^T k,  y = S'^T q,  s = k^T q
//     delta = beta (v - u)               (effective write of the delta rule)
//     S  <- S' + k delta^T
//     o  = S^T q = y + s * delta
//
// The step is HBM-bound: 64 KiB of state read and 64 KiB written per
// (sequence, head) against ~115 kFLOP. One CTA of 256 threads owns one state.
// Warp w holds rows 16w..16w+15; lane l holds columns 4l..4l+3 of each, so a
// warp's 16-byte loads cover a whole 512-byte row (fully coalesced), and each
// thread keeps its 64 state values in registers between the read and the write.
#pragma once

#include "kda_common.cuh"
#include "kda_sm100.cuh"

namespace kda {

constexpr int DEC_THREADS = 256;
constexpr int DEC_ROWS_PER_WARP = D / (DEC_THREADS / 32);  // 16

template <typename TQ, typename TG>
__global__ void __launch_bounds__(DEC_THREADS, 2)
kda_decode_step_kernel(const TQ* __restrict__ q, const TQ* __restrict__ k, const TQ* __restrict__ v,
                   const TG* __restrict__ log_alpha, const TG* __restrict__ beta,
                   float* __restrict__ state, TQ* __restrict__ o) {
  const int chain = blockIdx.x;          // (sequence, head) flattened
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  __shared__ float s_k[D], s_q[D], s_a[D], s_v[D];
  __shared__ float4 s_u[DEC_THREADS / 32][32], s_y[DEC_THREADS / 32][32];
  __shared__ float s_beta;

  float4* S = reinterpret_cast<float4*>(state + (size_t)chain * D * D);
  const int row0 = warp * DEC_ROWS_PER_WARP;

  // Issue all state loads first: 16 independent 16-byte loads per thread.
  float4 s[DEC_ROWS_PER_WARP];
#pragma unroll
  for (int i = 0; i < DEC_ROWS_PER_WARP; ++i) s[i] = __ldcs(&S[(row0 + i) * (D / 4) + lane]);

  if (tid < D) {
    const size_t base = (size_t)chain * D + tid;
    s_k[tid] = to_f32(k[base]);
    s_q[tid] = to_f32(q[base]);
    s_v[tid] = to_f32(v[base]);
    s_a[tid] = expf(to_f32(log_alpha[base]));
  }
  if (tid == 0) s_beta = to_f32(beta[chain]);
  __syncthreads();

  // Decay and the two partial projections over this warp's rows.
  float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < DEC_ROWS_PER_WARP; ++i) {
    const int r = row0 + i;
    const float a = s_a[r], kr = s_k[r], qr = s_q[r];
    s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
    u.x = fmaf(kr, s[i].x, u.x); u.y = fmaf(kr, s[i].y, u.y);
    u.z = fmaf(kr, s[i].z, u.z); u.w = fmaf(kr, s[i].w, u.w);
    y.x = fmaf(qr, s[i].x, y.x); y.y = fmaf(qr, s[i].y, y.y);
    y.z = fmaf(qr, s[i].z, y.z); y.w = fmaf(qr, s[i].w, y.w);
  }
  s_u[warp][lane] = u;
  s_y[warp][lane] = y;

  // s = k^T q, reduced within each warp (every warp gets the full sum).
  float kq = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) kq = fmaf(s_k[lane * 4 + i], s_q[lane * 4 + i], kq);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
  __syncthreads();

  u = make_float4(0.f, 0.f, 0.f, 0.f);
  y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int w = 0; w < DEC_THREADS / 32; ++w) {
    const float4 a = s_u[w][lane], b = s_y[w][lane];
    u.x += a.x; u.y += a.y; u.z += a.z; u.w += a.w;
    y.x += b.x; y.y += b.y; y.z += b.z; y.w += b.w;
  }
  const float bt = s_beta;
  const float4 vv = reinterpret_cast<const float4*>(s_v)[lane];
  float4 dl;
  dl.x = bt * (vv.x - u.x); dl.y = bt * (vv.y - u.y);
  dl.z = bt * (vv.z - u.z); dl.w = bt * (vv.w - u.w);

  if (warp == 0) {
    TQ* od = o + (size_t)chain * D + lane * 4;
    od[0] = from_f32<TQ>(fmaf(kq, dl.x, y.x));
    od[1] = from_f32<TQ>(fmaf(kq, dl.y, y.y));
    od[2] = from_f32<TQ>(fmaf(kq, dl.z, y.z));
    od[3] = from_f32<TQ>(fmaf(kq, dl.w, y.w));
  }
#pragma unroll
  for (int i = 0; i < DEC_ROWS_PER_WARP; ++i) {
    const float kr = s_k[row0 + i];
    float4 w;
    w.x = fmaf(kr, dl.x, s[i].x); w.y = fmaf(kr, dl.y, s[i].y);
    w.z = fmaf(kr, dl.z, s[i].z); w.w = fmaf(kr, dl.w, s[i].w);
    __stcs(&S[(row0 + i) * (D / 4) + lane], w);
  }
}

}  // namespace kda

namespace kda {

// Several consecutive tokens per (sequence, head) in one pass over the state: the
// recurrence of section 3 applied n_tokens times, with the state read once before the
// first token and written once after the last (speculative or multi-token decoding,
// where a few new tokens per sequence are verified at once). Per token the arithmetic
// is the single step's above, in the same order, so the result equals n_tokens
// consecutive single steps. Inputs are packed sequence-major like a prefill batch of
// equal lengths: [n_seqs, n_tokens, n_heads, 128] (beta [n_seqs, n_tokens, n_heads]).
//
// Two persistent CTAs per SM each walk the states blockIdx.x, + gridDim.x, ... While a
// CTA computes the tokens of one state from registers, a bulk copy brings the next state
// into a 64 KB shared-memory buffer, so its load no longer sits between two states. (Per
// CTA the load had taken 3.7 of a state's 7.5 us, with no other work to hide it.)
constexpr int DEC_MAX_TOKENS = 16;
constexpr uint32_t DEC_STATE_BYTES = D * D * sizeof(float);   // 64 KiB

// Untiled bulk copy global -> shared (both addresses 16-byte aligned, bytes a multiple
// of 16), completing `bytes` of the barrier's transaction count. No multicast.
__device__ __forceinline__ void bulk_load(void* dst_smem, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   sm100::smem_u32(dst_smem)),
               "l"(src), "r"(bytes), "r"(sm100::smem_u32(bar))
               : "memory");
}

// Dynamic shared memory of the multi-token step, in bytes, for n_tokens tokens: the state
// buffer, its barrier, the tokens' k, q, alpha, v in fp32, the partial projections and the
// reduced delta double-buffered by token parity, beta and k.q.
// With input prefetch, the next chain's inputs arrive raw (q, k, v in their storage type,
// log alpha in the gates' type) into a buffer of their own by 16-byte asynchronous copies.
__host__ __device__ constexpr size_t dec_tokens_raw_bytes(int n_tokens, size_t q_bytes, size_t g_bytes) {
  return (size_t)n_tokens * D * (3 * q_bytes + g_bytes);
}
__host__ __device__ constexpr size_t dec_tokens_smem_bytes(int n_tokens, size_t q_bytes, size_t g_bytes,
                                                           bool prefetch) {
  return DEC_STATE_BYTES + 16 + (size_t)4 * n_tokens * D * sizeof(float) +
         2 * 2 * (DEC_THREADS / 32) * 32 * sizeof(float4) + 2 * D * sizeof(float) +
         2 * DEC_MAX_TOKENS * sizeof(float) +
         (prefetch ? dec_tokens_raw_bytes(n_tokens, q_bytes, g_bytes) : 0);
}
__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sm100::smem_u32(dst_smem)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <typename TQ, typename TG, bool PF>
__global__ void __launch_bounds__(DEC_THREADS, 2)
kda_decode_tokens_kernel(const TQ* __restrict__ q, const TQ* __restrict__ k,
                         const TQ* __restrict__ v, const TG* __restrict__ log_alpha,
                         const TG* __restrict__ beta, float* __restrict__ state,
                         TQ* __restrict__ o, int n_heads, int n_tokens, int n_chains) {
  using namespace sm100;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  extern __shared__ __align__(128) unsigned char dec_smem[];
  const float4* sbuf = reinterpret_cast<const float4*>(dec_smem);
  uint64_t* bar = reinterpret_cast<uint64_t*>(dec_smem + DEC_STATE_BYTES);
  float* s_k = reinterpret_cast<float*>(dec_smem + DEC_STATE_BYTES + 16);   // [n_tokens][D]
  float* s_q = s_k + n_tokens * D;
  float* s_a = s_q + n_tokens * D;
  float* s_v = s_a + n_tokens * D;
  float4 (*s_u)[DEC_THREADS / 32][32] = reinterpret_cast<float4 (*)[DEC_THREADS / 32][32]>(s_v + n_tokens * D);
  float4 (*s_y)[DEC_THREADS / 32][32] = s_u + 2;
  float (*s_dl)[D] = reinterpret_cast<float (*)[D]>(s_y + 2);
  float* s_beta = reinterpret_cast<float*>(s_dl + 2);
  float* s_kq = s_beta + DEC_MAX_TOKENS;
  unsigned char* raw = reinterpret_cast<unsigned char*>(s_kq + DEC_MAX_TOKENS);   // 16-byte aligned
  TQ* r_q = reinterpret_cast<TQ*>(raw);
  TQ* r_k = r_q + n_tokens * D;
  TQ* r_v = r_k + n_tokens * D;
  TG* r_a = reinterpret_cast<TG*>(r_v + n_tokens * D);
  const int row0 = warp * DEC_ROWS_PER_WARP;
  // the inputs of chain ch: every (tensor, token) row of D elements is contiguous; 16-byte
  // pieces, all threads, one commit group. beta (n_tokens scalars) goes to a register.
  constexpr int QP = D * sizeof(TQ) / 16, GP = D * sizeof(TG) / 16;   // pieces per row
  auto prefetch_inputs = [&](int ch, float& beta_r) {
    const int sq = ch / n_heads, hd = ch - sq * n_heads;
    const int nq = n_tokens * QP, ng = n_tokens * GP;
#pragma unroll 1
    for (int i = tid; i < 3 * nq + ng; i += DEC_THREADS) {
      const int tensor = i < 3 * nq ? i / nq : 3;
      const int j = tensor < 3 ? i - tensor * nq : i - 3 * nq;
      const int per = tensor < 3 ? QP : GP;
      const int t = j / per, piece = j - t * per;
      const size_t row = ((size_t)sq * n_tokens + t) * n_heads + hd;
      if (tensor < 3) {
        const TQ* src = (tensor == 0 ? q : tensor == 1 ? k : v) + row * D;
        TQ* dst = (tensor == 0 ? r_q : tensor == 1 ? r_k : r_v) + t * D;
        cp_async16(reinterpret_cast<unsigned char*>(dst) + 16 * piece,
                   reinterpret_cast<const unsigned char*>(src) + 16 * piece);
      } else {
        cp_async16(reinterpret_cast<unsigned char*>(r_a + t * D) + 16 * piece,
                   reinterpret_cast<const unsigned char*>(log_alpha + row * D) + 16 * piece);
      }
    }
    cp_async_commit();
    beta_r = tid < n_tokens ? to_f32(beta[((size_t)sq * n_tokens + tid) * n_heads + hd]) : 0.f;
  };

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  int chain = blockIdx.x;          // (sequence, head) flattened, as the state
  if (tid == 0 && chain < n_chains) {
    mbar_arrive_expect_tx(bar, DEC_STATE_BYTES);
    bulk_load(dec_smem, state + (size_t)chain * D * D, DEC_STATE_BYTES, bar);
  }
  float beta_next = 0.f;
  if constexpr (PF) {
    if (chain < n_chains) prefetch_inputs(chain, beta_next);
  }
  uint32_t phase = 0;
#pragma unroll 1
  for (; chain < n_chains; chain += gridDim.x) {
    const int seq = chain / n_heads, h = chain - seq * n_heads;
    if constexpr (PF) {
      // this chain's inputs, copied while the previous chain computed: to fp32 (alpha
      // from its log), then the buffer takes the next chain's
      cp_async_wait_all();
      __syncthreads();
#pragma unroll 1
      for (int i = tid; i < n_tokens * D; i += DEC_THREADS) {
        s_k[i] = to_f32(r_k[i]);
        s_q[i] = to_f32(r_q[i]);
        s_v[i] = to_f32(r_v[i]);
        s_a[i] = expf(to_f32(r_a[i]));
      }
      if (tid < n_tokens) s_beta[tid] = beta_next;
      __syncthreads();
      if (chain + (int)gridDim.x < n_chains) prefetch_inputs(chain + gridDim.x, beta_next);
    } else {
      // this chain's inputs, loaded now (read after the barrier below)
#pragma unroll 1
      for (int i = tid; i < n_tokens * D; i += DEC_THREADS) {
        const int t = i / D, c = i - t * D;
        const size_t base = (((size_t)seq * n_tokens + t) * n_heads + h) * D + c;
        s_k[i] = to_f32(k[base]);
        s_q[i] = to_f32(q[base]);
        s_v[i] = to_f32(v[base]);
        s_a[i] = expf(to_f32(log_alpha[base]));
      }
      if (tid < n_tokens) s_beta[tid] = to_f32(beta[((size_t)seq * n_tokens + tid) * n_heads + h]);
    }
    // this chain's state, copied into the buffer while the previous chain computed
    const bool landed = mbar_wait(bar, phase);
    phase ^= 1u;
    float4 s[DEC_ROWS_PER_WARP];
#pragma unroll
    for (int i = 0; i < DEC_ROWS_PER_WARP; ++i) s[i] = sbuf[(row0 + i) * (D / 4) + lane];
    fence_proxy_async_smem();   // (these reads come before the next copy into the buffer)
    if (!__syncthreads_and(landed)) {   // (also the barrier before the staged inputs are read)
      if constexpr (PF) cp_async_wait_all();   // (nor with the next inputs' copies in flight)
      if (tid == 0) {
        flag_error(DEVERR_TIMEOUT);
        mbar_wait(bar, phase ^ 1u, 100000000ull);   // (never leave with the copy in flight)
      }
      break;
    }
    if (tid == 0 && chain + (int)gridDim.x < n_chains) {
      mbar_arrive_expect_tx(bar, DEC_STATE_BYTES);
      bulk_load(dec_smem, state + (size_t)(chain + gridDim.x) * D * D, DEC_STATE_BYTES, bar);
    }
    float4* S = reinterpret_cast<float4*>(state + (size_t)chain * D * D);
    // the output row of token 0; one token further is n_heads * D elements
    TQ* od = o + ((size_t)seq * n_tokens * n_heads + h) * D;
    const size_t o_step = (size_t)n_heads * D;
    // k^T q of every token once (warp w takes tokens w, w + 8), formed exactly as the
    // single step forms it; read after the first token's barrier
#pragma unroll 1
    for (int t = warp; t < n_tokens; t += DEC_THREADS / 32) {
      float kq = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) kq = fmaf(s_k[t * D + lane * 4 + i], s_q[t * D + lane * 4 + i], kq);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
      if (lane == 0) s_kq[t] = kq;
    }

#pragma unroll 1
    for (int t = 0; t < n_tokens; ++t, od += o_step) {
      const int buf = t & 1;
      const float* sa_t = s_a + t * D;
      const float* sk_t = s_k + t * D;
      const float* sq_t = s_q + t * D;
      // decay and the two partial projections over this warp's rows (4 rows of the
      // gates and keys per 16-byte read; rows in the single step's order). Two columns
      // per instruction: the paired multiply and FMA round each lane as the scalar ones do.
      float2 u0 = make_float2(0.f, 0.f), u1 = u0, y0 = u0, y1 = u0;
#pragma unroll
      for (int i4 = 0; i4 < DEC_ROWS_PER_WARP; i4 += 4) {
        const float4 a4 = *reinterpret_cast<const float4*>(&sa_t[row0 + i4]);
        const float4 k4 = *reinterpret_cast<const float4*>(&sk_t[row0 + i4]);
        const float4 q4 = *reinterpret_cast<const float4*>(&sq_t[row0 + i4]);
        const float av[4] = {a4.x, a4.y, a4.z, a4.w}, kv[4] = {k4.x, k4.y, k4.z, k4.w},
                    qv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = i4 + e;
          const float2 a2 = make_float2(av[e], av[e]), k2 = make_float2(kv[e], kv[e]),
                       q2 = make_float2(qv[e], qv[e]);
          const float2 lo = __fmul2_rn(make_float2(s[i].x, s[i].y), a2);
          const float2 hi = __fmul2_rn(make_float2(s[i].z, s[i].w), a2);
          s[i] = make_float4(lo.x, lo.y, hi.x, hi.y);
          u0 = __ffma2_rn(k2, lo, u0); u1 = __ffma2_rn(k2, hi, u1);
          y0 = __ffma2_rn(q2, lo, y0); y1 = __ffma2_rn(q2, hi, y1);
        }
      }
      s_u[buf][warp][lane] = make_float4(u0.x, u0.y, u1.x, u1.y);
      s_y[buf][warp][lane] = make_float4(y0.x, y0.y, y1.x, y1.y);
      // (this token's buffers were last read two tokens ago, before the previous barriers)
      __syncthreads();

      // thread c < 128 reduces column c over the warps, in the single step's order, and
      // leaves delta_c for all; the other threads wait at the next barrier. (Each thread
      // summing its own 4 columns, as the single step does, reads 8x the shared memory.)
      if (tid < D) {
        const int cl = tid >> 2, cc = tid & 3;
        float uc = 0.f, yc = 0.f;
#pragma unroll
        for (int w = 0; w < DEC_THREADS / 32; ++w) {
          uc += reinterpret_cast<const float*>(&s_u[buf][w][cl])[cc];
          yc += reinterpret_cast<const float*>(&s_y[buf][w][cl])[cc];
        }
        const float dc = s_beta[t] * (s_v[t * D + tid] - uc);
        s_dl[buf][tid] = dc;
        od[tid] = from_f32<TQ>(fmaf(s_kq[t], dc, yc));
      }
      __syncthreads();
      const float4 dl = reinterpret_cast<const float4*>(s_dl[buf])[lane];
      const float2 dl0 = make_float2(dl.x, dl.y), dl1 = make_float2(dl.z, dl.w);
#pragma unroll
      for (int i4 = 0; i4 < DEC_ROWS_PER_WARP; i4 += 4) {
        const float4 k4 = *reinterpret_cast<const float4*>(&sk_t[row0 + i4]);
        const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = i4 + e;
          const float2 k2 = make_float2(kv[e], kv[e]);
          const float2 lo = __ffma2_rn(k2, dl0, make_float2(s[i].x, s[i].y));
          const float2 hi = __ffma2_rn(k2, dl1, make_float2(s[i].z, s[i].w));
          s[i] = make_float4(lo.x, lo.y, hi.x, hi.y);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < DEC_ROWS_PER_WARP; ++i) __stcs(&S[(row0 + i) * (D / 4) + lane], s[i]);
    __syncthreads();   // (the staged inputs are rewritten for the next chain)
  }
}

// Host side: two persistent CTAs per SM (or one per state, if fewer); returns the
// launch's CUDA error. The next chain's inputs are prefetched from three tokens on, as
// long as two CTAs with the larger shared-memory layout still fit an SM: with one or two
// tokens a chain is bound by its state copies, and the prefetch's extra barriers cost
// more than the latency it hides.
template <typename TQ, typename TG, bool PF>
cudaError_t launch_decode_tokens_as(const TQ* q, const TQ* k, const TQ* v, const TG* log_alpha,
                                    const TG* beta, float* state, TQ* o, int n_tokens,
                                    int n_heads, int chains, int sms, cudaStream_t stream) {
  const size_t smem = dec_tokens_smem_bytes(n_tokens, sizeof(TQ), sizeof(TG), PF);
  cudaError_t e = cudaFuncSetAttribute(kda_decode_tokens_kernel<TQ, TG, PF>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = chains < 2 * sms ? chains : 2 * sms;
  kda_decode_tokens_kernel<TQ, TG, PF><<<grid, DEC_THREADS, smem, stream>>>(
      q, k, v, log_alpha, beta, state, o, n_heads, n_tokens, chains);
  return cudaGetLastError();
}

template <typename TQ, typename TG>
cudaError_t launch_decode_tokens(const TQ* q, const TQ* k, const TQ* v, const TG* log_alpha,
                                 const TG* beta, float* state, TQ* o, int n_seqs, int n_tokens,
                                 int n_heads, cudaStream_t stream) {
  const int chains = n_seqs * n_heads;
  int dev = 0, sms = 0, smem_sm = 0, reserved = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess)
    e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  if (e == cudaSuccess)
    e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  if (e != cudaSuccess) return e;
  const size_t pf_smem = dec_tokens_smem_bytes(n_tokens, sizeof(TQ), sizeof(TG), true);
  if (n_tokens >= 3 && 2 * (pf_smem + (size_t)reserved) <= (size_t)smem_sm)
    return launch_decode_tokens_as<TQ, TG, true>(q, k, v, log_alpha, beta, state, o, n_tokens,
                                                 n_heads, chains, sms, stream);
  return launch_decode_tokens_as<TQ, TG, false>(q, k, v, log_alpha, beta, state, o, n_tokens,
                                                n_heads, chains, sms, stream);
}

}  // namespace kda
