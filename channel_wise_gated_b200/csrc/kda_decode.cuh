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
