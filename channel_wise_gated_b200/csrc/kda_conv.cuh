// Short causal depthwise convolution (4 taps) + Swish over the tokens of each sequence:
// the step that produces q, k and v from their projections before the recurrence
// (Kimi Linear summary, section 4; Note, section "Other Components": "linear
// projection, short convolution, Swish"). For token t of a sequence starting at bos,
//     y_t[c] = swish( sum_{i=0..3} w[c][i] x_{t-3+i}[c] ),   x_s = 0 for s < bos,
// swish(u) = u * sigmoid(u). Streaming and HBM-bound: every input row is read once
// (plus a 3-row halo per run of tokens, mostly from L2) and every output row written
// once. At ~20 instructions per element the issue rate is close to the bandwidth too,
// so the swish takes the fast division.
//
// Layout: x, y [T, C] bf16 (C a multiple of 8, e.g. H * 128), w [C, 4] fp32.
// Thread = 8 channels (one 16-byte vector) x a run of CONV_RUN consecutive tokens; a
// warp covers 256 consecutive channels of the same token, so its loads and stores of a
// row are contiguous 512-byte segments. The three previous rows stay in registers, and
// the rows are loaded CONV_BATCH at a time ahead of their use, so that every thread has
// that many 16-byte loads in flight (one at a time leaves HBM mostly idle).
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace conv {

constexpr int CONV_THREADS = 256;
constexpr int CONV_RUN = 32;     // tokens per thread
constexpr int CONV_BATCH = 12;   // rows in flight per thread
constexpr int TAPS = 4;

__device__ __forceinline__ void unpack8(uint4 u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// First token of the sequence holding token t (cu_seqlens sorted; clamped like the
// chunk kernels clamp them): the largest n with cu[n] <= t, by bisection.
__device__ __forceinline__ int seq_of(const int32_t* __restrict__ cu, int n_seqs, int64_t t) {
  int lo = 0, hi = n_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int64_t)cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(CONV_THREADS)
kda_short_conv_swish_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ w,
                            const int32_t* __restrict__ cu_seqlens, int n_seqs, int64_t t_total,
                            int channels, __nv_bfloat16* __restrict__ y) {
  const int groups = channels >> 3;
  const int64_t gid = (int64_t)blockIdx.x * CONV_THREADS + threadIdx.x;
  const int g = (int)(gid % groups);
  const int64_t run = gid / groups;
  const int64_t t_begin = run * CONV_RUN;
  if (t_begin >= t_total) return;
  const int64_t t_end = t_begin + CONV_RUN < t_total ? t_begin + CONV_RUN : t_total;
  const int c0 = 8 * g;

  float wt[8][TAPS];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(w + (size_t)(c0 + i) * TAPS));
    wt[i][0] = v.x; wt[i][1] = v.y; wt[i][2] = v.z; wt[i][3] = v.w;
  }
  // sequence of the run's first token and where the next one starts
  int n = 0;
  int64_t bos = 0, next = t_total;
  if (cu_seqlens != nullptr) {
    n = seq_of(cu_seqlens, n_seqs, t_begin);
    bos = cu_seqlens[n];
    next = n + 1 <= n_seqs ? (int64_t)cu_seqlens[n + 1] : t_total;
    if (next > t_total) next = t_total;
    if (bos < 0) bos = 0;
  }
  // The stream of rows starts up to three rows before the run (not before the
  // sequence's first token), which only fill the history; zero history before that.
  const int64_t t_first = t_begin - 3 > bos ? t_begin - 3 : (bos < t_begin ? bos : t_begin);
  float h[3][8];
#pragma unroll
  for (int k = 0; k < 3; ++k)
#pragma unroll
    for (int i = 0; i < 8; ++i) h[k][i] = 0.f;
#pragma unroll 1
  for (int64_t tb = t_first; tb < t_end; tb += CONV_BATCH) {
    uint4 raw[CONV_BATCH];
#pragma unroll
    for (int b = 0; b < CONV_BATCH; ++b)
      raw[b] = tb + b < t_end ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)(tb + b) * channels + c0))
                              : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int b = 0; b < CONV_BATCH; ++b) {
      const int64_t t = tb + b;
      if (t >= t_end) break;
      while (t >= next && cu_seqlens != nullptr) {   // a new sequence: no history
        ++n;
        next = n + 1 <= n_seqs ? (int64_t)cu_seqlens[n + 1] : t_total;
        if (next > t_total || next < t) next = next < t ? t + 1 : t_total;
#pragma unroll
        for (int k = 0; k < 3; ++k)
#pragma unroll
          for (int i = 0; i < 8; ++i) h[k][i] = 0.f;
      }
      float cur[8];
      unpack8(raw[b], cur);
      if (t >= t_begin) {
        float out[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float u = wt[i][3] * cur[i];
          u = fmaf(wt[i][2], h[2][i], u);
          u = fmaf(wt[i][1], h[1][i], u);
          u = fmaf(wt[i][0], h[0][i], u);
          out[i] = __fdividef(u, 1.f + __expf(-u));   // swish (0 where exp(-u) overflows)
        }
        __stcs(reinterpret_cast<uint4*>(y + (size_t)t * channels + c0),
               make_uint4(pack2(out[0], out[1]), pack2(out[2], out[3]), pack2(out[4], out[5]),
                          pack2(out[6], out[7])));
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        h[0][i] = h[1][i];
        h[1][i] = h[2][i];
        h[2][i] = cur[i];
      }
    }
  }
}

}  // namespace conv
}  // namespace kda
