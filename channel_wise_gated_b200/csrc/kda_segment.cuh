// Time split of one long sequence: composition of the segments' state maps.
//
// Every step of the recurrence (Kimi Linear summary, section 3) is affine in the
// state, so a segment of chunks maps its entering state S to M S + R, with M the
// product of its per-token transitions (I - beta k k^T) Diag(alpha) and R its final
// state from a zero start. The chunk kernel's first pass of a split (PLAN_ZERO)
// leaves, per head, the exact state entering segment 1 in slot 0, R_j in slot j and
// M_j in slot n-2+j (j = 1 .. n-2; M_j is the final state from the identity with
// v = 0). This kernel
// then walks the segments in order,
//     S_{j+1} = M_j S_j + R_j,   j = 1 .. n-2   (S_1 = slot 0),
// writing S_{j+1} over R_j in slot j, all in fp32. One CTA per head; n-2 products
// of 128 x 128 matrices, about 20 us each. A transition chain that stopped early
// left M_j exactly zero: then S_{j+1} = R_j, already in place, and the step is skipped.
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace seg {

constexpr int SCAN_THREADS = 256;
constexpr int SP = D + 4;   // smem pitch of the row-major copies (keeps float4 rows aligned)
constexpr size_t SCAN_SMEM = 2 * (size_t)D * SP * sizeof(float);

// First chunk of segment j when n_chunks chunks are cut into n_seg segments balanced
// to within one chunk: seg_base = n_chunks / n_seg, seg_rem = n_chunks % n_seg, and
// the first seg_rem segments take one chunk more. Segment j covers chunks
// [seg_first_chunk(j), seg_first_chunk(j + 1)); seg_first_chunk(n_seg) = n_chunks.
__host__ __device__ inline int64_t seg_first_chunk(int j, int seg_base, int seg_rem) {
  return (int64_t)j * seg_base + (j < seg_rem ? j : seg_rem);
}

__global__ void __launch_bounds__(SCAN_THREADS)
kda_segment_scan_kernel(float* __restrict__ states, int n_heads, int n_seg) {
  extern __shared__ __align__(16) float sm[];
  float* Ms = sm;             // M_j, row-major, pitch SP
  float* Ss = sm + D * SP;    // S_j
  const int h = blockIdx.x, tid = threadIdx.x;
  const size_t E = (size_t)D * D;
  auto slot = [&](int s) { return states + ((size_t)s * n_heads + h) * E; };
  // thread tile: rows r0..r0+7, columns c0..c0+7 of the 128 x 128 result
  const int r0 = 8 * (tid >> 4), c0 = 8 * (tid & 15);
  for (int j = 1; j <= n_seg - 2; ++j) {
    const float* M = slot(n_seg - 2 + j);       // M_j
    const float* S = slot(j - 1);               // S_j (slot 0, or the previous result)
    float* RS = slot(j);                        // R_j in, S_{j+1} out
    int nz = 0;
    for (int i = tid; i < D * D / 4; i += SCAN_THREADS) {
      const int r = (4 * i) / D, c = (4 * i) % D;
      const float4 m4 = reinterpret_cast<const float4*>(M)[i];
      nz |= (m4.x != 0.f) | (m4.y != 0.f) | (m4.z != 0.f) | (m4.w != 0.f);
      *reinterpret_cast<float4*>(&Ms[r * SP + c]) = m4;
      *reinterpret_cast<float4*>(&Ss[r * SP + c]) = reinterpret_cast<const float4*>(S)[i];
    }
    if (!__syncthreads_or(nz)) continue;   // M_j = 0: S_{j+1} = R_j (the loop's barrier is passed)
    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
      float av[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) av[a] = Ms[(r0 + a) * SP + k];
      const float4 b0 = *reinterpret_cast<const float4*>(&Ss[k * SP + c0]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Ss[k * SP + c0 + 4]);
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
    }
    // each element of R_j is read and overwritten by the same thread
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const size_t e = (size_t)(r0 + a) * D + c0 + b;
        RS[e] = acc[a][b] + RS[e];
      }
    __syncthreads();
  }
}

// Launch order of a packed batch: order[rank] = sequence, ranked by decreasing
// length (ties by index), so that the chunk kernel starts the longest sequences
// first. Thread i ranks sequence i against all others; lengths are clamped like
// the chunk kernel clamps them (a bad cu_seqlens only changes the order).
constexpr int ORDER_THREADS = 256;
constexpr int ORDER_TILE = 1024;

__global__ void __launch_bounds__(ORDER_THREADS)
kda_seq_order_kernel(const int32_t* __restrict__ cu, int n_seqs, int64_t t_total,
                     int32_t* __restrict__ order) {
  __shared__ int64_t len_tile[ORDER_TILE];
  const int i = blockIdx.x * ORDER_THREADS + threadIdx.x;
  auto len_of = [&](int s) -> int64_t {
    const int64_t a = cu[s], b = cu[s + 1];
    const int64_t ca = a < 0 ? 0 : (a > t_total ? t_total : a);
    const int64_t cb = b < ca ? ca : (b > t_total ? t_total : b);
    return cb - ca;
  };
  const int64_t li = i < n_seqs ? len_of(i) : 0;
  int rank = 0;
  for (int t0 = 0; t0 < n_seqs; t0 += ORDER_TILE) {
    const int tn = (n_seqs - t0) < ORDER_TILE ? (n_seqs - t0) : ORDER_TILE;
    __syncthreads();
    for (int k = threadIdx.x; k < tn; k += ORDER_THREADS) len_tile[k] = len_of(t0 + k);
    __syncthreads();
    if (i < n_seqs)
      for (int k = 0; k < tn; ++k) {
        const int64_t lj = len_tile[k];
        rank += (lj > li || (lj == li && t0 + k < i)) ? 1 : 0;
      }
  }
  if (i < n_seqs) order[rank] = i;
}

}  // namespace seg
}  // namespace kda
