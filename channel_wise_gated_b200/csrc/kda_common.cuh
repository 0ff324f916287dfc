// Shared device helpers for the KDA kernels (one translation unit: kda_api.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

constexpr int D = 128;      // d_k = d_v
constexpr int CHUNK = 64;   // chunk length of the chunkwise form (appendix C: chunk_size = 64)

// Bits of the device-side error word read back by kda_device_status().
enum : int { DEVERR_SEQLENS = 1, DEVERR_TIMEOUT = 2 };

}  // namespace kda

// Device-side error word: kernels OR error bits in; the host reads and clears it.
static __device__ int g_kda_device_error;

namespace kda {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ void flag_error(int bits) { atomicOr(&g_kda_device_error, bits); }

// Token range [bos, eos) of sequence n. Values that are not monotone, negative,
// past t_total, or that do not start at 0 / end at t_total are clamped into
// range and flagged, so a bad cu_seqlens can never drive an access out of
// bounds.
__device__ __forceinline__ void seq_bounds(const int32_t* __restrict__ cu, int n, int n_seqs,
                                           int64_t t_total, int64_t& bos, int64_t& eos) {
  if (cu == nullptr) {
    bos = 0;
    eos = t_total;
    return;
  }
  const int64_t a = cu[n];
  const int64_t b = cu[n + 1];
  const int64_t ca = a < 0 ? 0 : (a > t_total ? t_total : a);
  const int64_t cb = b < ca ? ca : (b > t_total ? t_total : b);
  bool bad = (ca != a) || (cb != b);
  if (n == 0 && a != 0) bad = true;
  if (n == n_seqs - 1 && b != t_total) bad = true;
  if (bad) flag_error(DEVERR_SEQLENS);
  bos = ca;
  eos = cb;
}

}  // namespace kda
