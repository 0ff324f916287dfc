// C ABI of the KDA library (declared in include/kda.h): host-side validation and
// stream-ordered kernel launches. All device code lives in the included headers;
// this file is the library's single translation unit.

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "../../include/kda.h"
#include "kda_chunk_simt.cuh"
#include "kda_chunk_tc.cuh"
#include "kda_common.cuh"
#include "kda_conv.cuh"
#include "kda_decode.cuh"
#include "kda_dplr_simt.cuh"
#include "kda_segment.cuh"

// Scratch of kda_chunk_fwd_static, for callers that cannot allocate device memory:
// a fixed array in every GPU context that loads the library. The time split plans
// within it (on a 148-SM part the largest plan takes 18.2 MiB of a free workspace,
// so a few head counts split into fewer segments here); a packed batch's launch
// order needs 4 bytes per sequence.
static __device__ __align__(256) unsigned char g_kda_static_scratch[KDA_STATIC_SCRATCH_BYTES];

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

int validate_chunk_args(const void* q, const void* k, const void* v, const float* log_alpha,
                        const float* beta, const float* h0, const int32_t* cu_seqlens,
                        int32_t n_seqs, int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype,
                        const void* o, const float* hT) {
  if (qkv_dtype != KDA_F32 && qkv_dtype != KDA_BF16) return KDA_ERR_DTYPE;
  if (n_heads <= 0 || n_seqs <= 0 || t_total < 0) return KDA_ERR_SHAPE;
  if ((int64_t)n_seqs * n_heads > (int64_t)INT32_MAX / 4) return KDA_ERR_SHAPE;
  if (cu_seqlens == nullptr && n_seqs != 1) return KDA_ERR_SEQLENS;
  if (t_total > 0 && (!q || !k || !v || !log_alpha || !beta || !o)) return KDA_ERR_NULL;
  const void* ptrs[] = {q, k, v, log_alpha, beta, h0, o, hT, cu_seqlens};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_ALIGN;
  return KDA_OK;
}

template <typename TQ, bool SG>
int launch_chunk_simt(const void* q, const void* k, const void* v, const float* log_alpha,
                      const float* beta, const float* h0, const int32_t* cu_seqlens,
                      int32_t n_seqs, int64_t t_total, int32_t n_heads, void* o, float* hT,
                      cudaStream_t stream) {
  const size_t smem = sizeof(kda::SimtSmem);
  if (cudaFuncSetAttribute(kda::kda_chunk_simt_kernel<TQ, SG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return KDA_ERR_CUDA;
  dim3 grid((unsigned)(n_seqs * n_heads), kda::D / kda::SIMT_DV);
  kda::kda_chunk_simt_kernel<TQ, SG><<<grid, kda::SIMT_THREADS, smem, stream>>>(
      static_cast<const TQ*>(q), static_cast<const TQ*>(k), static_cast<const TQ*>(v), log_alpha,
      beta, h0, cu_seqlens, n_seqs, t_total, n_heads, static_cast<TQ*>(o), hT);
  return launch_status();
}

int chunk_simt_dispatch(const void* q, const void* k, const void* v, const float* log_alpha,
                        const float* beta, const float* h0, const int32_t* cu_seqlens,
                        int32_t n_seqs, int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype,
                        void* o, float* hT, bool sg, cudaStream_t stream) {
  if (qkv_dtype == KDA_F32)
    return sg ? launch_chunk_simt<float, true>(q, k, v, log_alpha, beta, h0, cu_seqlens, n_seqs,
                                               t_total, n_heads, o, hT, stream)
              : launch_chunk_simt<float, false>(q, k, v, log_alpha, beta, h0, cu_seqlens, n_seqs,
                                                t_total, n_heads, o, hT, stream);
  return sg ? launch_chunk_simt<__nv_bfloat16, true>(q, k, v, log_alpha, beta, h0, cu_seqlens,
                                                     n_seqs, t_total, n_heads, o, hT, stream)
            : launch_chunk_simt<__nv_bfloat16, false>(q, k, v, log_alpha, beta, h0, cu_seqlens,
                                                      n_seqs, t_total, n_heads, o, hT, stream);
}

// ---- tensor-core chunk kernel: TMA descriptors and launch ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn tensor_map_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D view [rows][cols] of a token-major tensor, box [box_r][box_c].
bool encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t cols,
               uint64_t rows, uint64_t elem_bytes, uint32_t box_c, uint32_t box_r,
               CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * elem_bytes};
  const cuuint32_t box[2] = {box_c, box_r};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Every segment keeps at least MIN_SEG_CHUNKS chunks; at most MAX_SEGMENTS.
constexpr int MIN_SEG_CHUNKS = 16;
constexpr int MAX_SEGMENTS = 64;
constexpr int64_t SPLIT_EARLY_CHUNKS = 128;

// Time split of one long sequence (the chunk kernel's PLAN_ZERO, the segment scan,
// PLAN_CORR; see the kernel's plans). A split into n segments of about len chunks runs
// the H n Z CTAs (all segments from zero states) in waves of one CTA per SM; the SMs
// the last wave leaves free take the H (n - 2) transition chains, the rest follow the
// Z CTAs. Then the scan (n - 2 products of 128 x 128 matrices per head, about two
// chunk periods each) and the H (n - 1) corrections. Transition chains and
// corrections both stop once their state is exactly zero; for segments of
// SPLIT_EARLY_CHUNKS chunks or more the plan counts on that within STOP_CHUNKS
// chunks, and otherwise on neither stopping. In chunk periods a split costs
//   waves(H n) len + (transition chains that do not fit) + 2 (n - 2) + waves(H (n - 1)) z
// and the single pass the whole sequence. Equal segments make the waves even: at 32
// heads over 1M tokens, 9 segments (two waves of 148 and 140 Z CTAs) measured 18.1 ms
// against 19.6 ms for 4 (one wave of 128), 20.0 for 8 and 23.5 for 10 (three waves).
// Every segment keeps at least MIN_SEG_CHUNKS chunks, and the plan's scratch must fit
// the bytes available.
constexpr int64_t STOP_CHUNKS = 64;
constexpr double SCAN_STEP_CHUNKS = 2.0;

size_t split_workspace_bytes(int n_seg, int32_t n_heads) {
  return n_seg >= 2 ? (size_t)(2 * n_seg - 2) * n_heads * kda::D * kda::D * sizeof(float) : 0;
}

int split_segments(int64_t n_chunks, int32_t n_heads, int sms, size_t max_bytes) {
  if (sms <= 0 || n_heads <= 0) return 0;
  int best = 0;
  double best_cost = (double)n_chunks * (double)((n_heads + sms - 1) / sms);
  for (int n = 2; n <= MAX_SEGMENTS; ++n) {
    if (n_chunks < (int64_t)n * MIN_SEG_CHUNKS) break;
    if (split_workspace_bytes(n, n_heads) > max_bytes) break;
    const int64_t len = (n_chunks + n - 1) / n;
    const double z = len >= SPLIT_EARLY_CHUNKS ? (double)std::min<int64_t>(len, STOP_CHUNKS) : (double)len;
    const int64_t zc = (int64_t)n_heads * n, waves = (zc + sms - 1) / sms;
    const int64_t trans = (int64_t)n_heads * (n - 2), free_sms = waves * sms - zc;
    const int64_t fit = free_sms * std::max<int64_t>(1, (int64_t)((double)len / z));
    const double extra = trans > fit ? z * (double)((trans - fit + sms - 1) / sms) : 0.0;
    const int64_t cwaves = ((int64_t)n_heads * (n - 1) + sms - 1) / sms;
    const double cost = (double)(waves * len) + extra + SCAN_STEP_CHUNKS * (n - 2) + (double)cwaves * z;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = n;
    }
  }
  return best;
}

int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return sms;
}

// Packed batches: a launch order by decreasing length (one int32 per sequence),
// worth it once the CTAs exceed one wave; ranking is O(n^2) so it stays bounded.
constexpr int32_t MAX_ORDERED_SEQS = 16384;
size_t order_workspace_bytes(int32_t n_seqs, int32_t n_heads) {
  if (n_seqs < 2 || n_seqs > MAX_ORDERED_SEQS) return 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  if ((int64_t)n_seqs * n_heads <= sms) return 0;
  return ((size_t)n_seqs * sizeof(int32_t) + 255) & ~(size_t)255;
}

// The fused variant's inputs (MODE_FUSED): pre-activations and the norm weight.
struct FusedIO {
  const void* decay_pre;
  const float* beta_pre;
  const void* gate_pre;
  const float* norm_w;
};

template <int MODE>
int launch_chunk_tc(const void* q, const void* k, const void* v, const float* log_alpha,
                    const float* beta, const float* h0, const int32_t* cu_seqlens, int32_t n_seqs,
                    int64_t t_total, int32_t n_heads, void* o, float* hT, int n_seg,
                    float* seg_states, int32_t* seq_order, const FusedIO* fu, cudaStream_t stream,
                    uint64_t wait_ns = 0, int debug_skip_tb = -1) {
  using namespace kda::tc;
  const uint64_t cols = (uint64_t)n_heads * kda::D;
  const uint64_t rows = (uint64_t)t_total;
  CUtensorMap mk, mq, mv, mla, mo;
  memset(&mla, 0, sizeof(mla));   // (a scalar gate has no tile map: prep A prefetches it)
  bool la_ok = true;
  if (MODE == MODE_KDA)
    la_ok = encode_2d(&mla, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, log_alpha, cols, rows, 4, 128, 64,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
  else if (MODE == MODE_FUSED)   // the bf16 decay pre-activation, prefetched the same way
    la_ok = encode_2d(&mla, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, fu->decay_pre, cols, rows, 2, 128, 64,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!la_ok ||
      !encode_2d(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k, cols, rows, 2, 64, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, cols, rows, 2, 64, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v, cols, rows, 2, 64, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&mo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, o, cols, rows, 2, 64, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return KDA_ERR_CUDA;
  if (cudaFuncSetAttribute(kda_chunk_tc_kernel<false, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)SMEM_BYTES) != cudaSuccess ||
      cudaFuncSetAttribute(kda_chunk_tc_kernel<true, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)SMEM_BYTES) != cudaSuccess)
    return KDA_ERR_CUDA;
  Args a;
  a.log_alpha = log_alpha;
  a.beta = beta;
  a.h0 = h0;
  a.cu_seqlens = cu_seqlens;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.hT = hT;
  a.n_seqs = n_seqs;
  a.n_heads = n_heads;
  a.t_total = t_total;
  a.plan = PLAN_SEQ;
  a.n_seg = 0;
  a.seg_base = 0;
  a.seg_rem = 0;
  a.seg_states = nullptr;
  a.seq_order = nullptr;
  a.decay_pre = fu ? static_cast<const __nv_bfloat16*>(fu->decay_pre) : nullptr;
  a.beta_pre = fu ? fu->beta_pre : nullptr;
  a.gate_pre = fu ? static_cast<const __nv_bfloat16*>(fu->gate_pre) : nullptr;
  a.norm_w = fu ? fu->norm_w : nullptr;
  a.wait_ns = wait_ns;
  a.debug_skip_tb = debug_skip_tb;
  if (seq_order != nullptr && cu_seqlens != nullptr && n_seqs > 1) {
    const unsigned blocks = (unsigned)((n_seqs + kda::seg::ORDER_THREADS - 1) / kda::seg::ORDER_THREADS);
    kda::seg::kda_seq_order_kernel<<<blocks, kda::seg::ORDER_THREADS, 0, stream>>>(
        cu_seqlens, n_seqs, t_total, seq_order);
    if (launch_status() != KDA_OK) return KDA_ERR_CUDA;
    a.seq_order = seq_order;
  }
  if (n_seg < 2 || seg_states == nullptr) {
    const int64_t grid = (int64_t)n_seqs * n_heads;   // one CTA per (sequence, head)
    kda_chunk_tc_kernel<false, MODE><<<(unsigned)grid, THREADS, SMEM_BYTES, stream>>>(mk, mq, mv, mla, mo, a);
    return launch_status();
  }
  // time split: every segment from a zero state (segment 0 from h0) with its output
  // and the transition chains, the scan over segments, then the corrections of
  // segments 1 .. n-1 (and for the fused variant the norm and gate of their outputs)
  const int64_t n_chunks = (t_total + kda::CHUNK - 1) / kda::CHUNK;
  a.n_seg = n_seg;
  a.seg_base = (int)(n_chunks / n_seg);
  a.seg_rem = (int)(n_chunks % n_seg);
  a.seg_states = seg_states;
  a.plan = PLAN_ZERO;
  kda_chunk_tc_kernel<true, MODE><<<(unsigned)(n_heads * (2 * n_seg - 2)), THREADS, SMEM_BYTES, stream>>>(
      mk, mq, mv, mla, mo, a);
  if (launch_status() != KDA_OK) return KDA_ERR_CUDA;
  if (n_seg >= 3) {
    if (cudaFuncSetAttribute(kda::seg::kda_segment_scan_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kda::seg::SCAN_SMEM) != cudaSuccess)
      return KDA_ERR_CUDA;
    kda::seg::kda_segment_scan_kernel<<<(unsigned)n_heads, kda::seg::SCAN_THREADS, kda::seg::SCAN_SMEM,
                                         stream>>>(seg_states, n_heads, n_seg);
    if (launch_status() != KDA_OK) return KDA_ERR_CUDA;
  }
  a.plan = PLAN_CORR;
  kda_chunk_tc_kernel<true, MODE><<<(unsigned)(n_heads * (n_seg - 1)), THREADS, SMEM_BYTES, stream>>>(
      mk, mq, mv, mla, mo, a);
  if (launch_status() != KDA_OK) return KDA_ERR_CUDA;
  if constexpr (MODE == MODE_FUSED) {
    const int64_t t1 = kda::seg::seg_first_chunk(1, a.seg_base, a.seg_rem) * kda::CHUNK;
    const int64_t rows = (t_total - t1) * n_heads;
    const int64_t want = (rows + NG_ROWS - 1) / NG_ROWS;
    const int sms = device_sms();
    const int64_t cap = (int64_t)(sms > 0 ? sms : 148) * 16;
    kda_norm_gate_kernel<<<(unsigned)(want < cap ? want : cap), NG_THREADS, 0, stream>>>(
        static_cast<__nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(fu->gate_pre), fu->norm_w,
        t1 * n_heads, rows);
    return launch_status();
  }
  return KDA_OK;
}

// Whether a call takes the tensor-core path and, if so, how many segments it splits into.
bool use_tc(const int32_t* cu_seqlens, int32_t n_seqs, int64_t t_total, int32_t n_heads,
            kda_dtype qkv_dtype) {
  (void)cu_seqlens;
  // bf16 inputs run on the tensor-core kernel; its TMA boxes span 64 tokens, so
  // inputs shorter than one chunk (and fp32 inputs) take the CUDA-core kernel.
  return qkv_dtype == KDA_BF16 && t_total >= kda::CHUNK &&
         t_total < (int64_t)INT32_MAX - 4 * kda::CHUNK && (int64_t)n_seqs * n_heads < (int64_t)INT32_MAX;
}
// Segments of the time split for a call with max_bytes of scratch (0: no split).
int plan_segments(const int32_t* cu_seqlens, int32_t n_seqs, int64_t t_total, int32_t n_heads,
                  kda_dtype qkv_dtype, size_t max_bytes) {
  if (!use_tc(cu_seqlens, n_seqs, t_total, n_heads, qkv_dtype) || cu_seqlens != nullptr || n_seqs != 1)
    return 0;
  return split_segments((t_total + kda::CHUNK - 1) / kda::CHUNK, n_heads, device_sms(), max_bytes);
}

template <typename TQ, typename TG>
int launch_decode(const void* q, const void* k, const void* v, const void* log_alpha,
                  const void* beta, float* state, void* o, int32_t n_seqs, int32_t n_heads,
                  cudaStream_t stream) {
  const unsigned chains = (unsigned)n_seqs * (unsigned)n_heads;
  kda::kda_decode_step_kernel<TQ, TG><<<chains, kda::DEC_THREADS, 0, stream>>>(
      static_cast<const TQ*>(q), static_cast<const TQ*>(k), static_cast<const TQ*>(v),
      static_cast<const TG*>(log_alpha), static_cast<const TG*>(beta), state, static_cast<TQ*>(o));
  return launch_status();
}

template <typename TQ, typename TG>
int launch_decode_tokens(const void* q, const void* k, const void* v, const void* log_alpha,
                         const void* beta, float* state, void* o, int32_t n_seqs, int32_t n_tokens,
                         int32_t n_heads, cudaStream_t stream) {
  const cudaError_t e = kda::launch_decode_tokens<TQ, TG>(
      static_cast<const TQ*>(q), static_cast<const TQ*>(k), static_cast<const TQ*>(v),
      static_cast<const TG*>(log_alpha), static_cast<const TG*>(beta), state, static_cast<TQ*>(o),
      n_seqs, n_tokens, n_heads, stream);
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
static_assert(KDA_DECODE_MAX_TOKENS == kda::DEC_MAX_TOKENS, "token limit of the ABI and the kernel");

// Device address of g_kda_static_scratch in the current context. In host code the
// array's name only stands in for the symbol, so the address is looked up once per
// device, with that device current, and kept together with the context it belongs
// to: a new context on the same device (after cudaDeviceReset, say) looks it up again.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

constexpr int MAX_STATIC_DEVICES = 64;
std::mutex g_static_mu;
void* g_static_addr[MAX_STATIC_DEVICES] = {};
CUcontext g_static_ctx[MAX_STATIC_DEVICES] = {};

int static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_STATIC_DEVICES)
    return KDA_ERR_CUDA;
  CtxGetCurrentFn get_ctx = ctx_get_current();
  CUcontext ctx = nullptr;
  if (get_ctx == nullptr || get_ctx(&ctx) != CUDA_SUCCESS) return KDA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (ctx == nullptr || g_static_addr[dev] == nullptr || g_static_ctx[dev] != ctx) {
    // (the look-up makes the device's primary context current if none was)
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kda_static_scratch) != cudaSuccess || p == nullptr)
      return KDA_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return KDA_ERR_CUDA;
    g_static_addr[dev] = p;
    g_static_ctx[dev] = ctx;
  }
  *out = g_static_addr[dev];
  return KDA_OK;
}

// The prefill for KDA (sg = false: log_alpha [T, H, 128]) or Gated DeltaNet (sg =
// true: one log-gate per token and head, [T, H]): validation, then the tensor-core
// kernel (time split when the workspace allows it) or the CUDA-core kernel.
int chunk_fwd_impl(const void* q, const void* k, const void* v, const float* log_alpha,
                   const float* beta, const float* h0, const int32_t* cu_seqlens, int32_t n_seqs,
                   int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype, void* o, float* hT,
                   void* workspace, size_t workspace_bytes, bool sg, cudaStream_t stream) {
  int st = validate_chunk_args(q, k, v, log_alpha, beta, h0, cu_seqlens, n_seqs, t_total, n_heads,
                               qkv_dtype, o, hT);
  if (st != KDA_OK) return st;
  if (workspace && !aligned16(workspace)) return KDA_ERR_ALIGN;
  if (use_tc(cu_seqlens, n_seqs, t_total, n_heads, qkv_dtype)) {
    const int n_seg = workspace == nullptr ? 0 : plan_segments(cu_seqlens, n_seqs, t_total, n_heads,
                                                               qkv_dtype, workspace_bytes);
    int32_t* order = nullptr;
    const size_t ob = order_workspace_bytes(n_seqs, n_heads);
    if (n_seg == 0 && cu_seqlens != nullptr && workspace != nullptr && ob > 0 && workspace_bytes >= ob)
      order = static_cast<int32_t*>(workspace);
    return sg ? launch_chunk_tc<kda::tc::MODE_GDN>(q, k, v, log_alpha, beta, h0, cu_seqlens,
                                                   n_seqs, t_total, n_heads, o, hT, n_seg,
                                                   static_cast<float*>(workspace), order, nullptr,
                                                   stream)
              : launch_chunk_tc<kda::tc::MODE_KDA>(q, k, v, log_alpha, beta, h0, cu_seqlens,
                                                   n_seqs, t_total, n_heads, o, hT, n_seg,
                                                   static_cast<float*>(workspace), order, nullptr,
                                                   stream);
  }
  return chunk_simt_dispatch(q, k, v, log_alpha, beta, h0, cu_seqlens, n_seqs, t_total, n_heads,
                             qkv_dtype, o, hT, sg, stream);
}

}  // namespace

extern "C" {

int kda_chunk_fwd_simt(const void* q, const void* k, const void* v, const float* log_alpha,
                       const float* beta, const float* h0, const int32_t* cu_seqlens,
                       int32_t n_seqs, int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype,
                       void* o, float* hT, cudaStream_t stream) {
  int st = validate_chunk_args(q, k, v, log_alpha, beta, h0, cu_seqlens, n_seqs, t_total, n_heads,
                               qkv_dtype, o, hT);
  if (st != KDA_OK) return st;
  return chunk_simt_dispatch(q, k, v, log_alpha, beta, h0, cu_seqlens, n_seqs, t_total, n_heads,
                             qkv_dtype, o, hT, false, stream);
}

int kda_chunk_fwd(const void* q, const void* k, const void* v, const float* log_alpha,
                  const float* beta, const float* h0, const int32_t* cu_seqlens, int32_t n_seqs,
                  int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype, void* o, float* hT,
                  cudaStream_t stream) {
  return kda_chunk_fwd_ws(q, k, v, log_alpha, beta, h0, cu_seqlens, n_seqs, t_total, n_heads,
                          qkv_dtype, o, hT, nullptr, 0, stream);
}

size_t kda_chunk_fwd_workspace_size(int32_t n_seqs, int64_t t_total, int32_t n_heads,
                                    kda_dtype qkv_dtype, int has_cu_seqlens) {
  if (n_heads <= 0 || n_seqs <= 0 || t_total < 0) return 0;
  static const int32_t dummy = 0;
  const int32_t* cu = has_cu_seqlens ? &dummy : nullptr;
  const int n_seg = plan_segments(cu, n_seqs, t_total, n_heads, qkv_dtype, SIZE_MAX);
  if (n_seg >= 2) return split_workspace_bytes(n_seg, n_heads);
  if (has_cu_seqlens && n_seqs > 1 &&
      use_tc(&dummy, n_seqs, t_total, n_heads, qkv_dtype))
    return order_workspace_bytes(n_seqs, n_heads);
  return 0;
}

int kda_chunk_fwd_split_plan(int32_t n_heads, int64_t t_total, int32_t n_sms,
                             size_t workspace_bytes, int64_t* seg_bounds) {
  if (n_heads <= 0 || t_total < 0) return KDA_ERR_SHAPE;
  if (n_sms <= 0) n_sms = device_sms();
  if (n_sms <= 0) return KDA_ERR_CUDA;
  if (!use_tc(nullptr, 1, t_total, n_heads, KDA_BF16)) return 0;
  const int64_t n_chunks = (t_total + kda::CHUNK - 1) / kda::CHUNK;
  const int n_seg = split_segments(n_chunks, n_heads, n_sms, workspace_bytes);
  if (n_seg >= 2 && seg_bounds != nullptr) {
    const int base = (int)(n_chunks / n_seg), rem = (int)(n_chunks % n_seg);
    for (int j = 0; j < n_seg; ++j) seg_bounds[j] = kda::seg::seg_first_chunk(j, base, rem) * kda::CHUNK;
    seg_bounds[n_seg] = t_total;
  }
  return n_seg;
}

int kda_chunk_fwd_ws(const void* q, const void* k, const void* v, const float* log_alpha,
                     const float* beta, const float* h0, const int32_t* cu_seqlens, int32_t n_seqs,
                     int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype, void* o, float* hT,
                     void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return chunk_fwd_impl(q, k, v, log_alpha, beta, h0, cu_seqlens, n_seqs, t_total, n_heads,
                        qkv_dtype, o, hT, workspace, workspace_bytes, false, stream);
}

int kda_chunk_fwd_fused(const void* q_pre, const void* k_pre, const void* v,
                        const void* decay_pre, const float* beta_pre, const void* gate_pre,
                        const float* norm_w, const float* h0, const int32_t* cu_seqlens,
                        int32_t n_seqs, int64_t t_total, int32_t n_heads, void* o, float* hT,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  // (beta_pre is checked as beta is; decay_pre and gate_pre below)
  int st = validate_chunk_args(q_pre, k_pre, v, static_cast<const float*>(decay_pre), beta_pre, h0,
                               cu_seqlens, n_seqs, t_total, n_heads, KDA_BF16, o, hT);
  if (st != KDA_OK) return st;
  if (t_total > 0 && (!gate_pre || !norm_w)) return KDA_ERR_NULL;
  if ((gate_pre && !aligned16(gate_pre)) || (norm_w && !aligned16(norm_w))) return KDA_ERR_ALIGN;
  if (workspace && !aligned16(workspace)) return KDA_ERR_ALIGN;
  if (t_total == 0) {   // nothing to compute: the final state is the initial one
    if (hT != nullptr) {
      const size_t bytes = (size_t)n_seqs * n_heads * kda::D * kda::D * sizeof(float);
      const cudaError_t e = h0 ? cudaMemcpyAsync(hT, h0, bytes, cudaMemcpyDeviceToDevice, stream)
                               : cudaMemsetAsync(hT, 0, bytes, stream);
      if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    return KDA_OK;
  }
  if (!use_tc(cu_seqlens, n_seqs, t_total, n_heads, KDA_BF16)) return KDA_ERR_SHAPE;
  const int n_seg = workspace == nullptr ? 0 : plan_segments(cu_seqlens, n_seqs, t_total, n_heads,
                                                             KDA_BF16, workspace_bytes);
  int32_t* order = nullptr;
  const size_t ob = order_workspace_bytes(n_seqs, n_heads);
  if (n_seg == 0 && cu_seqlens != nullptr && workspace != nullptr && ob > 0 && workspace_bytes >= ob)
    order = static_cast<int32_t*>(workspace);
  const FusedIO fu = {decay_pre, beta_pre, gate_pre, norm_w};
  return launch_chunk_tc<kda::tc::MODE_FUSED>(q_pre, k_pre, v, nullptr, nullptr, h0, cu_seqlens,
                                              n_seqs, t_total, n_heads, o, hT, n_seg,
                                              static_cast<float*>(workspace), order, &fu, stream);
}

int kda_dplr_chunk_fwd(const void* q, const void* k, const void* v, const void* a, const void* b,
                       const float* log_alpha, const float* h0, const int32_t* cu_seqlens,
                       int32_t n_seqs, int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype,
                       void* o, float* hT, cudaStream_t stream) {
  int st = validate_chunk_args(q, k, v, log_alpha, log_alpha, h0, cu_seqlens, n_seqs, t_total,
                               n_heads, qkv_dtype, o, hT);
  if (st != KDA_OK) return st;
  if (t_total > 0 && (!a || !b)) return KDA_ERR_NULL;
  if ((a && !aligned16(a)) || (b && !aligned16(b))) return KDA_ERR_ALIGN;
  const size_t smem = sizeof(kda::DplrSmem);
  dim3 grid((unsigned)(n_seqs * n_heads), kda::D / kda::DPLR_DV);
  if (qkv_dtype == KDA_F32) {
    if (cudaFuncSetAttribute(kda::kda_dplr_simt_kernel<float>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return KDA_ERR_CUDA;
    kda::kda_dplr_simt_kernel<float><<<grid, kda::DPLR_THREADS, smem, stream>>>(
        static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
        static_cast<const float*>(a), static_cast<const float*>(b), log_alpha, h0, cu_seqlens,
        n_seqs, t_total, n_heads, static_cast<float*>(o), hT);
  } else {
    using bf = __nv_bfloat16;
    if (cudaFuncSetAttribute(kda::kda_dplr_simt_kernel<bf>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return KDA_ERR_CUDA;
    kda::kda_dplr_simt_kernel<bf><<<grid, kda::DPLR_THREADS, smem, stream>>>(
        static_cast<const bf*>(q), static_cast<const bf*>(k), static_cast<const bf*>(v),
        static_cast<const bf*>(a), static_cast<const bf*>(b), log_alpha, h0, cu_seqlens, n_seqs,
        t_total, n_heads, static_cast<bf*>(o), hT);
  }
  return launch_status();
}

int kda_short_conv_swish(const void* x, const float* w, const int32_t* cu_seqlens, int32_t n_seqs,
                         int64_t t_total, int32_t channels, void* y, cudaStream_t stream) {
  if (t_total < 0 || channels <= 0 || (channels & 7) != 0 || n_seqs <= 0) return KDA_ERR_SHAPE;
  if (cu_seqlens == nullptr && n_seqs != 1) return KDA_ERR_SEQLENS;
  if (t_total == 0) return KDA_OK;
  if (!x || !w || !y) return KDA_ERR_NULL;
  const void* ptrs[] = {x, w, y, cu_seqlens};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_ALIGN;
  if (x == y) return KDA_ERR_SHAPE;   // (no in-place: runs read the rows before them)
  using namespace kda::conv;
  const int64_t runs = (t_total + CONV_RUN - 1) / CONV_RUN;
  const int64_t threads = runs * (channels / 8);
  const int64_t blocks = (threads + CONV_THREADS - 1) / CONV_THREADS;
  if (blocks > (int64_t)INT32_MAX) return KDA_ERR_SHAPE;
  kda_short_conv_swish_kernel<<<(unsigned)blocks, CONV_THREADS, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), w, cu_seqlens, n_seqs, t_total, channels,
      static_cast<__nv_bfloat16*>(y));
  return launch_status();
}

int kda_gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* log_a,
                      const float* beta, const float* h0, const int32_t* cu_seqlens, int32_t n_seqs,
                      int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype, void* o, float* hT,
                      cudaStream_t stream) {
  return chunk_fwd_impl(q, k, v, log_a, beta, h0, cu_seqlens, n_seqs, t_total, n_heads, qkv_dtype,
                        o, hT, nullptr, 0, true, stream);
}

int kda_gdn_chunk_fwd_ws(const void* q, const void* k, const void* v, const float* log_a,
                         const float* beta, const float* h0, const int32_t* cu_seqlens,
                         int32_t n_seqs, int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype,
                         void* o, float* hT, void* workspace, size_t workspace_bytes,
                         cudaStream_t stream) {
  return chunk_fwd_impl(q, k, v, log_a, beta, h0, cu_seqlens, n_seqs, t_total, n_heads, qkv_dtype,
                        o, hT, workspace, workspace_bytes, true, stream);
}

int kda_chunk_fwd_static(const void* q, const void* k, const void* v, const float* log_alpha,
                         const float* beta, const float* h0, const int32_t* cu_seqlens,
                         int32_t n_seqs, int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype,
                         void* o, float* hT, cudaStream_t stream) {
  const int st = validate_chunk_args(q, k, v, log_alpha, beta, h0, cu_seqlens, n_seqs, t_total,
                                     n_heads, qkv_dtype, o, hT);
  if (st != KDA_OK) return st;
  // (the time split plans within the array; only a packed batch's launch order could
  // need more than it holds)
  if (cu_seqlens != nullptr &&
      kda_chunk_fwd_workspace_size(n_seqs, t_total, n_heads, qkv_dtype, 1) > KDA_STATIC_SCRATCH_BYTES)
    return KDA_ERR_SCRATCH;
  void* scratch = nullptr;
  const int sst = static_scratch_address(&scratch);
  if (sst != KDA_OK) return sst;
  return kda_chunk_fwd_ws(q, k, v, log_alpha, beta, h0, cu_seqlens, n_seqs, t_total, n_heads,
                          qkv_dtype, o, hT, scratch, KDA_STATIC_SCRATCH_BYTES, stream);
}

int kda_decode_step(const void* q, const void* k, const void* v, const void* log_alpha,
                    const void* beta, float* state, void* o, int32_t n_seqs, int32_t n_heads,
                    kda_dtype qkv_dtype, kda_dtype gate_dtype, cudaStream_t stream) {
  if ((qkv_dtype != KDA_F32 && qkv_dtype != KDA_BF16) ||
      (gate_dtype != KDA_F32 && gate_dtype != KDA_BF16))
    return KDA_ERR_DTYPE;
  if (n_seqs <= 0 || n_heads <= 0 || (int64_t)n_seqs * n_heads > (int64_t)INT32_MAX)
    return KDA_ERR_SHAPE;
  if (!q || !k || !v || !log_alpha || !beta || !state || !o) return KDA_ERR_NULL;
  const void* ptrs[] = {q, k, v, log_alpha, state, o};
  for (const void* p : ptrs)
    if (!aligned16(p)) return KDA_ERR_ALIGN;
  if (qkv_dtype == KDA_BF16) {
    if (gate_dtype == KDA_BF16)
      return launch_decode<__nv_bfloat16, __nv_bfloat16>(q, k, v, log_alpha, beta, state, o,
                                                         n_seqs, n_heads, stream);
    return launch_decode<__nv_bfloat16, float>(q, k, v, log_alpha, beta, state, o, n_seqs,
                                               n_heads, stream);
  }
  if (gate_dtype == KDA_BF16)
    return launch_decode<float, __nv_bfloat16>(q, k, v, log_alpha, beta, state, o, n_seqs,
                                               n_heads, stream);
  return launch_decode<float, float>(q, k, v, log_alpha, beta, state, o, n_seqs, n_heads, stream);
}

int kda_decode_tokens(const void* q, const void* k, const void* v, const void* log_alpha,
                      const void* beta, float* state, void* o, int32_t n_seqs, int32_t n_tokens,
                      int32_t n_heads, kda_dtype qkv_dtype, kda_dtype gate_dtype,
                      cudaStream_t stream) {
  if ((qkv_dtype != KDA_F32 && qkv_dtype != KDA_BF16) ||
      (gate_dtype != KDA_F32 && gate_dtype != KDA_BF16))
    return KDA_ERR_DTYPE;
  if (n_seqs <= 0 || n_heads <= 0 || n_tokens <= 0 || n_tokens > KDA_DECODE_MAX_TOKENS ||
      (int64_t)n_seqs * n_heads > (int64_t)INT32_MAX)
    return KDA_ERR_SHAPE;
  if (!q || !k || !v || !log_alpha || !beta || !state || !o) return KDA_ERR_NULL;
  const void* ptrs[] = {q, k, v, log_alpha, state, o};
  for (const void* p : ptrs)
    if (!aligned16(p)) return KDA_ERR_ALIGN;
  if (qkv_dtype == KDA_BF16) {
    if (gate_dtype == KDA_BF16)
      return launch_decode_tokens<__nv_bfloat16, __nv_bfloat16>(q, k, v, log_alpha, beta, state, o,
                                                                n_seqs, n_tokens, n_heads, stream);
    return launch_decode_tokens<__nv_bfloat16, float>(q, k, v, log_alpha, beta, state, o, n_seqs,
                                                      n_tokens, n_heads, stream);
  }
  if (gate_dtype == KDA_BF16)
    return launch_decode_tokens<float, __nv_bfloat16>(q, k, v, log_alpha, beta, state, o, n_seqs,
                                                      n_tokens, n_heads, stream);
  return launch_decode_tokens<float, float>(q, k, v, log_alpha, beta, state, o, n_seqs, n_tokens,
                                            n_heads, stream);
}

int kda_testing_chunk_fwd_stall(const void* q, const void* k, const void* v,
                                const float* log_alpha, const float* beta, const float* h0,
                                int64_t t_total, int32_t n_heads, void* o, float* hT,
                                int32_t skip_chunk, uint32_t wait_us, cudaStream_t stream) {
  int st = validate_chunk_args(q, k, v, log_alpha, beta, h0, nullptr, 1, t_total, n_heads, KDA_BF16,
                               o, hT);
  if (st != KDA_OK) return st;
  if (!use_tc(nullptr, 1, t_total, n_heads, KDA_BF16) || wait_us == 0) return KDA_ERR_SHAPE;
  return launch_chunk_tc<kda::tc::MODE_KDA>(q, k, v, log_alpha, beta, h0, nullptr, 1, t_total,
                                            n_heads, o, hT, 0, nullptr, nullptr, nullptr, stream,
                                            (uint64_t)wait_us * 1000ull, skip_chunk);
}

int kda_device_status(cudaStream_t stream) {
  int h = 0;
  if (cudaMemcpyFromSymbolAsync(&h, g_kda_device_error, sizeof(int), 0, cudaMemcpyDeviceToHost,
                                stream) != cudaSuccess)
    return KDA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return KDA_ERR_CUDA;
  if (h != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_kda_device_error, &zero, sizeof(int), 0,
                                cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
      return KDA_ERR_CUDA;
  }
  if (h & kda::DEVERR_TIMEOUT) return KDA_ERR_TIMEOUT;
  if (h & kda::DEVERR_SEQLENS) return KDA_ERR_SEQLENS;
  return KDA_OK;
}

const char* kda_status_string(int status) {
  switch (status) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_NULL: return "KDA_ERR_NULL: a required pointer is NULL";
    case KDA_ERR_SHAPE: return "KDA_ERR_SHAPE: a size is out of range";
    case KDA_ERR_DTYPE: return "KDA_ERR_DTYPE: unsupported dtype";
    case KDA_ERR_ALIGN: return "KDA_ERR_ALIGN: a tensor pointer is not 16-byte aligned";
    case KDA_ERR_SEQLENS: return "KDA_ERR_SEQLENS: cu_seqlens inconsistent";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: a CUDA call or launch failed";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a kernel gave up a bounded wait";
    case KDA_ERR_SCRATCH:
      return "KDA_ERR_SCRATCH: the call needs more scratch than the library's static array holds";
    default: return "unknown kda_status";
  }
}

}  // extern "C"
