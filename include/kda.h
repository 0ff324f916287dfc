/*
 * kda.h - C ABI of the B200 (sm_100a) Kimi Delta Attention library.
 *
 * Kimi Delta Attention (KDA) is the channel-wise gated delta rule of Kimi Linear
 * (Kimi Linear summary, section 3 "Kimi Delta Attention"):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * S is a per-(sequence, head) 128 x 128 fp32 state (row = key channel, column =
 * value channel), alpha_t in (0,1]^128 is a per-channel decay passed in log
 * space (log_alpha = log alpha <= 0), beta_t is a scalar per token and head,
 * and q, k are expected to be L2-normalised already (section 4: queries and keys
 * are normalised to unit length before the recurrence; this library applies no
 * normalisation and no output scale).
 *
 * Two operations:
 *   kda_chunk_fwd    prefill: the chunkwise-parallel form (chunks of 64 tokens,
 *                    WY representation + UT transform, section 3.1
 *                    "Hardware-Efficient Chunkwise Algorithm"), with an optional
 *                    initial state and the final state returned (appendix C:
 *                    chunk_kda with initial_state and chunk_size = 64).
 *   kda_decode_step  generation: one recurrent update per (sequence, head) on a
 *                    state held in place (section 6.3: autoregressive generation
 *                    uses recurrent updates on a fixed 128 x 128 state).
 *
 * Conventions for every entry point:
 *   - Head dimension is fixed: d_k = d_v = 128.
 *   - Every pointer is a DEVICE pointer owned by the caller. The library
 *     allocates no device memory and keeps no per-call state (scratch, where an
 *     entry point can use it, is a caller-provided workspace, or for
 *     kda_chunk_fwd_static a fixed array compiled into the library).
 *   - Calls are asynchronous and ordered on `stream`. A return of KDA_OK means
 *     "arguments validated and kernel launched"; device-side problems (bad
 *     cu_seqlens contents) are reported later by kda_device_status().
 *   - Tensor pointers must be 16-byte aligned; tensors are dense, row-major,
 *     token-major with the strides implied by the shapes below.
 *   - Outputs may not alias inputs (except the decode state, updated in place).
 */
#ifndef KDA_B200_H
#define KDA_B200_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

typedef enum {
  KDA_OK = 0,
  KDA_ERR_NULL = -1,     /* a required pointer is NULL */
  KDA_ERR_SHAPE = -2,    /* a size is out of range (n_heads <= 0, t_total < 0, ...) */
  KDA_ERR_DTYPE = -3,    /* unsupported dtype enum */
  KDA_ERR_ALIGN = -4,    /* a tensor pointer is not 16-byte aligned */
  KDA_ERR_SEQLENS = -5,  /* cu_seqlens inconsistent (host check, or reported by the device) */
  KDA_ERR_CUDA = -6,     /* a CUDA runtime call or kernel launch failed */
  KDA_ERR_TIMEOUT = -7,  /* a kernel gave up a bounded wait and skipped its work */
  KDA_ERR_SCRATCH = -8   /* kda_chunk_fwd_static: the call needs more scratch than
                            KDA_STATIC_SCRATCH_BYTES; nothing was launched */
} kda_status;

/*
 * kda_chunk_fwd - chunkwise KDA prefill over a packed batch of sequences.
 *
 * Computes, for every sequence n and head h, the recurrence above over the
 * sequence's tokens starting from h0[n,h] (or zero), writes o for every token and
 * the state after the sequence's last token to hT[n,h]. The sequence is cut into
 * chunks of 64 tokens, restarting at each sequence's first token, so no chunk
 * crosses a sequence boundary; the last chunk of a sequence may be shorter.
 *
 * Arguments:
 *   q, k, v     [t_total, n_heads, 128], dtype qkv_dtype (KDA_F32 or KDA_BF16)
 *   log_alpha   [t_total, n_heads, 128] fp32, entries finite and <= 0
 *   beta        [t_total, n_heads] fp32, normally in [0, 1]
 *   h0          [n_seqs, n_heads, 128, 128] fp32, or NULL for a zero initial state
 *   cu_seqlens  [n_seqs + 1] int32 on the device: sequence n owns tokens
 *               [cu_seqlens[n], cu_seqlens[n+1]); must start at 0, be
 *               non-decreasing and end at t_total. NULL means one sequence of
 *               t_total tokens (then n_seqs must be 1).
 *   n_seqs, t_total, n_heads   sizes (t_total may be 0)
 *   qkv_dtype   dtype of q, k, v and o
 *   o           [t_total, n_heads, 128] output, dtype qkv_dtype
 *   hT          [n_seqs, n_heads, 128, 128] fp32 output, or NULL to skip
 *   stream      CUDA stream for the launch
 *
 * Precision: KDA_F32 inputs take the fp32 CUDA-core path throughout. KDA_BF16
 * inputs take the tensor-core path (bf16 operands, fp32 accumulation, fp32 state).
 * Device-side cu_seqlens errors are clamped to stay in bounds and flagged for
 * kda_device_status().
 * Returns KDA_OK or a negative kda_status.
 */
int kda_chunk_fwd(const void* q, const void* k, const void* v, const float* log_alpha,
                  const float* beta, const float* h0, const int32_t* cu_seqlens, int32_t n_seqs,
                  int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype, void* o, float* hT,
                  cudaStream_t stream);

/*
 * kda_chunk_fwd_ws - kda_chunk_fwd with a caller-provided workspace, which lets a
 * single long bf16 sequence (cu_seqlens == NULL, n_seqs == 1) be split in time.
 *
 * Every step of the recurrence is affine in the state, so a run of chunks maps
 * its entering state S to M S + R (M: product of the per-token transitions,
 * R: the final state from a zero start), and its output is its output from a zero
 * start plus that of the same run from S with v = 0. With the time split the
 * sequence is cut into n >= 2 segments of whole chunks (balanced to within one
 * chunk). A first pass runs every segment in parallel, segment 0 from h0 and the
 * others from a zero state, storing their outputs and final states, together with
 * the M_j of the middle segments (from the identity with v = 0). A scan composes
 * the maps into the state entering every segment, and a second pass runs segments
 * 1 .. n-1 from those states with v = 0, adding their outputs onto o, and sets hT.
 * The M_j runs and the second pass stop once their state is exactly zero, which
 * the erase and the decay bring about within some tens of chunks on typical
 * inputs; without decay or erase they run to the ends of their segments. n is
 * chosen for the current device's SM count (see kda_chunk_fwd_split_plan). The
 * result is the same recurrence (exact in real arithmetic; fp32 state throughout,
 * bf16 MMA operands as in kda_chunk_fwd; the outputs of segments 1 .. n-1 are
 * rounded to bf16 twice, once per pass).
 *
 * Arguments: as kda_chunk_fwd, plus
 *   workspace        16-byte aligned device scratch, or NULL
 *   workspace_bytes  its size. The split takes the best plan whose scratch fits
 *                    ((2n - 2) * n_heads * 64 KiB); with NULL, or too little for
 *                    any split, the call is exactly kda_chunk_fwd (single pass).
 *                    kda_chunk_fwd_workspace_size(...) bytes give the best plan.
 * The workspace must stay untouched until the stream has passed the call.
 * Returns KDA_OK or a negative kda_status (KDA_ERR_ALIGN for a misaligned workspace).
 */
int kda_chunk_fwd_ws(const void* q, const void* k, const void* v, const float* log_alpha,
                     const float* beta, const float* h0, const int32_t* cu_seqlens, int32_t n_seqs,
                     int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype, void* o, float* hT,
                     void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * kda_chunk_fwd_split_plan - the time split kda_chunk_fwd_ws would use for one bf16
 * sequence of t_total tokens and n_heads heads, given workspace_bytes of scratch
 * (SIZE_MAX: as much as it wants), on a GPU with n_sms SMs (0: the current
 * device's). Host-only arithmetic: it launches nothing and, with n_sms > 0,
 * touches no device.
 *
 * Returns the number of segments n (0: no split, the single pass runs), or a
 * negative kda_status (KDA_ERR_SHAPE for n_heads <= 0 or t_total < 0,
 * KDA_ERR_CUDA if n_sms is 0 and the device cannot be queried). If seg_bounds is
 * not NULL and n >= 2, it receives n + 1 token offsets: segment j covers tokens
 * [seg_bounds[j], seg_bounds[j+1]), seg_bounds[0] = 0, seg_bounds[n] = t_total,
 * every inner offset a multiple of 64, segments balanced to within one chunk, every
 * segment at least 16 chunks. At most KDA_MAX_SEGMENTS segments.
 */
#define KDA_MAX_SEGMENTS 64
int kda_chunk_fwd_split_plan(int32_t n_heads, int64_t t_total, int32_t n_sms,
                             size_t workspace_bytes, int64_t* seg_bounds);

/*
 * kda_chunk_fwd_workspace_size - bytes of workspace that give kda_chunk_fwd_ws (and
 * kda_gdn_chunk_fwd_ws, and for bf16 kda_chunk_fwd_fused, which split alike) their
 * best time split for these sizes on the current device (0: no time split applies).
 * has_cu_seqlens is nonzero when the call will pass a cu_seqlens array (then no split
 * applies, and a packed batch of more CTAs than SMs uses 4 bytes per sequence).
 */
size_t kda_chunk_fwd_workspace_size(int32_t n_seqs, int64_t t_total, int32_t n_heads,
                                    kda_dtype qkv_dtype, int has_cu_seqlens);

/*
 * kda_chunk_fwd_static - kda_chunk_fwd for callers that cannot allocate device
 * memory. The Kimi Linear pages have no counterpart to this entry point: it is a
 * deployment variant of kda_chunk_fwd_ws whose scratch is a fixed array compiled
 * into this library instead of a buffer from the caller.
 *
 * Who cannot allocate: an op that runs as a plugin or custom kernel inside an
 * inference engine which has already reserved the GPU's memory for its own pool
 * and hands the op only its inputs and outputs (a cudaMalloc there fails, or eats
 * into memory the engine has promised elsewhere), and code on a latency-critical
 * path, where cudaMalloc and cudaFree are ruled out because they can synchronise
 * the whole device. Such callers still pass q, k, v, the gates, o and hT.
 *
 * Scratch: one __device__ array of KDA_STATIC_SCRATCH_BYTES (16 MiB), 256-byte
 * aligned, in every GPU context that loads the library, held until the process
 * exits. The time split of one long sequence plans within it ((2n - 2) * n_heads
 * * 64 KiB for n segments: 12 MiB for 32 heads in 4 segments), so for a few head
 * counts it splits into fewer segments than kda_chunk_fwd_ws given a workspace of
 * kda_chunk_fwd_workspace_size(...) bytes would. A packed batch of more CTAs than
 * SMs uses 4 bytes per sequence.
 *
 * Limit: a packed batch whose launch order needs more than KDA_STATIC_SCRATCH_BYTES
 * is rejected with KDA_ERR_SCRATCH before anything is launched (the order is kept
 * for at most 16,384 sequences, 64 KiB, so no call reaches it).
 *
 * Set-up: the first call in each device context, made with that device current,
 * looks up the array's device address (cudaGetSymbolAddress, which may load this
 * library's kernels onto the device) and keeps it, with the context, for later
 * calls; make that first call before any stream capture on the device. A new
 * context on the device (after cudaDeviceReset, say) looks the address up again.
 * A failed look-up returns KDA_ERR_CUDA.
 *
 * Sharing: every call on a device, from any stream or host thread, uses the same
 * array and leaves its contents behind. Nothing in it has to start at zero (each
 * call writes every scratch byte it reads before reading it), but calls whose
 * kernels overlap on the GPU race on the array and give wrong results: issue them
 * on one stream, or order them with events.
 *
 * Arguments, layouts, results and other errors: as kda_chunk_fwd.
 */
#define KDA_STATIC_SCRATCH_BYTES ((size_t)16 << 20)
int kda_chunk_fwd_static(const void* q, const void* k, const void* v, const float* log_alpha,
                         const float* beta, const float* h0, const int32_t* cu_seqlens,
                         int32_t n_seqs, int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype,
                         void* o, float* hT, cudaStream_t stream);

/*
 * kda_chunk_fwd_simt - the same operation as kda_chunk_fwd, always on the fp32
 * CUDA-core chunk kernel (exact element-wise decay factors, fp32 math). Same
 * arguments, layouts and errors. It is the precision path for fp32 inputs and a
 * second, independent GPU implementation of the chunk form for bf16 inputs.
 */
int kda_chunk_fwd_simt(const void* q, const void* k, const void* v, const float* log_alpha,
                       const float* beta, const float* h0, const int32_t* cu_seqlens,
                       int32_t n_seqs, int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype,
                       void* o, float* hT, cudaStream_t stream);

/*
 * kda_chunk_fwd_fused - kda_chunk_fwd with the producing layer's activations and the
 * output's post-processing fused into the kernel (Kimi Linear summary, section 4 "The
 * Kimi Linear Model Architecture"; Note, section "Other Components"; Deep-Dive,
 * section 5.3 "Neural Parameterization"). Per head:
 *
 *     q = L2norm(q_pre),  k = L2norm(k_pre)          (x / sqrt(sum x^2 + 1e-12))
 *     log alpha = logsigmoid(decay_pre)              (per channel)
 *     beta = sigmoid(beta_pre)
 *     (o, hT) = the KDA recurrence on (q, k, v, alpha, beta) from h0
 *     o_out = o / sqrt(mean(o^2) + 1e-6) * norm_w * sigmoid(gate_pre)   (head-wise RMSNorm
 *             over the 128 values of a head, then the output gate)
 *
 * The pages give no formula for the decay function (they call it a decay function of
 * a low-rank projection, like those of Gated DeltaNet and Mamba); logsigmoid is the
 * function the synthetic workloads use to draw log alpha. The short convolution and
 * Swish that precede the normalisation are a separate call (kda_short_conv_swish).
 * The kernel reads 256 bytes of decay per token and head instead of 512 and writes
 * the gated output directly: no separate passes over q, k or o.
 *
 * Arguments (bf16 = KDA_BF16 storage; every pointer a 16-byte aligned device pointer):
 *   q_pre, k_pre, v   [t_total, n_heads, 128] bf16 (q and k before normalisation)
 *   decay_pre         [t_total, n_heads, 128] bf16
 *   beta_pre          [t_total, n_heads] fp32
 *   gate_pre          [t_total, n_heads, 128] bf16
 *   norm_w            [128] fp32, shared by the heads
 *   h0, cu_seqlens, n_seqs, t_total, n_heads, hT, workspace, workspace_bytes:
 *                     as kda_chunk_fwd_ws, with the same time split of one long
 *                     sequence. The gated output is not linear in the state, so in
 *                     the split only segment 0's output is normalised and gated by
 *                     the chunk kernel; segments 1 .. n-1 are stored raw, take their
 *                     corrections, and a last pass over them (one more read and write
 *                     of o, one read of gate_pre) applies the norm and the gate
 *   o                 [t_total, n_heads, 128] bf16, the gated output
 * t_total must be 0 or at least 64 (the tensor-core path); otherwise KDA_ERR_SHAPE.
 * Returns KDA_OK or a negative kda_status.
 */
int kda_chunk_fwd_fused(const void* q_pre, const void* k_pre, const void* v,
                        const void* decay_pre, const float* beta_pre, const void* gate_pre,
                        const float* norm_w, const float* h0, const int32_t* cu_seqlens,
                        int32_t n_seqs, int64_t t_total, int32_t n_heads, void* o, float* hT,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * kda_dplr_chunk_fwd - chunkwise prefill of the general DPLR recurrence, the operator
 * the pages compare KDA's kernel against (Rationalist Deep-Dive, section 3.2 "DPLR
 * Structure"; Kimi Linear summary, sections 3.2 "Efficiency Analysis" and 6.2
 * "Relation to DPLR"):
 *
 *     S_t = (Diag(alpha_t) - a_t b_t^T) S_{t-1} + k_t v_t^T,   o_t = S_t^T q_t
 *
 * with free low-rank factors a_t, b_t (KDA ties them, a = beta k and b = k * alpha,
 * which reduces the chunk form's four decayed Gram matrices to two). This is a
 * comparison kernel: fp32 CUDA-core arithmetic with exact pairwise decay factors, in
 * the style of kda_chunk_fwd_simt, so the two chunk algorithms can be timed on the
 * same footing.
 *
 * Arguments: as kda_chunk_fwd (q, k, v, h0, cu_seqlens, sizes, dtype, o, hT), plus
 *   a, b   [t_total, n_heads, 128], dtype qkv_dtype
 * log_alpha [t_total, n_heads, 128] fp32 as for KDA. Returns KDA_OK or a negative
 * kda_status.
 */
int kda_dplr_chunk_fwd(const void* q, const void* k, const void* v, const void* a, const void* b,
                       const float* log_alpha, const float* h0, const int32_t* cu_seqlens,
                       int32_t n_seqs, int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype,
                       void* o, float* hT, cudaStream_t stream);

/*
 * kda_short_conv_swish - the short causal depthwise convolution (4 taps) and Swish
 * that turn the projections into q, k and v (Kimi Linear summary, section 4; Note,
 * section "Other Components": projection, short convolution, Swish; q and k are then
 * L2-normalised, which kda_chunk_fwd_fused does in its loader). For token t of a
 * sequence starting at token bos and every channel c:
 *
 *     y_t[c] = swish(w[c][0] x_{t-3}[c] + w[c][1] x_{t-2}[c] + w[c][2] x_{t-1}[c] + w[c][3] x_t[c])
 *
 * with x_s = 0 for s < bos (each sequence starts without history) and swish(u) =
 * u / (1 + e^{-u}). One call serves one tensor; q, k and v take three calls.
 *
 * Arguments (device pointers, 16-byte aligned):
 *   x           [t_total, channels] bf16 (channels = n_heads * 128 for q, k, v)
 *   w           [channels, 4] fp32, one filter per channel (tap 3 = current token)
 *   cu_seqlens  [n_seqs + 1] int32 or NULL (one sequence), as kda_chunk_fwd
 *   channels    a positive multiple of 8
 *   y           [t_total, channels] bf16 output; must not be x
 * Returns KDA_OK or a negative kda_status.
 */
int kda_short_conv_swish(const void* x, const float* w, const int32_t* cu_seqlens, int32_t n_seqs,
                         int64_t t_total, int32_t channels, void* y, cudaStream_t stream);

/*
 * kda_gdn_chunk_fwd - chunkwise prefill of Gated DeltaNet, the scalar-gate
 * specialisation of the same operator (Rationalist Deep-Dive, section 2.3
 * "Gated DeltaNet: The Scalar Forget"; Kimi Linear summary, section 2.2):
 *
 *     S_t = a_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t
 *
 * with ONE gate a_t in (0, 1] per token and head instead of KDA's 128 per-channel
 * gates. The scalar commutes with the erase, so this is exactly KDA with the same
 * log-decay on every channel; the kernels read 64 gate values per chunk instead of
 * a 64 x 128 tile (4 bytes per token and head instead of 512) and evaluate each
 * row's decay factor once. The Summary's efficiency comparison (section 5.6) puts
 * the two gates side by side; this entry point lets a caller do the same.
 *
 * Arguments, layouts, chunking, precision and errors: as kda_chunk_fwd, except
 *   log_a   [t_total, n_heads] fp32, log a_t (finite, <= 0)
 */
int kda_gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* log_a,
                      const float* beta, const float* h0, const int32_t* cu_seqlens, int32_t n_seqs,
                      int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype, void* o, float* hT,
                      cudaStream_t stream);

/*
 * kda_gdn_chunk_fwd_ws - kda_gdn_chunk_fwd with a caller-provided workspace for the
 * time split of one long bf16 sequence, exactly as kda_chunk_fwd_ws (same plan,
 * same workspace size: kda_chunk_fwd_workspace_size).
 */
int kda_gdn_chunk_fwd_ws(const void* q, const void* k, const void* v, const float* log_a,
                         const float* beta, const float* h0, const int32_t* cu_seqlens,
                         int32_t n_seqs, int64_t t_total, int32_t n_heads, kda_dtype qkv_dtype,
                         void* o, float* hT, void* workspace, size_t workspace_bytes,
                         cudaStream_t stream);

/*
 * kda_decode_step - one recurrent KDA update per (sequence, head), in place.
 *
 * For each of the n_seqs * n_heads states (section 6.3 "Complexity Analysis":
 * generation uses recurrent updates on the fixed state), with
 * alpha = exp(log_alpha):
 *     S' = Diag(alpha) S;  delta = beta (v - S'^T k);  S <- S' + k delta^T;
 *     o = S^T q   (computed as S'^T q + (k^T q) delta)
 *
 * Arguments:
 *   q, k, v     [n_seqs, n_heads, 128], dtype qkv_dtype
 *   log_alpha   [n_seqs, n_heads, 128], dtype gate_dtype, entries <= 0
 *   beta        [n_seqs, n_heads], dtype gate_dtype
 *   state       [n_seqs, n_heads, 128, 128] fp32, read and overwritten in place
 *   o           [n_seqs, n_heads, 128] output, dtype qkv_dtype
 *   qkv_dtype, gate_dtype   KDA_F32 or KDA_BF16 each
 * Returns KDA_OK or a negative kda_status.
 */
int kda_decode_step(const void* q, const void* k, const void* v, const void* log_alpha,
                    const void* beta, float* state, void* o, int32_t n_seqs, int32_t n_heads,
                    kda_dtype qkv_dtype, kda_dtype gate_dtype, cudaStream_t stream);

/*
 * kda_decode_tokens - n_tokens consecutive recurrent KDA updates per (sequence,
 * head), in place, reading the state once and writing it once.
 *
 * The same recurrence as kda_decode_step, applied to n_tokens new tokens of every
 * sequence in order (section 3; section 6.3: generation runs the recurrent form on
 * the fixed state). It serves multi-token and speculative decoding, where a few
 * tokens per sequence are processed at once: the state traffic, which dominates a
 * decode step, is paid once per call instead of once per token. The result equals
 * n_tokens consecutive kda_decode_step calls.
 *
 * Arguments:
 *   q, k, v     [n_seqs, n_tokens, n_heads, 128], dtype qkv_dtype (sequence-major,
 *               as a packed prefill batch of equal lengths)
 *   log_alpha   [n_seqs, n_tokens, n_heads, 128], dtype gate_dtype, entries <= 0
 *   beta        [n_seqs, n_tokens, n_heads], dtype gate_dtype
 *   state       [n_seqs, n_heads, 128, 128] fp32, read and overwritten in place
 *   o           [n_seqs, n_tokens, n_heads, 128] output, dtype qkv_dtype
 *   n_tokens    1 .. KDA_DECODE_MAX_TOKENS (KDA_ERR_SHAPE otherwise)
 * Returns KDA_OK or a negative kda_status.
 */
#define KDA_DECODE_MAX_TOKENS 16
int kda_decode_tokens(const void* q, const void* k, const void* v, const void* log_alpha,
                      const void* beta, float* state, void* o, int32_t n_seqs, int32_t n_tokens,
                      int32_t n_heads, kda_dtype qkv_dtype, kda_dtype gate_dtype,
                      cudaStream_t stream);

/*
 * kda_device_status - read and clear the library's device-side error word.
 * Synchronises `stream`. Returns KDA_OK, KDA_ERR_SEQLENS (a kernel saw
 * cu_seqlens that were not monotone or ran past t_total, and clamped them),
 * KDA_ERR_TIMEOUT (a kernel gave up a bounded wait), or KDA_ERR_CUDA.
 *
 * The error word is one per GPU context and process, not per call or per stream:
 * every kernel of this library on the device ORs its errors into it, and any
 * caller's read clears it. A caller that runs the library on several streams
 * cannot tell from it which call failed, and one stream's read hides an error
 * from the others; synchronise the streams and read it once where that matters.
 */
int kda_device_status(cudaStream_t stream);

/*
 * kda_testing_chunk_fwd_stall - TESTING ONLY: exercises the kernels' bounded waits.
 * The pages have no counterpart; this entry point exists so that a test can make a wait
 * run out without faulting or hanging the GPU.
 *
 * Runs kda_chunk_fwd's tensor-core kernel (one bf16 sequence, single pass) with every
 * wait bounded by wait_us microseconds instead of 2 s, and with the producer of chunk
 * skip_chunk's "T*beta ready" signal (a software mbarrier arrive; no copy or tensor-core
 * completion is skipped) leaving that one arrive out. The consumer's wait then runs out:
 * the kernel records KDA_ERR_TIMEOUT, every role leaves its loop, copies in flight are
 * awaited and tensor memory is freed, and the call's outputs are undefined. Read the
 * result with kda_device_status(). skip_chunk = -1 leaves nothing out.
 * Arguments as kda_chunk_fwd for one sequence (cu_seqlens NULL, n_seqs 1, bf16).
 * Returns KDA_OK (launched), KDA_ERR_SHAPE (t_total < 64 or wait_us = 0), or another
 * negative kda_status.
 */
int kda_testing_chunk_fwd_stall(const void* q, const void* k, const void* v,
                                const float* log_alpha, const float* beta, const float* h0,
                                int64_t t_total, int32_t n_heads, void* o, float* hT,
                                int32_t skip_chunk, uint32_t wait_us, cudaStream_t stream);

/* kda_status_string - a static, human-readable name for a kda_status value. */
const char* kda_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* KDA_B200_H */
