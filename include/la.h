/*
 * la.h — C ABI of the Lightning Attention layer kernel for NVIDIA B200 (sm_100a).
 *
 * What it computes.  The linear-attention layer of the hybrid Lightning Attention + MLA stack
 * described in "Ling and Ring 2.6 Technical Report" (Chinese translation,
 * garden.houmin.site/digest/ling-ring-2.6): §2.1, Fig. 2 places a "Linear Attention Kernel" between
 * QK-Norm/RoPE and a grouped RMSNorm with a sigmoid gate; §4.1.1 ("Context Parallel for Lightning
 * Attention") describes it as an RNN-style recurrence whose per-rank hidden state is shaped
 * [B,H,D,D].  The recurrence itself is the decayed causal linear attention of Lightning Attention
 * (TransNormerLLM, the report's reference 7), which the pages name but do not print:
 *
 *     S_t = lambda_h * S_{t-1} + k_t^T v_t          (S is d x d, S_{-1} = 0)
 *     o_t = q_t S_t  =  sum_{s<=t} lambda_h^(t-s) (q_t . k_s) v_s
 *
 * with lambda_h = exp(-slope_h).  No softmax, normaliser or scale is applied inside the kernel (the
 * report normalises the output afterwards, in the grouped RMSNorm of Fig. 2).
 *
 * Conventions shared by every entry point.
 *   - All tensor pointers are DEVICE pointers (cudaMalloc / PyTorch CUDA memory) unless a
 *     parameter says otherwise.  The caller owns every buffer; the library keeps no allocations,
 *     handles or global state between calls (the one exception is the fixed scratch array behind
 *     la_prefill_noalloc).
 *   - Activations q, k, v, out are laid out token-major, [B, N, H, d] contiguous (d innermost),
 *     as a fused QKV projection writes them.  Element type is bf16 (LA_BF16) or fp32 (LA_F32).
 *   - The recurrent state is always fp32, [B, H, d, d] contiguous, S[b][h][i][j] with i over the
 *     key dimension and j over the value dimension.
 *   - slopes: fp32[H] device array, slope_h >= 0, the decay is lambda_h = exp(-slope_h).
 *   - stream: a cudaStream_t passed as void*; NULL means the legacy default stream.  Calls are
 *     stream-ordered and asynchronous: a return of LA_OK means the work was enqueued.
 *   - Base pointers of q, k, v, out must be 16-byte aligned (tensor-memory-accelerator rule);
 *     otherwise LA_ERR_ALIGN.  out must not overlap q, k or v, and a state that an entry point
 *     writes (state_out, state_inout) must not overlap q, k, v or out (LA_ERR_ALIAS).
 *   - Argument errors are reported synchronously before anything is enqueued.  Launch errors
 *     map to LA_ERR_CUDA.  Nothing in the library calls exit(), abort() or a device trap.
 *   - All sizes and index arithmetic are 64-bit.
 */
#ifndef LA_H_
#define LA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LA_VERSION 1004 /* major*1000 + minor */

typedef enum {
  LA_OK = 0,
  LA_ERR_NULL = -1,        /* a required pointer is NULL */
  LA_ERR_SHAPE = -2,       /* B, N, H or d out of range (N >= 1, d in {64,128}, ...) */
  LA_ERR_DTYPE = -3,       /* dtype not LA_BF16 / LA_F32 */
  LA_ERR_ALIGN = -4,       /* a base pointer is not 16-byte aligned */
  LA_ERR_OVERFLOW = -5,    /* B*N*H*d or a byte size does not fit the 64-bit / tensor-map limits */
  LA_ERR_WORKSPACE = -6,   /* workspace too small (see la_prefill_workspace_bytes) */
  LA_ERR_CUDA = -7,        /* a CUDA runtime/driver call failed */
  LA_ERR_TIMEOUT = -8,     /* a device-side bounded wait gave up (reported by la_workspace_status) */
  LA_ERR_UNSUPPORTED = -9, /* valid arguments, but no kernel for this combination (e.g. chunk) */
  LA_ERR_ALIAS = -10       /* out overlaps an input */
} la_status;

typedef enum { LA_BF16 = 0, LA_F32 = 1 } la_dtype;

/* Which prefill kernel runs.  AUTO picks the tensor-core chunked kernel for bf16 with d = 128 and
 * the recurrent kernel otherwise.  RECURRENT forces the token-by-token CUDA-core kernel (any dtype
 * and d), which is also the fp32 path; TENSOR forces the chunked tcgen05 kernel (bf16, d = 128). */
typedef enum { LA_PATH_AUTO = 0, LA_PATH_TENSOR = 1, LA_PATH_RECURRENT = 2 } la_path;

/* Problem descriptor for la_prefill. */
typedef struct {
  int64_t B;        /* batch (independent sequences), >= 1 */
  int64_t N;        /* tokens per sequence, >= 1 */
  int64_t H;        /* heads, >= 1 */
  int64_t d;        /* head dimension, d_k = d_v = d, 64 or 128 */
  int32_t dtype;    /* la_dtype of q, k, v, out */
  int32_t chunk;    /* chunk length C of the tensor-core path: 0 = default (128), or 64, 128,
                       256 (every C computes the same recurrence; they differ only in where
                       the bf16 roundings of the intra / inter split fall); the recurrent path
                       takes 0 or 1 */
  int32_t segments; /* segments per sequence: 0 = automatic; >= 1 explicit (clamped to chunks);
                       LA_SEGMENTS_BALANCED = the balanced range plan (the tiles of all
                       sequences cut into one contiguous range per SM), which the automatic
                       choice takes for few long sequences */
  int32_t path;     /* la_path */
} la_desc;

/* la_desc.segments value that selects the balanced range plan (tensor path of la_prefill). */
#define LA_SEGMENTS_BALANCED (-1)

/* Bytes of device workspace la_prefill needs for this descriptor (0 if none).  The workspace holds
 * the segment-state ring, the scan flags, a work counter and a device status word. */
size_t la_prefill_workspace_bytes(const la_desc* desc);

/*
 * la_prefill — the whole prefill of one layer: o for every token and the final state.
 *
 * Chunked evaluation of the recurrence above ("chunk QKV", Fig. 10 of §4.1.1): within a chunk of
 * C tokens (desc->chunk: 64, 128 or 256) the intra-chunk term (Q K^T ⊙ M) V with
 * M_ij = lambda^(i-j) (i >= j, else 0) and the inter-chunk term diag(lambda^(i+1)) Q KV are
 * tensor-core contractions (the state KV enters them rounded to bf16 once per chunk); the fp32
 * state is carried as KV <- lambda^C KV + (K ⊙ lambda^(C-1-i))^T V.  Long sequences are cut into segments whose
 * local states are combined by a decayed prefix scan, the single-GPU form of the report's
 * "local recurrence, then global correction" (§4.1.1, Fig. 10: local h, fused update h / O).
 *
 *   desc       problem shape and options (host pointer, read during the call only)
 *   q, k, v    [B, N, H, d] device, dtype desc->dtype, read only
 *   slopes     fp32[H] device, read only
 *   out        [B, N, H, d] device, dtype desc->dtype, written (o_t for every token)
 *   state_out  fp32 [B, H, d, d] device, written (S_{N-1}); may be NULL if not wanted
 *   workspace  device scratch of at least la_prefill_workspace_bytes(desc) bytes, 256-byte aligned,
 *              used exclusively by this call until it completes on `stream`.  May be NULL: the
 *              library then allocates and frees it on `stream` (cudaMallocAsync/cudaFreeAsync).
 *   stream     cudaStream_t as void*
 *
 * Returns LA_OK when enqueued.  A device-side timeout of the segment scan (a bounded wait that
 * gave up; it cannot occur unless the GPU is starved for seconds) is recorded in the workspace's
 * status word, readable with la_workspace_status().
 */
la_status la_prefill(const la_desc* desc, const void* q, const void* k, const void* v,
                     const float* slopes, void* out, float* state_out, void* workspace,
                     size_t workspace_bytes, void* stream);

/*
 * la_decode_step — one generated token for B sequences: for every (b, h)
 *     S <- lambda_h S + k^T v   (in place, fp32),   o = q S   (read out after the update)
 * This is the per-token RNN-style update of §4.1.1; the state it continues is la_prefill's
 * state_out (prefix caching in the report's serving path).
 *
 *   B, H, d       batch, heads, head dim (64 or 128)
 *   dtype         la_dtype of q, k, v, out
 *   q, k, v       [B, H, d] device, read only
 *   slopes        fp32[H] device
 *   state_inout   fp32 [B, H, d, d] device, read and written in place
 *   out           [B, H, d] device, written
 *   stream        cudaStream_t as void*
 */
la_status la_decode_step(int64_t B, int64_t H, int64_t d, int32_t dtype, const void* q,
                         const void* k, const void* v, const float* slopes, float* state_inout,
                         void* out, void* stream);

/* Optional output epilogue (la_prefill_varlen, la_decode_multi): the step the report's layer
 * runs right after this kernel, a grouped RMSNorm of each head's output vector followed by the
 * sigmoid gate (§2.1 Fig. 2: Linear Attention Kernel -> Grouped RMSNorm, times sigmoid(Gate
 * Projection); §4.3 fuses "group norm + sigmoid gate" into one operator).  With it, out receives,
 * per token t and head h,
 *     y_j = gamma[h, j] * o_j / sqrt(mean_j(o_j^2) + eps) * sigmoid(g[t, h, j])
 * computed from the fp32 o (each head is one norm group of d channels) and rounded once to the
 * output dtype.  In la_prefill_varlen: tensor-core path only (bf16, d = 128). */
typedef struct {
  const void* gate;   /* like out, device: the gate pre-activation g = x W_gate, read only */
  const float* gamma; /* fp32 [H, d] device: the norm's weight, read only */
  float eps;          /* epsilon under the root, >= 0 (the report's RMSNorm uses 1e-6) */
  /* NULL: y is stored in out's dtype.  Otherwise the quantize step the report fuses after the
   * gate (§4.3 "group norm + sigmoid gate + quantize", ahead of the FP8 out_proj): y goes out as
   * FP8 E4M3 codes, one byte per value (uint8 [T, H, d]), and fp8_scales (fp32, device, 16-byte
   * aligned) receives one scale per block of a token's d values of one head, stored head-major
   * [H, T].  With y' = y rounded to the I/O dtype (what the unfused chain stores before its
   * quantize step):  scale = max_j |y'_j| / 448,  code_j = E4M3(y'_j * (448 / max_j |y'_j|))
   * (the product in fp32, rounded to nearest even, saturating at 448; an all-zero block gets
   * scale 0 and signed-zero codes), so that y_j ~= value(code_j) * scale.  Produced by
   * la_gate_norm_apply, the report's stand-alone post-attention operator; la_prefill_varlen and
   * la_decode_multi return LA_ERR_UNSUPPORTED for it. */
  float* fp8_scales;
} la_gate_norm;

/*
 * la_gate_norm_apply — the report's post-kernel operator on its own: grouped RMSNorm + sigmoid
 * gate over the kernel's output (§2.1 Fig. 2; §4.3 runs "group norm + sigmoid gate" as one fused
 * operator after attention).  For every token t and head h:
 *     y = gamma[h] * o / sqrt(mean(o^2) + eps) * sigmoid(g)       (one norm group per head)
 * The same computation as the la_gate_norm epilogue of la_prefill_varlen / la_decode_multi, run
 * as a separate memory-bound pass over o, g and y.
 *
 *   T, H, d     tokens (>= 0), heads, head dim (64 or 128); dtype: la_dtype of o, gate and y
 *   o           [T, H, d] device, read only
 *   gn          gate ([T, H, d] of dtype), gamma (fp32 [H, d]) and eps (>= 0), and optionally
 *               fp8_scales (then y is FP8 E4M3 codes, uint8 [T, H, d]); host pointer
 *   y           [T, H, d] device, written; may be o itself (in place, not with fp8_scales), no
 *               other overlap
 *   stream      cudaStream_t as void*
 */
la_status la_gate_norm_apply(int64_t T, int64_t H, int64_t d, int32_t dtype, const void* o,
                             const la_gate_norm* gn, void* y, void* stream);

/*
 * la_decode_multi — n_tok generated tokens per sequence in one step, for speculative
 * verification ("attention with MTP" in the report's serving path, §4.3): for every (b, h) and
 * j = 0 .. n_tok-1 in order,
 *     S <- lambda_h S + k_j^T v_j,   o_j = q_j S        (the la_decode_step rule per token)
 * The state is read and written once for all n_tok tokens, so its HBM traffic per token falls
 * as 1/n_tok.  With n_tok = 1 and no epilogue it computes exactly what la_decode_step does.
 *
 *   B, H, d       sequences, heads, head dim (64 or 128); n_tok >= 1 tokens per sequence
 *   dtype         la_dtype of q, k, v, out (and of the gate)
 *   q, k, v       [B, n_tok, H, d] device, read only
 *   slopes        fp32[H] device
 *   state_inout   fp32 [B, H, d, d] device, updated in place with all n_tok tokens
 *   epilogue      NULL, or the fused grouped RMSNorm + sigmoid gate of la_gate_norm applied to
 *                 every output row (gate [B, n_tok, H, d] of dtype, gamma fp32 [H, d])
 *   out           [B, n_tok, H, d] device, written
 *   stream        cudaStream_t as void*
 * Errors as la_decode_step (LA_ERR_SHAPE also for n_tok < 1; LA_ERR_ALIAS when out or the gate
 * overlaps another operand).
 */
la_status la_decode_multi(int64_t B, int64_t H, int64_t d, int64_t n_tok, int32_t dtype,
                          const void* q, const void* k, const void* v, const float* slopes,
                          float* state_inout, const la_gate_norm* epilogue, void* out,
                          void* stream);

/*
 * la_prefill_noalloc — la_prefill for callers that cannot allocate device memory.
 *
 * The report has no counterpart to this call; it exists for callers of this library that must
 * not call cudaMalloc (or any allocating routine) once they are running: serving loops that
 * reserved all device memory for their own pool allocator at start-up (a stray cudaMalloc would
 * fail, or synchronise the whole device and stall other streams), and host frameworks or plugin
 * interfaces that hand a kernel library its inputs and outputs but no allocator.
 *
 * Same computation, arguments and errors as la_prefill, minus the workspace: the scratch memory
 * (work counter, status word, scan flags and segment-state ring) is a fixed array of
 * LA_NOALLOC_SCRATCH_BYTES bytes compiled into the library.  Every GPU that loads the library
 * holds that array until the process exits.  The caller still passes q, k, v, slopes, out and
 * state_out.
 *
 *   - Limit: problems whose scratch need (la_prefill_workspace_bytes) exceeds
 *     LA_NOALLOC_SCRATCH_BYTES are rejected with LA_ERR_WORKSPACE before anything is enqueued.
 *     Within the limit is every problem with the automatic plan (desc->segments = 0) or the
 *     balanced plan (LA_SEGMENTS_BALANCED) on a GPU of up to 256 SMs, whatever B, N and H: those
 *     plans need at most a header plus one flag and one d x d fp32 state per SM.  An explicit
 *     segment count needs two states per sequence when it cuts sequences, which fits for B*H up
 *     to 128.  The fp32 / recurrent path needs no
 *     scratch at all.
 *   - First call on a device: it looks up the device address of the array (cudaGetSymbolAddress)
 *     with that device current and caches it for that device's CUDA context; make that first
 *     call before any stream capture.  If the context is destroyed and recreated (for example by
 *     cudaDeviceReset), the next call sees a new context and looks the address up again, so make
 *     that call outside stream capture too.
 *   - Sharing: all calls on a device use the same array, which keeps the previous call's
 *     contents; each call zeroes the parts that must start at zero.  Calls whose executions
 *     overlap on the GPU (different streams, or threads without ordering) race on the array and
 *     give wrong results; order them on one stream or use la_prefill with separate workspaces.
 *   - Device status: a bounded device wait that gives up (it needs the GPU to be starved for
 *     seconds) leaves the outputs invalid and is recorded only in the array, which this call
 *     offers no way to read; callers that must observe it use la_prefill with their own
 *     workspace and la_workspace_status.  For the same reason the call returns
 *     LA_ERR_UNSUPPORTED while the test-only failure injection (environment variable
 *     LA_DEBUG_WITHHOLD_SEGMENT) is set.
 */
#define LA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u + 4096u)
la_status la_prefill_noalloc(const la_desc* desc, const void* q, const void* k, const void* v,
                             const float* slopes, void* out, float* state_out, void* stream);

/* Problem descriptor for la_prefill_varlen: n_seqs sequences packed back to back along one token
 * axis of length T. */
typedef struct {
  int64_t T;        /* total tokens of all sequences, >= 0 */
  int64_t n_seqs;   /* sequences, >= 1 */
  int64_t H;        /* heads, >= 1 */
  int64_t d;        /* head dimension, 64 or 128 */
  int32_t dtype;    /* la_dtype of q, k, v, out */
  int32_t chunk;    /* as in la_desc */
  int32_t segments; /* segments per non-empty sequence: 0 = automatic; >= 1 explicit (clamped) */
  int32_t path;     /* la_path */
} la_varlen_desc;


/* Bytes of device workspace la_prefill_varlen needs (0 only for invalid arguments): an upper
 * bound over every cu_seqlens of this shape (the work-unit table holds at most
 * H * (n_seqs + ceil(T / 128)) units). */
size_t la_prefill_varlen_workspace_bytes(const la_varlen_desc* desc);

/*
 * la_prefill_varlen — la_prefill over variable-length sequences packed along one token axis
 * ("varlen"), each continuing from an optional initial state (a cached prefix).
 *
 * The report trains on packed inputs of many short sub-sequences and folds every sub-sequence's
 * state correction into one fused launch (§4.1.2, kernel fusion for variable-length sequences);
 * at serving time a prefill continues from a cached prefix state (§4.3, prefix caching).  Here
 * sequence s owns tokens [cu_seqlens[s], cu_seqlens[s+1]) of the packed tensors.  For each s and
 * head h the recurrence of la_prefill runs from S = state_in[s, h] (zero if state_in is NULL):
 *     S <- lambda_h S + k_t^T v_t,   o_t = q_t S,   state_out[s, h] = S after the last token.
 * A sequence of length 0 writes no output and passes its initial state through to state_out.
 * The call stays on the device: a one-block planning kernel reads cu_seqlens, checks it and
 * writes the table of work units (one segment of one sequence and head each), then one launch
 * of the kernel la_prefill uses (tensor-core or recurrent, by desc->path) runs them all.
 *
 *   desc        shape and options (host pointer, read during the call only)
 *   q, k, v     [T, H, d] device, dtype desc->dtype, read only (a [B, N, H, d] tensor is the packed
 *               layout of B sequences of N tokens)
 *   slopes      fp32[H] device
 *   cu_seqlens  DEVICE int64[n_seqs + 1]: cu_seqlens[0] = 0, non-decreasing, cu_seqlens[n_seqs] = T
 *   state_in    fp32 [n_seqs, H, d, d] device, or NULL for zero initial states; read only
 *   epilogue    NULL (out receives o), or the fused norm + gate above (host pointer, read during
 *               the call; gate and gamma 16-byte aligned, gate must not overlap out)
 *   out         [T, H, d] device, written
 *   state_out   fp32 [n_seqs, H, d, d] device, or NULL.  It may be the same pointer as state_in
 *               (in-place continuation); any other overlap with state_in is LA_ERR_ALIAS.
 *   workspace   device scratch of at least la_prefill_varlen_workspace_bytes(desc) bytes, 256-byte
 *               aligned, used only by this call until it completes on `stream`; NULL: allocated
 *               and freed on `stream` (cudaMallocAsync / cudaFreeAsync)
 *   stream      cudaStream_t as void*
 *
 * Errors returned by the call: shape, dtype, NULL, alignment and aliasing errors as for
 * la_prefill (q, k, v, out, state_in, state_out must be 16-byte aligned).  cu_seqlens lives on the
 * device, so its contents are checked there: if it is not a non-decreasing run from 0 to T, the
 * planning kernel records LA_ERR_SHAPE in the workspace status word (la_workspace_status), no
 * kernel touches out or state_out, and the call itself has returned LA_OK.  A scan timeout is
 * reported the same way as for la_prefill.
 */
la_status la_prefill_varlen(const la_varlen_desc* desc, const void* q, const void* k,
                            const void* v, const float* slopes, const int64_t* cu_seqlens,
                            const float* state_in, const la_gate_norm* epilogue, void* out,
                            float* state_out, void* workspace, size_t workspace_bytes,
                            void* stream);

/* Shape and options of la_qk_norm_rope. */
typedef struct {
  int64_t T;          /* tokens (>= 0) */
  int64_t H;          /* heads (>= 1) */
  int64_t d;          /* head dimension, 64 or 128 */
  int64_t q_stride;   /* elements from token t to token t+1 of q, >= H*d, a multiple of 8 */
  int64_t k_stride;   /* the same for k (so q and k may be views into one fused projection) */
  int32_t rotary_dim; /* rotated dims r: a multiple of 16 in [16, d] (the report: 64) */
  float theta;        /* rotary base, > 0 (the report: 6,000,000) */
  float eps;          /* RMSNorm epsilon, >= 0 (the report: 1e-6) */
  int32_t pad;
} la_qk_norm_rope_desc;

/*
 * la_qk_norm_rope — the fused operator before the kernel: QK RMSNorm and partial rotary
 * embedding of q and k ("Ling and Ring 2.6 Technical Report", §2.1 Fig. 2: QK Norm -> RoPE ->
 * Linear Attention Kernel; §2.1.1: RMSNorm eps 1e-6, rotary dim 64 of 128, theta 6e6; §4.3: split +
 * QK norm + RoPE fused into one inference operator).  For every token t, head h and x in {q, k}:
 *     y = gamma_x * x / sqrt(mean(x^2) + eps)                      (norm over the d channels)
 *     (y_i, y_{i+r/2}) <- (y_i cos a - y_{i+r/2} sin a, y_{i+r/2} cos a + y_i sin a)
 *     with a = positions[t] * theta^(-2i/r) for i < r/2; dims >= r keep the normalised value.
 * The angle is formed and reduced modulo 2 pi in double precision before sin/cos.
 *
 *   desc        shape and options (host pointer, read during the call only)
 *   q, k        bf16 device, token t of head h at q + t*q_stride + h*d (16-byte aligned)
 *   gamma_q/_k  fp32 [d] device: the two norms' weights (shared by the heads)
 *   positions   int64 [T] device: each token's position in its sequence (for prefill of a
 *               cached prefix continuation, the prefix length is added by the caller)
 *   q_out/k_out bf16 [T, H, d] device, written; each may be its input itself (in place, when that
 *               input is contiguous), any other overlap with an input is LA_ERR_ALIAS
 *   stream      cudaStream_t as void*
 */
la_status la_qk_norm_rope(const la_qk_norm_rope_desc* desc, const void* q, const void* k,
                          const float* gamma_q, const float* gamma_k, const int64_t* positions,
                          void* q_out, void* k_out, void* stream);

/* The QK RMSNorm + partial RoPE of la_qk_norm_rope, applied by la_prefill_varlen_qk inside the
 * prefill kernel. */
typedef struct {
  const float* gamma_q;     /* fp32 [d] device, 16-byte aligned: q's norm weight (all heads) */
  const float* gamma_k;     /* fp32 [d] device, 16-byte aligned: k's norm weight */
  const int64_t* positions; /* int64 [T] device: each packed token's position in its sequence */
  int32_t rotary_dim;       /* rotated dims r: a multiple of 16 in [16, d] (the report: 64) */
  float theta;              /* rotary base, > 0 (the report: 6,000,000) */
  float eps;                /* RMSNorm epsilon, >= 0 (the report: 1e-6) */
  int32_t pad;
} la_qk_prologue;

/*
 * la_prefill_varlen_qk — la_prefill_varlen whose q and k are the raw projections: the kernel
 * applies the report's QK Norm and RoPE (§2.1 Fig. 2: QKV Projection -> QK Norm -> RoPE ->
 * Linear Attention Kernel; §2.1.1) to each q and k tile in shared memory before any product
 * reads it, so q_hat and k_hat never exist in device memory.  The result equals
 *     la_qk_norm_rope(q, k, ... positions ...) followed by la_prefill_varlen(q_hat, k_hat, v, ...)
 * exactly (the tiles hold the very bf16 rows la_qk_norm_rope stores), with the same segments.
 *
 *   desc        as for la_prefill_varlen; the tensor-core path only (bf16, d = 128, path AUTO or
 *               TENSOR, chunk 0 or 128), else LA_ERR_UNSUPPORTED
 *   qk          the norm + RoPE parameters (host pointer, read during the call); NULL:
 *               LA_ERR_NULL.  positions: 8-byte aligned, one entry per packed token
 *   q, k, v     [T, H, d] bf16 device (contiguous), read only: q and k are not modified
 *   other arguments, the workspace (la_prefill_varlen_workspace_bytes) and the errors as for
 *   la_prefill_varlen; there is no fused output epilogue here (out receives o).
 *
 * Speed: the transform runs on four warps between a tile's arrival and its first product, so
 * this call is currently slower than la_qk_norm_rope (which may write q_hat, k_hat in place over
 * q, k) followed by la_prefill_varlen.  It is for callers whose q and k must stay as they are and
 * who cannot hold a second copy of them.
 */
la_status la_prefill_varlen_qk(const la_varlen_desc* desc, const la_qk_prologue* qk,
                               const void* q, const void* k, const void* v, const float* slopes,
                               const int64_t* cu_seqlens, const float* state_in, void* out,
                               float* state_out, void* workspace, size_t workspace_bytes,
                               void* stream);

/* Bytes of device workspace la_prefill_state needs for this descriptor (0 for invalid
 * arguments or when the recurrent path runs, which needs none). */
size_t la_prefill_state_workspace_bytes(const la_desc* desc);

/*
 * la_prefill_state — the final state of a prefill without its outputs: for every (b, h)
 *     state_out = lambda^N state_in + sum_{t<N} lambda^(N-1-t) k_t^T v_t
 * (state_in NULL: zero).  This is the "local h" of the report's context-parallel forward (§4.1.1,
 * Fig. 10): each rank holding one part of a long sequence computes its part's state from its own
 * K, V, the states are gathered, and la_state_fold turns those of the earlier parts into the
 * rank's incoming state, from which la_prefill_varlen (state_in) computes the rank's outputs.
 * Reads K and V once (no q, no output); on the tensor path it is one row-scaled contraction
 * K~^T V per head (K~_t = lambda^(N-1-t) k_t) accumulated in fp32.
 *
 *   desc       as for la_prefill (B, N >= 1, H, d, dtype, path; chunk and segments ignored)
 *   k, v       [B, N, H, d] device, dtype desc->dtype, read only
 *   slopes     fp32[H] device
 *   state_in   fp32 [B, H, d, d] device or NULL, read only
 *   state_out  fp32 [B, H, d, d] device, written; may be state_in itself (in place)
 *   workspace  device scratch of la_prefill_state_workspace_bytes(desc) bytes, 256-byte aligned,
 *              or NULL (allocated and freed on `stream`)
 *   stream     cudaStream_t as void*
 * A device-side timeout is recorded in the workspace status word (la_workspace_status).
 */
la_status la_prefill_state(const la_desc* desc, const void* k, const void* v, const float* slopes,
                           const float* state_in, float* state_out, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * la_state_fold — the report's "fused update h" (§4.1.1, Fig. 10): the incoming state of part
 * n of a sequence cut into consecutive parts of lengths[0..n-1] tokens, from the parts' local
 * states h_j (la_prefill_state with no state_in) and the sequence's initial state:
 *     S = state_in (or 0);   S <- lambda^lengths[j] S + h_j   for j = 0 .. n_parts-1
 * per flat head (BH = batch * H of them).  n_parts = 0 copies state_in (or writes zeros).
 *
 *   n_parts    0 .. 256
 *   BH, H, d   flat heads (a multiple of H), heads, head dim (64 or 128)
 *   parts      fp32 [n_parts, BH, d, d] device, read only (may be NULL when n_parts = 0)
 *   lengths    int64 [n_parts] HOST, each >= 0
 *   slopes     fp32[H] device
 *   state_in   fp32 [BH, d, d] device or NULL
 *   state_out  fp32 [BH, d, d] device, written; may be state_in, must not overlap parts
 */
la_status la_state_fold(int64_t n_parts, int64_t BH, int64_t H, int64_t d, const float* parts,
                        const int64_t* lengths, const float* slopes, const float* state_in,
                        float* state_out, void* stream);

/* Synchronises `stream`, then returns the device status word of a workspace that la_prefill
 * used: LA_OK, or LA_ERR_TIMEOUT if a bounded device wait gave up during the last call. */
la_status la_workspace_status(const void* workspace, void* stream);

/* Static description of a status code (never NULL). */
const char* la_status_string(int status);

/* LA_VERSION of the built library. */
int la_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LA_H_ */
