// la_api.cu — the C ABI declared in include/la.h: argument validation, kernel selection and
// workspace handling.  No torch types cross this boundary; every pointer is a plain device
// pointer owned by the caller.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "la.h"
#include "la_internal.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

// a * b without signed overflow; false if it would exceed INT64_MAX.
bool mul_ok(int64_t a, int64_t b, int64_t* out) {
  if (a < 0 || b < 0) return false;
  if (a != 0 && b > INT64_MAX / a) return false;
  *out = a * b;
  return true;
}

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

bool use_tensor_path(int32_t path, int32_t dtype, int64_t d) {
  if (path == LA_PATH_RECURRENT) return false;
  if (path == LA_PATH_TENSOR) return true;
  return dtype == LA_BF16 && d == la::kHeadDim;
}
bool use_tensor_path(const la_desc* d) { return use_tensor_path(d->path, d->dtype, d->d); }

// The tensor path's chunk length for a descriptor's `chunk` field (0: the library's default).
int chunk_of(int32_t chunk) { return chunk == 0 ? la::kChunkDefault : chunk; }

// The work plan of la_prefill's tensor path: balanced ranges (returns true, fills *bal) when asked
// for or when the automatic choice prefers them, else equal segments per sequence (fills *seg).
bool compute_plan(const la_desc* d, int sms, la::BalancedPlan* bal, la::SegmentPlan* seg) {
  const int chunk = chunk_of(d->chunk);
  if (d->segments == LA_SEGMENTS_BALANCED) {
    *bal = la::plan_balanced(d->B, d->N, d->H, sms, chunk);
    return true;
  }
  if (d->segments == 0) return la::prefer_balanced(d->B, d->N, d->H, sms, chunk, bal, seg);
  *seg = la::plan_segments(d->B, d->N, d->H, d->segments, sms, chunk);
  return false;
}

// The balanced plan's search takes 0.1-0.25 ms of host time, as long as a short prefill itself, so
// the last few plans are kept, keyed by everything they depend on (shared by all host threads).
struct PlanCacheEntry {
  int64_t B = 0, N = 0, H = 0;
  int32_t sms = 0, chunk = 0, segments = 0;
  bool valid = false, balanced = false;
  la::BalancedPlan bal{};
  la::SegmentPlan seg{};
};
constexpr int kPlanCacheSize = 8;
std::mutex g_plan_mu;
PlanCacheEntry g_plan_cache[kPlanCacheSize];
int g_plan_next = 0;

bool choose_plan(const la_desc* d, int sms, la::BalancedPlan* bal, la::SegmentPlan* seg) {
  const int32_t chunk = chunk_of(d->chunk);
  {
    std::lock_guard<std::mutex> lk(g_plan_mu);
    for (const PlanCacheEntry& e : g_plan_cache) {
      if (e.valid && e.B == d->B && e.N == d->N && e.H == d->H && e.sms == sms &&
          e.chunk == chunk && e.segments == d->segments) {
        if (e.balanced) *bal = e.bal; else *seg = e.seg;
        return e.balanced;
      }
    }
  }
  PlanCacheEntry e;
  e.balanced = compute_plan(d, sms, &e.bal, &e.seg);
  e.B = d->B;
  e.N = d->N;
  e.H = d->H;
  e.sms = sms;
  e.chunk = chunk;
  e.segments = d->segments;
  e.valid = true;
  if (e.balanced) *bal = e.bal; else *seg = e.seg;
  std::lock_guard<std::mutex> lk(g_plan_mu);
  g_plan_cache[g_plan_next] = e;
  g_plan_next = (g_plan_next + 1) % kPlanCacheSize;
  return e.balanced;
}

// Workspace bytes of la_prefill's tensor path for its plan.
size_t prefill_workspace_need(const la_desc* d, int sms) {
  la::BalancedPlan bal{};
  la::SegmentPlan seg{};
  if (choose_plan(d, sms, &bal, &seg)) return la::balanced_workspace_bytes(bal);
  return la::workspace_layout(d->B, d->H, seg).total;
}

// Failure injection for tests, read on every call: LA_DEBUG_WITHHOLD_SEGMENT=k keeps segment k of
// every sequence from publishing its scan state, so segment k+1 waits until its bounded wait
// expires (LA_DEBUG_WAIT_LIMIT_MS, default 2000) and the call reports LA_ERR_TIMEOUT through
// la_workspace_status.  Unset in normal use.
void apply_debug_env(la::PrefillArgs& a) {
  if (const char* e = getenv("LA_DEBUG_WITHHOLD_SEGMENT")) a.withhold_segment = atoi(e);
  if (const char* e = getenv("LA_DEBUG_WAIT_LIMIT_MS")) {
    const long ms = atol(e);
    if (ms > 0 && ms <= 60000) a.wait_limit_ns = static_cast<uint64_t>(ms) * 1000000ull;
  }
}

// Validates a prefill descriptor; on success writes the element count of one activation tensor.
la_status check_desc(const la_desc* d, int64_t* numel) {
  if (d == nullptr) return LA_ERR_NULL;
  if (d->dtype != LA_BF16 && d->dtype != LA_F32) return LA_ERR_DTYPE;
  if (d->B < 1 || d->N < 1 || d->H < 1 || (d->d != 64 && d->d != 128)) return LA_ERR_SHAPE;
  if (d->path != LA_PATH_AUTO && d->path != LA_PATH_TENSOR && d->path != LA_PATH_RECURRENT)
    return LA_ERR_UNSUPPORTED;
  if (d->segments < LA_SEGMENTS_BALANCED) return LA_ERR_SHAPE;
  int64_t t = 0, bytes = 0;
  if (!mul_ok(d->B, d->N, &t) || !mul_ok(t, d->H, &t) || !mul_ok(t, d->d, &t))
    return LA_ERR_OVERFLOW;
  if (!mul_ok(t, d->dtype == LA_BF16 ? 2 : 4, &bytes)) return LA_ERR_OVERFLOW;
  int64_t st = 0;
  if (!mul_ok(d->B, d->H, &st) || !mul_ok(st, d->d * d->d * 4, &st)) return LA_ERR_OVERFLOW;
  if (d->B * d->H > INT32_MAX) return LA_ERR_OVERFLOW;  // grid / flat-head index range
  if (use_tensor_path(d)) {
    if (d->dtype != LA_BF16 || d->d != la::kHeadDim) return LA_ERR_UNSUPPORTED;
    if (d->chunk != 0 && !la::chunk_supported(d->chunk)) return LA_ERR_UNSUPPORTED;
    // tensor-map coordinates are 32-bit; byte strides below 2^40
    if (d->N > INT32_MAX - la::kChunk || d->H > INT32_MAX || d->B > INT32_MAX)
      return LA_ERR_OVERFLOW;
    int64_t row = 0;
    if (!mul_ok(d->N, d->H * d->d * 2, &row) || row >= (int64_t(1) << 40)) return LA_ERR_OVERFLOW;
  } else if (d->chunk != 0 && d->chunk != 1) {
    return LA_ERR_UNSUPPORTED;  // the recurrent path has no chunking
  }
  *numel = t;
  return LA_OK;
}

// Validates a varlen descriptor (cu_seqlens is a device array: its contents are checked by the
// planning kernel); on success writes the element count of one packed activation tensor.
la_status check_varlen(const la_varlen_desc* d, int64_t* numel) {
  if (d == nullptr) return LA_ERR_NULL;
  if (d->dtype != LA_BF16 && d->dtype != LA_F32) return LA_ERR_DTYPE;
  if (d->T < 0 || d->n_seqs < 1 || d->H < 1 || (d->d != 64 && d->d != 128)) return LA_ERR_SHAPE;
  if (d->path != LA_PATH_AUTO && d->path != LA_PATH_TENSOR && d->path != LA_PATH_RECURRENT)
    return LA_ERR_UNSUPPORTED;
  if (d->segments < 0) return LA_ERR_SHAPE;
  int64_t t = 0, bytes = 0, st = 0, nh = 0;
  if (!mul_ok(d->T, d->H, &t) || !mul_ok(t, d->d, &t)) return LA_ERR_OVERFLOW;
  if (!mul_ok(t, d->dtype == LA_BF16 ? 2 : 4, &bytes)) return LA_ERR_OVERFLOW;
  if (!mul_ok(d->n_seqs, d->H, &nh) || nh > INT32_MAX || !mul_ok(nh, d->d * d->d * 4, &st))
    return LA_ERR_OVERFLOW;
  if (use_tensor_path(d->path, d->dtype, d->d)) {
    if (d->dtype != LA_BF16 || d->d != la::kHeadDim) return LA_ERR_UNSUPPORTED;
    if (d->chunk != 0 && !la::chunk_supported(d->chunk)) return LA_ERR_UNSUPPORTED;
    // token coordinates of the tensor maps and work units are 32-bit, and so is the unit count
    if (d->T > INT32_MAX - la::kChunk) return LA_ERR_OVERFLOW;
    int64_t cap = 0;
    if (!mul_ok(d->H, d->n_seqs + (d->T + la::kChunk - 1) / la::kChunk, &cap) || cap > INT32_MAX)
      return LA_ERR_OVERFLOW;
    int64_t row = 0;
    if (!mul_ok(d->T, d->H * d->d * 2, &row) || row >= (int64_t(1) << 40)) return LA_ERR_OVERFLOW;
  } else if (d->chunk != 0 && d->chunk != 1) {
    return LA_ERR_UNSUPPORTED;
  }
  *numel = t;
  return LA_OK;
}

}  // namespace

extern "C" {

size_t la_prefill_workspace_bytes(const la_desc* desc) {
  int64_t numel = 0;
  if (check_desc(desc, &numel) != LA_OK) return 0;
  if (!use_tensor_path(desc)) return 0;
  return prefill_workspace_need(desc, device_sms() > 0 ? device_sms() : 148);
}

}  // extern "C"

namespace {

// Argument checks of la_prefill (and la_prefill_noalloc): descriptor, pointers, alignment and
// overlaps, all before any CUDA call.
la_status check_prefill_args(const la_desc* desc, const void* q, const void* k, const void* v,
                             const float* slopes, const void* out, const float* state_out) {
  int64_t numel = 0;
  const la_status st = check_desc(desc, &numel);
  if (st != LA_OK) return st;
  if (!q || !k || !v || !slopes || !out) return LA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return LA_ERR_ALIGN;
  if (state_out != nullptr && !aligned16(state_out)) return LA_ERR_ALIGN;
  const size_t bytes = static_cast<size_t>(numel) * (desc->dtype == LA_BF16 ? 2 : 4);
  if (overlaps(out, bytes, q, bytes) || overlaps(out, bytes, k, bytes) ||
      overlaps(out, bytes, v, bytes))
    return LA_ERR_ALIAS;
  if (state_out != nullptr) {
    // the final state is written while other CTAs still read q, k, v and write out
    const size_t sb = static_cast<size_t>(desc->B * desc->H) * static_cast<size_t>(desc->d * desc->d) * 4;
    if (overlaps(state_out, sb, q, bytes) || overlaps(state_out, sb, k, bytes) ||
        overlaps(state_out, sb, v, bytes) || overlaps(state_out, sb, out, bytes))
      return LA_ERR_ALIAS;
  }
  return LA_OK;
}

}  // namespace

extern "C" {

la_status la_prefill(const la_desc* desc, const void* q, const void* k, const void* v,
                     const float* slopes, void* out, float* state_out, void* workspace,
                     size_t workspace_bytes, void* stream) {
  const la_status st = check_prefill_args(desc, q, k, v, slopes, out, state_out);
  if (st != LA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  la::PrefillArgs a{desc->B, desc->N, desc->H, desc->d, desc->dtype, q, k, v, slopes, out,
                    state_out};
  a.chunk = chunk_of(desc->chunk);
  apply_debug_env(a);
  if (!use_tensor_path(desc)) {
    return la::launch_recurrent_prefill(a, s) == cudaSuccess ? LA_OK : LA_ERR_CUDA;
  }
  const int sms = device_sms();
  if (sms <= 0) return LA_ERR_CUDA;
  la::BalancedPlan bplan{};
  la::SegmentPlan splan{};
  const bool balanced = choose_plan(desc, sms, &bplan, &splan);
  const size_t need = balanced ? la::balanced_workspace_bytes(bplan)
                               : la::workspace_layout(desc->B, desc->H, splan).total;
  void* ws = workspace;
  bool owned = false;
  if (ws == nullptr) {
    if (cudaMallocAsync(&ws, need, s) != cudaSuccess) return LA_ERR_CUDA;
    owned = true;
  } else {
    if (workspace_bytes < need) return LA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return LA_ERR_ALIGN;
  }
  const cudaError_t e = balanced ? la::launch_chunked_prefill_balanced(a, bplan, ws, s, sms)
                                 : la::launch_chunked_prefill(a, splan, ws, s, sms);
  if (owned) cudaFreeAsync(ws, s);
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

size_t la_prefill_varlen_workspace_bytes(const la_varlen_desc* desc) {
  int64_t numel = 0;
  if (check_varlen(desc, &numel) != LA_OK) return 0;
  const bool tensor = use_tensor_path(desc->path, desc->dtype, desc->d);
  const int sms = device_sms() > 0 ? device_sms() : 148;
  return la::varlen_workspace_layout(desc->T, desc->n_seqs, desc->H, desc->segments, sms, tensor)
      .total;
}

}  // extern "C"

namespace {

// Rotary frequencies theta^(-2i / r), i < r / 2, in double (one routine for both QK operators,
// so that the in-tile form reproduces the stand-alone one exactly).
void rope_inv_freq(double* inv_freq, int rotary_dim, float theta) {
  const double log_theta = std::log(static_cast<double>(theta));
  for (int i = 0; i < rotary_dim / 2; ++i)
    inv_freq[i] = std::exp(-2.0 * i / rotary_dim * log_theta);
}

// The body of la_prefill_varlen and la_prefill_varlen_qk (qk: the in-tile QK norm + RoPE, or
// null).
la_status prefill_varlen_impl(const la_varlen_desc* desc, const la_qk_prologue* qk,
                              const void* q, const void* k, const void* v, const float* slopes,
                              const int64_t* cu_seqlens, const float* state_in,
                              const la_gate_norm* epilogue, void* out, float* state_out,
                              void* workspace, size_t workspace_bytes, void* stream) {
  int64_t numel = 0;
  const la_status st = check_varlen(desc, &numel);
  if (st != LA_OK) return st;
  if (!q || !k || !v || !slopes || !out || !cu_seqlens) return LA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return LA_ERR_ALIGN;
  if ((state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)))
    return LA_ERR_ALIGN;
  const size_t bytes = static_cast<size_t>(numel) * (desc->dtype == LA_BF16 ? 2 : 4);
  const size_t state_bytes =
      static_cast<size_t>(desc->n_seqs * desc->H) * static_cast<size_t>(desc->d * desc->d) * 4;
  if (bytes > 0 && (overlaps(out, bytes, q, bytes) || overlaps(out, bytes, k, bytes) ||
                    overlaps(out, bytes, v, bytes)))
    return LA_ERR_ALIAS;
  if (state_in && state_out && state_in != state_out &&
      overlaps(state_in, state_bytes, state_out, state_bytes))
    return LA_ERR_ALIAS;
  if (state_out && bytes > 0 && overlaps(state_out, state_bytes, out, bytes)) return LA_ERR_ALIAS;
  const bool tensor = use_tensor_path(desc->path, desc->dtype, desc->d);
  if (epilogue != nullptr) {
    if (!tensor) return LA_ERR_UNSUPPORTED;  // the fused norm + gate lives in the chunked kernel
    // the FP8 output is la_gate_norm_apply's (the report's separate post-attention operator)
    if (epilogue->fp8_scales != nullptr) return LA_ERR_UNSUPPORTED;
    if (!epilogue->gate || !epilogue->gamma) return LA_ERR_NULL;
    if (!aligned16(epilogue->gate) || !aligned16(epilogue->gamma)) return LA_ERR_ALIGN;
    if (!(epilogue->eps >= 0.f) || epilogue->eps > 3.0e38f) return LA_ERR_SHAPE;  // NaN, inf
    if (bytes > 0 && overlaps(epilogue->gate, bytes, out, bytes)) return LA_ERR_ALIAS;
  }
  if (qk != nullptr) {
    // one kernel instance carries it: tensor path, 128-token chunks, plain output
    if (!tensor || chunk_of(desc->chunk) != 128 || epilogue != nullptr) return LA_ERR_UNSUPPORTED;
    if (!qk->gamma_q || !qk->gamma_k || !qk->positions) return LA_ERR_NULL;
    if (!aligned16(qk->gamma_q) || !aligned16(qk->gamma_k) ||
        (reinterpret_cast<uintptr_t>(qk->positions) & 7u) != 0)
      return LA_ERR_ALIGN;
    if (qk->rotary_dim < 16 || qk->rotary_dim > desc->d || qk->rotary_dim % 16 != 0)
      return LA_ERR_SHAPE;
    if (!(qk->theta > 0.f) || qk->theta > 3.0e38f || !(qk->eps >= 0.f) || qk->eps > 3.0e38f)
      return LA_ERR_SHAPE;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = device_sms();
  if (sms <= 0) return LA_ERR_CUDA;
  const la::VarlenWorkspace layout =
      la::varlen_workspace_layout(desc->T, desc->n_seqs, desc->H, desc->segments, sms, tensor);
  void* ws = workspace;
  bool owned = false;
  if (ws == nullptr) {
    if (cudaMallocAsync(&ws, layout.total, s) != cudaSuccess) return LA_ERR_CUDA;
    owned = true;
  } else {
    if (workspace_bytes < layout.total) return LA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return LA_ERR_ALIGN;
  }
  la::PrefillArgs a{1, desc->T, desc->H, desc->d, desc->dtype, q, k, v, slopes, out, state_out};
  a.chunk = chunk_of(desc->chunk);
  a.n_seqs = desc->n_seqs;
  a.cu_dev = cu_seqlens;
  a.state_in = state_in;
  if (epilogue != nullptr) {
    a.gate = epilogue->gate;
    a.gamma = epilogue->gamma;
    a.eps = epilogue->eps;
  }
  if (qk != nullptr) {
    a.qk_gamma_q = qk->gamma_q;
    a.qk_gamma_k = qk->gamma_k;
    a.qk_positions = qk->positions;
    a.qk_rotary_dim = qk->rotary_dim;
    a.qk_eps = qk->eps;
    rope_inv_freq(a.qk_inv_freq, qk->rotary_dim, qk->theta);
  }
  apply_debug_env(a);
  const cudaError_t e =
      la::launch_prefill_varlen(a, layout, ws, desc->segments, tensor, s, sms);
  if (owned) cudaFreeAsync(ws, s);
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

}  // namespace

extern "C" {

la_status la_prefill_varlen(const la_varlen_desc* desc, const void* q, const void* k,
                            const void* v, const float* slopes, const int64_t* cu_seqlens,
                            const float* state_in, const la_gate_norm* epilogue, void* out,
                            float* state_out, void* workspace, size_t workspace_bytes,
                            void* stream) {
  return prefill_varlen_impl(desc, nullptr, q, k, v, slopes, cu_seqlens, state_in, epilogue, out,
                             state_out, workspace, workspace_bytes, stream);
}

la_status la_prefill_varlen_qk(const la_varlen_desc* desc, const la_qk_prologue* qk,
                               const void* q, const void* k, const void* v, const float* slopes,
                               const int64_t* cu_seqlens, const float* state_in, void* out,
                               float* state_out, void* workspace, size_t workspace_bytes,
                               void* stream) {
  if (qk == nullptr) return LA_ERR_NULL;
  return prefill_varlen_impl(desc, qk, q, k, v, slopes, cu_seqlens, state_in, nullptr, out,
                             state_out, workspace, workspace_bytes, stream);
}

la_status la_qk_norm_rope(const la_qk_norm_rope_desc* desc, const void* q, const void* k,
                          const float* gamma_q, const float* gamma_k, const int64_t* positions,
                          void* q_out, void* k_out, void* stream) {
  if (desc == nullptr) return LA_ERR_NULL;
  const la_qk_norm_rope_desc& d = *desc;
  if (d.T < 0 || d.H < 1 || (d.d != 64 && d.d != 128)) return LA_ERR_SHAPE;
  if (d.rotary_dim < 16 || d.rotary_dim > d.d || d.rotary_dim % 16 != 0) return LA_ERR_SHAPE;
  if (!(d.theta > 0.f) || d.theta > 3.0e38f || !(d.eps >= 0.f) || d.eps > 3.0e38f)
    return LA_ERR_SHAPE;
  int64_t hd = 0, n = 0, span_q = 0, span_k = 0;
  if (!mul_ok(d.H, d.d, &hd) || !mul_ok(d.T, hd, &n)) return LA_ERR_OVERFLOW;
  if (d.q_stride < hd || d.k_stride < hd || d.q_stride % 8 || d.k_stride % 8) return LA_ERR_SHAPE;
  if (!mul_ok(d.T, d.q_stride, &span_q) || !mul_ok(d.T, d.k_stride, &span_k))
    return LA_ERR_OVERFLOW;
  if (d.T > INT32_MAX) return LA_ERR_OVERFLOW;  // one CTA per token
  if (!q || !k || !gamma_q || !gamma_k || !positions || !q_out || !k_out) return LA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_out) || !aligned16(k_out) ||
      !aligned16(gamma_q) || !aligned16(gamma_k))
    return LA_ERR_ALIGN;
  const size_t out_bytes = static_cast<size_t>(n) * 2;
  const size_t qb = static_cast<size_t>(span_q) * 2, kb = static_cast<size_t>(span_k) * 2;
  if (n > 0) {
    // in place is allowed only onto a contiguous input itself
    const bool q_inplace = q_out == q && d.q_stride == hd;
    const bool k_inplace = k_out == k && d.k_stride == hd;
    if ((!q_inplace && overlaps(q_out, out_bytes, q, qb)) || overlaps(q_out, out_bytes, k, kb) ||
        (!k_inplace && overlaps(k_out, out_bytes, k, kb)) || overlaps(k_out, out_bytes, q, qb) ||
        overlaps(q_out, out_bytes, k_out, out_bytes))
      return LA_ERR_ALIAS;
  }
  la::QkNormRopeArgs a{};
  a.T = d.T;
  a.H = d.H;
  a.d = d.d;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.q_stride = d.q_stride;
  a.k_stride = d.k_stride;
  a.gamma_q = gamma_q;
  a.gamma_k = gamma_k;
  a.positions = positions;
  a.q_out = static_cast<__nv_bfloat16*>(q_out);
  a.k_out = static_cast<__nv_bfloat16*>(k_out);
  a.rotary_dim = d.rotary_dim;
  a.eps = d.eps;
  rope_inv_freq(a.inv_freq, d.rotary_dim, d.theta);
  return la::launch_qk_norm_rope(a, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? LA_OK
             : LA_ERR_CUDA;
}

la_status la_decode_multi(int64_t B, int64_t H, int64_t d, int64_t n_tok, int32_t dtype,
                          const void* q, const void* k, const void* v, const float* slopes,
                          float* state_inout, const la_gate_norm* epilogue, void* out,
                          void* stream) {
  if (dtype != LA_BF16 && dtype != LA_F32) return LA_ERR_DTYPE;
  if (B < 1 || H < 1 || n_tok < 1 || (d != 64 && d != 128)) return LA_ERR_SHAPE;
  if (!q || !k || !v || !slopes || !state_inout || !out) return LA_ERR_NULL;
  int64_t bh = 0, n = 0, sb = 0;
  if (!mul_ok(B, H, &bh) || bh > INT32_MAX || !mul_ok(bh, d, &n) || !mul_ok(n, n_tok, &n) ||
      !mul_ok(bh, d * d * 4, &sb))
    return LA_ERR_OVERFLOW;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      !aligned16(state_inout))
    return LA_ERR_ALIGN;
  const size_t bytes = static_cast<size_t>(n) * (dtype == LA_BF16 ? 2 : 4);
  if (overlaps(out, bytes, q, bytes) || overlaps(out, bytes, k, bytes) ||
      overlaps(out, bytes, v, bytes) || overlaps(out, bytes, state_inout, static_cast<size_t>(sb)))
    return LA_ERR_ALIAS;
  // the state is rewritten in place while the token rows are read
  if (overlaps(state_inout, static_cast<size_t>(sb), q, bytes) ||
      overlaps(state_inout, static_cast<size_t>(sb), k, bytes) ||
      overlaps(state_inout, static_cast<size_t>(sb), v, bytes))
    return LA_ERR_ALIAS;
  la::DecodeArgs a{B, H, d, dtype, q, k, v, slopes, state_inout, out};
  a.n_tok = n_tok;
  if (epilogue != nullptr) {
    if (epilogue->fp8_scales != nullptr) return LA_ERR_UNSUPPORTED;  // no FP8 output here
    if (!epilogue->gate || !epilogue->gamma) return LA_ERR_NULL;
    if (!aligned16(epilogue->gate) || !aligned16(epilogue->gamma)) return LA_ERR_ALIGN;
    if (!(epilogue->eps >= 0.f) || epilogue->eps > 3.0e38f) return LA_ERR_SHAPE;
    if (overlaps(epilogue->gate, bytes, out, bytes)) return LA_ERR_ALIAS;
    a.gate = epilogue->gate;
    a.gamma = epilogue->gamma;
    a.eps = epilogue->eps;
  }
  return la::launch_decode_multi(a, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? LA_OK
             : LA_ERR_CUDA;
}

la_status la_gate_norm_apply(int64_t T, int64_t H, int64_t d, int32_t dtype, const void* o,
                             const la_gate_norm* gn, void* y, void* stream) {
  if (dtype != LA_BF16 && dtype != LA_F32) return LA_ERR_DTYPE;
  if (T < 0 || H < 1 || (d != 64 && d != 128)) return LA_ERR_SHAPE;
  if (T > INT32_MAX) return LA_ERR_OVERFLOW;  // one CTA per token
  if (!o || !gn || !gn->gate || !gn->gamma || !y) return LA_ERR_NULL;
  if (!(gn->eps >= 0.f) || gn->eps > 3.0e38f) return LA_ERR_SHAPE;
  int64_t n = 0;
  if (!mul_ok(T, H, &n) || !mul_ok(n, d, &n)) return LA_ERR_OVERFLOW;
  if (!aligned16(o) || !aligned16(gn->gate) || !aligned16(gn->gamma) || !aligned16(y))
    return LA_ERR_ALIGN;
  const size_t bytes = static_cast<size_t>(n) * (dtype == LA_BF16 ? 2 : 4);
  const bool fp8 = gn->fp8_scales != nullptr;
  if (fp8) {
    // one byte per value plus [H, T] fp32 scales; y cannot be written over o in place
    const size_t y_bytes = static_cast<size_t>(n);
    const size_t s_bytes = static_cast<size_t>(T * H) * 4;
    if (!aligned16(gn->fp8_scales)) return LA_ERR_ALIGN;
    if (bytes > 0 && (overlaps(y, y_bytes, o, bytes) || overlaps(y, y_bytes, gn->gate, bytes) ||
                      overlaps(gn->fp8_scales, s_bytes, y, y_bytes) ||
                      overlaps(gn->fp8_scales, s_bytes, o, bytes) ||
                      overlaps(gn->fp8_scales, s_bytes, gn->gate, bytes)))
      return LA_ERR_ALIAS;
  } else if (bytes > 0 &&
             ((y != o && overlaps(y, bytes, o, bytes)) || overlaps(y, bytes, gn->gate, bytes))) {
    return LA_ERR_ALIAS;
  }
  la::GateNormArgs a{T, H, d, dtype, o, gn->gate, gn->gamma, gn->eps, y, gn->fp8_scales};
  return la::launch_gate_norm(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? LA_OK
                                                                                     : LA_ERR_CUDA;
}

size_t la_prefill_state_workspace_bytes(const la_desc* desc) {
  int64_t numel = 0;
  if (check_desc(desc, &numel) != LA_OK || !use_tensor_path(desc)) return 0;
  const int sms = device_sms() > 0 ? device_sms() : 148;
  return la::plan_state_pass(desc->B, desc->N, desc->H, sms).ws_bytes;
}

la_status la_prefill_state(const la_desc* desc, const void* k, const void* v, const float* slopes,
                           const float* state_in, float* state_out, void* workspace,
                           size_t workspace_bytes, void* stream) {
  int64_t numel = 0;
  const la_status st = check_desc(desc, &numel);
  if (st != LA_OK) return st;
  if (!k || !v || !slopes || !state_out) return LA_ERR_NULL;
  if (!aligned16(k) || !aligned16(v) || !aligned16(state_out) ||
      (state_in && !aligned16(state_in)))
    return LA_ERR_ALIGN;
  const size_t bytes = static_cast<size_t>(numel) * (desc->dtype == LA_BF16 ? 2 : 4);
  const size_t state_bytes =
      static_cast<size_t>(desc->B * desc->H) * static_cast<size_t>(desc->d * desc->d) * 4;
  if (overlaps(state_out, state_bytes, k, bytes) || overlaps(state_out, state_bytes, v, bytes))
    return LA_ERR_ALIAS;
  if (state_in && state_in != state_out && overlaps(state_in, state_bytes, state_out, state_bytes))
    return LA_ERR_ALIAS;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  la::PrefillArgs a{desc->B, desc->N, desc->H, desc->d, desc->dtype, nullptr, k, v, slopes,
                    nullptr, state_out};
  a.state_in = state_in;
  apply_debug_env(a);
  if (!use_tensor_path(desc)) {
    // token recurrence with no q and no read-out
    return la::launch_recurrent_prefill(a, s) == cudaSuccess ? LA_OK : LA_ERR_CUDA;
  }
  const int sms = device_sms();
  if (sms <= 0) return LA_ERR_CUDA;
  const la::StatePassPlan plan = la::plan_state_pass(desc->B, desc->N, desc->H, sms);
  void* ws = workspace;
  bool owned = false;
  if (ws == nullptr) {
    if (cudaMallocAsync(&ws, plan.ws_bytes, s) != cudaSuccess) return LA_ERR_CUDA;
    owned = true;
  } else {
    if (workspace_bytes < plan.ws_bytes) return LA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return LA_ERR_ALIGN;
  }
  const cudaError_t e = la::launch_state_pass(a, plan, ws, s);
  if (owned) cudaFreeAsync(ws, s);
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

la_status la_state_fold(int64_t n_parts, int64_t BH, int64_t H, int64_t d, const float* parts,
                        const int64_t* lengths, const float* slopes, const float* state_in,
                        float* state_out, void* stream) {
  if (n_parts < 0 || n_parts > la::kMaxFoldParts || BH < 1 || H < 1 || BH % H != 0 ||
      (d != 64 && d != 128))
    return LA_ERR_SHAPE;
  if (BH > INT32_MAX) return LA_ERR_OVERFLOW;  // grid
  if (!slopes || !state_out || (n_parts > 0 && (!parts || !lengths))) return LA_ERR_NULL;
  if (!aligned16(state_out) || (state_in && !aligned16(state_in)) || (parts && !aligned16(parts)))
    return LA_ERR_ALIGN;
  int64_t sb = 0, pb = 0;
  if (!mul_ok(BH, d * d * 4, &sb) || !mul_ok(sb, n_parts, &pb)) return LA_ERR_OVERFLOW;
  la::StateFoldArgs a{};
  for (int64_t j = 0; j < n_parts; ++j) {
    if (lengths[j] < 0) return LA_ERR_SHAPE;
    a.lengths[j] = lengths[j];
  }
  if (n_parts > 0 && overlaps(state_out, static_cast<size_t>(sb), parts, static_cast<size_t>(pb)))
    return LA_ERR_ALIAS;
  if (state_in && state_in != state_out &&
      overlaps(state_in, static_cast<size_t>(sb), state_out, static_cast<size_t>(sb)))
    return LA_ERR_ALIAS;
  a.n_parts = n_parts;
  a.BH = BH;
  a.H = H;
  a.d = d;
  a.parts = parts;
  a.slopes = slopes;
  a.state_in = state_in;
  a.state_out = state_out;
  return la::launch_state_fold(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? LA_OK
                                                                                    : LA_ERR_CUDA;
}

la_status la_decode_step(int64_t B, int64_t H, int64_t d, int32_t dtype, const void* q,
                         const void* k, const void* v, const float* slopes, float* state_inout,
                         void* out, void* stream) {
  if (dtype != LA_BF16 && dtype != LA_F32) return LA_ERR_DTYPE;
  if (B < 1 || H < 1 || (d != 64 && d != 128)) return LA_ERR_SHAPE;
  if (!q || !k || !v || !slopes || !state_inout || !out) return LA_ERR_NULL;
  int64_t bh = 0, n = 0, sb = 0;
  if (!mul_ok(B, H, &bh) || bh > INT32_MAX || !mul_ok(bh, d, &n) || !mul_ok(bh, d * d * 4, &sb))
    return LA_ERR_OVERFLOW;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      !aligned16(state_inout))
    return LA_ERR_ALIGN;
  const size_t bytes = static_cast<size_t>(n) * (dtype == LA_BF16 ? 2 : 4);
  if (overlaps(out, bytes, q, bytes) || overlaps(out, bytes, k, bytes) ||
      overlaps(out, bytes, v, bytes) || overlaps(out, bytes, state_inout, static_cast<size_t>(sb)))
    return LA_ERR_ALIAS;
  // the state is rewritten in place while the token rows are read
  if (overlaps(state_inout, static_cast<size_t>(sb), q, bytes) ||
      overlaps(state_inout, static_cast<size_t>(sb), k, bytes) ||
      overlaps(state_inout, static_cast<size_t>(sb), v, bytes))
    return LA_ERR_ALIAS;
  la::DecodeArgs a{B, H, d, dtype, q, k, v, slopes, state_inout, out};
  return la::launch_decode(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? LA_OK
                                                                                 : LA_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------------
// la_prefill_noalloc: la_prefill on a scratch array compiled into the library, for callers that
// cannot allocate device memory (see la.h).  The array is a device symbol; host code never uses
// its name as an address, it asks the runtime for the device address once per device.
// ---------------------------------------------------------------------------------------------
}  // extern "C"

static __device__ __align__(256) uint8_t g_noalloc_scratch[LA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 256;

// The scratch array's device address in one CUDA context.  A context that is destroyed and
// recreated (cudaDeviceReset, a primary-context reset) loads the module again, possibly at
// another address, so the cache is keyed by the context's unique id, not the device alone.
struct ScratchAddress {
  unsigned long long ctx_id;
  void* ptr;
};
ScratchAddress g_noalloc_addr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (the runtime's primary context of the
// current device once a runtime call has been made).
la_status current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (get_current == nullptr || get_id == nullptr) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess || f1 == nullptr ||
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess || f2 == nullptr)
      return LA_ERR_CUDA;
    get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    get_id = reinterpret_cast<CtxGetIdFn>(f2);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return LA_ERR_CUDA;
  if (get_id(ctx, id) != CUDA_SUCCESS) return LA_ERR_CUDA;
  return LA_OK;
}

// Device address of g_noalloc_scratch on the current device, looked up with cudaGetSymbolAddress
// once per device and context (the host-side name g_noalloc_scratch is not a device address).
la_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LA_ERR_UNSUPPORTED;
  // make the device's primary context current (since CUDA 12, cudaSetDevice initialises it;
  // a no-op once the runtime has used it); this allocates nothing
  if (cudaSetDevice(dev) != cudaSuccess) return LA_ERR_CUDA;
  unsigned long long ctx = 0;
  const la_status cs = current_context_id(&ctx);
  if (cs != LA_OK) return cs;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  ScratchAddress& a = g_noalloc_addr[dev];
  if (a.ptr == nullptr || a.ctx_id != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_noalloc_scratch) != cudaSuccess ||
        p == nullptr)
      return LA_ERR_CUDA;
    a.ptr = p;
    a.ctx_id = ctx;
  }
  *out = a.ptr;
  return LA_OK;
}

}  // namespace

extern "C" {

la_status la_prefill_noalloc(const la_desc* desc, const void* q, const void* k, const void* v,
                             const float* slopes, void* out, float* state_out, void* stream) {
  const la_status st = check_prefill_args(desc, q, k, v, slopes, out, state_out);
  if (st != LA_OK) return st;
  // The test-only failure injection (a withheld scan flag) can only be reported through the
  // workspace status word, which callers of this entry point cannot read: refuse it here rather
  // than return LA_OK with invalid outputs.
  if (getenv("LA_DEBUG_WITHHOLD_SEGMENT") != nullptr) return LA_ERR_UNSUPPORTED;
  if (!use_tensor_path(desc)) {
    // the recurrent kernel uses no scratch memory
    return la_prefill(desc, q, k, v, slopes, out, state_out, nullptr, 0, stream);
  }
  const int sms = device_sms();
  if (sms <= 0) return LA_ERR_CUDA;
  if (prefill_workspace_need(desc, sms) > LA_NOALLOC_SCRATCH_BYTES) return LA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const la_status sa = noalloc_scratch(&scratch);
  if (sa != LA_OK) return sa;
  return la_prefill(desc, q, k, v, slopes, out, state_out, scratch, LA_NOALLOC_SCRATCH_BYTES,
                    stream);
}

la_status la_workspace_status(const void* workspace, void* stream) {
  if (workspace == nullptr) return LA_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return LA_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, static_cast<const uint8_t*>(workspace) + la::kWsStatus, sizeof v,
                 cudaMemcpyDeviceToHost) != cudaSuccess)
    return LA_ERR_CUDA;
  return v == 0 ? LA_OK : static_cast<la_status>(v);
}

const char* la_status_string(int status) {
  switch (status) {
    case LA_OK: return "ok";
    case LA_ERR_NULL: return "a required pointer is NULL";
    case LA_ERR_SHAPE: return "shape out of range (B, N, H >= 1; d in {64, 128})";
    case LA_ERR_DTYPE: return "unknown dtype";
    case LA_ERR_ALIGN: return "pointer not 16-byte aligned (workspace: 256-byte)";
    case LA_ERR_OVERFLOW: return "size exceeds the 64-bit or tensor-map limits";
    case LA_ERR_WORKSPACE: return "workspace smaller than la_prefill_workspace_bytes()";
    case LA_ERR_CUDA: return "a CUDA call failed";
    case LA_ERR_TIMEOUT: return "a bounded device wait expired";
    case LA_ERR_UNSUPPORTED: return "no kernel for this combination of options";
    case LA_ERR_ALIAS: return "output overlaps an input";
    default: return "unknown status";
  }
}

int la_version(void) { return LA_VERSION; }

}  // extern "C"
