// la_recurrent.cu — token-by-token CUDA-core kernels: the fp32 prefill path and the decode step.
//
// Both evaluate the RNN-style form of linear attention ("Ling and Ring 2.6 Technical Report",
// §4.1.1, Context Parallel for Lightning Attention: a recurrence over the sequence with a per-head
// [D,D] hidden state), with Lightning Attention's per-head decay lambda = exp(-slope):
//     S <- lambda S + k^T v,    o = q S.
//
// Decay precision.  A plain fp32 multiply by a rounded lambda carries the rounding of lambda
// into every step (after n steps the relative error of lambda^n grows like n * 2^-24).  The kernels
// therefore split lambda = lam_hi + lam_lo (both fp32, computed from an fp64 exp) and apply
//     S' = lam_hi * S + (k v + lam_lo * S)
// with two fused multiply-adds, so the decay is exact to fp32 rounding of each step.
#include <cuda_bf16.h>

#include <algorithm>

#include "la_internal.h"
#include "la_sm100.cuh"

namespace la {
namespace {

template <typename T>
__device__ __forceinline__ float load_as_f32(const T* p, int64_t i);
template <>
__device__ __forceinline__ float load_as_f32<float>(const float* p, int64_t i) {
  return p[i];
}
template <>
__device__ __forceinline__ float load_as_f32<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}

template <typename T>
__device__ __forceinline__ void store_from_f32(T* p, int64_t i, float x);
template <>
__device__ __forceinline__ void store_from_f32<float>(float* p, int64_t i, float x) {
  p[i] = x;
}
template <>
__device__ __forceinline__ void store_from_f32<__nv_bfloat16>(__nv_bfloat16* p, int64_t i,
                                                              float x) {
  p[i] = __float2bfloat16_rn(x);
}

__device__ __forceinline__ void split_decay(float slope, float& hi, float& lo) {
  const double lam = exp(-static_cast<double>(slope));
  hi = static_cast<float>(lam);
  lo = static_cast<float>(lam - static_cast<double>(hi));
}

// ---------------------------------------------------------------------------------------------
// Recurrent prefill.  One CTA per flat head (b*H + h; for packed variable-length input,
// sequence*H + h with the sequence's tokens [cu[s], cu[s+1])), 4*D threads.  Thread t owns the state
// column j = t % D for rows [rg*R, rg*R + R), rg = t / D, R = D / 4; the read-out o_j is summed
// over the four row groups through shared memory.  q, k, v of the next token are prefetched into
// registers while the current token is processed.
// ---------------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(4 * D) recurrent_prefill_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const float* __restrict__ slopes, T* __restrict__ out, float* state_out, int64_t N,
    int64_t H, const int64_t* __restrict__ cu, const float* state_in, const int32_t* status) {
  constexpr int R = D / 4;
  __shared__ float tok[2][3][D];
  __shared__ float red[4][D];

  const int tid = threadIdx.x;
  const int j = tid % D;
  const int rg = tid / D;
  // packed input whose cu_seqlens failed the device check: touch nothing
  if (status != nullptr && *status != 0) return;
  const int64_t flat = blockIdx.x;
  const int64_t b = flat / H;  // batch index, or sequence index of packed input
  const int64_t h = flat % H;
  // rows [row0, row0 + len) of the token axis
  const int64_t row0 = cu != nullptr ? cu[b] : b * N;
  const int64_t len = cu != nullptr ? cu[b + 1] - cu[b] : N;

  float lam_hi, lam_lo;
  split_decay(slopes[h], lam_hi, lam_lo);

  // loader role: threads [0, 3D) each fetch one element of q, k or v of a token (state only,
  // q == nullptr and out == nullptr: the q loaders supply zeros and nothing is read out)
  const int which = tid / D;  // 0: q, 1: k, 2: v (3: idle)
  const int e = tid % D;
  const T* src = which == 0 ? q : (which == 1 ? k : v);
  auto fetch = [&](int64_t t) -> float {
    if (src == nullptr) return 0.f;
    return load_as_f32<T>(src, ((row0 + t) * H + h) * D + e);
  };

  float S[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    // the initial state (a cached prefix), read before any write: state_out may be this array
    S[r] = state_in != nullptr ? state_in[(flat * D + rg * R + r) * D + j] : 0.f;
  }

  if (which < 3 && len > 0) tok[0][which][e] = fetch(0);
  float pf = 0.f;
  if (which < 3 && len > 1) pf = fetch(1);
  __syncthreads();

  for (int64_t t = 0; t < len; ++t) {
    const int buf = static_cast<int>(t & 1);
    const float vj = tok[buf][2][j];
    float acc = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int i = rg * R + r;
      const float t1 = fmaf(tok[buf][1][i], vj, lam_lo * S[r]);
      S[r] = fmaf(lam_hi, S[r], t1);
      acc = fmaf(tok[buf][0][i], S[r], acc);
    }
    red[rg][j] = acc;
    if (which < 3 && t + 1 < len) tok[buf ^ 1][which][e] = pf;
    __syncthreads();
    if (rg == 0 && out != nullptr) {
      const float o = ((red[0][j] + red[1][j]) + red[2][j]) + red[3][j];
      store_from_f32<T>(out, ((row0 + t) * H + h) * D + j, o);
    }
    if (which < 3 && t + 2 < len) pf = fetch(t + 2);
    __syncthreads();
  }

  if (state_out != nullptr) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int i = rg * R + r;
      state_out[(flat * D + i) * D + j] = S[r];
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Decode step.  One CTA per flat head, 512 threads.  Thread t streams 128-bit quads of the fp32
// state: column quad c4 = t % (D/4), rows r0, r0 + RS, ... with r0 = t / (D/4), RS = 512/(D/4).
// All of a thread's state loads are issued before q, k, v are staged, so D*D*4/512 bytes per
// thread are in flight at once; the updated state is written back in place with streaming
// stores and the read-out o_j is reduced over the RS row slots through shared memory.
// ---------------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(512) decode_kernel(const T* __restrict__ q,
                                                     const T* __restrict__ k,
                                                     const T* __restrict__ v,
                                                     const float* __restrict__ slopes,
                                                     float* __restrict__ state,
                                                     T* __restrict__ out, int64_t H) {
  constexpr int NT = 512;
  constexpr int Q4 = D / 4;     // column quads per row
  constexpr int RS = NT / Q4;   // row slots
  constexpr int RPT = D / RS;   // rows per thread
  __shared__ float sq[D], sk[D], sv[D];
  __shared__ float red[RS][D];

  const int tid = threadIdx.x;
  const int c4 = tid % Q4;
  const int r0 = tid / Q4;
  const int64_t flat = blockIdx.x;
  const int64_t h = flat % H;
  float4* st = reinterpret_cast<float4*>(state + flat * D * D);

  float4 s[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) s[r] = __ldcs(st + (r0 + r * RS) * Q4 + c4);

  if (tid < 3 * D) {
    const int which = tid / D, e = tid % D;
    const T* src = which == 0 ? q : (which == 1 ? k : v);
    const float x = load_as_f32<T>(src, flat * D + e);
    (which == 0 ? sq : (which == 1 ? sk : sv))[e] = x;
  }
  float lam_hi, lam_lo;
  split_decay(slopes[h], lam_hi, lam_lo);
  __syncthreads();

  const float v0 = sv[4 * c4 + 0], v1 = sv[4 * c4 + 1], v2 = sv[4 * c4 + 2], v3 = sv[4 * c4 + 3];
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int i = r0 + r * RS;
    const float ki = sk[i], qi = sq[i];
    float4 x = s[r];
    x.x = fmaf(lam_hi, x.x, fmaf(ki, v0, lam_lo * x.x));
    x.y = fmaf(lam_hi, x.y, fmaf(ki, v1, lam_lo * x.y));
    x.z = fmaf(lam_hi, x.z, fmaf(ki, v2, lam_lo * x.z));
    x.w = fmaf(lam_hi, x.w, fmaf(ki, v3, lam_lo * x.w));
    a0 = fmaf(qi, x.x, a0);
    a1 = fmaf(qi, x.y, a1);
    a2 = fmaf(qi, x.z, a2);
    a3 = fmaf(qi, x.w, a3);
    __stcs(st + i * Q4 + c4, x);
  }
  red[r0][4 * c4 + 0] = a0;
  red[r0][4 * c4 + 1] = a1;
  red[r0][4 * c4 + 2] = a2;
  red[r0][4 * c4 + 3] = a3;
  __syncthreads();
  if (tid < D) {
    float o = 0.f;
#pragma unroll
    for (int rr = 0; rr < RS; ++rr) o += red[rr][tid];
    store_from_f32<T>(out, flat * D + tid, o);
  }
}

// ---------------------------------------------------------------------------------------------
// Multi-token decode step (speculative verification: the report's "attention with MTP", §4.3).
// For every (b, h), n tokens are applied in order, each one: S <- lambda S + k^T v, o = q S.
//
// The n tokens are one chunk of the recurrence, evaluated in its chunked form (the same algebra
// as the prefill's chunks): with S_0 the state before the step,
//     o_j = lambda^(j+1) q_j S_0 + sum_{m <= j} lambda^(j-m) (q_j . k_m) v_m
//     S_n = lambda^n S_0 + sum_m lambda^(n-1-m) k_m^T v_m
// so the state is read once for every read-out (one multiply-add per state element per token)
// and updated once (n + 1 per element), with a fixed number of block barriers per head instead
// of one per token.  Groups of at most 8 tokens are applied in turn.
//
// One CTA per (b, h), two resident per SM: each thread loads its quads of the state into
// registers with all its loads in flight at once (as in decode_kernel), the group's q, k, v (and
// gate) rows are staged in shared memory, and the updated state goes back with streaming stores.
// With a gate, each output row gets the fused grouped RMSNorm + sigmoid gate
// y = gamma * o / sqrt(mean(o^2) + eps) * sigmoid(g).
// ---------------------------------------------------------------------------------------------
template <typename T, int D>
struct MultiLayout {
  static constexpr int NG = 8;                                    // tokens per group
  static constexpr int RS = 512 / (D / 4);                        // row slots
  static constexpr size_t kTok = size_t(4) * NG * D * sizeof(T);  // q, k, v, gate rows
  static constexpr size_t kPart = size_t(NG) * RS * D * 4;        // q S_0 partial sums
  static constexpr size_t kCtrl = 512;                            // A, norms
  static constexpr size_t kTotal = kTok + kPart + kCtrl;
};

template <typename T>
__device__ __forceinline__ float smem_f32(const T* p);
template <>
__device__ __forceinline__ float smem_f32<float>(const float* p) {
  return *p;
}
template <>
__device__ __forceinline__ float smem_f32<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
// four consecutive elements (16-byte aligned for fp32, 8-byte for bf16) as fp32
template <typename T>
__device__ __forceinline__ float4 smem_f32x4(const T* p);
template <>
__device__ __forceinline__ float4 smem_f32x4<float>(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
template <>
__device__ __forceinline__ float4 smem_f32x4<__nv_bfloat16>(const __nv_bfloat16* p) {
  const uint2 w = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                     __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
}

template <typename T, int D>
__global__ void __launch_bounds__(512, 2) decode_multi_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const float* __restrict__ slopes, float* __restrict__ state, T* __restrict__ out, int64_t H,
    int64_t n_tok, const T* __restrict__ gate, const float* __restrict__ gamma, float eps) {
  using L = MultiLayout<T, D>;
  constexpr int NT = 512;
  constexpr int Q4 = D / 4;       // column quads per row
  constexpr int RS = L::RS;       // row slots
  constexpr int RPT = D / RS;     // rows per thread
  constexpr int NG = L::NG;
  constexpr int TPJ = NT / NG;    // output threads per token
  constexpr int CPT = D / TPJ;    // output columns per thread (2 at d = 128, 1 at d = 64)
  constexpr int EPP = 16 / static_cast<int>(sizeof(T));  // elements per 16-byte piece
  constexpr int PIECES = D / EPP;                        // pieces per token row
  constexpr float kLog2e = 1.4426950408889634f;
  extern __shared__ __align__(128) uint8_t sm[];
  T* tok = reinterpret_cast<T*>(sm);                                           // [4][NG][D]
  float(*part)[RS][D] = reinterpret_cast<float(*)[RS][D]>(sm + L::kTok);      // [NG][RS][D]
  float* A = reinterpret_cast<float*>(sm + L::kTok + L::kPart);               // [NG][NG]
  float* ssq = A + NG * NG;                                                    // [NG][TPJ / 32]

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int c4 = tid % Q4;
  const int r0 = tid / Q4;
  const int rows = gate != nullptr ? 4 : 3;
  const int64_t flat = blockIdx.x;  // b * H + h
  const int64_t b = flat / H, h = flat % H;
  float4* st = reinterpret_cast<float4*>(state + flat * D * D);

  // every state load of the thread in flight at once
  float4 s[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) s[r] = __ldcs(st + (r0 + r * RS) * Q4 + c4);
  const float alpha = slopes[h] * kLog2e;  // lambda^e = exp2(-alpha e)
  const T* tq = tok;
  const T* tkk = tok + NG * D;
  const T* tv = tok + 2 * NG * D;
  const T* tg = tok + 3 * NG * D;

  for (int64_t j0 = 0; j0 < n_tok; j0 += NG) {
    const int nn = static_cast<int>(min(static_cast<int64_t>(NG), n_tok - j0));
    if (j0 > 0) __syncthreads();  // the previous group's buffers are read
    // q, k, v (and gate) rows of the group, 16 bytes per copy
    for (int idx = tid; idx < rows * nn * PIECES; idx += NT) {
      const int which = idx / (nn * PIECES), rem = idx % (nn * PIECES);
      const int jj = rem / PIECES, pc = rem % PIECES;
      const T* src = which == 0 ? q : (which == 1 ? k : (which == 2 ? v : gate));
      cp_async16(tok + (which * NG + jj) * D + pc * EPP,
                 src + ((b * n_tok + j0 + jj) * H + h) * D + pc * EPP, true);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    // (1) partial read-outs q_j S_0 over this thread's rows, for every token of the group
#pragma unroll
    for (int jj = 0; jj < NG; ++jj) {
      if (jj < nn) {
        float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
          const float qi = smem_f32(tq + jj * D + r0 + r * RS);
          y.x = fmaf(qi, s[r].x, y.x);
          y.y = fmaf(qi, s[r].y, y.y);
          y.z = fmaf(qi, s[r].z, y.z);
          y.w = fmaf(qi, s[r].w, y.w);
        }
        *reinterpret_cast<float4*>(&part[jj][r0][4 * c4]) = y;
      }
    }
    // (2) intra weights A[j][m] = lambda^(j-m) (q_j . k_m), m <= j, one warp per pair
    for (int pidx = warp; pidx < nn * (nn + 1) / 2; pidx += NT / 32) {
      int jq = 0;
      while ((jq + 1) * (jq + 2) / 2 <= pidx) ++jq;
      const int m = pidx - jq * (jq + 1) / 2;
      float dot = 0.f;
#pragma unroll
      for (int e = lane; e < D; e += 32)
        dot = fmaf(smem_f32(tq + jq * D + e), smem_f32(tkk + m * D + e), dot);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (lane == 0) A[jq * NG + m] = exp2f(-alpha * static_cast<float>(jq - m)) * dot;
    }
    __syncthreads();
    // (3) outputs: thread (j, cols) sums the row slots, adds the intra terms, scales
    {
      const int jj = tid / TPJ;
      const int cbase = (tid % TPJ) * CPT;
      float o[CPT];
      if (jj < nn) {
        const float fq = exp2f(-alpha * static_cast<float>(jj + 1));
#pragma unroll
        for (int cc = 0; cc < CPT; ++cc) {
          const int c = cbase + cc;
          float acc = 0.f;
#pragma unroll
          for (int rr = 0; rr < RS; ++rr) acc += part[jj][rr][c];
          float intra = 0.f;
          for (int m = 0; m <= jj; ++m)
            intra = fmaf(A[jj * NG + m], smem_f32(tv + m * D + c), intra);
          o[cc] = fmaf(fq, acc, intra);
        }
      }
      if (gate != nullptr) {
        // grouped RMSNorm over the token's D outputs (TPJ threads), then the sigmoid gate
        float ss = 0.f;
        if (jj < nn) {
#pragma unroll
          for (int cc = 0; cc < CPT; ++cc) ss = fmaf(o[cc], o[cc], ss);
        }
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
        if (lane == 0) ssq[warp] = ss;  // the warps of token j are 2 j, 2 j + 1
        __syncthreads();
        if (jj < nn) {
          float tot = 0.f;
#pragma unroll
          for (int w = 0; w < TPJ / 32; ++w) tot += ssq[jj * (TPJ / 32) + w];
          const float rinv = rsqrtf(tot * (1.f / D) + eps);
#pragma unroll
          for (int cc = 0; cc < CPT; ++cc) {
            const int c = cbase + cc;
            const float sig = 1.f / (1.f + expf(-smem_f32(tg + jj * D + c)));
            o[cc] = gamma[h * D + c] * (o[cc] * rinv) * sig;
          }
        }
      }
      if (jj < nn) {
#pragma unroll
        for (int cc = 0; cc < CPT; ++cc)
          store_from_f32<T>(out, ((b * n_tok + j0 + jj) * H + h) * D + cbase + cc, o[cc]);
      }
    }
    // (4) state after the group: S <- lambda^nn S + sum_m lambda^(nn-1-m) k_m^T v_m
    {
      const float lam_n = exp2f(-alpha * static_cast<float>(nn));
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        s[r].x *= lam_n;
        s[r].y *= lam_n;
        s[r].z *= lam_n;
        s[r].w *= lam_n;
      }
      for (int m = 0; m < nn; ++m) {
        const float wm = exp2f(-alpha * static_cast<float>(nn - 1 - m));
        const float4 vm = smem_f32x4(tv + m * D + 4 * c4);
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
          const float km = wm * smem_f32(tkk + m * D + r0 + r * RS);
          s[r].x = fmaf(km, vm.x, s[r].x);
          s[r].y = fmaf(km, vm.y, s[r].y);
          s[r].z = fmaf(km, vm.z, s[r].z);
          s[r].w = fmaf(km, vm.w, s[r].w);
        }
      }
    }
  }
  // the updated state back in place (a warp writes whole 512-byte rows)
#pragma unroll
  for (int r = 0; r < RPT; ++r) __stcs(st + (r0 + r * RS) * Q4 + c4, s[r]);
}

template <typename T, int D>
cudaError_t launch_decode_multi_typed(const DecodeArgs& a, cudaStream_t stream) {
  using L = MultiLayout<T, D>;
  // set on every call: cheap, safe from any host thread, and it survives a context reset
  cudaError_t e = cudaFuncSetAttribute(decode_multi_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(L::kTotal));
  if (e != cudaSuccess) return e;
  decode_multi_kernel<T, D><<<static_cast<unsigned>(a.B * a.H), 512, L::kTotal, stream>>>(
      static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v),
      a.slopes, a.state, static_cast<T*>(a.out), a.H, a.n_tok, static_cast<const T*>(a.gate),
      a.gamma, a.eps);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_recurrent_typed(const PrefillArgs& a, cudaStream_t stream) {
  const int64_t grid = (a.n_seqs > 0 ? a.n_seqs : a.B) * a.H;
  if (grid == 0) return cudaSuccess;
  recurrent_prefill_kernel<T, D><<<static_cast<unsigned>(grid), 4 * D, 0, stream>>>(
      static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v),
      a.slopes, static_cast<T*>(a.out), a.state_out, a.N, a.H, a.cu_dev, a.state_in, a.status);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_decode_typed(const DecodeArgs& a, cudaStream_t stream) {
  const int64_t grid = a.B * a.H;
  decode_kernel<T, D><<<static_cast<unsigned>(grid), 512, 0, stream>>>(
      static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v),
      a.slopes, a.state, static_cast<T*>(a.out), a.H);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_recurrent_prefill(const PrefillArgs& a, cudaStream_t stream) {
  if (a.dtype == kF32) {
    return a.d == 64 ? launch_recurrent_typed<float, 64>(a, stream)
                     : launch_recurrent_typed<float, 128>(a, stream);
  }
  return a.d == 64 ? launch_recurrent_typed<__nv_bfloat16, 64>(a, stream)
                   : launch_recurrent_typed<__nv_bfloat16, 128>(a, stream);
}

cudaError_t launch_decode_multi(const DecodeArgs& a, cudaStream_t stream) {
  // one token and no epilogue is the plain decode step (same kernel, same bits)
  if (a.n_tok == 1 && a.gate == nullptr) return launch_decode(a, stream);
  if (a.dtype == kF32) {
    return a.d == 64 ? launch_decode_multi_typed<float, 64>(a, stream)
                     : launch_decode_multi_typed<float, 128>(a, stream);
  }
  return a.d == 64 ? launch_decode_multi_typed<__nv_bfloat16, 64>(a, stream)
                   : launch_decode_multi_typed<__nv_bfloat16, 128>(a, stream);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  if (a.dtype == kF32) {
    return a.d == 64 ? launch_decode_typed<float, 64>(a, stream)
                     : launch_decode_typed<float, 128>(a, stream);
  }
  return a.d == 64 ? launch_decode_typed<__nv_bfloat16, 64>(a, stream)
                   : launch_decode_typed<__nv_bfloat16, 128>(a, stream);
}

}  // namespace la
