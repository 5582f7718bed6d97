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

#include "la_internal.h"

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
// One CTA per (b, h), 512 threads, the state's quads held in registers as in decode_kernel, and
// n tokens applied in order, each one: S <- lambda S + k^T v, o = q S.  The state is read and
// written once for all n tokens.  The q, k, v (and gate) rows of up to 8 tokens are staged in
// shared memory at once, so a group costs one load latency, and each token then costs one block
// barrier.  With a gate, each output row gets the fused grouped RMSNorm + sigmoid gate:
// y = gamma * o / sqrt(mean(o^2) + eps) * sigmoid(g) (one norm group per head).
// ---------------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(512) decode_multi_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const float* __restrict__ slopes, float* __restrict__ state, T* __restrict__ out, int64_t H,
    int64_t n_tok, const T* __restrict__ gate, const float* __restrict__ gamma, float eps) {
  constexpr int NT = 512;
  constexpr int Q4 = D / 4;     // column quads per row
  constexpr int RS = NT / Q4;   // row slots
  constexpr int RPT = D / RS;   // rows per thread
  constexpr int NG = 8;         // tokens staged per group
  __shared__ float sqkv[3][NG][D];   // q, k, v of the group's tokens
  __shared__ float sg[NG][D];        // their gate pre-activations
  __shared__ float red[2][RS][D];    // read-out partial sums, double-buffered over tokens
  __shared__ float ss_part[D / 32];

  const int tid = threadIdx.x;
  const int c4 = tid % Q4;
  const int r0 = tid / Q4;
  const int64_t flat = blockIdx.x;  // b * H + h
  const int64_t b = flat / H;
  const int64_t h = flat % H;
  float4* st = reinterpret_cast<float4*>(state + flat * D * D);

  float4 s[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) s[r] = __ldcs(st + (r0 + r * RS) * Q4 + c4);
  float lam_hi, lam_lo;
  split_decay(slopes[h], lam_hi, lam_lo);

  // element offset of token j's row for this head in a [B, n_tok, H, D] tensor
  auto row_off = [&](int64_t j) { return ((b * n_tok + j) * H + h) * D; };
  int64_t tok = 0;  // tokens processed so far (selects the red buffer)
  for (int64_t j0 = 0; j0 < n_tok; j0 += NG) {
    const int nn = static_cast<int>(min(static_cast<int64_t>(NG), n_tok - j0));
    // stage the whole group (one load latency for nn tokens)
    for (int idx = tid; idx < 3 * nn * D; idx += NT) {
      const int which = idx / (nn * D), rem = idx % (nn * D), jj = rem / D, e = rem % D;
      const T* src = which == 0 ? q : (which == 1 ? k : v);
      sqkv[which][jj][e] = load_as_f32<T>(src, row_off(j0 + jj) + e);
    }
    if (gate != nullptr)
      for (int idx = tid; idx < nn * D; idx += NT)
        sg[idx / D][idx % D] = load_as_f32<T>(gate, row_off(j0 + idx / D) + idx % D);
    __syncthreads();
    for (int jj = 0; jj < nn; ++jj, ++tok) {
      const int rb = static_cast<int>(tok & 1);
      const float v0 = sqkv[2][jj][4 * c4 + 0], v1 = sqkv[2][jj][4 * c4 + 1];
      const float v2 = sqkv[2][jj][4 * c4 + 2], v3 = sqkv[2][jj][4 * c4 + 3];
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        const int i = r0 + r * RS;
        const float ki = sqkv[1][jj][i], qi = sqkv[0][jj][i];
        float4 x = s[r];
        x.x = fmaf(lam_hi, x.x, fmaf(ki, v0, lam_lo * x.x));
        x.y = fmaf(lam_hi, x.y, fmaf(ki, v1, lam_lo * x.y));
        x.z = fmaf(lam_hi, x.z, fmaf(ki, v2, lam_lo * x.z));
        x.w = fmaf(lam_hi, x.w, fmaf(ki, v3, lam_lo * x.w));
        a0 = fmaf(qi, x.x, a0);
        a1 = fmaf(qi, x.y, a1);
        a2 = fmaf(qi, x.z, a2);
        a3 = fmaf(qi, x.w, a3);
        s[r] = x;
      }
      red[rb][r0][4 * c4 + 0] = a0;
      red[rb][r0][4 * c4 + 1] = a1;
      red[rb][r0][4 * c4 + 2] = a2;
      red[rb][r0][4 * c4 + 3] = a3;
      // One barrier per token: red is double-buffered, and the read-out of this token finishes
      // before its threads reach the next token's barrier, so red[rb] is free again two tokens on.
      __syncthreads();
      if (tid < D) {
        float o = 0.f;
#pragma unroll
        for (int rr = 0; rr < RS; ++rr) o += red[rb][rr][tid];
        if (gate != nullptr) {
          float ss = o * o;
#pragma unroll
          for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
          if ((tid & 31) == 0) ss_part[tid >> 5] = ss;
          asm volatile("bar.sync 1, %0;" ::"r"(D) : "memory");  // the D read-out threads only
          float tot = 0.f;
#pragma unroll
          for (int w = 0; w < D / 32; ++w) tot += ss_part[w];
          const float sig = 1.f / (1.f + expf(-sg[jj][tid]));
          o = gamma[h * D + tid] * (o * rsqrtf(tot * (1.f / D) + eps)) * sig;
          asm volatile("bar.sync 1, %0;" ::"r"(D) : "memory");  // ss_part reused next token
        }
        store_from_f32<T>(out, row_off(j0 + jj) + tid, o);
      }
    }
    __syncthreads();  // the group's staging buffers are read; the next group may overwrite them
  }
#pragma unroll
  for (int r = 0; r < RPT; ++r) __stcs(st + (r0 + r * RS) * Q4 + c4, s[r]);
}

template <typename T, int D>
cudaError_t launch_decode_multi_typed(const DecodeArgs& a, cudaStream_t stream) {
  const int64_t grid = a.B * a.H;
  decode_multi_kernel<T, D><<<static_cast<unsigned>(grid), 512, 0, stream>>>(
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
