// la_gatenorm.cu — the fused operator after the kernel: grouped RMSNorm + sigmoid gate.
//
// "Ling and Ring 2.6 Technical Report", §2.1 Fig. 2 (Linear Attention Kernel -> Grouped RMSNorm,
// multiplied by sigmoid(Gate Projection) -> Output Projection) and §4.3 (group norm + sigmoid gate
// run as one fused inference operator).  Per token t and head h (each head is one norm group):
//     y = gamma[h] * o / sqrt(mean(o^2) + eps) * sigmoid(g)
// Memory bound: read o and g, write y (3 rows of d per token-head).  A row is handled by d/8
// threads of 16 bytes and its mean square is a shuffle reduction over them; o and g reach those
// threads through a shared-memory ring filled two items ahead by per-thread cp.async copies.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <cstdint>

#include <algorithm>

#include "la_internal.h"
#include "la_sm100.cuh"

namespace la {
namespace {

constexpr int kGnThreads = 512;

template <typename T>
struct Io;

template <>
struct Io<__nv_bfloat16> {  // 8 values = one 16-byte piece
  static __device__ __forceinline__ void unpack(const uint4& w, float (&x)[8]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[2 * e] = __uint_as_float(u[e] << 16);
      x[2 * e + 1] = __uint_as_float(u[e] & 0xffff0000u);
    }
  }
  // round to nearest even, one paired conversion; lo in the low half
  static __device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&p);
  }
  // the value as stored in this dtype (round to nearest even)
  static __device__ __forceinline__ float round(float x) {
    return __bfloat162float(__float2bfloat16_rn(x));
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* dst, const float (&y)[8]) {
    __stcs(reinterpret_cast<uint4*>(dst),
           make_uint4(pack2(y[0], y[1]), pack2(y[2], y[3]), pack2(y[4], y[5]), pack2(y[6], y[7])));
  }
};

template <>
struct Io<float> {  // 8 values = two 16-byte pieces
  static __device__ __forceinline__ float round(float x) { return x; }
  static __device__ __forceinline__ void store(float* dst, const float (&y)[8]) {
    __stcs(reinterpret_cast<float4*>(dst), make_float4(y[0], y[1], y[2], y[3]));
    __stcs(reinterpret_cast<float4*>(dst) + 1, make_float4(y[4], y[5], y[6], y[7]));
  }
};

// sigmoid(x).  bf16 output: (1 + tanh(x/2)) / 2 with one MUFU tanh (relative error about 2^-11,
// far below the bf16 rounding of y).  fp32 output: 1 / (1 + e^-x) with the approximate
// exponential and divide (a few ulp); an IEEE divide here would cost more issue slots than
// the memory system leaves per element.
template <typename T>
struct Sigmoid;
template <>
struct Sigmoid<__nv_bfloat16> {
  static __device__ __forceinline__ float f(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return fmaf(0.5f, t, 0.5f);
  }
};
template <>
struct Sigmoid<float> {
  static __device__ __forceinline__ float f(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }
};

// Pieces: a thread's 8 consecutive values of a row are kPieces 16-byte pieces (bf16 1, fp32 2).
template <typename T>
struct Piece {
  static constexpr int kPieces = sizeof(T) / 2;
  static constexpr int kElems = 16 / sizeof(T);  // elements per piece
  static __device__ __forceinline__ void unpack(const uint4 (&w)[kPieces], float (&x)[8]);
};
template <>
__device__ __forceinline__ void Piece<__nv_bfloat16>::unpack(const uint4 (&w)[1], float (&x)[8]) {
  Io<__nv_bfloat16>::unpack(w[0], x);
}
template <>
__device__ __forceinline__ void Piece<float>::unpack(const uint4 (&w)[2], float (&x)[8]) {
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    x[4 * p] = __uint_as_float(w[p].x);
    x[4 * p + 1] = __uint_as_float(w[p].y);
    x[4 * p + 2] = __uint_as_float(w[p].z);
    x[4 * p + 3] = __uint_as_float(w[p].w);
  }
}

// Work item: kSweeps x ROWS rows (head groups) of one token; a CTA takes a contiguous range of
// items.  The loads of each item go through a kStages-deep ring in shared memory with per-thread
// cp.async copies, two items ahead of the one being finished, so the bytes in flight are held by
// shared memory rather than registers.  Every thread reads back only the pieces it copied itself
// (slot [stage][piece][thread]), so the ring needs no block barrier.
constexpr int kStages = 3;
constexpr int kSweeps = 2;

template <typename T, int D>
__global__ void __launch_bounds__(kGnThreads, 2) gate_norm_kernel(const GateNormArgs a,
                                                               int64_t items_per_cta) {
  constexpr int TPR = D / 8;              // threads per row
  constexpr int ROWS = kGnThreads / TPR;  // rows per sweep
  constexpr int KP = Piece<T>::kPieces;
  constexpr int kPerItem = 2 * kSweeps * KP;  // o and g pieces per thread and item
  extern __shared__ uint4 ring[];             // [kStages][kPerItem][kGnThreads]
  const int tid = threadIdx.x;
  const int lt = tid % TPR;
  const int64_t per_token = (a.H + ROWS * kSweeps - 1) / (ROWS * kSweeps);
  const int64_t items = a.T * per_token;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * items_per_cta;
  const int64_t i1 = min(i0 + items_per_cta, items);
  const T* o = static_cast<const T*>(a.o);
  const T* g = static_cast<const T*>(a.gate);
  T* y = static_cast<T*>(a.y);

  auto slot = [&](int stage, int piece) -> uint4* {
    return ring + (stage * kPerItem + piece) * kGnThreads + tid;
  };
  // copy the pieces of item `it` into ring stage `st` (one commit group, empty past the range)
  auto issue = [&](int64_t it, const ItemCursor& c, int st) {
    if (it < i1) {
      const int64_t t = c.t;
      const int64_t hb = c.sub * (ROWS * kSweeps);
#pragma unroll
      for (int j = 0; j < kSweeps; ++j) {
        const int64_t h = hb + j * ROWS + tid / TPR;
        const bool valid = h < a.H;
        const int64_t off = valid ? (t * a.H + h) * D + lt * 8 : 0;
#pragma unroll
        for (int p = 0; p < KP; ++p) {
          cp_async16(slot(st, j * KP + p), o + off + p * Piece<T>::kElems, valid);
          cp_async16(slot(st, (kSweeps + j) * KP + p), g + off + p * Piece<T>::kElems, valid);
        }
      }
    }
    cp_async_commit();
  };

  ItemCursor cur = ItemCursor::at(i0, per_token);  // item it
  ItemCursor ahead = cur;                          // item it + 2
  issue(i0, ahead, 0);
  ahead.advance(per_token);
  issue(i0 + 1, ahead, 1);
  ahead.advance(per_token);
  int st = 0;
  for (int64_t it = i0; it < i1; ++it) {
    issue(it + 2, ahead, st == 0 ? 2 : st - 1);  // the stage item it - 1 used
    ahead.advance(per_token);
    cp_async_wait<2>();                          // item it's group has landed
    const int64_t t = cur.t;
    const int64_t hb = cur.sub * (ROWS * kSweeps);
    cur.advance(per_token);
#pragma unroll
    for (int j = 0; j < kSweeps; ++j) {
      const int64_t h = hb + j * ROWS + tid / TPR;
      uint4 wo[KP], wg[KP];
#pragma unroll
      for (int p = 0; p < KP; ++p) {
        wo[p] = *slot(st, j * KP + p);
        wg[p] = *slot(st, (kSweeps + j) * KP + p);
      }
      float xo[8];
      Piece<T>::unpack(wo, xo);
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(xo[e], xo[e], ss);
#pragma unroll
      for (int m = TPR / 2; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
      if (a.scales != nullptr) {
        // FP8 E4M3 output: y is rounded to the I/O dtype first (the value the unfused chain would
        // store before its quantize step); the row's (the block's) largest |y| sets its scale,
        // amax / 448, and each value is stored as E4M3(y * 448 / amax), rounded to nearest even
        // and saturated.  Every lane takes part in the max reduction; rows past H compute zeros.
        const bool row_ok = h < a.H;
        float xg[8];
        Piece<T>::unpack(wg, xg);
        const float rinv = rsqrtf(fmaf(ss, 1.f / D, a.eps));
        float gm[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (row_ok) {
          const float4 g0 = __ldg(reinterpret_cast<const float4*>(a.gamma + h * D + lt * 8));
          const float4 g1 = __ldg(reinterpret_cast<const float4*>(a.gamma + h * D + lt * 8) + 1);
          gm[0] = g0.x; gm[1] = g0.y; gm[2] = g0.z; gm[3] = g0.w;
          gm[4] = g1.x; gm[5] = g1.y; gm[6] = g1.z; gm[7] = g1.w;
        }
        float out[8];
        float am = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          out[e] = Io<T>::round(gm[e] * (xo[e] * rinv) * Sigmoid<T>::f(xg[e]));
          am = fmaxf(am, fabsf(out[e]));
        }
#pragma unroll
        for (int m = TPR / 2; m > 0; m >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, m));
        if (row_ok) {
          const float inv = am > 0.f ? 448.f / am : 0.f;
          uint32_t w[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2)
            w[e2] = __nv_cvt_float2_to_fp8x2(make_float2(out[2 * e2] * inv, out[2 * e2 + 1] * inv),
                                             __NV_SATFINITE, __NV_E4M3);
          uint8_t* y8 = static_cast<uint8_t*>(a.y) + (t * a.H + h) * D + lt * 8;
          __stcs(reinterpret_cast<uint2*>(y8), make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16)));
          if (lt == 0) a.scales[h * a.T + t] = am / 448.f;
        }
        continue;
      }
      if (h < a.H) {  // uniform across a row's threads
        float xg[8];
        Piece<T>::unpack(wg, xg);
        const float rinv = rsqrtf(fmaf(ss, 1.f / D, a.eps));
        const float4 g0 = __ldg(reinterpret_cast<const float4*>(a.gamma + h * D + lt * 8));
        const float4 g1 = __ldg(reinterpret_cast<const float4*>(a.gamma + h * D + lt * 8) + 1);
        const float gm[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        float out[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) out[e] = gm[e] * (xo[e] * rinv) * Sigmoid<T>::f(xg[e]);
        Io<T>::store(y + (t * a.H + h) * D + lt * 8, out);
      }
    }
    st = st == kStages - 1 ? 0 : st + 1;
  }
  cp_async_wait<0>();  // no copy outlives the CTA
}

template <typename T, int D>
cudaError_t launch_dim(const GateNormArgs& a, cudaStream_t stream) {
  constexpr int ROWS = kGnThreads / (D / 8);
  constexpr size_t kSmem = size_t(kStages) * 2 * kSweeps * Piece<T>::kPieces * kGnThreads * 16;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // set on every call: cheap, safe from any host thread, and it survives a context reset
  e = cudaFuncSetAttribute(gate_norm_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmem));
  if (e != cudaSuccess) return e;
  const int64_t per_token = (a.H + ROWS * kSweeps - 1) / (ROWS * kSweeps);
  const int64_t items = a.T * per_token;
  const int64_t resident = kSmem <= 100 * 1024 ? 2 : 1;  // CTAs per SM that the ring allows
  const int64_t grid0 = std::max<int64_t>(1, std::min<int64_t>(items, resident * sms));
  const int64_t per_cta = (items + grid0 - 1) / grid0;
  const int64_t grid = (items + per_cta - 1) / per_cta;
  gate_norm_kernel<T, D><<<static_cast<unsigned>(grid), kGnThreads, kSmem, stream>>>(a, per_cta);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_typed(const GateNormArgs& a, cudaStream_t stream) {
  return a.d == 64 ? launch_dim<T, 64>(a, stream) : launch_dim<T, 128>(a, stream);
}

}  // namespace

cudaError_t launch_gate_norm(const GateNormArgs& a, cudaStream_t stream) {
  if (a.T == 0) return cudaSuccess;
  return a.dtype == kF32 ? launch_typed<float>(a, stream) : launch_typed<__nv_bfloat16>(a, stream);
}

}  // namespace la
