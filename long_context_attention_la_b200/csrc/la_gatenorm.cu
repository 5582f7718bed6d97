// la_gatenorm.cu — the fused operator after the kernel: grouped RMSNorm + sigmoid gate.
//
// "Ling and Ring 2.6 Technical Report", §2.1 Fig. 2 (Linear Attention Kernel -> Grouped RMSNorm,
// multiplied by sigmoid(Gate Projection) -> Output Projection) and §4.3 (group norm + sigmoid gate
// run as one fused inference operator).  Per token t and head h (each head is one norm group):
//     y = gamma[h] * o / sqrt(mean(o^2) + eps) * sigmoid(g)
// Memory bound: read o and g, write y (3 rows of d per token-head).  One CTA per token; a row is
// handled by d/8 threads of 16 bytes, the mean square is a shuffle reduction over them, and every
// thread issues the loads of all its rows before using any.
#include <cuda_bf16.h>

#include <cstdint>

#include "la_internal.h"

namespace la {
namespace {

constexpr int kGnThreads = 256;

template <typename T>
struct Io;

template <>
struct Io<__nv_bfloat16> {  // 8 values = one 16-byte load
  using Vec = uint4;
  static __device__ __forceinline__ void unpack(const uint4& w, float (&x)[8]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[2 * e] = __uint_as_float(u[e] << 16);
      x[2 * e + 1] = __uint_as_float(u[e] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(lo))) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(hi))) << 16);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* dst, const float (&y)[8]) {
    __stcs(reinterpret_cast<uint4*>(dst),
           make_uint4(pack2(y[0], y[1]), pack2(y[2], y[3]), pack2(y[4], y[5]), pack2(y[6], y[7])));
  }
  static __device__ __forceinline__ void load(const __nv_bfloat16* src, float (&x)[8]) {
    unpack(__ldcs(reinterpret_cast<const uint4*>(src)), x);
  }
};

template <>
struct Io<float> {  // 8 values = two 16-byte loads
  static __device__ __forceinline__ void load(const float* src, float (&x)[8]) {
    const float4 a = __ldcs(reinterpret_cast<const float4*>(src));
    const float4 b = __ldcs(reinterpret_cast<const float4*>(src) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* dst, const float (&y)[8]) {
    __stcs(reinterpret_cast<float4*>(dst), make_float4(y[0], y[1], y[2], y[3]));
    __stcs(reinterpret_cast<float4*>(dst) + 1, make_float4(y[4], y[5], y[6], y[7]));
  }
};

// bf16 rows stay packed (one uint4 per 8 values) between load and use, so a thread keeps all its
// loads in flight with few registers; fp32 rows take two float4 each.
template <typename T>
struct Raw;
template <>
struct Raw<__nv_bfloat16> {
  uint4 w;
  __device__ __forceinline__ void load(const __nv_bfloat16* src) {
    w = __ldcs(reinterpret_cast<const uint4*>(src));
  }
  __device__ __forceinline__ void zero() { w = make_uint4(0u, 0u, 0u, 0u); }
  __device__ __forceinline__ void unpack(float (&x)[8]) const { Io<__nv_bfloat16>::unpack(w, x); }
};
template <>
struct Raw<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* src) {
    a = __ldcs(reinterpret_cast<const float4*>(src));
    b = __ldcs(reinterpret_cast<const float4*>(src) + 1);
  }
  __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void unpack(float (&x)[8]) const {
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};

template <typename T, int D>
__global__ void __launch_bounds__(kGnThreads) gate_norm_kernel(const GateNormArgs a) {
  constexpr int TPR = D / 8;                // threads per row
  constexpr int ROWS = kGnThreads / TPR;    // rows per sweep
  constexpr int kSweeps = 4;                // sweeps whose loads are issued together
  const int lt = threadIdx.x % TPR;
  const int64_t t = blockIdx.x;
  const T* o = static_cast<const T*>(a.o);
  const T* g = static_cast<const T*>(a.gate);
  T* y = static_cast<T*>(a.y);
  for (int64_t hb = 0; hb < a.H; hb += ROWS * kSweeps) {  // uniform trip count across the CTA
    Raw<T> ro[kSweeps], rg[kSweeps];
#pragma unroll
    for (int j = 0; j < kSweeps; ++j) {
      const int64_t h = hb + j * ROWS + threadIdx.x / TPR;
      if (h < a.H) {
        const int64_t off = (t * a.H + h) * D + lt * 8;
        ro[j].load(o + off);
        rg[j].load(g + off);
      } else {
        ro[j].zero();
        rg[j].zero();
      }
    }
#pragma unroll
    for (int j = 0; j < kSweeps; ++j) {
      const int64_t h = hb + j * ROWS + threadIdx.x / TPR;
      float xo[8];
      ro[j].unpack(xo);
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(xo[e], xo[e], ss);
#pragma unroll
      for (int m = TPR / 2; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
      if (h < a.H) {
        float xg[8];
        rg[j].unpack(xg);
        const float rinv = rsqrtf(fmaf(ss, 1.f / D, a.eps));
        const float* gam = a.gamma + h * D + lt * 8;
        float out[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float sig = 1.f / (1.f + __expf(-xg[e]));
          out[e] = __ldg(gam + e) * (xo[e] * rinv) * sig;
        }
        Io<T>::store(y + (t * a.H + h) * D + lt * 8, out);
      }
    }
  }
}

template <typename T>
cudaError_t launch_typed(const GateNormArgs& a, cudaStream_t stream) {
  if (a.d == 64)
    gate_norm_kernel<T, 64><<<static_cast<unsigned>(a.T), kGnThreads, 0, stream>>>(a);
  else
    gate_norm_kernel<T, 128><<<static_cast<unsigned>(a.T), kGnThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate_norm(const GateNormArgs& a, cudaStream_t stream) {
  if (a.T == 0) return cudaSuccess;
  return a.dtype == kF32 ? launch_typed<float>(a, stream) : launch_typed<__nv_bfloat16>(a, stream);
}

}  // namespace la
