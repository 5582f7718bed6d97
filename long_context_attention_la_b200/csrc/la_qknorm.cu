// la_qknorm.cu — the fused operator that feeds the kernel: QK RMSNorm + partial rotary embedding.
//
// "Ling and Ring 2.6 Technical Report", §2.1 Fig. 2 (QKV Projection -> QK Norm -> RoPE -> Linear
// Attention Kernel), §2.1.1 (RMSNorm eps = 1e-6; rotary dimension 64 of the 128 head dims;
// theta = 6,000,000) and §4.3 (split + QK norm + RoPE run as one fused inference operator).  Per
// token t and head h of q and of k:
//     y = gamma * x / sqrt(mean(x^2) + eps)
//     (y_i, y_{i+r/2}) <- (y_i cos a - y_{i+r/2} sin a, y_{i+r/2} cos a + y_i sin a),
//     a = pos_t * theta^(-2i/r), i < r/2 (rotate-half pairs); dims >= r pass through.
//
// Memory bound: one pass over q and k (read 2 rows, write 2 rows of d bf16 per token-head).  A row
// is handled by d/8 consecutive threads, 16 bytes each, so a warp reads whole rows; the mean
// square is a shuffle reduction over the row's threads and each rotary pair's partner value comes
// from the thread r/16 positions away.  The angle pos * w_i is formed and reduced modulo 2 pi in
// double precision (positions reach 2^18 and more, where a float angle would be off by ~0.03 rad),
// then sin and cos are taken in float, once per token and frequency.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "la_internal.h"

namespace la {
namespace {

constexpr int kQkThreads = 256;

// two floats -> bf16x2 (round to nearest even), lo in the low half
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
  const uint32_t u = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return l | (u << 16);
}

// Each CTA takes two tokens and issues the loads of both tokens' 2H rows before using any (enough
// bytes in flight per SM to stream), computes each token's r/2 rotation angles once
// (double-precision angle and reduction, float sin/cos) into shared memory, then sweeps the rows
// ROWS at a time.
template <int D>
__global__ void __launch_bounds__(kQkThreads) qk_norm_rope_kernel(const QkNormRopeArgs a) {
  constexpr int TPR = D / 8;                   // threads per row
  constexpr int ROWS = kQkThreads / TPR;       // rows per sweep step
  constexpr int kBatch = 8;                    // sweeps per token held in registers
  __shared__ float cs_sh[2][64], sn_sh[2][64];
  const int lt = threadIdx.x % TPR;            // position of this thread in its row
  const int64_t rows = 2 * a.H;                // q heads, then k heads
  const int half = a.rotary_dim / 2;

  auto load_rows = [&](int64_t t, int64_t rb, uint4 (&raw)[kBatch]) {
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int64_t row = rb + j * ROWS + threadIdx.x / TPR;
      raw[j] = make_uint4(0u, 0u, 0u, 0u);
      if (t < a.T && row < rows) {
        const bool is_k = row >= a.H;
        const int64_t h = is_k ? row - a.H : row;
        const __nv_bfloat16* src =
            (is_k ? a.k : a.q) + t * (is_k ? a.k_stride : a.q_stride) + h * D + lt * 8;
        raw[j] = __ldcs(reinterpret_cast<const uint4*>(src));
      }
    }
  };
  auto angles = [&](int64_t t, int buf) {
    if (t < a.T && threadIdx.x < half) {
      constexpr double kTwoPi = 6.283185307179586476925286766559;
      constexpr double kInvTwoPi = 0.15915494309189533576888376337251;
      double ang = static_cast<double>(a.positions[t]) * a.inv_freq[threadIdx.x];
      ang -= kTwoPi * rint(ang * kInvTwoPi);
      float sn, cs;
      sincosf(static_cast<float>(ang), &sn, &cs);
      cs_sh[buf][threadIdx.x] = cs;
      sn_sh[buf][threadIdx.x] = sn;
    }
  };

  const int half_threads = a.rotary_dim / 16;  // threads per half of the rotary dims
  const bool rotary = lt < 2 * half_threads;
  const bool first = lt < half_threads;
  const int lane = threadIdx.x & 31;
  const int partner_lane = rotary ? (first ? lane + half_threads : lane - half_threads) : lane;
  const int i0 = (first ? lt : lt - half_threads) * 8;  // frequency index of element 0

  // normalise + rotate the rows held in raw (sweeps rb .. rb + kBatch - 1 of token t)
  auto finish = [&](int64_t t, int64_t rb, const uint4 (&raw)[kBatch], int buf) {
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int64_t row = rb + j * ROWS + threadIdx.x / TPR;
      const bool valid = row < rows;  // uniform across a row's threads
      const bool is_k = row >= a.H;
      const int64_t h = is_k ? row - a.H : row;
      const uint32_t u[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
      float x[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[2 * e] = __uint_as_float(u[e] << 16);
        x[2 * e + 1] = __uint_as_float(u[e] & 0xffff0000u);
      }
      // mean square over the row: reduce across the TPR threads of the row (aligned groups)
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
      for (int o = TPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float rinv = rsqrtf(fmaf(ss, 1.f / D, a.eps));
      const float* gam = (is_k ? a.gamma_k : a.gamma_q) + lt * 8;
      float y[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = __ldg(gam + e) * (x[e] * rinv);
      // rotate-half over the first r dims: the partner of element j is j +- r/2, held by the
      // thread r/16 positions away in the same row
      float pv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) pv[e] = __shfl_sync(0xffffffffu, y[e], partner_lane);
      if (rotary) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float cs = cs_sh[buf][i0 + e], sn = sn_sh[buf][i0 + e];
          y[e] = first ? fmaf(y[e], cs, -pv[e] * sn) : fmaf(y[e], cs, pv[e] * sn);
        }
      }
      if (valid) {
        __nv_bfloat16* dst = (is_k ? a.k_out : a.q_out) + (t * a.H + h) * D + lt * 8;
        uint4 w;
        w.x = pack2(y[0], y[1]);
        w.y = pack2(y[2], y[3]);
        w.z = pack2(y[4], y[5]);
        w.w = pack2(y[6], y[7]);
        __stcs(reinterpret_cast<uint4*>(dst), w);
      }
    }
  };

  // two tokens per CTA, all of their row loads issued before any is used
  const int64_t t0 = 2 * static_cast<int64_t>(blockIdx.x), t1 = t0 + 1;
  uint4 ra[kBatch], rb_[kBatch];
  load_rows(t0, 0, ra);
  load_rows(t1, 0, rb_);
  angles(t0, 0);
  angles(t1, 1);
  __syncthreads();
  finish(t0, 0, ra, 0);
  for (int64_t rb = ROWS * kBatch; rb < rows; rb += ROWS * kBatch) {  // H > 64: more sweeps
    load_rows(t0, rb, ra);
    finish(t0, rb, ra, 0);
  }
  if (t1 < a.T) {  // uniform across the CTA
    finish(t1, 0, rb_, 1);
    for (int64_t rb = ROWS * kBatch; rb < rows; rb += ROWS * kBatch) {
      load_rows(t1, rb, rb_);
      finish(t1, rb, rb_, 1);
    }
  }
}

}  // namespace

cudaError_t launch_qk_norm_rope(const QkNormRopeArgs& a, cudaStream_t stream) {
  if (a.T == 0) return cudaSuccess;
  const int64_t grid = (a.T + 1) / 2;  // two tokens per CTA
  if (a.d == 64)
    qk_norm_rope_kernel<64><<<static_cast<unsigned>(grid), kQkThreads, 0, stream>>>(a);
  else
    qk_norm_rope_kernel<128><<<static_cast<unsigned>(grid), kQkThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace la
