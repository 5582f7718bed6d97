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
// is handled by d/16 consecutive threads with two 16-byte pieces each, chosen so that both
// members of every rotary pair sit in one thread (no exchange between threads), staged through
// a shared-memory ring by per-thread cp.async copies; the mean square is a shuffle reduction over
// the row's threads.  The norm weights sit in shared memory (per-row loads of them through L1
// doubled the L1 traffic), and the row arithmetic runs on paired fp32 operations (two lanes per
// instruction; the sum of squares keeps two partial sums).  The angle pos * w_i is formed and reduced modulo 2 pi in
// double precision (positions reach 2^18 and more, where a float angle would be off by ~0.03 rad),
// then sin and cos are taken in float, once per token and frequency by each warp.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "la_internal.h"
#include "la_sm100.cuh"

namespace la {
namespace {

constexpr int kQkThreads = 512;

// two floats -> bf16x2 (round to nearest even, one paired conversion), lo in the low half
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

// Work item: ROWS x kBatch rows of one token (q heads first, then k heads); a CTA takes a
// contiguous range of items.  A row is handled by D/16 threads, each holding two 16-byte pieces
// (8 dims each) that are r/2 dims apart inside the rotary span (so both members of every
// rotate-half pair sit in one thread) and (D - r)/2 dims apart beyond it; a warp's copies still
// cover whole 32-byte sectors.  Row loads go through a kStages-deep shared-memory ring filled two
// items ahead with per-thread cp.async copies (each thread reads back only its own pieces), so
// the bytes in flight are held by shared memory rather than registers.  Every warp computes the
// rotation angles of its item's token itself (all of a warp's rows belong to one token) into a
// table of its own, so no block barrier is needed anywhere: a barrier per item made every warp
// wait for the slowest warp's copies.
constexpr int kStages = 3;
constexpr int kBatch = 2;  // sweeps of ROWS rows per item

template <int D>
__global__ void __launch_bounds__(kQkThreads, 2) qk_norm_rope_kernel(const QkNormRopeArgs a,
                                                                  int64_t items_per_cta) {
  constexpr int TPR = D / 16;                  // threads per row
  constexpr int ROWS = kQkThreads / TPR;       // rows per sweep
  extern __shared__ uint4 ring[];              // [kStages][kBatch][2][kQkThreads]
  __shared__ __align__(16) float cs_sh[kQkThreads / 32][64];  // per warp: cos, sin of the token
  __shared__ __align__(16) float sn_sh[kQkThreads / 32][64];
  // gamma_q, gamma_k; 4 floats of padding after every 64, so the 16-byte reads of one row's
  // threads (pieces 0..3 and 8..11 of the row, 256 bytes apart) fall in different banks
  constexpr int kGamStride = D + 4 * (D / 64);
  __shared__ __align__(16) float gam_sh[2][kGamStride];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int u = tid % TPR;                     // position of this thread in its row
  const int64_t rows = 2 * a.H;                // q heads, then k heads
  const int64_t per_token = (rows + ROWS * kBatch - 1) / (ROWS * kBatch);
  const int64_t items = a.T * per_token;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * items_per_cta;
  const int64_t i1 = min(i0 + items_per_cta, items);
  const int half = a.rotary_dim / 2;
  const int rot_threads = a.rotary_dim / 16;   // threads holding rotary pairs
  const bool rotary = u < rot_threads;
  // the thread's two pieces (8-dim units): (u, u + r/16) in the rotary span, else
  // (r/8 + m, r/8 + m + (D - r)/16) with m = u - r/16
  const int pa = rotary ? u : a.rotary_dim / 8 + (u - rot_threads);
  const int pb = rotary ? u + rot_threads : pa + (D - a.rotary_dim) / 16;

  for (int i = threadIdx.x; i < 2 * D; i += kQkThreads) {
    const int dd = i % D;
    gam_sh[i / D][dd + 4 * (dd / 64)] = i < D ? a.gamma_q[i] : a.gamma_k[i - D];
  }
  __syncthreads();
  auto slot = [&](int stage, int j, int w) -> uint4* {
    return ring + ((stage * kBatch + j) * 2 + w) * kQkThreads + tid;
  };
  auto issue = [&](int64_t it, const ItemCursor& c, int st) {
    if (it < i1) {
      const int64_t t = c.t;
      const int64_t rb = c.sub * (ROWS * kBatch);
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int64_t row = rb + j * ROWS + tid / TPR;
        const bool valid = row < rows;
        const bool is_k = row >= a.H;
        const int64_t h = is_k ? row - a.H : row;
        const __nv_bfloat16* src =
            valid ? (is_k ? a.k : a.q) + t * (is_k ? a.k_stride : a.q_stride) + h * D : a.q;
        cp_async16(slot(st, j, 0), valid ? src + pa * 8 : src, valid);
        cp_async16(slot(st, j, 1), valid ? src + pb * 8 : src, valid);
      }
    }
    cp_async_commit();
  };
  // cos / sin at position `pos` into this warp's table, frequency f by lane f % 32.  The angle is
  // reduced to [-pi, pi] in fp64 first, where the fast sin/cos (absolute error about 2^-21) is
  // far below the bf16 rounding of the output.
  auto angles = [&](int64_t pos) {
    constexpr double kTwoPi = 6.283185307179586476925286766559;
    constexpr double kInvTwoPi = 0.15915494309189533576888376337251;
    for (int f = lane; f < half; f += 32) {
      // explicit roundings (no contraction left to the compiler), so that the prefill kernel's
      // in-tile form of this operator reproduces the angles bit for bit
      const double a0 = __dmul_rn(static_cast<double>(pos), a.inv_freq[f]);
      float sn, cs;
      __sincosf(static_cast<float>(__fma_rn(-kTwoPi, rint(__dmul_rn(a0, kInvTwoPi)), a0)), &sn,
                &cs);
      cs_sh[warp][f] = cs;
      sn_sh[warp][f] = sn;
    }
  };
  auto unpack = [](const uint4& w, float2 (&x)[4]) {
    const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      x[e] = make_float2(__uint_as_float(v[e] << 16), __uint_as_float(v[e] & 0xffff0000u));
  };
  auto pack_row = [](const float2 (&y)[4]) {
    uint4 w;
    w.x = pack2(y[0].x, y[0].y);
    w.y = pack2(y[1].x, y[1].y);
    w.z = pack2(y[2].x, y[2].y);
    w.w = pack2(y[3].x, y[3].y);
    return w;
  };


  ItemCursor cur = ItemCursor::at(i0, per_token);  // item it
  ItemCursor ahead = cur;                          // item it + 2
  issue(i0, ahead, 0);
  ahead.advance(per_token);
  issue(i0 + 1, ahead, 1);
  ahead.advance(per_token);
  int st = 0;
  int64_t pos = i0 < i1 ? a.positions[cur.t] : 0;
  for (int64_t it = i0; it < i1; ++it) {
    issue(it + 2, ahead, st == 0 ? 2 : st - 1);  // the stage item it - 1 used
    ahead.advance(per_token);
    const int64_t t = cur.t;
    const int64_t rb = cur.sub * (ROWS * kBatch);
    cur.advance(per_token);
    // the next item's position, one item ahead of its use
    const int64_t pos_next = it + 1 < i1 ? a.positions[cur.t] : 0;
    __syncwarp();                         // the warp is done reading the previous token's table
    angles(pos);
    __syncwarp();                         // ... and this token's table is written
    cp_async_wait<2>();                   // item it's rows have landed (this thread's pieces)
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int64_t row = rb + j * ROWS + tid / TPR;
      const bool valid = row < rows;  // uniform across a row's threads
      const bool is_k = row >= a.H;
      const int64_t h = is_k ? row - a.H : row;
      float2 xa[4], xb[4];
      unpack(*slot(st, j, 0), xa);
      unpack(*slot(st, j, 1), xb);
      // mean square over the row: reduce across the TPR threads of the row (aligned groups)
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc = __ffma2_rn(xb[e], xb[e], __ffma2_rn(xa[e], xa[e], acc));
      float ss = acc.x + acc.y;
#pragma unroll
      for (int o = TPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float rinv = rsqrtf(fmaf(ss, 1.f / D, a.eps));
      const float2 r2 = make_float2(rinv, rinv);
      const float* gam = gam_sh[is_k ? 1 : 0];
      const float4* gpa = reinterpret_cast<const float4*>(gam + pa * 8 + 4 * (pa / 8));
      const float4* gpb = reinterpret_cast<const float4*>(gam + pb * 8 + 4 * (pb / 8));
      const float4 ga0 = gpa[0], ga1 = gpa[1];
      const float4 gb0 = gpb[0], gb1 = gpb[1];
      const float2 gma[4] = {make_float2(ga0.x, ga0.y), make_float2(ga0.z, ga0.w),
                             make_float2(ga1.x, ga1.y), make_float2(ga1.z, ga1.w)};
      const float2 gmb[4] = {make_float2(gb0.x, gb0.y), make_float2(gb0.z, gb0.w),
                             make_float2(gb1.x, gb1.y), make_float2(gb1.z, gb1.w)};
      float2 ya[4], yb[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ya[e] = __fmul2_rn(gma[e], __fmul2_rn(xa[e], r2));
        yb[e] = __fmul2_rn(gmb[e], __fmul2_rn(xb[e], r2));
      }
      if (rotary) {
        // rotate-half: dims (8 pa + e, 8 pa + e + r/2) with frequency index 8 pa + e
        const float4* c4 = reinterpret_cast<const float4*>(&cs_sh[warp][pa * 8]);
        const float4* s4 = reinterpret_cast<const float4*>(&sn_sh[warp][pa * 8]);
        const float4 c0 = c4[0], c1 = c4[1], s0 = s4[0], s1 = s4[1];
        const float2 cs[4] = {make_float2(c0.x, c0.y), make_float2(c0.z, c0.w),
                              make_float2(c1.x, c1.y), make_float2(c1.z, c1.w)};
        const float2 sn[4] = {make_float2(s0.x, s0.y), make_float2(s0.z, s0.w),
                              make_float2(s1.x, s1.y), make_float2(s1.z, s1.w)};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 y0 = ya[e], y1 = yb[e];
          const float2 nsn = make_float2(-sn[e].x, -sn[e].y);
          ya[e] = __ffma2_rn(y0, cs[e], __fmul2_rn(y1, nsn));
          yb[e] = __ffma2_rn(y1, cs[e], __fmul2_rn(y0, sn[e]));
        }
      }
      if (valid) {
        __nv_bfloat16* dst = (is_k ? a.k_out : a.q_out) + (t * a.H + h) * D;
        __stcs(reinterpret_cast<uint4*>(dst + pa * 8), pack_row(ya));
        __stcs(reinterpret_cast<uint4*>(dst + pb * 8), pack_row(yb));
      }
    }
    st = st == kStages - 1 ? 0 : st + 1;
    pos = pos_next;
  }
  cp_async_wait<0>();  // no copy outlives the CTA
}

template <int D>
cudaError_t launch_dim(const QkNormRopeArgs& a, cudaStream_t stream) {
  constexpr int ROWS = kQkThreads / (D / 16);
  constexpr size_t kSmem = size_t(kStages) * kBatch * 2 * kQkThreads * 16;  // 96 KiB: 2 per SM
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // set on every call: cheap, safe from any host thread, and it survives a context reset
  e = cudaFuncSetAttribute(qk_norm_rope_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmem));
  if (e != cudaSuccess) return e;
  const int64_t per_token = (2 * a.H + ROWS * kBatch - 1) / (ROWS * kBatch);
  const int64_t items = a.T * per_token;
  const int64_t grid0 = std::max<int64_t>(1, std::min<int64_t>(items, 2 * int64_t(sms)));
  const int64_t per_cta = (items + grid0 - 1) / grid0;
  const int64_t grid = (items + per_cta - 1) / per_cta;
  qk_norm_rope_kernel<D><<<static_cast<unsigned>(grid), kQkThreads, kSmem, stream>>>(a, per_cta);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qk_norm_rope(const QkNormRopeArgs& a, cudaStream_t stream) {
  if (a.T == 0) return cudaSuccess;
  return a.d == 64 ? launch_dim<64>(a, stream) : launch_dim<128>(a, stream);
}

}  // namespace la
