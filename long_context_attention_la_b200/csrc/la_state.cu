// la_state.cu — the state-only prefill on the sm_100a tensor cores, and the fold of per-part
// states.
//
// Context-parallel forward of Lightning Attention ("Ling and Ring 2.6 Technical Report", §4.1.1
// Context Parallel for Lightning Attention, Fig. 10): every rank holds one contiguous part of the
// sequence, computes that part's local state h from its own K, V ("local h"), exchanges the states
// (AllGather), and folds the states of the parts before it into its incoming state ("fused update
// h").  The two device steps here:
//
//   state pass   per (b, h) of a fixed-length batch of N tokens
//                    S_out = lambda^N S_in + sum_{t<N} lambda^(N-1-t) k_t^T v_t
//                i.e. the final state of the prefill without its outputs (q is not read).  The
//                sum is one [d x N] x [N x d] contraction with the rows of K pre-scaled,
//                    K~_t = lambda^(N-1-t) k_t,   S_out - lambda^N S_in = K~^T V,
//                so a whole range of chunks accumulates in one TMEM tile with no rescaling in
//                between (weights below the fp32 range belong to terms that no longer matter).
//   fold         S <- lambda^(L_j) S + h_j over parts j = 0 .. n-1, starting from S_in.
//
// State pass work split: the B*H*ceil(N/C) chunk-loads, head-major, are cut into one contiguous
// range per CTA (one CTA per SM; ranges differ by at most one chunk).  A range covers whole
// heads and at most two partial ones.  A whole head goes straight to state_out; a partial one
// goes to a workspace slot, and a second small kernel adds a split head's partials in range
// order (the result does not depend on timing) together with lambda^N S_in.
// Roles (384 threads):
//   warp 0      TMA producer: three-stage ring of K, V tiles (64 KiB per stage)
//   warp 1      tcgen05.mma issuer: acc[piece % 2] (+)= K~^T V, one chunk at a time
//   warp 2      TMEM allocator (256 columns: two accumulators)
//   warps 4-7   K -> K~ in shared memory, one thread per row
//   warps 8-11  read-out: accumulator -> fp32 global, 16-byte pieces exchanged within 4-lane
//               groups so that every store writes whole 32-byte sectors
// Every wait is bounded in time; on expiry the CTA records LA_ERR_TIMEOUT in the workspace status
// word, unwinds, frees its TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "la_internal.h"
#include "la_sm100.cuh"

namespace la {
namespace {

constexpr int C = kChunk;       // 128 tokens per chunk
constexpr int D = kHeadDim;     // 128
constexpr int kThreads = 384;   // 12 warps
constexpr int kStages = 3;
constexpr uint32_t kWarpK0 = 4;  // warps 4..7: K scaling
constexpr uint32_t kWarpR0 = 8;  // warps 8..11: read-out
constexpr uint32_t kTileBytes = C * D * 2;       // one bf16 [128 x 128] tile
constexpr uint32_t kHalfBytes = kTileBytes / 2;  // [128 rows x 64 cols], 128-byte rows
constexpr uint32_t kOffK = 0;
constexpr uint32_t kOffV = kTileBytes;
constexpr uint32_t kStageBytes = 2 * kTileBytes;  // 64 KiB
constexpr uint32_t kOffCtrl = kStages * kStageBytes;
constexpr uint32_t kCtrlBytes = 256;
constexpr uint32_t kSmemAlloc = kOffCtrl + kCtrlBytes + 1024;  // slack for 1024-byte alignment
constexpr uint32_t kTmemCols = 256;
constexpr int32_t kErrTimeout = -8;  // LA_ERR_TIMEOUT
constexpr float kLog2e = 1.4426950408889634f;

struct Ctrl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t kt_ready[kStages];
  uint64_t acc_full[2];
  uint64_t acc_free[2];
  uint64_t mma_final;
  uint32_t tmem_base;
  uint32_t abort;
};
static_assert(sizeof(Ctrl) <= kCtrlBytes, "control block too large");

struct StateParams {
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  const float* slopes;
  const float* state_in;  // fp32 [B*H, D, D] or null
  float* state_out;       // fp32 [B*H, D, D]
  float* partial;         // fp32 [2 * grid, D, D]: slot 2i + (head == first head of range i ? 0 : 1)
  int32_t* status;
  int64_t N, H, n_chunks, total, width;  // width: chunk-loads per CTA
  uint64_t timeout_ns;
};

// lambda^n in fp64, rounded once to fp32
__device__ __forceinline__ float decay_pow(float slope, int64_t n) {
  return static_cast<float>(exp(-static_cast<double>(slope) * static_cast<double>(n)));
}

// Multiplies the 64 bf16 of one half-row (row r of a swizzled [128 x 64] half-tile) by w, in
// fp32 with one rounding; the 8 rows of a swizzle atom touch 8 different bank groups per step.
__device__ __forceinline__ void scale_half_row(uint8_t* half_tile, uint32_t r, float w) {
  uint8_t* row = half_tile + (r >> 3) * 1024u + (r & 7u) * 128u;
#pragma unroll
  for (uint32_t c0 = 0; c0 < 8; c0 += 4) {
    uint4 x[4];
#pragma unroll
    for (uint32_t c = 0; c < 4; ++c)
      x[c] = *reinterpret_cast<const uint4*>(row + (((c0 + c) ^ (r & 7u)) << 4));
#pragma unroll
    for (uint32_t c = 0; c < 4; ++c) {
      x[c].x = pack_bf16x2(bf16lo_to_f32(x[c].x) * w, bf16hi_to_f32(x[c].x) * w);
      x[c].y = pack_bf16x2(bf16lo_to_f32(x[c].y) * w, bf16hi_to_f32(x[c].y) * w);
      x[c].z = pack_bf16x2(bf16lo_to_f32(x[c].z) * w, bf16hi_to_f32(x[c].z) * w);
      x[c].w = pack_bf16x2(bf16lo_to_f32(x[c].w) * w, bf16hi_to_f32(x[c].w) * w);
      *reinterpret_cast<uint4*>(row + (((c0 + c) ^ (r & 7u)) << 4)) = x[c];
    }
  }
}

__device__ __forceinline__ float4 shfl_xor_f4(float4 v, int m) {
  v.x = __shfl_xor_sync(0xffffffffu, v.x, m);
  v.y = __shfl_xor_sync(0xffffffffu, v.y, m);
  v.z = __shfl_xor_sync(0xffffffffu, v.z, m);
  v.w = __shfl_xor_sync(0xffffffffu, v.w, m);
  return v;
}
// 4 x 4 transpose of 16-byte pieces within each group of 4 lanes: on entry lane t holds pieces
// x[0..3] of its own row; on exit it holds piece t of the group's rows 0..3.
__device__ __forceinline__ void transpose4x4_lanes(float4 (&x)[4], uint32_t t) {
  const bool hi = (t & 2u) != 0;
  float4 a = shfl_xor_f4(hi ? x[0] : x[2], 2);
  float4 b = shfl_xor_f4(hi ? x[1] : x[3], 2);
  if (hi) {
    x[0] = a;
    x[1] = b;
  } else {
    x[2] = a;
    x[3] = b;
  }
  const bool odd = (t & 1u) != 0;
  a = shfl_xor_f4(odd ? x[0] : x[1], 1);
  b = shfl_xor_f4(odd ? x[2] : x[3], 1);
  if (odd) {
    x[0] = a;
    x[2] = b;
  } else {
    x[1] = a;
    x[3] = b;
  }
}

__global__ void __launch_bounds__(kThreads, 1) state_pass_kernel(const __grid_constant__ StateParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + kOffCtrl);
  volatile uint32_t* abort_flag = &ctrl->abort;
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const uint64_t T = p.timeout_ns;

  // this CTA's chunk-loads [f0, f1), head-major: load f is chunk f % n_chunks of head f / n_chunks
  const int64_t f0 = static_cast<int64_t>(blockIdx.x) * p.width;
  const int64_t f1 = min(f0 + p.width, p.total);
  const int64_t head0 = f0 / p.n_chunks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->empty[s], 1);
      mbar_init(&ctrl->kt_ready[s], 128);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctrl->acc_full[b], 1);
      mbar_init(&ctrl->acc_free[b], 128);
    }
    mbar_init(&ctrl->mma_final, 1);
    ctrl->abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
  }
  if (warp == 2) {
    tmem_alloc(&ctrl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;

  if (warp == 0) {
    // TMA producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      uint32_t issued[kStages] = {0, 0, 0};
      bool ok = true;
      for (int64_t f = f0; f < f1; ++f) {
        const uint32_t it = static_cast<uint32_t>(f - f0);
        const uint32_t s = it % kStages;
        if (!mbar_wait_bounded(&ctrl->empty[s], ((it / kStages) & 1) ^ 1, abort_flag, T)) {
          ok = false;
          break;
        }
        const int64_t bh = f / p.n_chunks;
        const int32_t c = static_cast<int32_t>(f - bh * p.n_chunks);
        const int32_t b = static_cast<int32_t>(bh / p.H);
        const int32_t h = static_cast<int32_t>(bh - static_cast<int64_t>(b) * p.H);
        uint8_t* st = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&ctrl->full[s], 2 * kTileBytes);  // rows past N are zero-filled
        tma_load_4d(st + kOffK, &p.tm_k, &ctrl->full[s], 0, h, c * C, b, pol);
        tma_load_4d(st + kOffK + kHalfBytes, &p.tm_k, &ctrl->full[s], 64, h, c * C, b, pol);
        tma_load_4d(st + kOffV, &p.tm_v, &ctrl->full[s], 0, h, c * C, b, pol);
        tma_load_4d(st + kOffV + kHalfBytes, &p.tm_v, &ctrl->full[s], 64, h, c * C, b, pol);
        issued[s] += 1;
      }
      if (!ok) {
        // every fill already issued must land before the CTA's shared memory goes away
        for (uint32_t s = 0; s < kStages; ++s) {
          if (issued[s] > 0) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&ctrl->full[s], (issued[s] - 1) & 1) &&
                   globaltimer_ns() - t0 < T) {
            }
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // tcgen05.mma issuer
    if (lane == 0) {
      constexpr uint32_t idKV = make_idesc_bf16(128, 128, 1, 1);  // K~^T (MN) x V (MN)
      uint32_t piece = 0;
      for (int64_t f = f0; f < f1; ++f) {
        const uint32_t it = static_cast<uint32_t>(f - f0);
        const uint32_t s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        const int64_t bh = f / p.n_chunks;
        const bool first = f == f0 || f == bh * p.n_chunks;
        const bool last = f + 1 == f1 || f + 1 == (bh + 1) * p.n_chunks;
        const uint32_t acc = tmem + (piece & 1) * 128;
        if (first && piece >= 2 &&
            !mbar_wait_bounded(&ctrl->acc_free[piece & 1], ((piece >> 1) - 1) & 1, abort_flag, T))
          break;
        if (!mbar_wait_bounded(&ctrl->full[s], ph, abort_flag, T) ||
            !mbar_wait_bounded(&ctrl->kt_ready[s], ph, abort_flag, T))
          break;
        tc_fence_after();
        const uint32_t kb = smem_base + s * kStageBytes + kOffK;
        const uint32_t vb = smem_base + s * kStageBytes + kOffV;
#pragma unroll
        for (uint32_t kk = 0; kk < 8; ++kk) {
          umma_ss(acc, make_sdesc_sw128(kb + kk * 2048, kHalfBytes, 1024),
                  make_sdesc_sw128(vb + kk * 2048, kHalfBytes, 1024), idKV,
                  (!first || kk > 0) ? 1u : 0u);
        }
        umma_commit(&ctrl->empty[s]);
        if (last) {
          umma_commit(&ctrl->acc_full[piece & 1]);
          ++piece;
        }
      }
      // all issued MMAs must finish before TMEM is released
      umma_commit(&ctrl->mma_final);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&ctrl->mma_final, 0) && globaltimer_ns() - t0 < T) {
      }
    }
    __syncwarp();
  } else if (warp >= kWarpK0 && warp < kWarpR0) {
    // K -> K~: row r of chunk c (token t = c*C + r) is scaled by lambda^(N-1-t); rows past N
    // (zero-filled) by 0
    const uint32_t r = threadIdx.x - kWarpK0 * 32;
    for (int64_t f = f0; f < f1; ++f) {
      const uint32_t it = static_cast<uint32_t>(f - f0);
      const uint32_t s = it % kStages;
      if (!mbar_wait_bounded(&ctrl->full[s], (it / kStages) & 1, abort_flag, T)) break;
      const int64_t bh = f / p.n_chunks;
      const int64_t t = (f - bh * p.n_chunks) * C + r;
      const float alpha = p.slopes[bh % p.H] * kLog2e;
      const float w = t < p.N ? exp2f(-alpha * static_cast<float>(p.N - 1 - t)) : 0.f;
      uint8_t* kt = smem + s * kStageBytes + kOffK;
      scale_half_row(kt, r, w);
      scale_half_row(kt + kHalfBytes, r, w);
      fence_proxy_async_smem();
      mbar_arrive(&ctrl->kt_ready[s]);
    }
  } else if (warp >= kWarpR0) {
    // read-out: thread (warp quarter wq, lane) owns state row i = 32 wq + lane
    const uint32_t wq = warp & 3;
    const uint32_t t4 = lane & 3;
    const uint32_t i0 = wq * 32 + (lane & ~3u);  // first row of this lane's group of four
    const uint32_t trow = tmem + ((wq * 32) << 16);
    uint32_t piece = 0;
    for (int64_t f = f0; f < f1; ++f) {
      const int64_t bh = f / p.n_chunks;
      const bool last = f + 1 == f1 || f + 1 == (bh + 1) * p.n_chunks;
      if (!last) continue;
      const bool whole = (f0 <= bh * p.n_chunks) && (f1 >= (bh + 1) * p.n_chunks);
      if (!mbar_wait_bounded(&ctrl->acc_full[piece & 1], (piece >> 1) & 1, abort_flag, T)) break;
      tc_fence_after();
      float* dst = whole ? p.state_out + bh * D * D
                         : p.partial + (2 * static_cast<int64_t>(blockIdx.x) + (bh == head0 ? 0 : 1)) * D * D;
      const float* sin = whole && p.state_in != nullptr ? p.state_in + bh * D * D : nullptr;
      const float lam_n = sin != nullptr ? decay_pow(p.slopes[bh % p.H], p.N) : 0.f;
      const uint32_t col0 = (piece & 1) * 128;
#pragma unroll 1
      for (uint32_t cb = 0; cb < 8; ++cb) {  // 16-column blocks
        uint32_t r16[16];
        tmem_ld16(trow + col0 + cb * 16, r16);
        tmem_wait_ld();
        if (cb == 7) {
          // every column of this accumulator has been read: it may be overwritten
          tc_fence_before();
          mbar_arrive(&ctrl->acc_free[piece & 1]);
        }
        float4 x[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          x[q] = make_float4(__uint_as_float(r16[4 * q]), __uint_as_float(r16[4 * q + 1]),
                             __uint_as_float(r16[4 * q + 2]), __uint_as_float(r16[4 * q + 3]));
        transpose4x4_lanes(x, t4);  // x[k] = piece t4 of row i0 + k
#pragma unroll
        for (uint32_t k = 0; k < 4; ++k) {
          const int64_t off = static_cast<int64_t>(i0 + k) * D + cb * 16 + 4 * t4;
          float4 y = x[k];
          if (sin != nullptr) {
            const float4 s0 = __ldcs(reinterpret_cast<const float4*>(sin + off));
            y.x = fmaf(lam_n, s0.x, y.x);
            y.y = fmaf(lam_n, s0.y, y.y);
            y.z = fmaf(lam_n, s0.z, y.z);
            y.w = fmaf(lam_n, s0.w, y.w);
          }
          *reinterpret_cast<float4*>(dst + off) = y;
        }
      }
      ++piece;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && ctrl->abort) atomicExch(p.status, kErrTimeout);
  if (warp == 2) tmem_dealloc(tmem, kTmemCols);
}

// Heads split over several ranges: S_out = lambda^N S_in + partials in range order.  One CTA per
// (head, 1024-float slice); heads that one range covers whole were written by the state pass.
__global__ void __launch_bounds__(256) state_combine_kernel(const StateParams p) {
  const int64_t bh = blockIdx.x;
  const int64_t i0 = bh * p.n_chunks / p.width;            // range holding the head's first chunk
  const int64_t i1 = ((bh + 1) * p.n_chunks - 1) / p.width;  // ... and its last
  if (i0 == i1) return;  // whole in one range
  if (*p.status != 0) return;
  const int64_t e = (static_cast<int64_t>(blockIdx.y) * 256 + threadIdx.x) * 4;  // float index
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (p.state_in != nullptr) {
    const float lam_n = decay_pow(p.slopes[bh % p.H], p.N);
    const float4 s0 = *reinterpret_cast<const float4*>(p.state_in + bh * D * D + e);
    acc = make_float4(lam_n * s0.x, lam_n * s0.y, lam_n * s0.z, lam_n * s0.w);
  }
  for (int64_t i = i0; i <= i1; ++i) {
    const int64_t head_first = i * p.width / p.n_chunks;
    const float4 x = *reinterpret_cast<const float4*>(
        p.partial + (2 * i + (bh == head_first ? 0 : 1)) * D * D + e);
    acc.x += x.x;
    acc.y += x.y;
    acc.z += x.z;
    acc.w += x.w;
  }
  *reinterpret_cast<float4*>(p.state_out + bh * D * D + e) = acc;
}

// Fold: S = S_in (or 0); S <- lambda^(L_j) S + h_j for j < n.  One thread per 4 state entries.
template <int DD>
__global__ void __launch_bounds__(256) state_fold_kernel(const StateFoldArgs a) {
  const int64_t bh = blockIdx.x;
  const int64_t e = (static_cast<int64_t>(blockIdx.y) * 256 + threadIdx.x) * 4;
  if (e >= DD * DD) return;
  const float slope = a.slopes[bh % a.H];
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  if (a.state_in != nullptr) s = *reinterpret_cast<const float4*>(a.state_in + bh * DD * DD + e);
  for (int64_t j = 0; j < a.n_parts; ++j) {
    const float lam = decay_pow(slope, a.lengths[j]);
    const float4 h = *reinterpret_cast<const float4*>(a.parts + (j * a.BH + bh) * DD * DD + e);
    s.x = fmaf(lam, s.x, h.x);
    s.y = fmaf(lam, s.y, h.y);
    s.z = fmaf(lam, s.z, h.z);
    s.w = fmaf(lam, s.w, h.w);
  }
  *reinterpret_cast<float4*>(a.state_out + bh * DD * DD + e) = s;
}

}  // namespace

StatePassPlan plan_state_pass(int64_t B, int64_t N, int64_t H, int num_sms) {
  StatePassPlan pl{};
  pl.n_chunks = (N + C - 1) / C;
  pl.total = B * H * pl.n_chunks;
  const int64_t grid0 = std::max<int64_t>(1, std::min<int64_t>(num_sms, pl.total));
  pl.width = (pl.total + grid0 - 1) / grid0;
  pl.grid = (pl.total + pl.width - 1) / pl.width;
  pl.ws_bytes = 256 + static_cast<size_t>(2 * pl.grid) * D * D * sizeof(float);
  return pl;
}

cudaError_t launch_state_pass(const PrefillArgs& a, const StatePassPlan& plan, void* workspace,
                              cudaStream_t stream) {
  // set on every call: cheap, safe from any host thread, and it survives a context reset
  cudaError_t e = cudaFuncSetAttribute(state_pass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemAlloc));
  if (e != cudaSuccess) return e;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  e = cudaMemsetAsync(ws, 0, 256, stream);  // status word
  if (e != cudaSuccess) return e;
  if (plan.total == 0) return cudaSuccess;
  StateParams prm{};
  if (!encode_map(&prm.tm_k, a.k, a.B, a.N, a.H) || !encode_map(&prm.tm_v, a.v, a.B, a.N, a.H))
    return cudaErrorInvalidValue;
  prm.slopes = a.slopes;
  prm.state_in = a.state_in;
  prm.state_out = a.state_out;
  prm.partial = reinterpret_cast<float*>(ws + 256);
  prm.status = reinterpret_cast<int32_t*>(ws + kWsStatus);
  prm.N = a.N;
  prm.H = a.H;
  prm.n_chunks = plan.n_chunks;
  prm.total = plan.total;
  prm.width = plan.width;
  prm.timeout_ns = a.wait_limit_ns;
  state_pass_kernel<<<static_cast<unsigned>(plan.grid), kThreads, kSmemAlloc, stream>>>(prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (plan.grid > 1 && plan.width % plan.n_chunks != 0) {
    // a range boundary falls inside some head: combine the split heads (the others return)
    const dim3 grid(static_cast<unsigned>(a.B * a.H), D * D / (256 * 4));
    state_combine_kernel<<<grid, 256, 0, stream>>>(prm);
    e = cudaGetLastError();
  }
  return e;
}

cudaError_t launch_state_fold(const StateFoldArgs& a, cudaStream_t stream) {
  if (a.BH == 0) return cudaSuccess;
  if (a.d == 64) {
    const dim3 grid(static_cast<unsigned>(a.BH), (64 * 64 / 4 + 255) / 256);
    state_fold_kernel<64><<<grid, 256, 0, stream>>>(a);
  } else {
    const dim3 grid(static_cast<unsigned>(a.BH), (128 * 128 / 4 + 255) / 256);
    state_fold_kernel<128><<<grid, 256, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace la
