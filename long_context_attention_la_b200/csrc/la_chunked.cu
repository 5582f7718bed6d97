// la_chunked.cu — chunked Lightning Attention prefill on the sm_100a tensor cores.
//
// Method ("Ling and Ring 2.6 Technical Report", Chinese translation, garden.houmin.site;
// §4.1.1 Context Parallel for Lightning Attention, Fig. 10): each (b, h) sequence is evaluated as
// chunks of C tokens ("chunk QKV").  For chunk c with rows i, j in [0, C):
//     S      = Q K^T                                   (tensor cores, fp32 in TMEM)
//     P_ij   = lambda^(i-j) S_ij  (i >= j), 0 otherwise  (CUDA cores, bf16 back into TMEM)
//     O      = P V + diag(lambda^(i+1)) Q KV_in          (two tensor-core accumulators)
//     KV_out = lambda^n KV_in + (K ⊙ lambda^(n-1-j))^T V  (tensor cores, fp32 state in TMEM)
// where n is the chunk's token count and KV_in the d x d state before the chunk.  The kernel moves
// and multiplies 128-token tiles (every MMA is M = 128); the chunk length C in {64, 128, 256} is
// how a tile's rows split between the intra- and the inter-chunk term:
//   C = 128  one chunk per tile (the code below calls a tile a "chunk" where C = 128 is meant);
//   C = 64   two chunks per tile: P is block-diagonal (two 64 x 64 causal blocks), rows 0..63 read
//            the state before the tile and rows 64..127 the state after its first half, which the
//            state warps round to bf16 in the middle of the tile (a second Q KV product whose
//            accumulator reuses the S columns once P V has read P);
//   C = 256  two tiles per chunk: the second tile B adds the block below the diagonal directly,
//            P_BA = lambda^(128+i-j) Q_B K_A^T = diag(lambda^(i+1)) Q_B K~_A^T with K~_A the first
//            tile's keys already scaled for the state update, so the bf16 state operand is
//            refreshed once per 256 tokens and B's inter term is lambda^(i+129) Q_B KV_in.
// All three are the same recurrence; they differ only in where bf16 roundings fall.  Long sequences
// are cut into segments ("local recurrence, then global correction"): a segment first computes its
// local state h (the "local h" of Fig. 10) from K, V alone, obtains its incoming state from its
// predecessor through a decayed prefix scan over segments (S_{k+1} = lambda^L S_k + h_k, the
// "fused update h"), and then runs its output chunks starting from that state (the "fused
// update O", folded into the inter-chunk term instead of a separate correction pass).
//
// Execution: one persistent CTA per SM (640 threads, ~226 KB shared memory, all 512 TMEM
// columns).  Work units (segment, b, h) are taken in segment-major order from an atomic counter,
// so a unit only ever waits on units that running CTAs already hold.  Roles:
//   warp 0       TMA producer: two-stage ring of Q/K/V tiles (optional L2 prefetch ahead)
//   warp 1       tcgen05.mma issuer; per chunk c: S_c, O_inter_c, the state update with chunk c,
//                O_intra_c; the stage is released when O_intra_c completes
//   warp 2       TMEM allocator
//   warps 4-11   P = decay-mask(S) into TMEM (two warps per TMEM lane quarter, alternate
//                32-column blocks); K -> K~ in the local-state pass
//   warps 12-15  state: look-back scan, K -> K~ (row-scaled, as soon as S_c is done) in the
//                output pass, KV -> bf16 operand, decay rescale, final state
//   warps 16-19  output epilogue: O = O_intra + lambda^(i+1) O_inter -> bf16 -> global, in
//                whole 32-byte sectors
// Two instances regroup warps 8-11: the fused norm + gate instance gives them half the epilogue's
// columns, and the in-tile QK instance (raw q and k in) has them apply the QK RMSNorm + RoPE to
// each tile's q and k rows in shared memory before any product reads them (and scale the keys in
// the local-state pass); both run the decay mask on warps 4-7 alone.
// Every wait (mbarrier or scan flag) is bounded in time; on expiry the CTA records
// LA_ERR_TIMEOUT in the workspace status word, unwinds, frees its TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>

#include "la_internal.h"
#include "la_sm100.cuh"

namespace la {
namespace {

constexpr int C = kChunk;      // 128 tokens per chunk
constexpr int D = kHeadDim;    // 128
constexpr int kThreads = 640;  // 20 warps
constexpr uint32_t kWarpP0 = 4;    // warps 4..11: decay mask / local-pass K scaling
constexpr uint32_t kWarpS0 = 12;   // warps 12..15: state
constexpr uint32_t kWarpO0 = 16;   // warps 16..19: output epilogue
constexpr uint32_t kBarP = 1, kBarS = 2, kBarO = 3;  // named barriers of the three groups
constexpr uint32_t kBarT = 4;                        // ... and of the in-tile QK transform warps
constexpr uint32_t kTileBytes = C * D * 2;           // one bf16 [128 x 128] tile
constexpr uint32_t kHalfBytes = kTileBytes / 2;      // [128 rows x 64 cols], 128-byte rows
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kTileBytes;
constexpr uint32_t kOffV = 2 * kTileBytes;
constexpr uint32_t kStageBytes = 3 * kTileBytes;     // 96 KiB
constexpr uint32_t kOffKVb = 2 * kStageBytes;        // bf16 state operand, 32 KiB
constexpr uint32_t kOffCtrl = kOffKVb + kTileBytes;  // barriers and unit ring
constexpr uint32_t kCtrlBytes = 1024;
constexpr uint32_t kSmemBytes = kOffCtrl + kCtrlBytes;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;   // slack for 1024-byte alignment

// TMEM columns (128 lanes x 512 columns of 32 bit).
constexpr uint32_t kColS = 0;        // S (fp32, 128 cols); P (bf16 pairs) aliases cols 0..63
constexpr uint32_t kColOintra = 128;
constexpr uint32_t kColOinter = 256;
constexpr uint32_t kColKV = 384;     // carried state / segment-local state h

constexpr int32_t kErrTimeout = -8;  // LA_ERR_TIMEOUT

using UnitInfo = WorkUnit;  // one (segment, sequence, head) work unit

// Chunk length of a kernel instance: C = 128 (one chunk per tile), C = 64 (two per tile) or
// C = 256 (two tiles per chunk).
enum ChunkMode : int { kC128 = 0, kC64 = 1, kC256 = 2 };

struct Ctrl {
  uint64_t full[2];
  uint64_t empty[2];
  uint64_t kt_ready[2];
  uint64_t unit_full[2];
  uint64_t unit_empty[2];
  uint64_t s_full;
  uint64_t p_ready;
  uint64_t s2_full;   // C = 256: the cross scores Q_B K~_A^T of a chunk's second tile are in TMEM
  uint64_t p2_ready;  // C = 256: their scaled bf16 P_BA is in TMEM
  uint64_t gate_full[2];  // fused norm + gate: the tile's gate rows are in its stage's Q slot
  uint64_t qk_ready[2];   // in-tile QK norm + RoPE: the stage's q and k rows are transformed
  float row_x[128];       // fused norm + gate: a row's sum of squares / 1/rms between its two warps
  uint64_t o_full;
  uint64_t o_free;
  uint64_t kv_done;
  uint64_t kvb_ready;
  uint64_t kv_free;
  uint64_t h_done;
  uint64_t mma_final;
  uint32_t tmem_base;
  uint32_t abort;
  uint32_t pad[2];
  UnitInfo units[2];
};
static_assert(sizeof(Ctrl) <= kCtrlBytes, "control block too large");

struct Params {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_gate;  // fused norm + gate only: the gate pre-activation, for L2 prefetches
  __nv_bfloat16* out;
  const float* slopes;
  float* state_out;
  uint32_t* counter;
  int32_t* status;
  uint32_t* flags;
  float* ring;
  const WorkUnit* unit_table;  // variable-length plan (device), or null: units follow from N, BH
  const volatile int32_t* units_dev;  // its unit count (device), written by the planning kernel
  const float* state_in;       // fp32 [sequences, H, D, D] initial states, or null (zero)
  const __nv_bfloat16* gate;   // fused norm + gate: gate pre-activation like out, or null
  const float* gamma;          // fp32 [H, D] norm weight
  float eps;
  // in-tile QK RMSNorm + RoPE (kQk instance): weights fp32 [D], positions int64 [B * N]
  const float* qk_gamma_q;
  const float* qk_gamma_k;
  const int64_t* qk_positions;
  int32_t qk_rotary_dim;
  float qk_eps;
  double qk_inv_freq[64];      // theta^(-2i / rotary_dim), i < rotary_dim / 2
  int64_t N, H, BH;
  int64_t n_chunks, seg_chunks, segments, units;
  uint64_t timeout_ns;
  int32_t prefetch_depth;
  int32_t withhold_segment;  // failure injection: this segment never publishes (-1: none)
  // balanced plan (n_ranges > 0): range r covers flat tiles [range_start[r], range_start[r+1])
  // of the head-major list of B*H sequences of n_chunks tiles
  int32_t n_ranges;
  int32_t range_start[kMaxRanges + 1];
};

constexpr float kLog2e = 1.4426950408889634f;

// All `count` threads of a role group agree on `ok` (logical AND) at named barrier `id`.
__device__ __forceinline__ bool group_all(bool ok, uint32_t id, uint32_t count) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(ok ? 1u : 0u), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int32_t ld_volatile_s32(const int32_t* p) {
  int32_t v;
  asm volatile("ld.volatile.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Byte offset of 16-byte chunk `c16` (0..7) of row `r` in a [rows x 64] bf16 half-tile stored
// with the 128-byte swizzle (8-row, 1024-byte atoms; chunk index XOR row-in-atom).
__device__ __forceinline__ uint32_t sw128_off(uint32_t r, uint32_t c16) {
  return (r >> 3) * 1024u + (r & 7u) * 128u + ((c16 ^ (r & 7u)) << 4);
}

// Multiplies the 64 bf16 of one half-row (row r of a swizzled [128 x 64] half-tile) by w, in
// fp32 with one rounding.  Step c touches physical chunk c ^ (r & 7), so the 8 rows of a swizzle
// atom hit 8 different 16-byte bank groups at every step.
__device__ __forceinline__ void scale_half_row(uint8_t* half_tile, uint32_t r, float w) {
  uint8_t* row = half_tile + (r >> 3) * 1024u + (r & 7u) * 128u;
#pragma unroll
  for (uint32_t c0 = 0; c0 < 8; c0 += 4) {  // four loads in flight, then four stores
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

// 16-byte chunk gc (0..15, dims 8 gc .. 8 gc + 7) of row r of a swizzled [128 x 128] tile
__device__ __forceinline__ uint8_t* tile_chunk(uint8_t* tile, uint32_t r, uint32_t gc) {
  return tile + (gc >> 3) * kHalfBytes + sw128_off(r, gc & 7u);
}

// the 8 bf16 of a chunk as 4 fp32 pairs
__device__ __forceinline__ void unpack_chunk(const uint4& w, float2 (&x)[4]) {
  const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) x[e] = make_float2(bf16lo_to_f32(v[e]), bf16hi_to_f32(v[e]));
}

// QK RMSNorm + partial rotate-half RoPE, in place, of row r of the k tile and (kWithQ) of the q
// tile in the same stage: both rows are one token's, so they share its rotation angles.
//     y = gamma * x / sqrt(mean(x^2) + eps);  (y_i, y_{i+R/2}) <- (y_i cos a - y_{i+R/2} sin a,
//     y_{i+R/2} cos a + y_i sin a), a = pos * theta^(-2i/R), i < R/2 (R = rotary_dim)
// ("Ling and Ring 2.6 Technical Report", §2.1 Fig. 2 and §2.1.1).  The row's 16 chunks are taken
// in the pairs the stand-alone operator (la_qknorm.cu) gives to each of a row's 8 threads,
// piece (u, u + R/16) for u < R/16, else two chunks (128 - R)/16 apart past the rotary span, and
// every rounding follows that operator: per-pair partial sums of squares on paired fp32 FMAs,
// added in its shuffle-tree order; y = gamma (x rinv); the rotation and the angle reduction as
// there.  The tiles therefore hold exactly the bf16 rows that operator would have stored.
template <bool kWithQ>
__device__ __forceinline__ void qk_norm_rope_rows(uint8_t* q_tile, uint8_t* k_tile, uint32_t r,
                                                  int64_t pos, const float* gamma_q,
                                                  const float* gamma_k, const double* inv_freq,
                                                  int32_t rotary_dim, float eps) {
  const int rot = rotary_dim / 16;      // chunk pairs inside the rotary span
  const int rd8 = rotary_dim / 8;       // first chunk past it
  const int far = 8 - rot;              // distance of a pass-through pair's two chunks
  auto piece_a = [&](int u) { return u < rot ? u : rd8 + (u - rot); };
  auto piece_b = [&](int u) { return u < rot ? u + rot : rd8 + (u - rot) + far; };
  auto pair_ss = [&](uint8_t* tile, int u) {
    float2 xa[4], xb[4];
    unpack_chunk(*reinterpret_cast<const uint4*>(tile_chunk(tile, r, piece_a(u))), xa);
    unpack_chunk(*reinterpret_cast<const uint4*>(tile_chunk(tile, r, piece_b(u))), xb);
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
    for (int e = 0; e < 4; ++e) acc = __ffma2_rn(xb[e], xb[e], __ffma2_rn(xa[e], xa[e], acc));
    return acc.x + acc.y;
  };
  // the pairs' partial sums in the order of a butterfly over 8 lanes (xor 4, then 2, then 1)
  auto tree = [](const float (&s)[8]) {
    return ((s[0] + s[4]) + (s[2] + s[6])) + ((s[1] + s[5]) + (s[3] + s[7]));
  };
  float sq[8] = {}, sk[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    if constexpr (kWithQ) sq[u] = pair_ss(q_tile, u);
    sk[u] = pair_ss(k_tile, u);
  }
  float rq = 0.f;
  if constexpr (kWithQ) rq = rsqrtf(fmaf(tree(sq), 1.f / D, eps));
  const float rk = rsqrtf(fmaf(tree(sk), 1.f / D, eps));

  // one pair of chunks of one row: normalise, weight, rotate (rotary pairs), store as bf16
  auto apply = [&](uint8_t* tile, const float* gamma, float rinv, int ca, int cb, bool rotary,
                   const float2 (&cs)[4], const float2 (&sn)[4]) {
    uint4* pa = reinterpret_cast<uint4*>(tile_chunk(tile, r, ca));
    uint4* pb = reinterpret_cast<uint4*>(tile_chunk(tile, r, cb));
    float2 ya[4], yb[4];
    unpack_chunk(*pa, ya);
    unpack_chunk(*pb, yb);
    const float4* gpa = reinterpret_cast<const float4*>(gamma + 8 * ca);
    const float4* gpb = reinterpret_cast<const float4*>(gamma + 8 * cb);
    const float4 ga0 = __ldg(gpa), ga1 = __ldg(gpa + 1), gb0 = __ldg(gpb), gb1 = __ldg(gpb + 1);
    const float2 gma[4] = {make_float2(ga0.x, ga0.y), make_float2(ga0.z, ga0.w),
                           make_float2(ga1.x, ga1.y), make_float2(ga1.z, ga1.w)};
    const float2 gmb[4] = {make_float2(gb0.x, gb0.y), make_float2(gb0.z, gb0.w),
                           make_float2(gb1.x, gb1.y), make_float2(gb1.z, gb1.w)};
    const float2 r2 = make_float2(rinv, rinv);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      ya[e] = __fmul2_rn(gma[e], __fmul2_rn(ya[e], r2));
      yb[e] = __fmul2_rn(gmb[e], __fmul2_rn(yb[e], r2));
    }
    if (rotary) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 y0 = ya[e], y1 = yb[e];
        const float2 nsn = make_float2(-sn[e].x, -sn[e].y);
        ya[e] = __ffma2_rn(y0, cs[e], __fmul2_rn(y1, nsn));
        yb[e] = __ffma2_rn(y1, cs[e], __fmul2_rn(y0, sn[e]));
      }
    }
    uint4 wa, wb;
    wa.x = pack_bf16x2(ya[0].x, ya[0].y);
    wa.y = pack_bf16x2(ya[1].x, ya[1].y);
    wa.z = pack_bf16x2(ya[2].x, ya[2].y);
    wa.w = pack_bf16x2(ya[3].x, ya[3].y);
    wb.x = pack_bf16x2(yb[0].x, yb[0].y);
    wb.y = pack_bf16x2(yb[1].x, yb[1].y);
    wb.z = pack_bf16x2(yb[2].x, yb[2].y);
    wb.w = pack_bf16x2(yb[3].x, yb[3].y);
    *pa = wa;
    *pb = wb;
  };
#pragma unroll 1
  for (int u = 0; u < 8; ++u) {
    const bool rotary = u < rot;
    float2 cs[4], sn[4];
    if (rotary) {
      // the angle pos * w_f, reduced modulo 2 pi in fp64, then sin and cos in fp32
      constexpr double kTwoPi = 6.283185307179586476925286766559;
      constexpr double kInvTwoPi = 0.15915494309189533576888376337251;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float s0, c0, s1, c1;
        const double a0 = __dmul_rn(static_cast<double>(pos), inv_freq[8 * u + 2 * e]);
        const double a1 = __dmul_rn(static_cast<double>(pos), inv_freq[8 * u + 2 * e + 1]);
        __sincosf(static_cast<float>(__fma_rn(-kTwoPi, rint(__dmul_rn(a0, kInvTwoPi)), a0)), &s0,
                  &c0);
        __sincosf(static_cast<float>(__fma_rn(-kTwoPi, rint(__dmul_rn(a1, kInvTwoPi)), a1)), &s1,
                  &c1);
        cs[e] = make_float2(c0, c1);
        sn[e] = make_float2(s0, s1);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) cs[e] = sn[e] = make_float2(0.f, 0.f);
    }
    const int ca = piece_a(u), cb = piece_b(u);
    if constexpr (kWithQ) apply(q_tile, gamma_q, rq, ca, cb, rotary, cs, sn);
    apply(k_tile, gamma_k, rk, ca, cb, rotary, cs, sn);
  }
}

// 4 x 4 transpose of 16-byte pieces within each group of 4 lanes: on entry lane t of a group
// holds pieces x[0..3] of its own row; on exit it holds piece t of the group's rows 0..3.  Two
// butterfly exchanges: swap the off-diagonal 2 x 2 blocks (partner t ^ 2), then transpose each
// 2 x 2 block (partner t ^ 1).
__device__ __forceinline__ uint4 shfl_xor_u4(uint4 v, int m) {
  v.x = __shfl_xor_sync(0xffffffffu, v.x, m);
  v.y = __shfl_xor_sync(0xffffffffu, v.y, m);
  v.z = __shfl_xor_sync(0xffffffffu, v.z, m);
  v.w = __shfl_xor_sync(0xffffffffu, v.w, m);
  return v;
}
__device__ __forceinline__ void transpose4x4_lanes(uint4 (&x)[4], uint32_t t) {
  const bool hi = (t & 2u) != 0;
  uint4 a = shfl_xor_u4(hi ? x[0] : x[2], 2);
  uint4 b = shfl_xor_u4(hi ? x[1] : x[3], 2);
  if (hi) {
    x[0] = a;
    x[1] = b;
  } else {
    x[2] = a;
    x[3] = b;
  }
  const bool odd = (t & 1u) != 0;
  a = shfl_xor_u4(odd ? x[0] : x[1], 1);
  b = shfl_xor_u4(odd ? x[2] : x[3], 1);
  if (odd) {
    x[0] = a;
    x[2] = b;
  } else {
    x[1] = a;
    x[3] = b;
  }
}

__device__ __forceinline__ void decode_unit(const Params& p, int64_t u, UnitInfo& ui) {
  if (p.unit_table != nullptr) {
    // written by the planning kernel earlier on the stream: coherent loads
    const int4* src = reinterpret_cast<const int4*>(p.unit_table + u);
    const int4 w0 = __ldcg(src), w1 = __ldcg(src + 1), w2 = __ldcg(src + 2);
    ui.bh = w0.x;
    ui.seg = w0.y;
    ui.c0 = w0.z;
    ui.nc = w0.w;
    ui.len = w1.x;
    ui.flags = w1.y;
    ui.b = w1.z;
    ui.tok0 = w1.w;
    ui.slot = w2.x;
    ui.in_slot = w2.y;
    ui.in_val = w2.z;
    ui.pub_val = w2.w;
    return;
  }
  // fixed length: unit u = segment k of flat head bh, segment-major; a two-slot state ring per
  // sequence, segment k publishing into slot k & 1 with flag value k + 1
  const int64_t k = u / p.BH;
  const int64_t bh = u % p.BH;
  const int64_t c0 = k * p.seg_chunks;
  const int64_t nc = min(p.seg_chunks, p.n_chunks - c0);
  const int64_t end = min(p.N, (c0 + nc) * C);
  ui.bh = static_cast<int32_t>(bh);
  ui.seg = static_cast<int32_t>(k);
  ui.c0 = static_cast<int32_t>(c0);
  ui.nc = static_cast<int32_t>(nc);
  ui.len = static_cast<int32_t>(end - c0 * C);
  ui.flags = (k + 1 < p.segments ? kUnitLocal : 0) | (k + 1 == p.segments ? kUnitFinal : 0);
  ui.b = static_cast<int32_t>(bh / p.H);
  ui.tok0 = 0;
  ui.slot = static_cast<int32_t>(bh * 2 + (k & 1));
  ui.in_slot = k > 0 ? static_cast<int32_t>(bh * 2 + ((k - 1) & 1)) : -1;
  ui.in_val = static_cast<int32_t>(k);
  ui.pub_val = static_cast<int32_t>(k + 1);
}

// Balanced plan: the units of range r, in order.  Cursor state lives with the producer thread.
struct RangeCursor {
  int32_t r = -1;           // current range (-1: none yet)
  int32_t phase = 0;        // 0: cut piece's local state, 1: its outputs, 2: whole sequences,
                            // 3: the piece that continues the previous range
  int64_t a = 0, end = 0;   // the range's flat tiles [a, end)
  int64_t cut = 0;          // first tile of the piece the range's end cuts (end: none)
  int64_t cont_end = 0;     // end of the continuing first piece (a: none)
  int64_t next = 0;         // next tile of phase 2 (whole sequences in [cont_end, cut))
};

// Fills ui with the piece of flat tiles [t0, t1) of one sequence (t1 inside or at its end).
__device__ __forceinline__ void piece_unit(const Params& p, int64_t t0, int64_t t1, UnitInfo& ui) {
  const int64_t n = p.n_chunks;
  const int64_t sq = t0 / n;
  const int64_t c0 = t0 - sq * n;
  const int64_t nc = t1 - t0;
  ui.bh = static_cast<int32_t>(sq);
  ui.seg = c0 > 0 ? 1 : 0;
  ui.c0 = static_cast<int32_t>(c0);
  ui.nc = static_cast<int32_t>(nc);
  ui.len = static_cast<int32_t>(min(p.N, (c0 + nc) * C) - c0 * C);
  ui.b = static_cast<int32_t>(sq / p.H);
  ui.tok0 = 0;
  ui.flags = (c0 + nc == n) ? kUnitFinal : 0;
  ui.slot = -1;
  ui.pub_val = 0;
  // a piece that starts inside its sequence begins its range; its predecessor is the cut last
  // piece of the previous range, whose local-state unit published into ring slot r - 1
  ui.in_slot = -1;
  ui.in_val = 1;
}

// Next unit of the balanced plan (ui.bh = -1 once every range has been taken).  A range runs,
// in this order: the local-state pass of its cut last piece (publishing that piece's outgoing
// state into ring slot r for the next range), that piece's outputs (its incoming state is at hand:
// zero at a sequence start, else already awaited by the local-state unit), the outputs of the
// whole sequences inside it, and last the piece that continues the previous range's cut, whose
// publication (ring slot r - 1) it may have to wait for.
__device__ __forceinline__ void next_balanced_unit(const Params& p, RangeCursor& cur,
                                                   UnitInfo& ui) {
  const int64_t n = p.n_chunks;
  while (true) {
    if (cur.r >= 0) {
      if (cur.phase == 0) {
        cur.phase = 1;
        if (cur.cut < cur.end) {
          piece_unit(p, cur.cut, cur.end, ui);
          ui.flags = kUnitLocal | kUnitNoOutput;
          ui.slot = cur.r;
          ui.pub_val = 1;
          if (ui.c0 > 0) ui.in_slot = cur.r - 1;
          return;
        }
      }
      if (cur.phase == 1) {
        cur.phase = 2;
        if (cur.cut < cur.end) {
          piece_unit(p, cur.cut, cur.end, ui);
          if (ui.c0 > 0) ui.in_slot = cur.r - 1;
          return;
        }
      }
      if (cur.phase == 2) {
        if (cur.next < cur.cut) {
          const int64_t t0 = cur.next;
          const int64_t t1 = min(cur.cut, (t0 / n + 1) * n);
          piece_unit(p, t0, t1, ui);
          cur.next = t1;
          return;
        }
        cur.phase = 3;
      }
      if (cur.phase == 3) {
        cur.phase = 4;
        if (cur.cont_end > cur.a) {
          piece_unit(p, cur.a, cur.cont_end, ui);
          ui.in_slot = cur.r - 1;
          return;
        }
      }
    }
    const int32_t r = static_cast<int32_t>(atomicAdd(p.counter, 1u));
    if (r >= p.n_ranges) {
      ui.bh = -1;
      ui.seg = ui.c0 = ui.nc = ui.len = ui.flags = ui.b = ui.tok0 = ui.slot = 0;
      ui.in_slot = -1;
      ui.in_val = ui.pub_val = 0;
      return;
    }
    cur.r = r;
    cur.phase = 0;
    cur.a = p.range_start[r];
    cur.end = p.range_start[r + 1];
    // the range's end inside a sequence cuts its last piece
    cur.cut = cur.end % n != 0 ? max(cur.a, ((cur.end - 1) / n) * n) : cur.end;
    // a start inside a sequence continues the previous range's cut piece; when that piece is
    // also this range's cut piece, phases 0 and 1 handle it
    cur.cont_end = (cur.a % n != 0 && cur.cut > cur.a) ? min(cur.cut, (cur.a / n + 1) * n) : cur.a;
    cur.next = cur.cont_end;
  }
}

// Output epilogue with the fused grouped RMSNorm and sigmoid gate ("Ling and Ring 2.6 Technical
// Report", §2.1 Fig. 2; §4.3): thread i's row of O (one head, D channels) is one norm group,
//     y_j = gamma_j * O_j / sqrt(mean(O^2) + eps) * sigmoid(g_j).
// Pass 1 reads the row's fp32 accumulators once: it sums the squares and keeps O rounded to bf16
// (the precision the unfused layer hands to its norm) in registers.  Pass 2 exchanges 16-byte
// pieces of that O within each 4-lane group as the plain epilogue does, and then finishes each
// piece in the store layout: lane t holds piece t of rows i0..i0+3, so its gate reads and stores
// cover whole sectors and its gamma slice is the same for all four rows.
// sigmoid(x) = (1 + tanh(x / 2)) / 2 takes one MUFU operation (tanh.approx, max relative error
// about 2^-11) instead of an exponential and a reciprocal.
__device__ __forceinline__ float tanhf_fast(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(x));
  return t;
}

// Gate pieces of 32-column block cb in the 4-lane store layout, from the tile's gate rows staged
// in shared memory (two [128 x 64] halves, 128-byte swizzle): g[k] = piece t of tile row i0 + k.
__device__ __forceinline__ void load_gate_pieces(const uint8_t* gate_tile, uint32_t i0, uint32_t t,
                                                 uint32_t cb, uint4 (&g)[4]) {
  const uint32_t piece = cb * 4 + t;  // 16-byte piece of the 256-byte row
  const uint8_t* half = gate_tile + (piece >> 3) * kHalfBytes;
#pragma unroll
  for (uint32_t k = 0; k < 4; ++k)
    g[k] = *reinterpret_cast<const uint4*>(half + sw128_off(i0 + k, piece & 7u));
}

// Pass 1: columns [64 eh, 64 eh + 64) of this thread's row i; the other half of the row is
// another warp's.  Returns the half row's sum of squares and its O rounded to bf16 (pairs of
// columns 64 eh + 2m, 64 eh + 2m + 1), then gives O back to the MMA warp.
__device__ __forceinline__ float gated_epilogue_read(Ctrl* ctrl, uint32_t trow, uint32_t col_inter,
                                                     float f, uint32_t eh, uint32_t (&ob)[32]) {
  float ss = 0.f;
#pragma unroll
  for (uint32_t c = 0; c < 4; ++c) {  // 16-column blocks
    const uint32_t cb = 4 * eh + c;
    uint32_t ra[16], re[16];
    tmem_ld16(trow + kColOintra + cb * 16, ra);
    tmem_ld16(trow + col_inter + cb * 16, re);
    tmem_wait_ld();
#pragma unroll
    for (int m = 0; m < 16; m += 2) {
      const float o0 = fmaf(f, __uint_as_float(re[m]), __uint_as_float(ra[m]));
      const float o1 = fmaf(f, __uint_as_float(re[m + 1]), __uint_as_float(ra[m + 1]));
      ss = fmaf(o0, o0, ss);
      ss = fmaf(o1, o1, ss);
      ob[c * 8 + m / 2] = pack_bf16x2(o0, o1);
    }
  }
  tc_fence_before();
  mbar_arrive(&ctrl->o_free);  // every O column of this thread's half row has been read
  return ss;
}

// Pass 2: completes the row's mean square through ctrl->row_x with the warp that holds the other
// half, then writes y for this thread's half row from the gate rows staged in shared memory.
__device__ __forceinline__ void gated_epilogue_write(const Params& p, Ctrl* ctrl, float ss,
                                                     const uint32_t (&ob)[32],
                                                     const UnitInfo& ui, int64_t h,
                                                     const uint8_t* gate_tile,
                                                     __nv_bfloat16* out_h, uint32_t t, int32_t r0,
                                                     uint32_t i0, int64_t n0, int64_t row_stride,
                                                     uint32_t i, uint32_t eh, uint32_t n_threads) {
  if (eh == 1) ctrl->row_x[i] = ss;
  named_bar_sync(kBarO, n_threads);
  float rinv = 0.f;
  if (eh == 0) {
    rinv = rsqrtf(fmaf(ss + ctrl->row_x[i], 1.f / D, p.eps));
    ctrl->row_x[i] = rinv;
  }
  named_bar_sync(kBarO, n_threads);
  if (eh == 1) rinv = ctrl->row_x[i];
  float rk[4];  // 1 / rms of rows i0 + k, held by lanes 4a + k
  const uint32_t lane0 = (threadIdx.x & 31u) & ~3u;
#pragma unroll
  for (uint32_t k = 0; k < 4; ++k) rk[k] = __shfl_sync(0xffffffffu, rinv, lane0 + k);
#pragma unroll
  for (uint32_t cc = 0; cc < 2; ++cc) {  // 32-column blocks of the half row
    const uint32_t cb = 2 * eh + cc;
    uint4 g[4];
    load_gate_pieces(gate_tile, i0, t, cb, g);
    uint4 x[4];  // bf16 O, pieces q = 0..3 of this row's 32 columns
#pragma unroll
    for (uint32_t q = 0; q < 4; ++q)
      x[q] = make_uint4(ob[cc * 16 + q * 4], ob[cc * 16 + q * 4 + 1], ob[cc * 16 + q * 4 + 2],
                        ob[cc * 16 + q * 4 + 3]);
    transpose4x4_lanes(x, t);  // now x[k] = piece t of row i0 + k
    const float4 g0 = __ldg(reinterpret_cast<const float4*>(p.gamma + h * D + cb * 32 + 8 * t));
    const float4 g1 = __ldg(reinterpret_cast<const float4*>(p.gamma + h * D + cb * 32 + 8 * t) + 1);
    const float gm[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
    for (uint32_t k = 0; k < 4; ++k) {
      if (r0 + static_cast<int32_t>(k) < ui.len) {
        const uint32_t gw[4] = {g[k].x, g[k].y, g[k].z, g[k].w};
        const uint32_t ow[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
        // y = gamma * (O * rinv) * sigmoid(g) on paired fp32 operations (two columns per
        // instruction, the same roundings as the scalar form); the sigmoid is
        // 1/2 + tanh(g/2)/2 with one MUFU tanh per column
        uint32_t yw[4];
        const float2 rk2 = make_float2(rk[k], rk[k]);
        const float2 half2 = make_float2(0.5f, 0.5f);
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const float2 ov = make_float2(bf16lo_to_f32(ow[e2]), bf16hi_to_f32(ow[e2]));
          const float2 hg =
              __fmul2_rn(half2, make_float2(bf16lo_to_f32(gw[e2]), bf16hi_to_f32(gw[e2])));
          const float2 sg = __ffma2_rn(half2, make_float2(tanhf_fast(hg.x), tanhf_fast(hg.y)),
                                       half2);
          const float2 y = __fmul2_rn(
              __fmul2_rn(make_float2(gm[2 * e2], gm[2 * e2 + 1]), __fmul2_rn(ov, rk2)), sg);
          yw[e2] = pack_bf16x2(y.x, y.y);
        }
        uint4* dst = reinterpret_cast<uint4*>(out_h + (n0 + k) * row_stride + cb * 32) + t;
        __stcs(dst, make_uint4(yw[0], yw[1], yw[2], yw[3]));
      }
    }
  }
}

// kGated: the output epilogue applies the fused norm + gate (p.gate != null).  Separate instances,
// so that the plain kernel's register allocation carries none of the gated epilogue's pressure.
// kCM: the chunk length (ChunkMode).  kQk: q and k arrive raw and get their QK RMSNorm + RoPE in
// shared memory first (C = 128, plain output only).
template <bool kGated, int kCM, bool kQk = false>
__global__ void __launch_bounds__(kThreads, 1)
    chunked_prefill_kernel(const __grid_constant__ Params p) {
  static_assert(!kQk || (!kGated && kCM == kC128), "in-tile QK norm: C = 128, plain output");
  // The fused norm + gate instance runs the decay mask on 4 warps (one per TMEM lane quarter)
  // and its heavier epilogue on 8 (warps 16-19 take columns 0..63, warps 8-11 columns 64..127);
  // the in-tile QK instance gives warps 8-11 the QK transform instead; the plain instance has 8
  // mask warps and 4 epilogue warps.
  constexpr uint32_t kMaskWarps = (kGated || kQk) ? 4 : 8;
  constexpr uint32_t kQkThreads = kQk ? 128 : 0;
  constexpr uint32_t kMaskThreads = 32 * kMaskWarps;
  constexpr uint32_t kEpiThreads = kGated ? 256 : 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + kOffCtrl);
  volatile uint32_t* abort_flag = &ctrl->abort;
  const uint32_t smem_base = smem_u32(smem);

  const uint32_t warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;
  const uint64_t T = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctrl->full[s], 1);
      // with the fused norm + gate a stage is free once the MMAs are done with it and the
      // epilogue has read the gate rows staged in its Q slot
      mbar_init(&ctrl->empty[s], kGated ? 2 : 1);
      mbar_init(&ctrl->gate_full[s], 1);
      mbar_init(&ctrl->qk_ready[s], 128);
      mbar_init(&ctrl->kt_ready[s], 128);
      mbar_init(&ctrl->unit_full[s], 1);
      mbar_init(&ctrl->unit_empty[s], 1 + kMaskThreads + 128 + kEpiThreads + kQkThreads);
    }
    mbar_init(&ctrl->s_full, 1);
    mbar_init(&ctrl->p_ready, kMaskThreads);
    mbar_init(&ctrl->s2_full, 1);
    mbar_init(&ctrl->p2_ready, kMaskThreads);
    mbar_init(&ctrl->o_full, 1);
    mbar_init(&ctrl->o_free, kEpiThreads);
    mbar_init(&ctrl->kv_done, 1);
    mbar_init(&ctrl->kvb_ready, 128);
    mbar_init(&ctrl->kv_free, 128);
    mbar_init(&ctrl->h_done, 1);
    mbar_init(&ctrl->mma_final, 1);
    ctrl->abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
    if (kGated) tma_prefetch_desc(&p.tm_gate);
  }
  if (warp == 2) {
    tmem_alloc(&ctrl->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctrl->tmem_base;

  if (warp == 0) {
    // =========================================================================================
    // TMA producer
    // =========================================================================================
    if (lane == 0) {
      const uint64_t pol_first = policy_evict_first();
      const uint64_t pol_last = policy_evict_last();
      const uint64_t pol_normal = policy_evict_normal();
      const int32_t depth = p.prefetch_depth;  // chunk-loads brought into L2 ahead of time

      // A unit is a stream of chunk-loads: nc local-state loads (K, V) if it has that pass,
      // then nc output loads (Q, K, V).
      RangeCursor rcur;
      auto fetch = [&](UnitInfo& ui) {
        if (p.n_ranges > 0) {
          next_balanced_unit(p, rcur, ui);
          return;
        }
        const int64_t u = static_cast<int64_t>(atomicAdd(p.counter, 1u));
        const int64_t units = p.units_dev != nullptr ? *p.units_dev : p.units;
        if (u < units) {
          decode_unit(p, u, ui);
        } else {
          ui.bh = -1;
          ui.seg = ui.c0 = ui.nc = ui.len = ui.flags = ui.b = ui.tok0 = ui.slot = 0;
          ui.in_slot = -1;
          ui.in_val = ui.pub_val = 0;
        }
      };
      auto n_loads = [](const UnitInfo& ui) -> int32_t {
        if (ui.bh < 0) return 0;
        if (!(ui.flags & kUnitLocal)) return ui.nc;
        return (ui.flags & kUnitNoOutput) ? ui.nc : 2 * ui.nc;
      };
      // L2 prefetch of chunk-load `pos` of `ui` (the part of it that comes from DRAM)
      auto prefetch = [&](const UnitInfo& ui, int32_t pos) {
        const int32_t b = ui.b;
        const int32_t h = static_cast<int32_t>(ui.bh % p.H);
        const bool two_pass = (ui.flags & 1) != 0;
        const bool local_pass = two_pass && pos < ui.nc;
        const int32_t c = two_pass && !local_pass ? pos - ui.nc : pos;
        const int32_t n0 = ui.tok0 + (ui.c0 + c) * C;
        if (!local_pass) {
          tma_prefetch_l2_4d(&p.tm_q, 0, h, n0, b, pol_normal);
          tma_prefetch_l2_4d(&p.tm_q, 64, h, n0, b, pol_normal);
        }
        if (local_pass || !two_pass) {
          const uint64_t pol = local_pass ? pol_last : pol_normal;
          tma_prefetch_l2_4d(&p.tm_k, 0, h, n0, b, pol);
          tma_prefetch_l2_4d(&p.tm_k, 64, h, n0, b, pol);
          tma_prefetch_l2_4d(&p.tm_v, 0, h, n0, b, pol);
          tma_prefetch_l2_4d(&p.tm_v, 64, h, n0, b, pol);
        }
      };

      uint32_t g = 0;
      uint32_t j = 0;
      uint32_t issued[2] = {0, 0};  // fills issued per stage (for the abort drain)
      bool ok = true;
      UnitInfo cur, nxt;
      bool have_nxt = false;
      while (ok) {
        const uint32_t slot = j & 1;
        if (!mbar_wait_bounded(&ctrl->unit_empty[slot], ((j >> 1) & 1) ^ 1, abort_flag, T)) {
          ok = false;
          break;
        }
        if (have_nxt) {
          cur = nxt;
          have_nxt = false;
        } else {
          fetch(cur);
          for (int32_t q = 0; q < min(depth, n_loads(cur)); ++q) prefetch(cur, q);
        }
        ctrl->units[slot] = cur;
        mbar_arrive(&ctrl->unit_full[slot]);
        if (cur.bh < 0) break;
        const int32_t b = cur.b;
        const int32_t h = static_cast<int32_t>(cur.bh % p.H);
        const int32_t n_cur = n_loads(cur);
        for (int32_t pos = 0; pos < n_cur; ++pos) {
          // keep `depth` chunk-loads ahead in L2, running into the next unit near the end
          if (depth > 0) {
            const int32_t q = pos + depth;
            if (q < n_cur) {
              prefetch(cur, q);
            } else {
              if (!have_nxt) {
                fetch(nxt);
                have_nxt = true;
              }
              if (q - n_cur < n_loads(nxt)) prefetch(nxt, q - n_cur);
            }
          }
          if (pos + 1 == n_cur && p.state_in != nullptr) {
            // at the unit's last load, claim the next unit and bring its initial state into L2
            // for the state warps (64 KiB per head, read when that unit starts)
            if (!have_nxt) {
              fetch(nxt);
              have_nxt = true;
            }
            if (nxt.bh >= 0 && nxt.seg == 0)
              bulk_prefetch_l2(p.state_in + static_cast<int64_t>(nxt.bh) * D * D, D * D * 4);
          }
          const uint32_t s = g & 1;
          if (!mbar_wait_bounded(&ctrl->empty[s], ((g >> 1) & 1) ^ 1, abort_flag, T)) {
            ok = false;
            break;
          }
          const bool local_state_pass = (cur.flags & 1) && pos < cur.nc;
          const int32_t c = (cur.flags & 1) && !local_state_pass ? pos - cur.nc : pos;
          uint8_t* st = smem + s * kStageBytes;
          const int32_t n0 = cur.tok0 + (cur.c0 + c) * C;
          const uint64_t kv_pol = local_state_pass ? pol_last : pol_first;
          if (local_state_pass) {
            mbar_arrive_expect_tx(&ctrl->full[s], 2 * kTileBytes);
          } else {
            mbar_arrive_expect_tx(&ctrl->full[s], 3 * kTileBytes);
            tma_load_4d(st + kOffQ, &p.tm_q, &ctrl->full[s], 0, h, n0, b, pol_first);
            tma_load_4d(st + kOffQ + kHalfBytes, &p.tm_q, &ctrl->full[s], 64, h, n0, b,
                        pol_first);
          }
          if (kGated && !local_state_pass) {
            // the epilogue reads this chunk's gate rows about one chunk period from now
            tma_prefetch_l2_4d(&p.tm_gate, 0, h, n0, b, pol_normal);
            tma_prefetch_l2_4d(&p.tm_gate, 64, h, n0, b, pol_normal);
          }
          tma_load_4d(st + kOffK, &p.tm_k, &ctrl->full[s], 0, h, n0, b, kv_pol);
          tma_load_4d(st + kOffK + kHalfBytes, &p.tm_k, &ctrl->full[s], 64, h, n0, b, kv_pol);
          tma_load_4d(st + kOffV, &p.tm_v, &ctrl->full[s], 0, h, n0, b, kv_pol);
          tma_load_4d(st + kOffV + kHalfBytes, &p.tm_v, &ctrl->full[s], 64, h, n0, b, kv_pol);
          issued[s] += 1;
          ++g;
        }
        ++j;
      }
      if (!ok) {
        // Let every fill already issued land before the CTA's shared memory goes away.
        for (uint32_t s = 0; s < 2; ++s) {
          if (issued[s] > 0) {
            const uint32_t last_parity = (issued[s] - 1) & 1;
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&ctrl->full[s], last_parity) && globaltimer_ns() - t0 < T) {
            }
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // =========================================================================================
    // tcgen05.mma issuer
    // =========================================================================================
    if (lane == 0) {
      constexpr uint32_t idS = make_idesc_bf16(128, 128, 0, 0);   // Q (K-major) x K (K-major)
      constexpr uint32_t idQK = make_idesc_bf16(128, 128, 0, 1);  // Q x KVb (MN-major)
      constexpr uint32_t idPV = make_idesc_bf16(128, 128, 0, 1);  // P (TMEM) x V (MN-major)
      constexpr uint32_t idKV = make_idesc_bf16(128, 128, 1, 1);  // K~^T (MN) x V (MN)
      uint32_t g = 0, j = 0;
      uint32_t n_kvb = 0, n_ofree = 0, n_p = 0, n_p2 = 0;
      bool ok = true;
      // KV (+)= K~^T V over token rows [16 kk0, 16 kk1) of the tile held in stage (gg & 1)
      auto issue_state_update_rows = [&](uint32_t gg, uint32_t kk0, uint32_t kk1) {
        const uint32_t kb = smem_base + (gg & 1) * kStageBytes + kOffK;
        const uint32_t vb = smem_base + (gg & 1) * kStageBytes + kOffV;
#pragma unroll
        for (uint32_t kk = kk0; kk < kk1; ++kk) {
          umma_ss(tmem + kColKV, make_sdesc_sw128(kb + kk * 2048, kHalfBytes, 1024),
                  make_sdesc_sw128(vb + kk * 2048, kHalfBytes, 1024), idKV, 1u);
        }
      };
      // KV (+)= K~^T V for the whole tile held in stage (gg & 1)
      auto issue_state_update = [&](uint32_t gg, bool accumulate_first) {
        const uint32_t kb = smem_base + (gg & 1) * kStageBytes + kOffK;
        const uint32_t vb = smem_base + (gg & 1) * kStageBytes + kOffV;
#pragma unroll
        for (uint32_t kk = 0; kk < 8; ++kk) {
          umma_ss(tmem + kColKV, make_sdesc_sw128(kb + kk * 2048, kHalfBytes, 1024),
                  make_sdesc_sw128(vb + kk * 2048, kHalfBytes, 1024), idKV,
                  (accumulate_first || kk > 0) ? 1u : 0u);
        }
      };
      while (ok) {
        const uint32_t slot = j & 1;
        if (!mbar_wait_bounded(&ctrl->unit_full[slot], (j >> 1) & 1, abort_flag, T)) break;
        const UnitInfo ui = ctrl->units[slot];
        mbar_arrive(&ctrl->unit_empty[slot]);
        if (ui.bh < 0) break;
        // A local-state pass writes the state columns first, so it waits for the previous unit's
        // read-out.  Otherwise the state warps write them first themselves (the incoming state),
        // after their own read-out, and every state-column MMA here waits for that; S_0 need not.
        // Skipping the wait keeps the barrier's phases unambiguous: when this warp starts unit j,
        // the state warps have finished unit j-2 (it waited either here or for their operand of
        // unit j-1's first chunk), so the phase it waits for next is never two behind.  A unit
        // without chunks gives no such operand, so it waits here too.
        if ((ui.flags & 1) || ui.nc == 0) {
          if (!mbar_wait_bounded(&ctrl->kv_free, j & 1, abort_flag, T)) break;
          tc_fence_after();
        }
        if (ui.flags & 1) {
          // local segment state h = sum_j lambda^(L-1-j) k_j^T v_j into the KV columns
          for (int32_t c = 0; c < ui.nc && ok; ++c) {
            const uint32_t s = g & 1;
            const uint32_t ph = (g >> 1) & 1;
            if (!mbar_wait_bounded(&ctrl->full[s], ph, abort_flag, T) ||
                !mbar_wait_bounded(&ctrl->kt_ready[s], ph, abort_flag, T)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_state_update(g, c > 0);
            umma_commit(&ctrl->empty[s]);
            // (with the fused norm + gate a stage takes two arrivals; a local-state tile has no
            // epilogue, so both come from here)
            if (kGated) umma_commit(&ctrl->empty[s]);
            ++g;
          }
          if (!ok) break;
          umma_commit(&ctrl->h_done);
        }
        const int32_t n_out = (ui.flags & kUnitNoOutput) ? 0 : ui.nc;
        for (int32_t c = 0; c < n_out && ok; ++c) {
          const uint32_t s = g & 1;
          const uint32_t ph = (g >> 1) & 1;
          if (!mbar_wait_bounded(&ctrl->full[s], ph, abort_flag, T) ||
              (kQk && !mbar_wait_bounded(&ctrl->qk_ready[s], ph, abort_flag, T))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t qb = smem_base + s * kStageBytes + kOffQ;
          const uint32_t kb = smem_base + s * kStageBytes + kOffK;
          const uint32_t vb = smem_base + s * kStageBytes + kOffV;
          const uint32_t kvb = smem_base + kOffKVb;
          // C = 256: the first tile A (even c) of a two-tile chunk keeps its stage until the second
          // tile B (odd c) has read K~_A and V_A from it (stage s ^ 1).
          const bool tile_b = kCM == kC256 && (c & 1) != 0;
          const bool keep_stage = kCM == kC256 && (c & 1) == 0 && c + 1 < n_out;
          // D (+)= Q K^T over d = 128 (both K-major), from this tile's Q and the keys at kbase
          auto issue_qk = [&](uint32_t d_col, uint32_t kbase) {
#pragma unroll
            for (uint32_t kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
              umma_ss(tmem + d_col, make_sdesc_sw128(qb + off, 16, 1024),
                      make_sdesc_sw128(kbase + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
            }
          };
          // D = Q KVb (the bf16 state operand)
          auto issue_qkv = [&](uint32_t d_col) {
#pragma unroll
            for (uint32_t kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
              umma_ss(tmem + d_col, make_sdesc_sw128(qb + off, 16, 1024),
                      make_sdesc_sw128(kvb + kk * 2048, kHalfBytes, 1024), idQK,
                      kk > 0 ? 1u : 0u);
            }
          };
          // O_intra (+)= P V with P read from TMEM and the values at vbase
          auto issue_pv = [&](uint32_t vbase, bool accumulate) {
#pragma unroll
            for (uint32_t kk = 0; kk < 8; ++kk) {
              umma_ts(tmem + kColOintra, tmem + kColS + kk * 8,
                      make_sdesc_sw128(vbase + kk * 2048, kHalfBytes, 1024), idPV,
                      (accumulate || kk > 0) ? 1u : 0u);
            }
          };
          if (kCM == kC64) {
            // the S columns held the previous tile's second inter product until the epilogue read
            // it, so S waits for the free accumulators here rather than before O_inter
            if (!mbar_wait_bounded(&ctrl->o_free, n_ofree & 1, abort_flag, T)) {
              ok = false;
              break;
            }
            ++n_ofree;
            tc_fence_after();
          }
          if (tile_b) {
            // S_BA = Q_B K~_A^T, the scores of this tile's queries against the chunk's first tile
            issue_qk(kColS, smem_base + (s ^ 1) * kStageBytes + kOffK);
            umma_commit(&ctrl->s2_full);
          } else {
            issue_qk(kColS, kb);  // S_c = Q K^T
            umma_commit(&ctrl->s_full);
          }
          // O_inter = Q KV_in (needs the bf16 state operand and a free O accumulator)
          if (!mbar_wait_bounded(&ctrl->kvb_ready, n_kvb & 1, abort_flag, T)) {
            ok = false;
            break;
          }
          ++n_kvb;
          if (kCM != kC64) {
            if (!mbar_wait_bounded(&ctrl->o_free, n_ofree & 1, abort_flag, T)) {
              ok = false;
              break;
            }
            ++n_ofree;
          }
          tc_fence_after();
          issue_qkv(kColOinter);
          if (kCM == kC64) {
            // first chunk of the tile: KV += K~_A^T V_A (token rows 0..63)
            if (!mbar_wait_bounded(&ctrl->kt_ready[s], ph, abort_flag, T)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_state_update_rows(g, 0, 4);
            umma_commit(&ctrl->kv_done);
            // O_intra = P V with the block-diagonal P
            if (!mbar_wait_bounded(&ctrl->p_ready, n_p & 1, abort_flag, T)) {
              ok = false;
              break;
            }
            ++n_p;
            tc_fence_after();
            issue_pv(vb, false);
            // second chunk: its inter product from the state after the first chunk (rows 64..127
            // of this D are the ones used), written over the S columns now that P has been read;
            // then KV += K~_B^T V_B
            if (!mbar_wait_bounded(&ctrl->kvb_ready, n_kvb & 1, abort_flag, T)) {
              ok = false;
              break;
            }
            ++n_kvb;
            tc_fence_after();
            issue_qkv(kColS);
            issue_state_update_rows(g, 4, 8);
            umma_commit(&ctrl->kv_done);
            umma_commit(&ctrl->o_full);
            umma_commit(&ctrl->empty[s]);
          } else if (tile_b) {
            // O_intra = P_BA V_A; then tile A's stage is free
            if (!mbar_wait_bounded(&ctrl->p2_ready, n_p2 & 1, abort_flag, T)) {
              ok = false;
              break;
            }
            ++n_p2;
            tc_fence_after();
            issue_pv(smem_base + (s ^ 1) * kStageBytes + kOffV, false);
            umma_commit(&ctrl->empty[s ^ 1]);
            // S_BB = Q_B K_B^T over the S columns (in issue order after P_BA V_A read P_BA)
            issue_qk(kColS, kb);
            umma_commit(&ctrl->s_full);
            if (!mbar_wait_bounded(&ctrl->kt_ready[s], ph, abort_flag, T)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_state_update(g, true);
            umma_commit(&ctrl->kv_done);
            if (!mbar_wait_bounded(&ctrl->p_ready, n_p & 1, abort_flag, T)) {
              ok = false;
              break;
            }
            ++n_p;
            tc_fence_after();
            issue_pv(vb, true);  // O_intra += P_BB V_B
            umma_commit(&ctrl->o_full);
            umma_commit(&ctrl->empty[s]);
          } else {
            // KV += K~_c^T V_c once K_c is row-scaled (after S_c, which read K_c unscaled).  It
            // follows O_inter_c, so kv_done also tells the state warps that the bf16 operand
            // O_inter read is free again.
            if (!mbar_wait_bounded(&ctrl->kt_ready[s], ph, abort_flag, T)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_state_update(g, true);
            umma_commit(&ctrl->kv_done);
            // O_intra = P V, P read from TMEM
            if (!mbar_wait_bounded(&ctrl->p_ready, n_p & 1, abort_flag, T)) {
              ok = false;
              break;
            }
            ++n_p;
            tc_fence_after();
            issue_pv(vb, false);
            umma_commit(&ctrl->o_full);
            if (!keep_stage) umma_commit(&ctrl->empty[s]);
          }
          ++g;
        }
        if (!ok) break;
        ++j;
      }
      // all issued MMAs must finish before TMEM is released
      umma_commit(&ctrl->mma_final);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&ctrl->mma_final, 0) && globaltimer_ns() - t0 < T) {
      }
    }
    __syncwarp();
  } else if (warp >= kWarpP0 && warp < kWarpP0 + kMaskWarps) {
    // =========================================================================================
    // P = decay-mask(S) -> TMEM (bf16); K -> K~ in the local-state pass
    // =========================================================================================
    const uint32_t pw = warp - kWarpP0;          // 0..kMaskWarps-1
    const uint32_t wq = warp & 3;                // TMEM lane quarter
    const uint32_t hf = pw >> 2;                 // 8 warps: column blocks hf and hf + 2
    const uint32_t i = wq * 32 + lane;           // row of the chunk (query token)
    const uint32_t tp = threadIdx.x - kWarpP0 * 32;  // 0..kMaskThreads-1
    const uint32_t trow = tmem + ((wq * 32) << 16);
    uint32_t g = 0, j = 0, n_s = 0, n_s2 = 0;
    while (true) {
      const uint32_t slot = j & 1;
      bool ok = mbar_wait_bounded(&ctrl->unit_full[slot], (j >> 1) & 1, abort_flag, T);
      if (!group_all(ok, kBarP, kMaskThreads)) break;
      const UnitInfo ui = ctrl->units[slot];
      mbar_arrive(&ctrl->unit_empty[slot]);
      if (ui.bh < 0) break;
      const float alpha = p.slopes[ui.bh % p.H] * kLog2e;  // lambda^n = exp2(-alpha n)
      const float lam1 = ex2_approx(-alpha);                 // lambda

      if ((ui.flags & 1) && kQk) {
        g += static_cast<uint32_t>(ui.nc);  // (the QK transform warps scale these tiles' keys)
      } else if (ui.flags & 1) {
        // local-state pass: K~_j = lambda^(L-1-j) k_j (8 warps: two threads per row, one per
        // half; 4 warps: one thread per row)
        const uint32_t r = tp & 127;
        const uint32_t half = tp >> 7;
        for (int32_t c = 0; c < ui.nc; ++c) {
          const uint32_t s = g & 1;
          ok = mbar_wait_bounded(&ctrl->full[s], (g >> 1) & 1, abort_flag, T);
          if (!group_all(ok, kBarP, kMaskThreads)) goto p_out;
          const int32_t pos = c * C + static_cast<int32_t>(r);  // token within the segment
          const float w =
              pos < ui.len ? exp2f(-alpha * static_cast<float>(ui.len - 1 - pos)) : 0.f;
          if (kMaskWarps == 8) {
            scale_half_row(smem + s * kStageBytes + kOffK + half * kHalfBytes, r, w);
          } else {
            scale_half_row(smem + s * kStageBytes + kOffK, r, w);
            scale_half_row(smem + s * kStageBytes + kOffK + kHalfBytes, r, w);
          }
          fence_proxy_async_smem();
          named_bar_sync(kBarP, kMaskThreads);
          if (tp < 128) mbar_arrive(&ctrl->kt_ready[s]);
          ++g;
        }
      }
      // P_ij = lambda^(i-j) S_ij for j <= i, else 0, over S columns j = 32 jb + m.  The factor
      // lambda^max(i-j, 0) is built per 16-column half by walking m downward from the half's
      // last column and multiplying by lambda <= 1 once j <= i: no intermediate can overflow,
      // for any slope, and underflow only drops terms below fp32 range.
      auto make_p = [&](uint32_t jb, const uint32_t (&r)[32], uint32_t (&pk)[16]) {
        const int32_t dbase = static_cast<int32_t>(i) - static_cast<int32_t>(jb * 32);
        const int mlim = jb == wq ? static_cast<int>(lane) : 31;  // columns m > mlim: j > i
#pragma unroll
        for (int h = 1; h >= 0; --h) {
          const int mtop = 16 * h + 15;
          float f = ex2_approx(-alpha * static_cast<float>(max(dbase - mtop, 0)));
#pragma unroll
          for (int m = mtop; m > 16 * h; m -= 2) {
            const float x1 = m <= mlim ? __uint_as_float(r[m]) * f : 0.f;
            if (dbase - m >= 0) f *= lam1;
            const float x0 = m - 1 <= mlim ? __uint_as_float(r[m - 1]) * f : 0.f;
            if (dbase - (m - 1) >= 0) f *= lam1;
            pk[(m - 1) >> 1] = pack_bf16x2(x0, x1);
          }
        }
      };
      // C = 64: P is block-diagonal, so rows 64..127 (lane quarters 2, 3) keep nothing of
      // columns 0..63 (S blocks 0, 1)
      auto live = [&](uint32_t jb) { return jb <= wq && !(kCM == kC64 && wq >= 2 && jb < 2); };
      const int32_t n_out = (ui.flags & kUnitNoOutput) ? 0 : ui.nc;
      for (int32_t c = 0; c < n_out; ++c) {
        if (kCM == kC256 && (c & 1) != 0) {
          // Second tile of a 256-token chunk: P_BA = lambda^(i+1) S~_BA over all 128 columns
          // (S~_BA = Q_B K~_A^T already carries lambda^(127-j)), no causal mask.  The block split
          // and the barrier before the first store are those of the causal pass below.
          ok = mbar_wait_bounded(&ctrl->s2_full, n_s2 & 1, abort_flag, T);
          if (!group_all(ok, kBarP, kMaskThreads)) goto p_out;
          ++n_s2;
          tc_fence_after();
          const float fr = ex2_approx(-alpha * static_cast<float>(i + 1));
          uint32_t r[32];
          uint32_t pk[16];
          if (kMaskWarps == 8) {
            tmem_ld32(trow + kColS + hf * 32, r);
            tmem_wait_ld();
            tc_fence_before();
            named_bar_sync(kBarP, kMaskThreads);
            tc_fence_after();
#pragma unroll
            for (int m = 0; m < 16; ++m)
              pk[m] =
                  pack_bf16x2(__uint_as_float(r[2 * m]) * fr, __uint_as_float(r[2 * m + 1]) * fr);
            tmem_st16(trow + kColS + hf * 16, pk);
            tmem_ld32(trow + kColS + (hf + 2) * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int m = 0; m < 16; ++m)
              pk[m] =
                  pack_bf16x2(__uint_as_float(r[2 * m]) * fr, __uint_as_float(r[2 * m + 1]) * fr);
            tmem_st16(trow + kColS + (hf + 2) * 16, pk);
          } else {
            // one warp owns the lane quarter: the blocks in order, each read before the P
            // store that overlaps it (P block jb lands in S block jb / 2 <= jb)
#pragma unroll 1
            for (uint32_t jb = 0; jb < 4; ++jb) {
              tmem_ld32(trow + kColS + jb * 32, r);
              tmem_wait_ld();
#pragma unroll
              for (int m = 0; m < 16; ++m)
                pk[m] = pack_bf16x2(__uint_as_float(r[2 * m]) * fr,
                                    __uint_as_float(r[2 * m + 1]) * fr);
              tmem_st16(trow + kColS + jb * 16, pk);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&ctrl->p2_ready);
        }
        ok = mbar_wait_bounded(&ctrl->s_full, n_s & 1, abort_flag, T);
        if (!group_all(ok, kBarP, kMaskThreads)) goto p_out;
        ++n_s;
        tc_fence_after();
        // P is written over S in place: P block jb -> columns [16 jb, 16 jb + 16), inside S block
        // jb / 2.  With 8 warps, the two warps of a lane quarter take S blocks {hf, hf + 2}; the
        // only S blocks a P store can overwrite are 0 and 1, which the warps read first, before a
        // barrier that precedes every P store.  With 4 warps, each warp walks its quarter's
        // blocks in order, reading each before the store that overlaps it.
        {
          uint32_t r[32];
          uint32_t pk[16];
          if (kMaskWarps == 8) {
            const uint32_t jb0 = hf;
            const bool live0 = live(jb0);
            if (live0) {
              tmem_ld32(trow + kColS + jb0 * 32, r);
              tmem_wait_ld();
            }
            tc_fence_before();
            named_bar_sync(kBarP, kMaskThreads);
            tc_fence_after();
            if (live0) {
              make_p(jb0, r, pk);
            } else {
#pragma unroll
              for (int m = 0; m < 16; ++m) pk[m] = 0u;
            }
            tmem_st16(trow + kColS + jb0 * 16, pk);
            const uint32_t jb1 = hf + 2;
            if (jb1 <= wq) {
              tmem_ld32(trow + kColS + jb1 * 32, r);
              tmem_wait_ld();
              make_p(jb1, r, pk);
            } else {
#pragma unroll
              for (int m = 0; m < 16; ++m) pk[m] = 0u;
            }
            tmem_st16(trow + kColS + jb1 * 16, pk);
          } else {
#pragma unroll 1
            for (uint32_t jb = 0; jb < 4; ++jb) {
              if (live(jb)) {
                tmem_ld32(trow + kColS + jb * 32, r);
                tmem_wait_ld();
                make_p(jb, r, pk);
              } else {
#pragma unroll
                for (int m = 0; m < 16; ++m) pk[m] = 0u;
              }
              tmem_st16(trow + kColS + jb * 16, pk);
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ctrl->p_ready);
        ++g;
      }
      ++j;
    }
  p_out:;
  } else if (kQk && warp >= kWarpP0 + kMaskWarps && warp < kWarpS0) {
    // =========================================================================================
    // in-tile QK RMSNorm + RoPE: thread r transforms row r of the stage's q and k tiles as soon
    // as they land, before any product reads them; in the local-state pass it also scales its
    // key row to K~ (the mask warps' job in the other instances)
    // =========================================================================================
    const uint32_t r = (warp - (kWarpP0 + kMaskWarps)) * 32 + lane;  // tile row 0..127
    uint32_t g = 0, j = 0;
    while (true) {
      const uint32_t slot = j & 1;
      bool ok = mbar_wait_bounded(&ctrl->unit_full[slot], (j >> 1) & 1, abort_flag, T);
      if (!group_all(ok, kBarT, kQkThreads)) break;
      const UnitInfo ui = ctrl->units[slot];
      mbar_arrive(&ctrl->unit_empty[slot]);
      if (ui.bh < 0) break;
      const float alpha = p.slopes[ui.bh % p.H] * kLog2e;
      const int32_t n_local = (ui.flags & kUnitLocal) ? ui.nc : 0;
      const int32_t n_tiles = n_local + ((ui.flags & kUnitNoOutput) ? 0 : ui.nc);
      // index along the B * N token axis of row r of the piece's first tile
      const int64_t tok_r = static_cast<int64_t>(ui.b) * p.N + ui.tok0 +
                            static_cast<int64_t>(ui.c0) * C + r;
      for (int32_t q = 0; q < n_tiles; ++q) {
        const bool local = q < n_local;
        const int32_t c = local ? q : q - n_local;
        const int32_t row = c * C + static_cast<int32_t>(r);  // token of the piece
        const bool valid = row < ui.len;  // rows past the piece are never output nor summed
        const int64_t pos = valid ? p.qk_positions[tok_r + static_cast<int64_t>(c) * C] : 0;
        const uint32_t s = g & 1;
        ok = mbar_wait_bounded(&ctrl->full[s], (g >> 1) & 1, abort_flag, T);
        if (!group_all(ok, kBarT, kQkThreads)) goto t_out;
        uint8_t* st = smem + s * kStageBytes;
        if (local) {
          // K~_j = lambda^(L-1-j) k_hat_j: the transformed row is rounded to bf16 and then
          // scaled with one more rounding, as when k_hat comes from memory
          if (valid)
            qk_norm_rope_rows<false>(nullptr, st + kOffK, r, pos, p.qk_gamma_q, p.qk_gamma_k,
                                     p.qk_inv_freq, p.qk_rotary_dim, p.qk_eps);
          const float w = valid ? exp2f(-alpha * static_cast<float>(ui.len - 1 - row)) : 0.f;
          scale_half_row(st + kOffK, r, w);
          scale_half_row(st + kOffK + kHalfBytes, r, w);
        } else if (valid) {
          qk_norm_rope_rows<true>(st + kOffQ, st + kOffK, r, pos, p.qk_gamma_q, p.qk_gamma_k,
                                  p.qk_inv_freq, p.qk_rotary_dim, p.qk_eps);
        }
        fence_proxy_async_smem();
        mbar_arrive(&ctrl->qk_ready[s]);
        if (local) mbar_arrive(&ctrl->kt_ready[s]);
        ++g;
      }
      ++j;
    }
  t_out:;
  } else if (warp >= kWarpS0 && warp < kWarpO0) {
    // =========================================================================================
    // state: look-back scan over segments, bf16 operand, decay rescale, final state; K -> K~
    // during the output pass
    // =========================================================================================
    const uint32_t wq = warp & 3;
    const uint32_t i = wq * 32 + lane;  // key-dimension row of the state / key token of K~
    const uint32_t trow = tmem + ((wq * 32) << 16);
    uint8_t* kvb = smem + kOffKVb;
    uint32_t g = 0, j = 0, n_kvd = 0, n_h = 0, n_s = 0;
    uint32_t gate_issued[2] = {0u, 0u};  // fused norm + gate: gate tiles loaded per stage
    tc_fence_before();
    mbar_arrive(&ctrl->kv_free);  // the KV columns start out free

    // bf16 copy of 32 state columns [32 cb, 32 cb + 32) of row i into the MN-major operand
    // (x holds fp32 bit patterns)
    auto write_kvb = [&](uint32_t cb, const uint32_t (&x)[32]) {
      const uint32_t half = cb >> 1;
#pragma unroll
      for (uint32_t q = 0; q < 4; ++q) {
        const uint32_t c16 = (cb & 1) * 4 + q;
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(x[8 * q + 0]), __uint_as_float(x[8 * q + 1]));
        w.y = pack_bf16x2(__uint_as_float(x[8 * q + 2]), __uint_as_float(x[8 * q + 3]));
        w.z = pack_bf16x2(__uint_as_float(x[8 * q + 4]), __uint_as_float(x[8 * q + 5]));
        w.w = pack_bf16x2(__uint_as_float(x[8 * q + 6]), __uint_as_float(x[8 * q + 7]));
        *reinterpret_cast<uint4*>(kvb + half * kHalfBytes + sw128_off(i, c16)) = w;
      }
    };

    while (true) {
      const uint32_t slot = j & 1;
      bool ok = mbar_wait_bounded(&ctrl->unit_full[slot], (j >> 1) & 1, abort_flag, T);
      if (!group_all(ok, kBarS, 128)) break;
      const UnitInfo ui = ctrl->units[slot];
      mbar_arrive(&ctrl->unit_empty[slot]);
      if (ui.bh < 0) break;
      const float alpha = p.slopes[ui.bh % p.H] * kLog2e;
      const int64_t bh = ui.bh;    // state_in / state_out index
      const int32_t k = ui.seg;
      const bool publish = (ui.flags & kUnitLocal) != 0;
      const bool outputs = (ui.flags & kUnitNoOutput) == 0;

      if (publish) {
        ok = mbar_wait_bounded(&ctrl->h_done, n_h & 1, abort_flag, T);
        if (!group_all(ok, kBarS, 128)) break;
        ++n_h;
        tc_fence_after();
        g += static_cast<uint32_t>(ui.nc);  // the local-state pass used these stages
      }
      // incoming state of this piece: published by the previous piece of the same sequence
      if (ui.in_slot >= 0) {
        const uint32_t* fl = p.flags + ui.in_slot;
        const uint64_t t0 = globaltimer_ns();
        ok = true;
        while (ld_acquire_u32(fl) != static_cast<uint32_t>(ui.in_val)) {
          if (*abort_flag || ld_volatile_s32(p.status) != 0 || globaltimer_ns() - t0 > T) {
            ok = false;
            *abort_flag = 1u;
            break;
          }
        }
        if (!group_all(ok, kBarS, 128)) break;
      }
      // ring layout: float4 (state row i, columns 4q..4q+3) at index q * 128 + i
      const float4* ring_in = reinterpret_cast<const float4*>(
          p.ring + static_cast<int64_t>(ui.in_slot >= 0 ? ui.in_slot : 0) * (D * D));
      float4* ring_out = reinterpret_cast<float4*>(
          p.ring + static_cast<int64_t>(publish ? ui.slot : 0) * (D * D));
      const float lam_len = exp2f(-alpha * static_cast<float>(ui.len));
      // decay of the incoming state over the first chunk (C = 64: the first half of tile 0)
      const float lam_n0 =
          exp2f(-alpha * static_cast<float>(min(kCM == kC64 ? 64 : C, ui.len)));
#pragma unroll 1
      for (uint32_t cb = 0; cb < 4; ++cb) {
        uint32_t sin[32];  // fp32 bits of the incoming state, columns [32 cb, 32 cb + 32)
        if (ui.in_slot >= 0) {
#pragma unroll
          for (uint32_t q = 0; q < 8; ++q) {
            const float4 x = __ldcg(ring_in + (cb * 8 + q) * 128 + i);
            sin[4 * q + 0] = __float_as_uint(x.x);
            sin[4 * q + 1] = __float_as_uint(x.y);
            sin[4 * q + 2] = __float_as_uint(x.z);
            sin[4 * q + 3] = __float_as_uint(x.w);
          }
        } else if (p.state_in != nullptr) {
          // the first segment continues from the caller's state: row i, columns [32 cb, +32)
          const float4* sr = reinterpret_cast<const float4*>(p.state_in + (bh * D + i) * D) + cb * 8;
#pragma unroll
          for (uint32_t q = 0; q < 8; ++q) {
            const float4 x = __ldcg(sr + q);  // coherent: state_out may be this same array
            sin[4 * q + 0] = __float_as_uint(x.x);
            sin[4 * q + 1] = __float_as_uint(x.y);
            sin[4 * q + 2] = __float_as_uint(x.z);
            sin[4 * q + 3] = __float_as_uint(x.w);
          }
        } else {
#pragma unroll
          for (int m = 0; m < 32; ++m) sin[m] = 0u;
        }
        if (publish) {
          // inclusive state S_{k+1} = lambda^L S_k + h_k, published for the next piece
          uint32_t r[32];
          tmem_ld32(trow + kColKV + cb * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (uint32_t q = 0; q < 8; ++q) {
            float4 x;
            x.x = fmaf(lam_len, __uint_as_float(sin[4 * q + 0]), __uint_as_float(r[4 * q + 0]));
            x.y = fmaf(lam_len, __uint_as_float(sin[4 * q + 1]), __uint_as_float(r[4 * q + 1]));
            x.z = fmaf(lam_len, __uint_as_float(sin[4 * q + 2]), __uint_as_float(r[4 * q + 2]));
            x.w = fmaf(lam_len, __uint_as_float(sin[4 * q + 3]), __uint_as_float(r[4 * q + 3]));
            __stcg(ring_out + (cb * 8 + q) * 128 + i, x);
          }
        }
        if (ui.nc == 0 && p.state_out != nullptr) {
          // a sequence without tokens: its final state is its initial state
          float4* so = reinterpret_cast<float4*>(p.state_out + (bh * D + i) * D) + cb * 8;
#pragma unroll
          for (uint32_t q = 0; q < 8; ++q)
            so[q] = make_float4(__uint_as_float(sin[4 * q]), __uint_as_float(sin[4 * q + 1]),
                                __uint_as_float(sin[4 * q + 2]), __uint_as_float(sin[4 * q + 3]));
        }
        if (outputs) {
          // the incoming state: bf16 operand of the first tile's inter product, and the fp32
          // state the tiles carry (already decayed over the first chunk)
          write_kvb(cb, sin);
#pragma unroll
          for (int m = 0; m < 32; ++m) sin[m] = __float_as_uint(lam_n0 * __uint_as_float(sin[m]));
          tmem_st32(trow + kColKV + cb * 32, sin);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      if (publish) {
        __threadfence();
        named_bar_sync(kBarS, 128);
        if (wq == 0 && lane == 0 && k != p.withhold_segment) {
          __threadfence();
          st_release_u32(p.flags + ui.slot, static_cast<uint32_t>(ui.pub_val));
        }
      }

      // carry the state through the segment's tiles
      bool good = true;
      // TMEM KV <- lambda^n KV, and (write_operand) its bf16 copy -> the MMA operand beforehand
      auto refresh = [&](bool write_operand, float lam) {
#pragma unroll 1
        for (uint32_t cb = 0; cb < 4; ++cb) {
          uint32_t r[32];
          tmem_ld32(trow + kColKV + cb * 32, r);
          tmem_wait_ld();
          if (write_operand) write_kvb(cb, r);
#pragma unroll
          for (int m = 0; m < 32; ++m) r[m] = __float_as_uint(lam * __uint_as_float(r[m]));
          tmem_st32(trow + kColKV + cb * 32, r);
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
      };
      const int32_t n_out = outputs ? ui.nc : 0;
      for (int32_t c = 0; c < n_out; ++c) {
        const uint32_t s = g & 1;
        const int32_t n_c = min(C, ui.len - c * C);  // tokens in this tile
        // the state operand for tile c is in place (written before the loop or by the previous
        // iteration's update)
        mbar_arrive(&ctrl->kvb_ready);
        // K~_c = diag(lambda^(n-1-j)) K_c for the state update, once S_c (the only other reader of
        // K_c) is complete; thread i scales key row i.  C = 64: each half of the tile is a chunk
        // of its own, scaled to its own end.
        ok = mbar_wait_bounded(&ctrl->s_full, n_s & 1, abort_flag, T);
        if (!group_all(ok, kBarS, 128)) {
          good = false;
          break;
        }
        ++n_s;
        {
          int32_t r = static_cast<int32_t>(i);
          int32_t n_r = n_c;
          if (kCM == kC64) {
            n_r = i < 64 ? min(64, n_c) : max(0, n_c - 64);
            r = static_cast<int32_t>(i & 63u);
          }
          const float w = r < n_r ? exp2f(-alpha * static_cast<float>(n_r - 1 - r)) : 0.f;
          uint8_t* kt = smem + s * kStageBytes + kOffK;
          // in-tile QK instance: the transform of this tile completed before S_c was issued, so
          // this wait returns at once; it orders those shared-memory writes before this row's
          if (kQk) (void)mbar_wait_bounded(&ctrl->qk_ready[s], (g >> 1) & 1, abort_flag, T);
          scale_half_row(kt, i, w);
          scale_half_row(kt + kHalfBytes, i, w);
          fence_proxy_async_smem();
          mbar_arrive(&ctrl->kt_ready[s]);
        }
        ok = mbar_wait_bounded(&ctrl->kv_done, n_kvd & 1, abort_flag, T);
        if (!group_all(ok, kBarS, 128)) {
          good = false;
          break;
        }
        ++n_kvd;
        tc_fence_after();
        if (kCM == kC64) {
          // the state after the tile's first chunk: its bf16 copy is the second chunk's operand
          // (the first chunk's inter product has completed: it precedes the update just waited
          // for); the fp32 state then decays over the second chunk's tokens
          refresh(true, exp2f(-alpha * static_cast<float>(max(0, n_c - 64))));
          mbar_arrive(&ctrl->kvb_ready);
          ok = mbar_wait_bounded(&ctrl->kv_done, n_kvd & 1, abort_flag, T);
          if (!group_all(ok, kBarS, 128)) {
            good = false;
            break;
          }
          ++n_kvd;
          tc_fence_after();
        }
        if (kGated && wq == 0 && lane == 0) {
          // every product that reads this tile's Q is complete (the update just waited for comes
          // after them): its Q slot takes the tile's gate rows for the fused epilogue
          const int32_t gn0 = ui.tok0 + (ui.c0 + c) * C;
          const int32_t gh = static_cast<int32_t>(ui.bh % p.H);
          const uint64_t pol = policy_evict_first();
          uint8_t* qslot = smem + s * kStageBytes + kOffQ;
          mbar_arrive_expect_tx(&ctrl->gate_full[s], kTileBytes);
          tma_load_4d(qslot, &p.tm_gate, &ctrl->gate_full[s], 0, gh, gn0, ui.b, pol);
          tma_load_4d(qslot + kHalfBytes, &p.tm_gate, &ctrl->gate_full[s], 64, gh, gn0, ui.b, pol);
          ++gate_issued[s];
        }
        if (c + 1 < n_out) {
          int32_t n_next = min(C, ui.len - (c + 1) * C);
          if (kCM == kC64) n_next = min(64, n_next);  // the next tile's first chunk
          // C = 256: after a chunk's first tile the operand stays the chunk's initial state
          refresh(!(kCM == kC256 && (c & 1) == 0), exp2f(-alpha * static_cast<float>(n_next)));
        } else if ((ui.flags & 2) && p.state_out != nullptr) {
          float4* so = reinterpret_cast<float4*>(p.state_out + (bh * D + i) * D);
#pragma unroll 1
          for (uint32_t cb = 0; cb < 4; ++cb) {
            uint32_t r[32];
            tmem_ld32(trow + kColKV + cb * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (uint32_t q = 0; q < 8; ++q) {
              so[cb * 8 + q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                           __uint_as_float(r[4 * q + 2]),
                                           __uint_as_float(r[4 * q + 3]));
            }
          }
        }
        ++g;
      }
      if (!good) break;
      tc_fence_before();
      mbar_arrive(&ctrl->kv_free);
      ++j;
    }
    if (kGated && wq == 0 && lane == 0 && *abort_flag) {
      // gate loads still in flight land before the CTA's shared memory goes away
      for (uint32_t st = 0; st < 2; ++st) {
        if (gate_issued[st] > 0) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&ctrl->gate_full[st], (gate_issued[st] - 1) & 1) &&
                 globaltimer_ns() - t0 < T) {
          }
        }
      }
    }
  } else if (warp >= kWarpO0 || (kGated && warp >= kWarpP0 + kMaskWarps && warp < kWarpS0)) {
    // =========================================================================================
    // output epilogue: thread i owns token row i of the chunk and writes its 256-byte output row
    // straight to global memory (no shared-memory staging, so the stage is released by the MMA
    // warp alone)
    // =========================================================================================
    const uint32_t wq = warp & 3;
    const uint32_t i = wq * 32 + lane;  // token row of the chunk
    const uint32_t trow = tmem + ((wq * 32) << 16);
    uint32_t j = 0, n_o = 0;
    uint32_t eg = 0;                  // tile loads so far (the stage of a tile is eg & 1)
    uint32_t n_gate[2] = {0u, 0u};    // gate tiles consumed per stage
    const uint32_t eh = warp >= kWarpO0 ? 0u : 1u;  // fused norm + gate: column half
    tc_fence_before();
    mbar_arrive(&ctrl->o_free);  // the O accumulators start out free
    while (true) {
      const uint32_t slot = j & 1;
      bool ok = mbar_wait_bounded(&ctrl->unit_full[slot], (j >> 1) & 1, abort_flag, T);
      if (!group_all(ok, kBarO, kEpiThreads)) break;
      const UnitInfo ui = ctrl->units[slot];
      mbar_arrive(&ctrl->unit_empty[slot]);
      if (ui.bh < 0) break;
      const float alpha = p.slopes[ui.bh % p.H] * kLog2e;
      // row i's inter-term factor lambda^(i'+1), i' its position in its chunk (C = 64: rows
      // 64..127 start the tile's second chunk); C = 256 adds lambda^128 on a chunk's second tile
      const float f_a = exp2f(-alpha * static_cast<float>((kCM == kC64 ? (i & 63u) : i) + 1));
      const float f_b = kCM == kC256 ? exp2f(-alpha * static_cast<float>(i + 129)) : f_a;
      // C = 64: rows 64..127 take their inter product from the S columns
      const uint32_t col_inter = (kCM == kC64 && i >= 64) ? kColS : kColOinter;
      const int64_t b = ui.b;
      const int64_t h = ui.bh % p.H;
      bool good = true;
      if (ui.flags & kUnitLocal) eg += static_cast<uint32_t>(ui.nc);  // local-state pass loads
      const int32_t n_out = (ui.flags & kUnitNoOutput) ? 0 : ui.nc;
      for (int32_t c = 0; c < n_out; ++c) {
        const float f = (c & 1) ? f_b : f_a;
        // Stores go out in 4-lane groups: after a 4 x 4 exchange of 16-byte pieces among lanes
        // 4a..4a+3 (rows i0..i0+3 of the chunk), store k writes 64 contiguous bytes of row i0 + k,
        // so every 32-byte sector is written whole by one instruction.
        const uint32_t t = lane & 3;
        const int32_t r0 = c * C + static_cast<int32_t>(i & ~3u);  // row i0, from segment start
        const int64_t n0 = static_cast<int64_t>(ui.tok0) + static_cast<int64_t>(ui.c0) * C + r0;
        __nv_bfloat16* out_h = p.out + (b * p.N * p.H + h) * D;
        const int64_t row_stride = p.H * D;
        if (kGated) {
          // the tile's gate rows are staged in its stage's Q slot (the state warps load them once
          // the tile's last Q product is done); once read, the stage may be refilled
          const uint32_t s = eg & 1;
          ++eg;
          ok = mbar_wait_bounded(&ctrl->o_full, n_o & 1, abort_flag, T);
          if (!group_all(ok, kBarO, kEpiThreads)) {
            good = false;
            break;
          }
          ++n_o;
          tc_fence_after();
          uint32_t ob[32];
          const float ss = gated_epilogue_read(ctrl, trow, col_inter, f, eh, ob);
          // the gate rows land while O is read
          ok = mbar_wait_bounded(&ctrl->gate_full[s], n_gate[s] & 1, abort_flag, T);
          if (!group_all(ok, kBarO, kEpiThreads)) {
            good = false;
            break;
          }
          ++n_gate[s];
          gated_epilogue_write(p, ctrl, ss, ob, ui, h, smem + s * kStageBytes + kOffQ, out_h, t,
                               r0, i & ~3u, n0, row_stride, i, eh, kEpiThreads);
          named_bar_sync(kBarO, kEpiThreads);
          if (warp == kWarpO0 && lane == 0) mbar_arrive(&ctrl->empty[s]);
          continue;
        }
        ok = mbar_wait_bounded(&ctrl->o_full, n_o & 1, abort_flag, T);
        if (!group_all(ok, kBarO, kEpiThreads)) {
          good = false;
          break;
        }
        ++n_o;
        tc_fence_after();
#pragma unroll 1
        for (uint32_t cb = 0; cb < 4; ++cb) {  // 32-column blocks
          uint32_t ra[32], re[32];
          tmem_ld32(trow + kColOintra + cb * 32, ra);
          tmem_ld32(trow + col_inter + cb * 32, re);
          tmem_wait_ld();
          if (cb == 3) {
            // every O column of this row has been read: the accumulators may be overwritten
            tc_fence_before();
            mbar_arrive(&ctrl->o_free);
          }
          uint4 x[4];  // 16-byte pieces q = 0..3 of this row's 64 bytes
#pragma unroll
          for (uint32_t q = 0; q < 4; ++q) {
            float o[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              o[e] = fmaf(f, __uint_as_float(re[8 * q + e]), __uint_as_float(ra[8 * q + e]));
            x[q].x = pack_bf16x2(o[0], o[1]);
            x[q].y = pack_bf16x2(o[2], o[3]);
            x[q].z = pack_bf16x2(o[4], o[5]);
            x[q].w = pack_bf16x2(o[6], o[7]);
          }
          transpose4x4_lanes(x, t);  // now x[k] = piece t of row i0 + k
#pragma unroll
          for (uint32_t k = 0; k < 4; ++k) {
            if (r0 + static_cast<int32_t>(k) < ui.len) {  // rows past the segment end: none
              uint4* dst = reinterpret_cast<uint4*>(out_h + (n0 + k) * row_stride + cb * 32) + t;
              __stcs(dst, x[k]);
            }
          }
        }
      }
      if (!good) break;
      ++j;
    }
  }

  // ===========================================================================================
  // teardown
  // ===========================================================================================
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && ctrl->abort) atomicExch(p.status, kErrTimeout);
  if (warp == 2) tmem_dealloc(tmem, 512);
}

// Chunk-loads the producer keeps in flight as L2 prefetches ahead of its shared-memory fills.
// LA_PREFETCH_DEPTH overrides the default (a tuning knob; every value computes the same result).
int32_t prefetch_depth() {
  static int32_t v = -1;
  if (v < 0) {
    const char* e = getenv("LA_PREFETCH_DEPTH");
    int32_t d = 0;  // measured: prefetching ahead did not beat the two-stage TMA ring alone
    if (e != nullptr) d = std::max(0, std::min(16, atoi(e)));
    v = d;
  }
  return v;
}

}  // namespace

bool encode_map(CUtensorMap* map, const void* base, int64_t B, int64_t N, int64_t H) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (encode == nullptr) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr) {
      return false;
    }
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2,
                                 static_cast<cuuint64_t>(H) * D * 2,
                                 static_cast<cuuint64_t>(N) * H * D * 2};
  const cuuint32_t box[4] = {64, 1, C, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base),
                            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

SegmentPlan plan_segments(int64_t B, int64_t N, int64_t H, int requested_segments, int num_sms,
                          int chunk) {
  SegmentPlan pl{};
  pl.n_chunks = (N + C - 1) / C;
  const int64_t bh = B * H;
  int64_t want;
  if (requested_segments > 0) {
    want = requested_segments;
  } else if (2 * bh > static_cast<int64_t>(num_sms)) {
    // More than half the SMs already hold a whole sequence: splitting cannot shorten the
    // longest unit without adding the local-state pass to every split sequence.
    want = 1;
  } else {
    // One wave of equal segments, one per SM.  All segments then finish together: each runs
    // its local-state pass, the scan hands every segment its incoming state right after, and
    // each runs its output pass (the last segment has no local-state pass but waits for the
    // scan instead).  Segments keep at least 4 chunks.
    want = std::max<int64_t>(1, std::min<int64_t>(num_sms / bh, pl.n_chunks / 4));
  }
  want = std::max<int64_t>(1, std::min<int64_t>(want, pl.n_chunks));
  pl.seg_chunks = (pl.n_chunks + want - 1) / want;
  if (chunk == 256) pl.seg_chunks += pl.seg_chunks & 1;  // whole 256-token chunks per segment
  pl.segments = (pl.n_chunks + pl.seg_chunks - 1) / pl.seg_chunks;
  pl.units = pl.segments * bh;
  return pl;
}

namespace {

// Relative time of a local-state tile (K and V only) against an output tile (Q, K, V in, O out).
// LA_BALANCE_LOCAL_COST (percent) overrides it: a tuning knob; every value computes the same
// result.
double local_pass_cost() {
  static double v = -1.0;
  if (v < 0.0) {
    double c = 0.46;
    if (const char* e = getenv("LA_BALANCE_LOCAL_COST")) c = std::max(0, std::min(300, atoi(e))) / 100.0;
    v = c;
  }
  return v;
}

// Finish time, in output-tile units, of the range [a, b) of the head-major tile list (sequences
// of n tiles), and the time its cut last piece publishes its outgoing state (-1: no cut).  The
// range runs the cut piece's local-state pass (rho per tile), that piece's outputs, the outputs
// of the whole sequences inside it and last the piece that continues the previous range's cut,
// which cannot start before that cut was published at pub_prev.  A range that is one piece cut
// at both ends publishes only once its own local pass and its predecessor's publication are done.
struct RangeTiming {
  double finish, pub;
};
RangeTiming range_timing(int64_t a, int64_t b, int64_t n, double rho, double pub_prev) {
  const int64_t sa = a / n, sb = (b - 1) / n;
  const bool cont = a % n != 0;  // the first piece continues the previous range's cut
  const bool cut = b % n != 0;   // the last piece is cut off from the rest of its sequence
  RangeTiming t{0.0, -1.0};
  if (sa == sb && cont && cut) {  // one piece, cut at both ends
    const double y = static_cast<double>(b - a);
    t.pub = std::max(rho * y, pub_prev);
    t.finish = t.pub + y;
    return t;
  }
  const double x = cont ? static_cast<double>(std::min(b, (sa + 1) * n) - a) : 0.0;
  const double y = cut ? static_cast<double>(b - std::max(a, sb * n)) : 0.0;
  const double m = static_cast<double>(b - a) - x - y;
  double time = (1.0 + rho) * y + m;
  if (cut) t.pub = rho * y;
  if (cont) time = std::max(time, pub_prev) + x;
  t.finish = time;
  return t;
}

// The furthest end b > a of a range that finishes by `cap`; ends at sequence boundaries are
// considered first (no local pass), then ends inside the next sequence (binary search; the
// finish time grows with the cut piece).  Inside a sequence the end falls on an even tile offset
// when `pair` (256-token chunks).
int64_t range_end(int64_t a, double cap, int64_t n, int64_t total, double rho, bool pair,
                  double pub_prev) {
  int64_t best = a;
  // whole sequences: ends at seq_end(a), seq_end(a) + n, ...
  int64_t e = (a / n + 1) * n;
  while (e <= total && range_timing(a, e, n, rho, pub_prev).finish <= cap) {
    best = e;
    e += n;
  }
  // an end inside the sequence that starts at q0
  const int64_t q0 = best > a ? best : (a / n) * n;
  if (q0 < total) {
    int64_t lo = std::max(a, q0), hi = std::min(q0 + n - 1, total);  // candidate ends (lo, hi]
    while (hi > lo) {
      int64_t mid = lo + (hi - lo + 1) / 2;
      if (pair) mid = q0 + ((mid - q0) & ~int64_t(1));
      if (mid <= lo) break;
      if (range_timing(a, mid, n, rho, pub_prev).finish <= cap)
        lo = mid;
      else
        hi = mid - 1;
    }
    if (pair) lo = q0 + ((lo - q0) & ~int64_t(1));
    if (lo > std::max(a, q0) && lo > best) best = lo;
  }
  return std::min(best, total);
}

}  // namespace

BalancedPlan plan_balanced(int64_t B, int64_t N, int64_t H, int num_sms, int chunk) {
  BalancedPlan pl{};
  const int64_t n = (N + C - 1) / C;
  const int64_t total = B * H * n;
  pl.seq_tiles = static_cast<int32_t>(n);
  pl.total_tiles = total;
  const int64_t r_max = std::max<int64_t>(
      1, std::min<int64_t>({static_cast<int64_t>(std::max(num_sms, 1)), int64_t(kMaxRanges), total}));
  const double rho = local_pass_cost();
  const bool pair = chunk == 256;
  // greedy cut with a finish-time cap; true when it covers every tile in r_max ranges or fewer
  auto cut = [&](double cap, BalancedPlan* out) -> bool {
    int64_t a = 0;
    int32_t r = 0;
    double pub_prev = 0.0;
    if (out) out->start[0] = 0;
    while (a < total) {
      if (r >= r_max) return false;
      int64_t b = range_end(a, cap, n, total, rho, pair, pub_prev);
      if (b <= a) {  // always make progress: one tile (two inside a sequence for pairs)
        const int64_t se = (a / n + 1) * n;
        b = std::min(se, a + (pair ? 2 : 1));
      }
      const RangeTiming t = range_timing(a, b, n, rho, pub_prev);
      pub_prev = t.pub >= 0.0 ? t.pub : 0.0;
      a = b;
      ++r;
      if (out) out->start[r] = static_cast<int32_t>(a);
    }
    if (out) out->n_ranges = r;
    return true;
  };
  double lo = static_cast<double>(total) / static_cast<double>(r_max);
  double hi = (1.0 + rho) * (lo + static_cast<double>(n)) + 2.0;
  while (!cut(hi, nullptr)) hi *= 2.0;
  for (int it = 0; it < 48 && hi - lo > 0.25; ++it) {
    const double mid = 0.5 * (lo + hi);
    if (cut(mid, nullptr)) hi = mid; else lo = mid;
  }
  cut(hi, &pl);
  pl.makespan = hi;
  return pl;
}

double segments_makespan(const SegmentPlan& plan, int64_t B, int64_t H, int num_sms) {
  const double rho = local_pass_cost();
  const double L = static_cast<double>(plan.seg_chunks);
  if (plan.segments <= 1) {
    // whole sequences handed out dynamically to the CTAs
    const double waves = std::ceil(static_cast<double>(B * H) / std::max(num_sms, 1));
    return waves * static_cast<double>(plan.n_chunks);
  }
  // every segment in one wave: a cut segment runs its local pass and its outputs; the others
  // wait for their predecessor's publication (after its local pass) and run their outputs
  return (1.0 + rho) * L;
}

bool prefer_balanced(int64_t B, int64_t N, int64_t H, int num_sms, int chunk, BalancedPlan* bal,
                     SegmentPlan* seg) {
  *seg = plan_segments(B, N, H, 0, num_sms, chunk);
  *bal = plan_balanced(B, N, H, num_sms, chunk);
  // Short ranges pay each unit's pipeline fill and drain, which the model leaves out (measured:
  // the balanced plan loses at 14 tiles per range and gains about 8 % at 886), so they stay on
  // equal segments.
  const double tiles_per_range =
      static_cast<double>(bal->total_tiles) / std::max(bal->n_ranges, 1);
  return tiles_per_range >= 64.0 &&
         bal->makespan < 0.9 * segments_makespan(*seg, B, H, num_sms);
}

size_t balanced_workspace_bytes(const BalancedPlan& plan) {
  const size_t flags = (static_cast<size_t>(plan.n_ranges) * 4 + 255) / 256 * 256;
  return 256 + flags + static_cast<size_t>(plan.n_ranges) * D * D * sizeof(float);
}

WorkspaceLayout workspace_layout(int64_t B, int64_t H, const SegmentPlan& plan) {
  WorkspaceLayout w{};
  const int64_t bh = B * H;
  w.header_bytes = 256;
  w.flags_off = 256;
  w.flags_bytes = plan.segments > 1 ? static_cast<size_t>(bh) * 2 * sizeof(uint32_t) : 0;
  w.ring_off = (w.flags_off + w.flags_bytes + 255) / 256 * 256;
  w.ring_bytes =
      plan.segments > 1 ? static_cast<size_t>(bh) * 2 * D * D * sizeof(float) : 0;
  w.total = w.ring_off + w.ring_bytes;
  return w;
}

namespace {

// Shared launch: fills the parameters common to both forms and runs the kernel.  With
// clear_header the counter, status word and scan flags are first cleared on `stream`.
cudaError_t launch_common(const PrefillArgs& a, Params& prm, uint8_t* ws,
                          const WorkspaceLayout& wl, int64_t units, cudaStream_t stream,
                          int num_sms, bool clear_header = true) {
  // the kernel instance for this chunk length and epilogue
  void (*kernel)(Params) = nullptr;
  const bool gated = a.gate != nullptr;
  switch (a.chunk) {
    case 64:
      kernel = gated ? chunked_prefill_kernel<true, kC64> : chunked_prefill_kernel<false, kC64>;
      break;
    case 128:
      kernel = gated ? chunked_prefill_kernel<true, kC128> : chunked_prefill_kernel<false, kC128>;
      break;
    case 256:
      kernel = gated ? chunked_prefill_kernel<true, kC256> : chunked_prefill_kernel<false, kC256>;
      break;
    default:
      return cudaErrorInvalidValue;
  }
  const bool qk = a.qk_positions != nullptr;
  if (qk) {
    // the in-tile QK norm + RoPE instance: C = 128, plain output, 16-row chunk pairs
    if (a.chunk != 128 || gated || a.qk_gamma_q == nullptr || a.qk_gamma_k == nullptr ||
        a.qk_rotary_dim < 16 || a.qk_rotary_dim > D || a.qk_rotary_dim % 16 != 0)
      return cudaErrorInvalidValue;
    kernel = chunked_prefill_kernel<false, kC128, true>;
  }
  // set on every call: cheap, safe from any host thread, and it survives a context reset
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemAlloc));
  if (e != cudaSuccess) return e;
  // counter, status and scan flags start at zero for every call
  if (clear_header) {
    e = cudaMemsetAsync(ws, 0, wl.flags_off + wl.flags_bytes, stream);
    if (e != cudaSuccess) return e;
  }
  if (units == 0) return cudaSuccess;
  // (an all-empty packed batch has N = 0 tokens: its units load nothing, but a map needs N >= 1)
  const int64_t n_map = std::max<int64_t>(a.N, 1);
  if (!encode_map(&prm.tm_q, a.q, a.B, n_map, a.H) || !encode_map(&prm.tm_k, a.k, a.B, n_map, a.H) ||
      !encode_map(&prm.tm_v, a.v, a.B, n_map, a.H)) {
    return cudaErrorInvalidValue;
  }
  prm.out = static_cast<__nv_bfloat16*>(a.out);
  prm.slopes = a.slopes;
  prm.state_out = a.state_out;
  prm.state_in = a.state_in;
  prm.gate = static_cast<const __nv_bfloat16*>(a.gate);
  if (a.gate != nullptr && !encode_map(&prm.tm_gate, a.gate, a.B, n_map, a.H))
    return cudaErrorInvalidValue;
  prm.gamma = a.gamma;
  prm.eps = a.eps;
  prm.qk_gamma_q = a.qk_gamma_q;
  prm.qk_gamma_k = a.qk_gamma_k;
  prm.qk_positions = a.qk_positions;
  prm.qk_rotary_dim = a.qk_rotary_dim;
  prm.qk_eps = a.qk_eps;
  for (int f = 0; f < 64; ++f) prm.qk_inv_freq[f] = a.qk_inv_freq[f];
  prm.counter = reinterpret_cast<uint32_t*>(ws + kWsCounter);
  prm.status = reinterpret_cast<int32_t*>(ws + kWsStatus);
  prm.flags = reinterpret_cast<uint32_t*>(ws + wl.flags_off);
  prm.ring = reinterpret_cast<float*>(ws + wl.ring_off);
  prm.N = a.N;
  prm.H = a.H;
  prm.units = units;
  prm.timeout_ns = a.wait_limit_ns;
  prm.withhold_segment = a.withhold_segment;
  prm.prefetch_depth = prefetch_depth();
  const int64_t grid = std::min<int64_t>(units, num_sms);
  kernel<<<static_cast<unsigned>(grid), kThreads, kSmemAlloc, stream>>>(prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunked_prefill(const PrefillArgs& a, const SegmentPlan& plan,
                                   void* workspace, cudaStream_t stream, int num_sms) {
  Params prm{};
  prm.unit_table = nullptr;
  prm.n_ranges = 0;
  prm.BH = a.B * a.H;
  prm.n_chunks = plan.n_chunks;
  prm.seg_chunks = plan.seg_chunks;
  prm.segments = plan.segments;
  return launch_common(a, prm, static_cast<uint8_t*>(workspace), workspace_layout(a.B, a.H, plan),
                       plan.units, stream, num_sms);
}

cudaError_t launch_chunked_prefill_balanced(const PrefillArgs& a, const BalancedPlan& plan,
                                            void* workspace, cudaStream_t stream, int num_sms) {
  // the plan must cover the tile list with increasing range starts; inside a sequence a range
  // starts on an even tile for 256-token chunks (checked here, since the kernel trusts it)
  if (plan.n_ranges < 1 || plan.n_ranges > kMaxRanges || plan.start[0] != 0 ||
      plan.start[plan.n_ranges] != plan.total_tiles || plan.seq_tiles < 1)
    return cudaErrorInvalidValue;
  for (int r = 0; r < plan.n_ranges; ++r) {
    if (plan.start[r + 1] <= plan.start[r]) return cudaErrorInvalidValue;
    if (a.chunk == 256 && (plan.start[r] % plan.seq_tiles) % 2 != 0) return cudaErrorInvalidValue;
  }
  Params prm{};
  prm.unit_table = nullptr;
  prm.BH = a.B * a.H;
  prm.n_chunks = plan.seq_tiles;
  prm.n_ranges = plan.n_ranges;
  for (int r = 0; r <= plan.n_ranges; ++r) prm.range_start[r] = plan.start[r];
  WorkspaceLayout wl{};
  wl.header_bytes = 256;
  wl.flags_off = 256;
  wl.flags_bytes = (static_cast<size_t>(plan.n_ranges) * 4 + 255) / 256 * 256;
  wl.ring_off = wl.flags_off + wl.flags_bytes;
  wl.ring_bytes = static_cast<size_t>(plan.n_ranges) * D * D * sizeof(float);
  wl.total = wl.ring_off + wl.ring_bytes;
  // one CTA per range at most; a CTA that finishes its range takes the next untaken one
  return launch_common(a, prm, static_cast<uint8_t*>(workspace), wl, plan.n_ranges, stream,
                       num_sms);
}

// ---------------------------------------------------------------------------------------------
// Variable-length plan, built on the device from cu_seqlens by one block of 1024 threads.
// ---------------------------------------------------------------------------------------------
namespace {

constexpr int kPlanThreads = 1024;
constexpr int kPlanSortMax = 8192;  // sequences ordered longest first up to this count

struct PlanArgs {
  const int64_t* cu;
  int64_t n_seqs, T, H;
  int32_t requested, num_sms;
  int32_t pair;  // 256-token chunks: segments hold whole chunks (an even number of tiles)
  int64_t unit_cap, slot_cap;
  WorkUnit* table;  // null: only check cu (recurrent path)
  int32_t* status;
  int32_t* units_out;
};

// Segments of a sequence of n_chunks chunks: the fixed-length rule of plan_segments, with B*H
// counted over the non-empty sequences, so equal lengths plan exactly as la_prefill does.  An
// empty sequence is one unit without chunks.
__device__ __forceinline__ int64_t seg_chunks_of(int64_t n_chunks, int64_t nonempty_heads,
                                                 int32_t requested, int32_t sms, bool pair) {
  int64_t want;
  if (requested > 0) {
    want = requested;
  } else if (2 * nonempty_heads > sms) {
    want = 1;
  } else {
    want = max(int64_t(1), min(int64_t(sms) / nonempty_heads, n_chunks / 4));
  }
  want = max(int64_t(1), min(want, n_chunks));
  int64_t seg_chunks = (n_chunks + want - 1) / want;
  if (pair) seg_chunks += seg_chunks & 1;  // whole 256-token chunks per segment
  return seg_chunks;
}

__device__ __forceinline__ int64_t segments_of(int64_t n_chunks, int64_t nonempty_heads,
                                               int32_t requested, int32_t sms, bool pair) {
  if (n_chunks == 0) return 1;
  const int64_t seg_chunks = seg_chunks_of(n_chunks, nonempty_heads, requested, sms, pair);
  return (n_chunks + seg_chunks - 1) / seg_chunks;
}

// Exclusive block-wide prefix sum of one int64 per thread; also returns the block total.
__device__ int64_t block_exclusive_scan(int64_t x, int64_t* total, int64_t* sh /* [33] */) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int64_t incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sh[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int64_t v = lane < (kPlanThreads / 32) ? sh[lane] : 0;
    int64_t vi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, vi, o);
      if (lane >= o) vi += y;
    }
    sh[lane] = vi - v;  // exclusive prefix of the warp totals
    if (lane == 31) sh[32] = vi;
  }
  __syncthreads();
  const int64_t r = sh[w] + incl - x;
  *total = sh[32];
  __syncthreads();
  return r;
}

// Sorts keys[0, n) ascending in shared memory (bitonic network; n a power of two).
__device__ void block_bitonic_sort(unsigned long long* keys, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int i = threadIdx.x; i < n / 2; i += kPlanThreads) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const unsigned long long x = keys[lo], y = keys[hi];
        if ((x > y) == up) {
          keys[lo] = y;
          keys[hi] = x;
        }
      }
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kPlanThreads) plan_varlen_kernel(const PlanArgs a) {
  extern __shared__ unsigned long long order[];  // [n_pad]: (longest first, then index) keys
  __shared__ int64_t sh[33];
  __shared__ int bad;
  __shared__ unsigned long long nonempty, max_seg;
  if (threadIdx.x == 0) {
    bad = (a.cu[0] != 0 || a.cu[a.n_seqs] != a.T) ? 1 : 0;
    nonempty = 0;
    max_seg = 0;
  }
  __syncthreads();
  // check cu and count the non-empty sequences
  unsigned long long my_nonempty = 0;
  for (int64_t s = threadIdx.x; s < a.n_seqs; s += kPlanThreads) {
    const int64_t x0 = a.cu[s], x1 = a.cu[s + 1];
    if (x1 < x0 || x0 < 0 || x1 > a.T) bad = 1;
    my_nonempty += x1 > x0 ? 1 : 0;
  }
  atomicAdd(&nonempty, my_nonempty);
  __syncthreads();
  if (bad) {
    if (threadIdx.x == 0) {
      *a.status = -2;  // LA_ERR_SHAPE
      *a.units_out = 0;
    }
    return;
  }
  if (a.table == nullptr) {
    if (threadIdx.x == 0) *a.units_out = 0;
    return;
  }
  const int64_t nonempty_heads = max(int64_t(1), static_cast<int64_t>(nonempty)) * a.H;
  unsigned long long my_max = 0;
  for (int64_t s = threadIdx.x; s < a.n_seqs; s += kPlanThreads) {
    const int64_t nch = (a.cu[s + 1] - a.cu[s] + C - 1) / C;
    my_max = max(my_max, static_cast<unsigned long long>(segments_of(
                             nch, nonempty_heads, a.requested, a.num_sms, a.pair != 0)));
  }
  atomicMax(&max_seg, my_max);
  __syncthreads();
  const int64_t levels = static_cast<int64_t>(max_seg);

  // Within a level, sequences go longest first (ties by index), so the persistent CTAs, which
  // take units in table order, start the long units early and finish together.  Beyond
  // kPlanSortMax sequences the table keeps sequence order.
  const bool sorted = a.n_seqs <= kPlanSortMax;
  int n_pad = 1;
  while (n_pad < a.n_seqs) n_pad <<= 1;
  if (sorted) {
    for (int64_t p = threadIdx.x; p < n_pad; p += kPlanThreads) {
      if (p < a.n_seqs) {
        const int64_t nch = (a.cu[p + 1] - a.cu[p] + C - 1) / C;
        order[p] = (static_cast<unsigned long long>(0x7fffffff - nch) << 32) |
                   static_cast<unsigned long long>(p);
      } else {
        order[p] = ~0ull;  // padding sorts last
      }
    }
    block_bitonic_sort(order, n_pad);
  }

  // Units go out segment-major: all units of segment k precede those of segment k + 1, so a
  // unit only ever waits on a unit taken before it.  Within a level: sequences in order, H heads
  // each.  Sequences with more than one segment get a ring slot, in sequence order.
  int64_t base = 0;
  int status = 0;
  for (int64_t k = 0; k < levels; ++k) {
    int64_t slot_base = 0;
    for (int64_t s0 = 0; s0 < a.n_seqs; s0 += kPlanThreads) {
      const int64_t p = s0 + threadIdx.x;  // position in the level's order
      const int64_t s = p < a.n_seqs ? (sorted ? static_cast<int64_t>(order[p] & 0xffffffffull) : p)
                                     : a.n_seqs;
      int64_t len = 0, nch = 0, segs = 0;
      if (s < a.n_seqs) {
        len = a.cu[s + 1] - a.cu[s];
        nch = (len + C - 1) / C;
        segs = segments_of(nch, nonempty_heads, a.requested, a.num_sms, a.pair != 0);
      }
      const int64_t active = (s < a.n_seqs && k < segs) ? 1 : 0;
      const int64_t multi = (s < a.n_seqs && segs > 1) ? 1 : 0;
      int64_t n_active = 0, n_multi = 0;
      const int64_t pos = block_exclusive_scan(active, &n_active, sh);
      const int64_t mpos = block_exclusive_scan(multi, &n_multi, sh);
      if (active) {
        const int64_t u0 = base + pos * a.H;
        const int64_t slot = slot_base + mpos;
        if (u0 + a.H > a.unit_cap || (multi && slot >= a.slot_cap)) {
          status = -6;  // LA_ERR_WORKSPACE (cannot happen with the host's capacities)
        } else {
          const int64_t seg_chunks =
              nch > 0 ? seg_chunks_of(nch, nonempty_heads, a.requested, a.num_sms, a.pair != 0) : 0;
          const int64_t c0 = k * seg_chunks;
          const int64_t nc = nch > 0 ? min(seg_chunks, nch - c0) : 0;
          const int64_t end = min(len, (c0 + nc) * C);
          WorkUnit w;
          w.seg = static_cast<int32_t>(k);
          w.c0 = static_cast<int32_t>(c0);
          w.nc = static_cast<int32_t>(nc);
          w.len = static_cast<int32_t>(end - c0 * C);
          w.flags = (k + 1 < segs ? 1 : 0) | (k + 1 == segs ? 2 : 0);
          w.b = 0;
          w.tok0 = static_cast<int32_t>(a.cu[s]);
          // a sequence cut into segments has a two-slot state ring per head: segment k
          // publishes into slot k & 1 with flag value k + 1
          w.in_val = static_cast<int32_t>(k);
          w.pub_val = static_cast<int32_t>(k + 1);
          for (int64_t h = 0; h < a.H; ++h) {
            w.bh = static_cast<int32_t>(s * a.H + h);
            const int64_t rs = slot * a.H + h;
            w.slot = multi ? static_cast<int32_t>(rs * 2 + (k & 1)) : -1;
            w.in_slot = (multi && k > 0) ? static_cast<int32_t>(rs * 2 + ((k - 1) & 1)) : -1;
            a.table[u0 + h] = w;
          }
        }
      }
      base += n_active * a.H;
      slot_base += n_multi;
    }
  }
  if (status != 0) atomicExch(a.status, status);
  __syncthreads();
  if (threadIdx.x == 0) *a.units_out = static_cast<int32_t>(min(base, a.unit_cap));
}

}  // namespace

VarlenWorkspace varlen_workspace_layout(int64_t T, int64_t n_seqs, int64_t H,
                                        int requested_segments, int num_sms, bool tensor_path) {
  VarlenWorkspace w{};
  w.unit_cap = tensor_path ? H * (n_seqs + (T + C - 1) / C) : 0;
  // Sequences cut into segments need a ring slot.  Automatic plans cut only when the non-empty
  // sequences times H fit in half the SMs; an explicit request may cut every sequence.
  if (!tensor_path || requested_segments == 1) {
    w.slot_cap = 0;
  } else if (requested_segments > 1) {
    w.slot_cap = n_seqs;
  } else {
    w.slot_cap = std::min<int64_t>(n_seqs, std::max(0, num_sms) / std::max<int64_t>(1, 2 * H));
  }
  SegmentPlan sp{};
  sp.segments = w.slot_cap > 0 ? 2 : 1;  // only "more than one segment" matters for the size
  w.base = workspace_layout(w.slot_cap, H, sp);
  w.table_off = (w.base.total + 255) / 256 * 256;
  w.total = w.table_off + static_cast<size_t>(w.unit_cap) * sizeof(WorkUnit);
  return w;
}

cudaError_t launch_prefill_varlen(const PrefillArgs& a, const VarlenWorkspace& layout,
                                  void* workspace, int requested_segments, bool tensor_path,
                                  cudaStream_t stream, int num_sms) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaError_t e = cudaMemsetAsync(ws, 0, layout.base.flags_off + layout.base.flags_bytes, stream);
  if (e != cudaSuccess) return e;
  PlanArgs pa{};
  pa.cu = a.cu_dev;
  pa.n_seqs = a.n_seqs;
  pa.T = a.N;
  pa.H = a.H;
  pa.requested = requested_segments;
  pa.num_sms = num_sms;
  pa.pair = a.chunk == 256 ? 1 : 0;
  pa.unit_cap = layout.unit_cap;
  pa.slot_cap = layout.slot_cap;
  pa.table = tensor_path ? reinterpret_cast<WorkUnit*>(ws + layout.table_off) : nullptr;
  pa.status = reinterpret_cast<int32_t*>(ws + kWsStatus);
  pa.units_out = reinterpret_cast<int32_t*>(ws + kWsUnits);
  size_t sort_bytes = 0;
  if (a.n_seqs <= kPlanSortMax) {
    int64_t n_pad = 1;
    while (n_pad < a.n_seqs) n_pad <<= 1;
    sort_bytes = static_cast<size_t>(n_pad) * sizeof(unsigned long long);
  }
  e = cudaFuncSetAttribute(plan_varlen_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kPlanSortMax * sizeof(unsigned long long)));
  if (e != cudaSuccess) return e;
  plan_varlen_kernel<<<1, kPlanThreads, sort_bytes, stream>>>(pa);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (!tensor_path) {
    PrefillArgs r = a;
    r.status = pa.status;
    return launch_recurrent_prefill(r, stream);
  }
  Params prm{};
  prm.unit_table = pa.table;
  prm.units_dev = pa.units_out;
  prm.BH = a.n_seqs * a.H;
  // The plan's unit count is only known on the device: launch for the capacity (one CTA per SM
  // at most); CTAs that find no unit exit.
  return launch_common(a, prm, ws, layout.base, layout.unit_cap, stream, num_sms,
                       /*clear_header=*/false);
}

}  // namespace la
