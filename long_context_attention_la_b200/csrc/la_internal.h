// la_internal.h — launch interfaces shared by the C ABI (la_api.cu) and the kernel files.
// Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace la {

enum DType : int { kBF16 = 0, kF32 = 1 };

struct PrefillArgs {
  int64_t B, N, H, d;
  int dtype;
  const void* q;
  const void* k;
  const void* v;
  const float* slopes;
  void* out;
  float* state_out;  // may be null
  // Packed variable-length form (la_prefill_varlen): B = 1, N = total tokens; sequence s owns
  // tokens [cu[s], cu[s+1]) of the device array cu_dev; state_in is an optional fp32
  // [n_seqs, H, d, d] initial state.  n_seqs = 0 means the fixed [B, N] form.  status (device)
  // is the workspace status word, which the recurrent kernel checks before doing any work.
  int64_t n_seqs = 0;
  const int64_t* cu_dev = nullptr;
  const float* state_in = nullptr;
  const int32_t* status = nullptr;
  // Fused grouped RMSNorm + sigmoid gate on the output (tensor path): gate [.., H, d] bf16 and
  // gamma fp32 [H, d]; gate == nullptr stores o itself.
  const void* gate = nullptr;
  const float* gamma = nullptr;
  float eps = 0.f;
  // QK RMSNorm + partial rotate-half RoPE applied to each q and k tile inside the chunked kernel
  // before any product reads it (la_prefill_varlen_qk; tensor path, C = 128, no gate): weights
  // fp32 [d], positions int64 over the token axis (index b * N + n).  Null: q and k as given.
  const float* qk_gamma_q = nullptr;
  const float* qk_gamma_k = nullptr;
  const int64_t* qk_positions = nullptr;
  int32_t qk_rotary_dim = 0;
  float qk_eps = 0.f;
  double qk_inv_freq[64] = {};  // theta^(-2i / rotary_dim), i < rotary_dim / 2
  // Chunk length of the tensor-core path: 64, 128 or 256 (the 128-token tile is fixed).
  int32_t chunk = 128;
  // Failure injection for tests (host-side switch, see la_api.cu): the segment index whose scan
  // flag is never published (-1: none) and the limit of every device wait.
  int32_t withhold_segment = -1;
  uint64_t wait_limit_ns = 2000000000ull;
};

struct DecodeArgs {
  int64_t B, H, d;
  int dtype;
  const void* q;
  const void* k;
  const void* v;
  const float* slopes;
  float* state;
  void* out;
  // multi-token step (la_decode_multi): n_tok tokens per sequence, [B, n_tok, H, d] operands;
  // optional fused grouped RMSNorm + sigmoid gate on each output (gate like out, gamma [H, d])
  int64_t n_tok = 1;
  const void* gate = nullptr;
  const float* gamma = nullptr;
  float eps = 0.f;
};

// n_tok tokens per sequence in one pass over the state (la_decode_multi).
cudaError_t launch_decode_multi(const DecodeArgs& a, cudaStream_t stream);

// Token-by-token CUDA-core prefill (any dtype, d in {64, 128}); one CTA per (b, h).
cudaError_t launch_recurrent_prefill(const PrefillArgs& a, cudaStream_t stream);

// Fused decode step; one CTA per (b, h).
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);

// QK RMSNorm + partial rotate-half RoPE over bf16 q and k rows (la_qknorm.cu).
struct QkNormRopeArgs {
  int64_t T, H, d;                  // tokens, heads, head dim (64 or 128)
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  int64_t q_stride, k_stride;       // elements between consecutive tokens
  const float* gamma_q;             // [d]
  const float* gamma_k;             // [d]
  const int64_t* positions;         // [T]
  __nv_bfloat16* q_out;             // [T, H, d]
  __nv_bfloat16* k_out;             // [T, H, d]
  int32_t rotary_dim;               // multiple of 16, <= d
  float eps;
  double inv_freq[64];              // theta^(-2i / rotary_dim), i < rotary_dim / 2
};
cudaError_t launch_qk_norm_rope(const QkNormRopeArgs& a, cudaStream_t stream);

// Grouped RMSNorm + sigmoid gate over [T, H, d] rows (la_gatenorm.cu).
struct GateNormArgs {
  int64_t T, H, d;
  int dtype;
  const void* o;
  const void* gate;
  const float* gamma;  // [H, d]
  float eps;
  void* y;             // [T, H, d] of dtype, or uint8 E4M3 codes when scales is set
  float* scales;       // FP8 output: fp32 [H, T] block scales (nullptr: y in dtype)
};
cudaError_t launch_gate_norm(const GateNormArgs& a, cudaStream_t stream);

// Fold of per-part states (la_state.cu): S = S_in (or 0); S <- lambda^(L_j) S + h_j for the
// parts j < n_parts in order.  parts: fp32 [n_parts, BH, d, d]; lengths travel by value.
constexpr int kMaxFoldParts = 256;
struct StateFoldArgs {
  int64_t n_parts, BH, H, d;
  const float* parts;
  const float* slopes;
  const float* state_in;  // [BH, d, d] or null
  float* state_out;       // [BH, d, d]; may be state_in
  int64_t lengths[kMaxFoldParts];
};
cudaError_t launch_state_fold(const StateFoldArgs& a, cudaStream_t stream);

// ---------------------------------------------------------------------------------------------
// Chunked tensor-core prefill (bf16, d = 128, chunk C = 128).
// ---------------------------------------------------------------------------------------------
constexpr int kChunk = 128;  // the tile: tokens per TMA load and per M = 128 MMA
constexpr int kHeadDim = 128;
// Chunk lengths the tensor-core prefill supports, and the one it uses when the caller leaves
// the choice to the library.
constexpr int kChunkDefault = 128;
inline bool chunk_supported(int64_t c) { return c == 64 || c == 128 || c == 256; }

// One work unit of the chunked prefill, as the kernel reads it: one piece (a run of consecutive
// tiles) of one (sequence, head).  A unit with kUnitLocal first computes the piece's local state
// h = sum_j lambda^(L-1-j) k_j^T v_j, takes its incoming state S from ring slot in_slot, and
// publishes S_out = lambda^L S + h into ring slot `slot` (flag value pub_val), so that the next
// piece can start before this one's outputs exist; with kUnitNoOutput it stops there.  Every
// other unit runs the output pass from its incoming state.
constexpr int32_t kUnitLocal = 1;     // local-state pass and publish first
constexpr int32_t kUnitFinal = 2;     // last piece of the sequence: write state_out
constexpr int32_t kUnitNoOutput = 4;  // publish only (the outputs are another unit's)
struct WorkUnit {
  int32_t bh;       // state index: sequence * H + head (-1: no more work)
  int32_t seg;      // piece index within the sequence (0: its first piece)
  int32_t c0;       // first tile of the piece, counted from the sequence start
  int32_t nc;       // tiles in the piece (0: an empty sequence, whose state passes through)
  int32_t len;      // tokens in the piece
  int32_t flags;    // kUnitLocal | kUnitFinal | kUnitNoOutput
  int32_t b;        // batch coordinate of the sequence in the [B, N, H, d] tensors
  int32_t tok0;     // token coordinate (along N) of the sequence's first token
  int32_t slot;     // ring slot this unit publishes into (with kUnitLocal)
  int32_t in_slot;  // ring slot of the incoming state (-1: state_in, or zero)
  int32_t in_val;   // flag value that marks in_slot as published
  int32_t pub_val;  // flag value this unit publishes with
};
static_assert(sizeof(WorkUnit) == 48, "WorkUnit is read as three 16-byte words");

// How a prefill is cut into work units: each (b, h) sequence of N tokens becomes `segments`
// segments of `seg_chunks` 128-token tiles (the last may be shorter); one unit = one
// (segment, b, h).  With 256-token chunks a segment holds an even number of tiles, so that no
// chunk straddles two segments.
struct SegmentPlan {
  int64_t n_chunks;    // ceil(N / 128)
  int64_t seg_chunks;  // tiles per segment
  int64_t segments;    // ceil(n_chunks / seg_chunks)
  int64_t units;       // segments * B * H
};

SegmentPlan plan_segments(int64_t B, int64_t N, int64_t H, int requested_segments, int num_sms,
                          int chunk = kChunkDefault);

// Balanced plan (the automatic plan of la_prefill): the B*H sequences' tiles, head-major, are cut
// into at most one range per SM such that every range costs about the same, counting a tile of a
// piece that the range's end cuts off from the rest of its sequence (1 + rho) times, since that
// piece needs a local-state pass.  Range r runs [start[r], start[r+1]) as: the local-state pass of
// its last piece when that piece is cut (publishing into ring slot r), then the outputs of its
// pieces in order.  A range ends at an even tile offset within a sequence for 256-token chunks.
constexpr int kMaxRanges = 256;
struct BalancedPlan {
  int32_t n_ranges;
  int32_t seq_tiles;                  // tiles per sequence
  int64_t total_tiles;                // B * H * seq_tiles
  double makespan;                    // modelled finish time of the slowest range, in tile times
  int32_t start[kMaxRanges + 1];
};
BalancedPlan plan_balanced(int64_t B, int64_t N, int64_t H, int num_sms, int chunk);
// Modelled finish time of the equal-segment plan, in the same units.
double segments_makespan(const SegmentPlan& plan, int64_t B, int64_t H, int num_sms);
// The automatic plan: balanced ranges when their modelled finish time beats the equal-segment
// plan's by a clear margin, else equal segments (sets exactly one of the two outputs).
bool prefer_balanced(int64_t B, int64_t N, int64_t H, int num_sms, int chunk, BalancedPlan* bal,
                     SegmentPlan* seg);
// workspace: header, one scan flag and one d x d fp32 ring slot per range
size_t balanced_workspace_bytes(const BalancedPlan& plan);
cudaError_t launch_chunked_prefill_balanced(const PrefillArgs& a, const BalancedPlan& plan,
                                            void* workspace, cudaStream_t stream, int num_sms);

// Workspace layout of the chunked prefill (byte offsets from the workspace base).
struct WorkspaceLayout {
  size_t header_bytes;  // [0, 256): counter, status
  size_t flags_off;     // uint32 [B*H*2] scan flags
  size_t flags_bytes;
  size_t ring_off;      // float [B*H*2][d*d] segment-state ring (two slots per sequence)
  size_t ring_bytes;
  size_t total;
};

WorkspaceLayout workspace_layout(int64_t B, int64_t H, const SegmentPlan& plan);

// Offsets inside the 256-byte header.
constexpr size_t kWsCounter = 0;   // uint32 work-unit counter
constexpr size_t kWsStatus = 64;   // uint32 device status (0 = ok, else a la_status code)

// Tensor map of a bf16 [B, N, H, 128] activation as 4-D (d, H, N, B) tiles of 64 x 1 x C x 1
// elements with the 128-byte swizzle (two boxes make one [C x 128] tile).
bool encode_map(CUtensorMap* map, const void* base, int64_t B, int64_t N, int64_t H);

// State-only prefill on the tensor cores (la_state.cu): the B*H*n_chunks chunk-loads, head-major,
// in one contiguous range of `width` per CTA (`grid` CTAs).  Workspace: a 256-byte header (status
// word at kWsStatus) and two fp32 d x d partial-state slots per CTA.
struct StatePassPlan {
  int64_t n_chunks;  // ceil(N / C)
  int64_t total;     // B * H * n_chunks
  int64_t width;     // chunk-loads per CTA
  int64_t grid;      // CTAs
  size_t ws_bytes;
};
StatePassPlan plan_state_pass(int64_t B, int64_t N, int64_t H, int num_sms);
cudaError_t launch_state_pass(const PrefillArgs& a, const StatePassPlan& plan, void* workspace,
                              cudaStream_t stream);

cudaError_t launch_chunked_prefill(const PrefillArgs& a, const SegmentPlan& plan,
                                   void* workspace, cudaStream_t stream, int num_sms);

// Variable-length form.  Capacities the host sizes the workspace with (cu_seqlens stays on the
// device, so only its shape is known here): at most H * (n_seqs + ceil(T / C)) work units, and
// ring slots for the sequences that may be cut into segments.
struct VarlenWorkspace {
  int64_t unit_cap;     // work units
  int64_t slot_cap;     // sequences with a state-ring slot (times H heads each)
  WorkspaceLayout base; // header, scan flags and ring for slot_cap * H states
  size_t table_off;     // work-unit table
  size_t total;
};
VarlenWorkspace varlen_workspace_layout(int64_t T, int64_t n_seqs, int64_t H,
                                        int requested_segments, int num_sms, bool tensor_path);
// (the chunk length travels in PrefillArgs::chunk)

// Offset of the device-written work-unit count in the workspace header.
constexpr size_t kWsUnits = 128;

// Clears the header and flags, runs the one-block planning kernel (checks cu, writes the unit
// table and count; with tensor_path false it only checks cu), then the prefill kernel.
cudaError_t launch_prefill_varlen(const PrefillArgs& a, const VarlenWorkspace& layout,
                                  void* workspace, int requested_segments, bool tensor_path,
                                  cudaStream_t stream, int num_sms);

}  // namespace la
