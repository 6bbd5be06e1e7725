// cpattn_internal.h -- launch plans shared by the host planner (cpattn_api.cu)
// and the kernels.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace cpattn {

// ---------------------------------------------------------------- attention
//
// The attention kernel sees every Q/K/V tensor as a 3-D array [rows, H, D]
// (D contiguous).  A full BSHD tensor has rows = B*S with row = b*S + s; the
// rank-buffer layouts used by the Ulysses/unified flows are also [rows, H, D]
// with other row formulas.  Work is described with row ranges:
//   problem : one (Q, K, V, out, lse) tensor set with its head count H,
//   group   : (problem, batch index b) -- the set of Q segments sharing
//             K/V row numbering; units are ordered head-major inside it,
//   segment : a range of Q rows (one sequence shard) with its list of K/V
//             row ranges, visited in order (ring order for ring attention),
//   kv      : a K/V row range (one chunk).
// Segments and K/V ranges carry the sequence position of their first row; a
// causal plan masks by positions (no mask tensor), and a unit never walks a
// K/V tile that lies wholly after its last query.
// One CTA processes one unit = (group, head, segment, pair of 128-row Q tiles).

constexpr int kMaxProblems = 8;
constexpr int kMaxRanks = 64;   // sequence / head ranks of a permutation or an output map
constexpr int kMaxGroups = 64;
constexpr int kMaxSegs = 128;
constexpr int kMaxKV = 512;
constexpr int kQTile = 128;     // rows per Q tile (one TMEM lane per row)
constexpr int kKVTile = 128;    // keys per K/V tile
constexpr int kQTilesPerCTA = 2;

struct alignas(64) AttnProblem {
  CUtensorMap tm_q, tm_k, tm_v;   // 3-D maps over [rows, H, D] bf16, box {64, 1, 128}, 128B swizzle
  void *out;                      // [rows, H, D] bf16 or float32 (same rows as Q)
  float *lse;                     // may be null; index b*lse_b + (h + lse_h0)*lse_h + (s - lse_pos0)
  const float *prev;              // null, or a previous partial state to merge into: float32 [rows, H, D]
                                  // (same rows as Q, normalised over its keys) with its LSE read from
                                  // `lse` before it is overwritten; may alias `out` when out is float32
  long long lse_b;
  long long lse_h;
  int lse_h0;
  int lse_pos0;                   // sequence position of LSE column 0
  int H;
  // Where a row of out goes (batch b, sequence position s, head h):
  //   out_mode 0: the row of Q (out has Q's layout);
  //   out_mode 1: the sequence-side rank buffers (B, len_r, out_H, D) of the
  //               Ulysses exchange, row out_B*off_r + b*len_r + (s - off_r),
  //               head out_h0 + h (the second all-to-all, fused);
  //   out_mode 2: a full (B, out_S, out_H, D) tensor, row b*out_S + s, head
  //               out_h0 + h.
  int out_mode;
  int out_H, out_h0, out_B, out_S;
  int out_nseq;
  int out_seq_off[kMaxRanks + 1];
};

struct AttnGroup {
  int prob;
  int b;
  int seg_first;
  int seg_count;
  int tiles_per_head;   // sum over the group's segments of their CTA tile pairs
  int unit_base;        // first unit (blockIdx) of this group
  int head_block;       // causal plans: heads whose units interleave pair by pair
};

struct AttnSeg {
  int row0;       // first Q row
  int nrows;      // Q rows in the segment
  int s0;         // sequence position of row0 (for the LSE index)
  int kv_first;   // index into kv[]
  int kv_count;   // number of K/V ranges (0: empty -> out 0, lse -inf)
  int tile_base;  // first tile pair of this segment within the group's head
  int split;      // 1: a lone Q tile whose K/V tiles are split between the two slots
  // q1_rows > 0: a lone tile of rows [row0, row0 + nrows) paired with another
  // shard's lone tile (q1_rows rows from q1_row0, position q1_s0) in slot 1;
  // both walk this segment's K/V list (no causal mask, so both see every key).
  int q1_row0, q1_s0, q1_rows;
};

struct AttnKV {
  int row0;
  int nrows;
  int s0;         // sequence position of row0 (for the causal mask)
};

struct AttnParams {
  AttnProblem prob[kMaxProblems];
  AttnGroup group[kMaxGroups];
  AttnSeg seg[kMaxSegs];
  AttnKV kv[kMaxKV];
  int num_groups;
  int total_units;
  int causal;                    // 1: key visible to a query iff its position <= the query's
  float scale_log2;              // D**-0.5 * log2(e)
  unsigned long long timeout_ns; // bound for every pipeline wait
};

// Launches the attention kernel for a plan.  D in {64, 128}; out_f32 selects
// float32 partial outputs (ring step) instead of bf16.
cudaError_t launch_attention(const AttnParams &p, int D, bool out_f32, cudaStream_t stream);

// ---------------------------------------------------------------- backward
// Gradient of attention.  A problem is one (Q, K, V, dO) tensor set laid out
// [B, S, H, D] (rows = B*S) with its own head count: the full tensors, or one
// head rank's head-side buffer of the Ulysses flow.
struct alignas(64) BwdProblem {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;   // 3-D maps over [rows, H, D] bf16, box {64, 1, 128}, 128B swizzle
  const float *lse;                      // natural log, from the forward: index b*lse_b + (h + lse_h0)*lse_h + s
  long long lse_b;
  long long lse_h;
  int lse_h0;
  int H;                                 // heads of the tensors
  int h0, nh;                            // the heads [h0, h0 + nh) that this problem's units cover
  float *delta;                          // [B, H, S] rowsum(dO * O) of this problem
  void *dq, *dk, *dv;                    // bf16 gradients, rows placed by the output map below
  // Where a gradient row goes (batch b, sequence position s, head h):
  //   out_mode 0: [B, S, H, D], the inputs' layout;
  //   out_mode 1: the sequence-side rank buffers (B, len_r, out_H, D) of the
  //               Ulysses exchange, row B*off_r + b*len_r + (s - off_r), head
  //               out_h0 + h (the backward flow's second all-to-all, fused).
  int out_mode;
  int out_H, out_h0;
  int out_nseq;
  int out_seq_off[kMaxRanks + 1];
  // dS tiles of heads [h0, h0 + nh): written by the dK/dV kernel, read by the
  // dQ GEMM (null: the dQ kernel recomputes S and dP instead).  Tile (b, h,
  // q tile, k tile) at bwd_ds_tile_index * kBwdDsTileBytes, each tile
  // [4 quarters of 32 keys][16 groups of 8 queries][32 keys][8 queries] bf16;
  // 256-byte aligned.
  unsigned char *ds;
  int unit_base;                         // first unit (blockIdx) of this problem
};
constexpr int kBwdDsTileBytes = 128 * 128 * 2;
// dS tiles per (b, h): every (q tile, k tile) pair, or under the causal mask
// only the pairs with kt <= qt (the dK/dV kernel walks no others).  A Q tile's
// k tiles are consecutive either way.
__host__ __device__ inline long long bwd_ds_tiles_per_head(int nt, bool causal) {
  return causal ? static_cast<long long>(nt) * (nt + 1) / 2 : static_cast<long long>(nt) * nt;
}
__host__ __device__ inline long long bwd_ds_tile_index(int b, int hl, int nh, int nt, int qt, int kt, bool causal) {
  const long long within = causal ? static_cast<long long>(qt) * (qt + 1) / 2 + kt : static_cast<long long>(qt) * nt + kt;
  return (static_cast<long long>(b) * nh + hl) * bwd_ds_tiles_per_head(nt, causal) + within;
}
struct BwdParams {
  BwdProblem prob[kMaxProblems];
  int n_prob;
  int B, S;
  int causal;
  float scale_log2;                      // D**-0.5 * log2(e)
  float scale;                           // D**-0.5
  unsigned long long timeout_ns;
};
// Delta = rowsum(dO * O) over [B, S, H, D] tensors into delta[B, H, S].
cudaError_t launch_bwd_delta(const void *out, const void *dout, float *delta, int B, int S, int H, int D,
                             cudaStream_t stream);
// The gradient kernels over every problem of p (Delta already computed): with
// dS tiles (every problem's ds set) the dK/dV kernel stores dS and the dQ
// GEMM follows; without, the dQ and dK/dV kernels.
cudaError_t launch_bwd_kernels(const BwdParams &p, int D, cudaStream_t stream);

// ---------------------------------------------------------------- LSE merge
struct MergeParams {
  const float *part_out;  // P x [B, S, H, D]
  const float *part_lse;  // P x [B, H, S]
  float *out_f32;         // may be null
  __nv_bfloat16 *out_bf16; // may be null
  float *lse_out;         // may be null
  int P, B, H, S, D;
};
cudaError_t launch_lse_merge(const MergeParams &p, cudaStream_t stream);

// ----------------------------------------------------------------- permute
//
// Moves token rows between a sequence-side layout and a head-side layout.
// Every token (b, s) owns one source row of H*D elements on the sequence side;
// on the head side it owns, for every head rank u, a row of H_u*D elements.
//   sequence side row:  seq_mode 0 (full BSHD):     b*S + s
//                       seq_mode 1 (rank buffers):   B*off_r + b*len_r + (s - off_r)
//   head side row in buffer u (groups = outer sequence ranges, one group for
//   plain Ulysses):     B*goff_i + b*glen_i + (s - goff_i)
//   head buffer u starts at element B*S*hoff_u*D.
constexpr int kMaxHeads = 1024;

constexpr int kMaxPermuteTensors = 3;   // Q, K and V move in one launch

struct PermuteParams {
  const unsigned char *src[kMaxPermuteTensors];
  unsigned char *dst[kMaxPermuteTensors];
  int n_tensors;        // tensors with the same shape and splits, 1..kMaxPermuteTensors
  int B, S, H;
  int row_bytes;        // D * elem_bytes (multiple of 16)
  int direction;        // 0: sequence side -> head side, 1: head side -> sequence side
  int seq_mode;         // 0 full BSHD, 1 rank buffers
  int n_seq;            // sequence ranks (seq_mode 1)
  int seq_off[kMaxRanks + 1];
  int n_groups;         // head-side groups
  int group_off[kMaxRanks + 1];
  int n_head;           // head ranks
  int head_off[kMaxRanks + 1];
};
cudaError_t launch_permute(const PermuteParams &p, cudaStream_t stream);

// ------------------------------------------------------------------- misc
cudaError_t launch_debug_wait(unsigned long long timeout_ns, cudaStream_t stream);
cudaError_t read_and_clear_device_status(unsigned int *code, cudaStream_t stream);

}  // namespace cpattn
