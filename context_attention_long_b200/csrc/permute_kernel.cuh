// permute_kernel.cuh -- Ulysses sequence-sharded <-> head-sharded permutation.
//
// diffusers "Context parallelism", "Ulysses Attention": the first all-to-all
// regroups the data so that each GPU holds every token for a subset of the
// heads, the second regroups the results by token; "Ulysses Anything
// Attention" allows uneven sequence and head splits.  Emulated on one GPU, the
// all-to-all is a permutation of token rows:
//     y_{u}[b, s, h - hoff_u, :] = x_{r(s)}[b, s - off_{r(s)}, h, :]
// Each token (b, s) owns one contiguous run of H*D elements on the sequence
// side and, for every head rank u, one contiguous run of H_u*D elements on the
// head side, so the permutation never splits a (token, head) row of D
// elements: every moved unit is a contiguous run of >= 128 bytes and no
// shared-memory transpose is needed to keep both sides coalesced.
//
// Up to three tensors of the same shape (Q, K and V of the first all-to-all)
// move in one launch: every warp takes its tokens of each tensor in turn.
// One warp moves one token per iteration: lanes take consecutive 16-byte
// vectors of the token's H*D run (coalesced on the sequence side, and on the
// head side within each head rank's contiguous block), kPermuteBatch vectors in
// flight per lane; per-head offsets and strides sit in shared memory, so a vector's
// head-side address costs one multiply-add.  Bit-exact (plain 16-byte loads
// and stores).
#pragma once

#include "cpattn_internal.h"

namespace cpattn {

constexpr int kPermuteThreads = 256;
// 16-byte vectors a lane loads before it stores them (8 measured slower: the
// registers they take cost occupancy).
constexpr int kPermuteBatch = 4;

__device__ __forceinline__ int find_range(const int *off, int n, int x) {
  // largest i in [0, n) with off[i] <= x < off[i+1] (empty ranges skipped)
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(kPermuteThreads) permute_kernel(const __grid_constant__ PermuteParams p) {
  // Per head h: the byte offset of its first (token, head) row on the head
  // side, and the stride between consecutive head-side token rows of its
  // head rank (H_u * row_bytes), so that a vector's address is one
  // multiply-add from the token's head-side row index.
  __shared__ long long s_base[kMaxHeads];
  __shared__ int s_stride[kMaxHeads];   // <= kMaxHeads * 1 MiB < 2^31
  for (int h = threadIdx.x; h < p.H; h += blockDim.x) {
    const int u = find_range(p.head_off, p.n_head, h);
    const int hu0 = p.head_off[u];
    const int Hu = p.head_off[u + 1] - hu0;
    s_base[h] = (static_cast<long long>(p.B) * p.S * hu0 + (h - hu0)) * p.row_bytes;
    s_stride[h] = Hu * p.row_bytes;
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const long long warp_id = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const long long ntok = static_cast<long long>(p.B) * p.S;
  const int vpr = p.row_bytes >> 4;                 // 16-byte vectors per (token, head) row
  const int nvec = p.H * vpr;                       // vectors per token
  const long long seq_row_bytes = static_cast<long long>(p.H) * p.row_bytes;
  // Vector v of a token is (head v / vpr, piece v % vpr).  A lane starts at
  // v = lane and steps by 32: the (head, piece) pair advances by (32 / vpr,
  // 32 % vpr) with one carry, so no division runs per vector.
  const int h_lane = lane / vpr, w_lane = lane - h_lane * vpr;
  const int dh = 32 / vpr, dw = 32 - dh * vpr;

  for (int t = 0; t < p.n_tensors; ++t)
  for (long long tok = warp_id; tok < ntok; tok += nwarps) {
    const int b = static_cast<int>(tok / p.S);
    const int s = static_cast<int>(tok - static_cast<long long>(b) * p.S);
    long long seq_row;
    if (p.seq_mode == 0) {
      seq_row = tok;
    } else {
      const int r = find_range(p.seq_off, p.n_seq, s);
      const int off = p.seq_off[r], len = p.seq_off[r + 1] - off;
      seq_row = static_cast<long long>(p.B) * off + static_cast<long long>(b) * len + (s - off);
    }
    const int gi = find_range(p.group_off, p.n_groups, s);
    const int goff = p.group_off[gi], glen = p.group_off[gi + 1] - goff;
    const long long head_row = static_cast<long long>(p.B) * goff + static_cast<long long>(b) * glen + (s - goff);
    const unsigned char *seq_base = (p.direction == 0 ? p.src[t] : p.dst[t]) + seq_row * seq_row_bytes;
    unsigned char *const head_buf = p.direction == 0 ? p.dst[t] : const_cast<unsigned char *>(p.src[t]);

    int h = h_lane, w = w_lane;
    for (int v0 = lane; v0 < nvec; v0 += 32 * kPermuteBatch) {
      uint4 val[kPermuteBatch];
      long long head_off[kPermuteBatch];
#pragma unroll
      for (int k = 0; k < kPermuteBatch; ++k) {
        const int v = v0 + 32 * k;
        if (v < nvec)              // then h < H
          head_off[k] = s_base[h] + head_row * s_stride[h] + static_cast<long long>(w) * 16;
        w += dw;
        h += dh;
        if (w >= vpr) {
          w -= vpr;
          ++h;
        }
      }
#pragma unroll
      for (int k = 0; k < kPermuteBatch; ++k) {
        const int v = v0 + 32 * k;
        if (v < nvec) {
          if (p.direction == 0) val[k] = __ldcs(reinterpret_cast<const uint4 *>(seq_base + static_cast<long long>(v) * 16));
          else val[k] = __ldcs(reinterpret_cast<const uint4 *>(head_buf + head_off[k]));
        }
      }
#pragma unroll
      for (int k = 0; k < kPermuteBatch; ++k) {
        const int v = v0 + 32 * k;
        if (v < nvec) {
          if (p.direction == 0) __stcs(reinterpret_cast<uint4 *>(head_buf + head_off[k]), val[k]);
          else __stcs(reinterpret_cast<uint4 *>(const_cast<unsigned char *>(seq_base) + static_cast<long long>(v) * 16), val[k]);
        }
      }
    }
  }
}

}  // namespace cpattn
