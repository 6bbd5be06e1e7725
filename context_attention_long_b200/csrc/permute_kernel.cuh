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
// head side within each head rank's contiguous block), four vectors in flight
// per lane.  Bit-exact (plain 16-byte loads and stores).
#pragma once

#include "cpattn_internal.h"

namespace cpattn {

constexpr int kPermuteThreads = 256;

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
  __shared__ int s_rank[kMaxHeads];   // head -> head rank
  for (int h = threadIdx.x; h < p.H; h += blockDim.x) s_rank[h] = find_range(p.head_off, p.n_head, h);
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const long long warp_id = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const long long ntok = static_cast<long long>(p.B) * p.S;
  const int vpr = p.row_bytes >> 4;                 // 16-byte vectors per (token, head) row
  const int nvec = p.H * vpr;                       // vectors per token
  const long long seq_row_bytes = static_cast<long long>(p.H) * p.row_bytes;

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

    for (int v0 = lane; v0 < nvec; v0 += 32 * 4) {
      uint4 val[4];
      long long seq_off[4], head_off[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int v = v0 + 32 * k;
        seq_off[k] = -1;
        if (v < nvec) {
          const int h = v / vpr;
          const int w = v - h * vpr;
          const int u = s_rank[h];
          const int hu0 = p.head_off[u];
          const int Hu = p.head_off[u + 1] - hu0;
          seq_off[k] = static_cast<long long>(v) * 16;
          head_off[k] = (static_cast<long long>(p.B) * p.S * hu0 + head_row * Hu + (h - hu0)) * p.row_bytes +
                        static_cast<long long>(w) * 16;
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (seq_off[k] >= 0) {
          if (p.direction == 0) val[k] = __ldcs(reinterpret_cast<const uint4 *>(seq_base + seq_off[k]));
          else val[k] = __ldcs(reinterpret_cast<const uint4 *>(head_buf + head_off[k]));
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (seq_off[k] >= 0) {
          if (p.direction == 0) __stcs(reinterpret_cast<uint4 *>(head_buf + head_off[k]), val[k]);
          else __stcs(reinterpret_cast<uint4 *>(const_cast<unsigned char *>(seq_base) + seq_off[k]), val[k]);
        }
      }
    }
  }
}

}  // namespace cpattn
