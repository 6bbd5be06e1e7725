// merge_kernel.cuh -- P-way LSE merge of float32 partial attention results.
//
// SGLang "Sequence Parallelism", "Numerics across node boundaries" (the ring's
// partial results are combined by an online-softmax merge) and diffusers
// "parallel", convert_to_fp32 (partial output and LSE in float32):
//   M = max_p LSE_p, LSE = M + ln sum_p e^(LSE_p - M), out = sum_p e^(LSE_p - LSE) out_p
//
// HBM-bound: per (b, h, s) row it reads P*(4D + 4) bytes and writes 4D and/or
// 2D bytes plus 4.  Rows are visited in (b, h, s) order so that the LSE reads
// and writes of a warp are contiguous; each row's D floats are read as float4
// by D/4 lanes (one 512-byte or 256-byte contiguous run per partial).  All P
// loads of a row are issued before any is consumed.
#pragma once

#include "cpattn_internal.h"
#include "cpattn_ptx.cuh"

namespace cpattn {

constexpr int kMergeThreads = 256;

// Rows are visited in (b, h, s) order, grid-stride; each thread carries its
// row's (b, h, s) and advances it by the constant stride, so no row needs a
// division (the stride is split into whole sequences and a remainder once).
struct RowCursor {
  int s, h, b;
  int ds, dh, db;   // stride in rows = ((db * H) + dh) * S + ds
  int S, H;
  __device__ __forceinline__ void init(long long r, long long stride, int S_, int H_) {
    S = S_;
    H = H_;
    s = static_cast<int>(r % S);
    const long long bh = r / S;
    h = static_cast<int>(bh % H);
    b = static_cast<int>(bh / H);
    ds = static_cast<int>(stride % S);
    const long long sbh = stride / S;
    dh = static_cast<int>(sbh % H);
    db = static_cast<int>(sbh / H);
  }
  __device__ __forceinline__ void advance() {
    s += ds;
    int carry = 0;
    if (s >= S) {
      s -= S;
      carry = 1;
    }
    h += dh + carry;
    b += db;
    if (h >= H) {
      h -= H;
      b += 1;
    }
  }
};

template <int D, int MAXP>
__global__ void __launch_bounds__(kMergeThreads) lse_merge_kernel(const MergeParams p) {
  constexpr int LPR = D / 4;            // lanes per row
  constexpr int RPW = 32 / LPR;         // rows per warp per iteration
  const long long nrows = static_cast<long long>(p.B) * p.H * p.S;
  const long long tensor = nrows * D;   // elements of one partial output
  const int lane = threadIdx.x & 31;
  const int col = (lane % LPR) * 4;
  const long long warp_id = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const long long stride = nwarps * RPW;
  const int P = p.P;
  long long r = warp_id * RPW + lane / LPR;   // row index in (b, h, s) order
  RowCursor cur;
  cur.init(r, stride, p.S, p.H);
  for (; r < nrows; r += stride, cur.advance()) {
    const long long o_off = ((static_cast<long long>(cur.b) * p.S + cur.s) * p.H + cur.h) * D + col;
    float lse_p[MAXP];
    float4 o_p[MAXP];
#pragma unroll
    for (int i = 0; i < MAXP; ++i) {
      if (i < P) {
        lse_p[i] = __ldcs(p.part_lse + i * nrows + r);
        o_p[i] = __ldcs(reinterpret_cast<const float4 *>(p.part_out + i * tensor + o_off));
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int i = 0; i < MAXP; ++i)
      if (i < P) M = fmaxf(M, lse_p[i]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lse = -INFINITY;
    if (M != -INFINITY) {
      float w[MAXP];
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < MAXP; ++i) {
        w[i] = 0.f;
        if (i < P) {
          w[i] = expf(lse_p[i] - M);  // LSE_p = -inf gives 0
          sum += w[i];
        }
      }
      const float inv = 1.0f / sum;
#pragma unroll
      for (int i = 0; i < MAXP; ++i) {
        if (i < P) {
          const float a = w[i] * inv;
          acc.x = fmaf(a, o_p[i].x, acc.x);
          acc.y = fmaf(a, o_p[i].y, acc.y);
          acc.z = fmaf(a, o_p[i].z, acc.z);
          acc.w = fmaf(a, o_p[i].w, acc.w);
        }
      }
      lse = M + logf(sum);
    }
    if (p.out_f32 != nullptr) __stcs(reinterpret_cast<float4 *>(p.out_f32 + o_off), acc);
    if (p.out_bf16 != nullptr) {
      uint2 v = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
      __stcs(reinterpret_cast<uint2 *>(p.out_bf16 + o_off), v);
    }
    if (p.lse_out != nullptr && (lane % LPR) == 0) p.lse_out[r] = lse;
  }
}

// Any P: two passes over the partials of a row (max, then weighted sum).
template <int D>
__global__ void __launch_bounds__(kMergeThreads) lse_merge_kernel_anyp(const MergeParams p) {
  constexpr int LPR = D / 4;
  constexpr int RPW = 32 / LPR;
  const long long nrows = static_cast<long long>(p.B) * p.H * p.S;
  const long long tensor = nrows * D;
  const int lane = threadIdx.x & 31;
  const int col = (lane % LPR) * 4;
  const long long warp_id = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const long long stride = nwarps * RPW;
  long long r = warp_id * RPW + lane / LPR;
  RowCursor cur;
  cur.init(r, stride, p.S, p.H);
  for (; r < nrows; r += stride, cur.advance()) {
    const long long o_off = ((static_cast<long long>(cur.b) * p.S + cur.s) * p.H + cur.h) * D + col;
    float M = -INFINITY;
    for (int i = 0; i < p.P; ++i) M = fmaxf(M, p.part_lse[i * nrows + r]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lse = -INFINITY;
    if (M != -INFINITY) {
      float sum = 0.f;
      for (int i = 0; i < p.P; ++i) sum += expf(p.part_lse[i * nrows + r] - M);
      const float inv = 1.0f / sum;
      for (int i = 0; i < p.P; ++i) {
        const float a = expf(p.part_lse[i * nrows + r] - M) * inv;
        const float4 o = *reinterpret_cast<const float4 *>(p.part_out + i * tensor + o_off);
        acc.x = fmaf(a, o.x, acc.x);
        acc.y = fmaf(a, o.y, acc.y);
        acc.z = fmaf(a, o.z, acc.z);
        acc.w = fmaf(a, o.w, acc.w);
      }
      lse = M + logf(sum);
    }
    if (p.out_f32 != nullptr) *reinterpret_cast<float4 *>(p.out_f32 + o_off) = acc;
    if (p.out_bf16 != nullptr)
      *reinterpret_cast<uint2 *>(p.out_bf16 + o_off) = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
    if (p.lse_out != nullptr && (lane % LPR) == 0) p.lse_out[r] = lse;
  }
}

}  // namespace cpattn
