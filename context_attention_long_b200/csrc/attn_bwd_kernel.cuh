// attn_bwd_kernel.cuh -- gradient of softmax attention for sm_100a.
//
// The derivative of the forward definition (attn_kernel.cuh), per (batch,
// head), with S = Q K^T * scale, P = softmax(S) recomputed from the forward's
// log-sum-exp, and the upstream gradient dO of the output O:
//   Delta = rowsum(dO * O)                       (attn_bwd_delta_kernel)
//   dP    = dO V^T,   dS = P * (dP - Delta)
//   dQ    = dS K * scale                         (attn_bwd_dq_kernel)
//   dV    = P^T dO,   dK = dS^T Q * scale        (attn_bwd_dkv_kernel)
// The pages train with Ulysses over long contexts (the Ulysses Sequence
// Parallelism article, sections 1 and 7, causal masking by position ids); the
// causal mask here is the forward's: key j is visible to query i iff j <= i.
//
// No gradient needs atomics.  The dK/dV kernel owns a K/V tile and walks the
// Q tiles.  dQ comes one of two ways:
//   - with dS scratch (the default of the bindings): the dK/dV kernel also
//     stores dS in bf16 (a shared-memory staging tile and asynchronous bulk
//     stores), and the dQ GEMM (attn_bwd_dq_gemm_kernel) computes dS K from
//     it, bound by the HBM reads of dS -- S and dP are formed once;
//   - without: the dQ kernel owns a Q tile, walks the K/V tiles and forms S,
//     P, dP and dS again (the same values, bit for bit).
// A launch covers up to 8 problems (the full tensors, the head ranks' buffers
// of the Ulysses flow, or groups of their heads whose dS fits the scratch),
// each with its own tensor maps, LSE strides and Delta slice.  CTA
// organisation of the dQ and dK/dV kernels (320 threads, one CTA per SM):
//   warp 0      TMA producer: the owned tiles once, the walked tiles through
//               rings of 3 stages (K or Q) and 2 stages (V or dO); the dK/dV
//               kernel that stores dS has 2 Q stages and a dS staging tile
//   warp 1      TMEM allocator + single-thread MMA issuer (tcgen05.mma)
//   warps 2-9   two threads per row of the owned tile (TMEM lane), one per
//               half of the walked tile's 128 columns (warps 2-5 the first
//               half, 6-9 the second): P and dS in registers, bf16 results
//               back into TMEM (and dS to the staging tile, whose 4 KB part
//               each warp then bulk-stores), the epilogue.  Two row warps share each
//               sub-partition, so one's exponentials overlap the other's
//               loads, stores and waits.
// TMEM columns: S [0,128) (later P), dP [128,256) (later dS), then the
// accumulators (dQ; or dV and dK); the dQ kernel keeps a second dP buffer in
// [384,512), so dP(j+1) is computed while dS(j) still waits for the dQ MMA.
// Half h of a row packs its bf16 results
// into columns [64h, 64h + 32) of its region -- the start of the columns it
// read itself, so the two halves never overwrite each other's inputs -- and
// the MMAs read K block kk (16 keys or queries) at (kk / 4) * 64 + (kk % 4) * 8.
// The next tile's S (and, in the dQ kernel, dP) is issued as soon as the row
// threads have read the current S (dQ kernel) or the current P has been
// consumed (dK/dV kernel), so the tensor core works while the row threads
// exponentiate.  Every wait is bounded as in the forward.
#pragma once

#include "cpattn_internal.h"
#include "cpattn_ptx.cuh"

namespace cpattn {

// Device status bit of a backward kernel that found its shared-memory window
// misaligned (it then returns without touching memory).
constexpr unsigned int SITE_LAYOUT = 1u << 6;

template <int D, int kQStages = 3, bool kStaging = false>
struct BwdSmem {
  static constexpr int kHalves = D / 64;
  static constexpr int kBoxBytes = 128 * 128;          // [128 rows][64 bf16], 128B-swizzled
  static constexpr int kTileBytes = kHalves * kBoxBytes;
  // The walked tile a step needs first (K in the dQ kernel, Q in the dK/dV
  // kernel) is also the one released last (after the step's final MMA), so
  // it gets three stages: its load starts two steps ahead and its TMA latency
  // stays off the pipeline.  The other walked tile (V, dO) is released
  // mid-step, after its last MMA, and two stages are enough.  The dK/dV
  // kernel that stores dS gives the third stage up for the dS staging tile.
  static constexpr int kStagesC = kQStages;
  static constexpr int kStagesE = 2;
  static constexpr int kOffA = 0;                       // owned tile 0: Q (dq) or K (dkv)
  static constexpr int kOffB = kOffA + kTileBytes;      // owned tile 1: dO (dq) or V (dkv)
  static constexpr int kOffC = kOffB + kTileBytes;      // walked tile 0 per stage: K (dq) or Q (dkv)
  static constexpr int kOffE = kOffC + kStagesC * kTileBytes;   // walked tile 1 per stage: V or dO
  static constexpr int kOffStaging = kOffE + kStagesE * kTileBytes;   // dkv with dS stores: one dS tile
  static constexpr int kOffVec = kOffStaging + (kStaging ? kBwdDsTileBytes : 0);  // dkv: [2][lse2 128 | delta 128] floats
  static constexpr int kOffBar = kOffVec + 2 * 2 * 128 * 4;
  static constexpr int kNumBars = 24;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 16;
  // No alignment slack: seven D = 128 tiles leave too little room for one.
  // The dynamic window starts 1024-aligned (declared so, and checked at
  // kernel entry: a misaligned window records SITE_LAYOUT and the kernel
  // returns without touching memory).
  static constexpr int kAllocBytes = kBytes;
};
static_assert(BwdSmem<128>::kAllocBytes <= 232448 && BwdSmem<128, 2, true>::kAllocBytes <= 232448,
              "backward shared memory exceeds the per-CTA limit");

// Pins a value in a register at this point of the program: an empty volatile
// asm that reads and "writes" it, so the computation of the value cannot sink
// past a later volatile asm (a barrier wait).
__device__ __forceinline__ void reg_pin(uint32_t &v) { asm volatile("" : "+r"(v)); }

constexpr int kBwdRowWarps = 8;
constexpr int kBwdThreads = 64 + 32 * kBwdRowWarps;

// TMEM column of the bf16 pairs of K-block kk (16 rows of the contraction)
// inside a packed region (see the layout above).
__device__ __forceinline__ uint32_t bwd_packed_col(int kk) { return static_cast<uint32_t>((kk >> 2) * 64 + (kk & 3) * 8); }
constexpr uint32_t kBwdTmemCols = 512;
// dQ kernel: TMEM column of dP buffer b (dP(j) uses buffer j % 2); dQ sits
// at [256, 256 + D) between them.
__device__ __forceinline__ uint32_t bwd_dq_dp_col(int b) { return b ? 384u : 128u; }

// Delta[b, h, s] = sum_d dO[b, s, h, d] * O[b, s, h, d].  A (token, head) row
// is D / 8 lanes, each on one 16-byte piece of both rows (coalesced); a warp
// covers 32 / (D / 8) rows per pass and issues the loads of kDeltaPasses passes
// before it reduces any of them, so that many rows' loads are in flight at
// once.  The sum order is fixed: the result is deterministic.
constexpr int kDeltaPasses = 4;
__global__ void __launch_bounds__(256, 3) attn_bwd_delta_kernel(const __nv_bfloat16 *__restrict__ out,
                                                                const __nv_bfloat16 *__restrict__ dout,
                                                                float *__restrict__ delta, int B, int S, int H,
                                                                int D) {
  // Rows are (token, head) pairs, B*S*H < 2^31 (checked on the host).
  const int lane = threadIdx.x & 31;
  const int lpr = D >> 3;                    // lanes per row (16 for D = 128, 8 for D = 64)
  const int rpp = 32 / lpr;                  // rows per warp pass
  const int sub = lane / lpr, piece = lane - sub * lpr;
  const unsigned warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const unsigned nwarps = (gridDim.x * blockDim.x) >> 5;
  const unsigned nrows = static_cast<unsigned>(B) * S * H;
  const unsigned per_iter = static_cast<unsigned>(rpp) * kDeltaPasses;
  for (unsigned r0 = warp * per_iter; r0 < nrows; r0 += nwarps * per_iter) {
    uint4 ov[kDeltaPasses], gv[kDeltaPasses];
#pragma unroll
    for (int u = 0; u < kDeltaPasses; ++u) {
      const unsigned r = r0 + u * rpp + sub;
      ov[u] = make_uint4(0u, 0u, 0u, 0u);
      gv[u] = ov[u];
      if (r < nrows) {
        ov[u] = __ldcs(reinterpret_cast<const uint4 *>(out + static_cast<size_t>(r) * D) + piece);
        gv[u] = __ldcs(reinterpret_cast<const uint4 *>(dout + static_cast<size_t>(r) * D) + piece);
      }
    }
    // (token, head) of row r0 and (batch, position) of that token, once per
    // iteration; each row below steps from them without dividing.
    const unsigned tok0 = r0 / H;
    const int h0 = static_cast<int>(r0 - tok0 * H);
    const unsigned b0 = tok0 / S;
    const int s0 = static_cast<int>(tok0 - b0 * S);
#pragma unroll
    for (int u = 0; u < kDeltaPasses; ++u) {
      const uint32_t o4[4] = {ov[u].x, ov[u].y, ov[u].z, ov[u].w};
      const uint32_t g4[4] = {gv[u].x, gv[u].y, gv[u].z, gv[u].w};
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 o = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&o4[e]));
        const float2 g = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&g4[e]));
        acc = fmaf(o.x, g.x, fmaf(o.y, g.y, acc));
      }
      for (int off = lpr >> 1; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      const unsigned r = r0 + u * rpp + sub;
      if (piece == 0 && r < nrows) {
        int h = h0 + u * rpp + sub, s = s0;
        unsigned b = b0;
        while (h >= H) {         // at most kDeltaPasses * rpp / H + 1 steps
          h -= H;
          if (++s == S) {
            s = 0;
            ++b;
          }
        }
        delta[(static_cast<size_t>(b) * H + h) * S + s] = acc;
      }
    }
  }
}

// Units: (problem, b, h, 128-row tile) over the problem's heads [h0, h0 + nh),
// the tile index fastest (with last_first, the last tile of a head first);
// problems occupy consecutive unit ranges.  hl = h - h0.
struct BwdUnit {
  int pi, b, h, hl, t;
};
__device__ __forceinline__ BwdUnit bwd_unit_at(const BwdParams &p, int idx, bool last_first) {
  const int nt = (p.S + 127) / 128;
  BwdUnit u;
  int pi = 0;
  while (pi + 1 < p.n_prob && p.prob[pi + 1].unit_base <= idx) ++pi;
  const int local = idx - p.prob[pi].unit_base;
  const int NH = p.prob[pi].nh;
  const int t_in = local % nt;
  const int bh = local / nt;
  u.pi = pi;
  u.hl = bh % NH;
  u.h = p.prob[pi].h0 + u.hl;
  u.b = bh / NH;
  u.t = last_first ? nt - 1 - t_in : t_in;
  return u;
}
__device__ __forceinline__ BwdUnit bwd_unit(const BwdParams &p, bool last_first) {
  return bwd_unit_at(p, static_cast<int>(blockIdx.x), last_first);
}

// Element offset of the gradient row of (batch b, sequence position s, head
// h) by the problem's output map (see BwdProblem).
template <int D>
__device__ __forceinline__ long long bwd_out_elems(const BwdProblem &PB, int B, int S, int b, int s, int h) {
  if (PB.out_mode == 0) return ((static_cast<long long>(b) * S + s) * PB.H + h) * D;
  int lo = 0, hi = PB.out_nseq - 1;   // the sequence rank holding s (empty ranks are never found)
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (PB.out_seq_off[mid] <= s) lo = mid; else hi = mid - 1;
  }
  const int off = PB.out_seq_off[lo], len = PB.out_seq_off[lo + 1] - off;
  const long long row = static_cast<long long>(B) * off + static_cast<long long>(b) * len + (s - off);
  return (row * PB.out_H + PB.out_h0 + h) * D;
}

// ===================================================================== dQ
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) attn_bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  using L = BwdSmem<D>;
  constexpr uint32_t IDESC_SS = idesc_bf16_f32(128, 128, false);   // S = Q K^T, dP = dO V^T
  constexpr uint32_t IDESC_DQ = idesc_bf16_f32(128, D, true);      // dQ += dS K, K MN-major
  extern __shared__ __align__(1024) uint8_t bwd_smem[];
  const uint32_t sb = smem_u32(bwd_smem);
  if (sb & 1023u) {
    if (threadIdx.x == 0) atomicOr(&g_device_status, SITE_LAYOUT);
    return;
  }
  constexpr int KS = L::kStagesC, VS = L::kStagesE;
  constexpr uint32_t BAR_QD = L::kOffBar;          // Q and dO loaded
  constexpr uint32_t BAR_KF = BAR_QD + 8;          // [KS]
  constexpr uint32_t BAR_KE = BAR_KF + 8 * KS;     // [KS]
  constexpr uint32_t BAR_VF = BAR_KE + 8 * KS;     // [VS]
  constexpr uint32_t BAR_VE = BAR_VF + 8 * VS;     // [VS]
  constexpr uint32_t BAR_S = BAR_VE + 8 * VS;      // S(j) in TMEM
  constexpr uint32_t BAR_SC = BAR_S + 8;           // S(j) read by the row threads
  constexpr uint32_t BAR_DP = BAR_SC + 8;          // [2] dP(j) in TMEM buffer j % 2
  constexpr uint32_t BAR_DS = BAR_DP + 16;         // [2] dS(j) in TMEM buffer j % 2
  constexpr uint32_t BAR_DQ = BAR_DS + 16;         // dQ complete
  constexpr uint32_t BAR_TAIL = BAR_DQ + 8;
  constexpr uint32_t TMEM_SLOT = L::kOffMisc;
  constexpr uint32_t ABORT = L::kOffMisc + 4;
  static_assert(BAR_TAIL + 8 <= L::kOffMisc, "barrier area");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t tmo = p.timeout_ns;
  const BwdUnit U = bwd_unit(p, p.causal != 0);   // causal: heavier (later) Q tiles first
  const BwdProblem &PB = p.prob[U.pi];
  const int q0 = U.t * 128;
  const int q_rows = min(128, p.S - q0);
  const int kv_len = p.causal ? min(p.S, q0 + q_rows) : p.S;   // keys at positions < kv_len
  const int n = (kv_len + 127) / 128;
  const int row_base = U.b * p.S;

  if (threadIdx.x == 0) {
    mbar_init(sb + BAR_QD, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(sb + BAR_KF + 8 * s, 1);
      mbar_init(sb + BAR_KE + 8 * s, 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(sb + BAR_VF + 8 * s, 1);
      mbar_init(sb + BAR_VE + 8 * s, 1);
    }
    mbar_init(sb + BAR_S, 1);
    mbar_init(sb + BAR_SC, kBwdRowWarps);
    for (int s = 0; s < 2; ++s) {
      mbar_init(sb + BAR_DP + 8 * s, 1);
      mbar_init(sb + BAR_DS + 8 * s, kBwdRowWarps);
    }
    mbar_init(sb + BAR_DQ, 1);
    mbar_init(sb + BAR_TAIL, 1);
    st_shared_volatile(sb + ABORT, 0u);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sb + TMEM_SLOT, kBwdTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ld_shared_volatile(sb + TMEM_SLOT);
  const uint32_t abort_flag = sb + ABORT;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&PB.tm_q);
      tma_prefetch_desc(&PB.tm_k);
      tma_prefetch_desc(&PB.tm_v);
      tma_prefetch_desc(&PB.tm_do);
      mbar_arrive_expect_tx(sb + BAR_QD, 2 * L::kTileBytes);
      for (int hf = 0; hf < L::kHalves; ++hf) {
        tma_load_3d(sb + L::kOffA + hf * L::kBoxBytes, &PB.tm_q, hf * 64, U.h, row_base + q0, sb + BAR_QD);
        tma_load_3d(sb + L::kOffB + hf * L::kBoxBytes, &PB.tm_do, hf * 64, U.h, row_base + q0, sb + BAR_QD);
      }
      for (int j = 0; j < n; ++j) {
        const int ks = j % KS, vs = j % VS;
        const uint32_t kph = (j / KS) & 1, vph = (j / VS) & 1;
        if (!mbar_wait(sb + BAR_KE + 8 * ks, kph ^ 1, abort_flag, tmo, SITE_PRODUCER)) break;
        mbar_arrive_expect_tx(sb + BAR_KF + 8 * ks, L::kTileBytes);
        for (int hf = 0; hf < L::kHalves; ++hf)
          tma_load_3d(sb + L::kOffC + ks * L::kTileBytes + hf * L::kBoxBytes, &PB.tm_k, hf * 64, U.h,
                      row_base + j * 128, sb + BAR_KF + 8 * ks);
        if (!mbar_wait(sb + BAR_VE + 8 * vs, vph ^ 1, abort_flag, tmo, SITE_PRODUCER)) break;
        mbar_arrive_expect_tx(sb + BAR_VF + 8 * vs, L::kTileBytes);
        for (int hf = 0; hf < L::kHalves; ++hf)
          tma_load_3d(sb + L::kOffE + vs * L::kTileBytes + hf * L::kBoxBytes, &PB.tm_v, hf * 64, U.h,
                      row_base + j * 128, sb + BAR_VF + 8 * vs);
      }
      // every stage's last release must arrive before the CTA exits
      for (int st = 0; st < KS; ++st) {
        const int uses = n > st ? (n - 1 - st) / KS + 1 : 0;
        if (uses > 0) mbar_wait(sb + BAR_KE + 8 * st, (uses - 1) & 1, 0u, tmo, SITE_TAIL);
      }
      for (int st = 0; st < VS; ++st) {
        const int uses = n > st ? (n - 1 - st) / VS + 1 : 0;
        if (uses > 0) mbar_wait(sb + BAR_VE + 8 * st, (uses - 1) & 1, 0u, tmo, SITE_TAIL);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t dQo = smem_desc_sw128(sb + L::kOffA, 16, 1024);
      const uint64_t dDO = smem_desc_sw128(sb + L::kOffB, 16, 1024);
      const uint64_t dK = smem_desc_sw128(sb + L::kOffC, 16, 1024);                  // K-major (S)
      const uint64_t dKmn = smem_desc_sw128(sb + L::kOffC, L::kBoxBytes, 1024);       // MN-major (dQ)
      const uint64_t dV = smem_desc_sw128(sb + L::kOffE, 16, 1024);
      auto issue_ss = [&](uint32_t d, uint64_t a0, uint64_t b0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * L::kBoxBytes + (kk & 3) * 32) >> 4;
          mma_ss(d, a0 + off, b0 + off, IDESC_SS, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_s = [&](int ks) { issue_ss(tmem, opaque_u64(dQo), opaque_u64(dK + ((ks * L::kTileBytes) >> 4))); };
      auto issue_dp = [&](int buf, int vs) {
        issue_ss(tmem + bwd_dq_dp_col(buf), opaque_u64(dDO), opaque_u64(dV + ((vs * L::kTileBytes) >> 4)));
      };
      // dQ (+)= dS K: dS (bf16 pairs) from TMEM over dP, K MN-major (keys
      // are rows of 128 bytes): 16 keys = 2048 bytes per MMA.
      auto issue_dq = [&](int buf, int ks, bool acc) {
        const uint64_t b0 = opaque_u64(dKmn + ((ks * L::kTileBytes) >> 4));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + 256, tmem + bwd_dq_dp_col(buf) + bwd_packed_col(kk), b0 + ((kk * 2048) >> 4), IDESC_DQ,
                 (acc || kk > 0) ? 1u : 0u);
      };
      // S(j+1) and dP(j+1) are issued as soon as the row threads have read
      // S(j): dP alternates between two TMEM buffers, so dP(j+1) does not wait
      // for dQ(j) to consume dS(j).  dQ(j) follows dS(j).  The tensor core runs
      // the three MMAs of a step while the row threads work on the previous one.
      bool ok = n > 0 && mbar_wait_spin(sb + BAR_QD, 0, abort_flag, tmo, SITE_MMA);
      if (ok) ok = mbar_wait_spin(sb + BAR_KF, 0, abort_flag, tmo, SITE_MMA);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        mma_commit(sb + BAR_S);
      }
      if (ok) ok = mbar_wait_spin(sb + BAR_VF, 0, abort_flag, tmo, SITE_MMA);
      if (ok) {
        tc_fence_after();
        issue_dp(0, 0);
        mma_commit(sb + BAR_DP);
        mma_commit(sb + BAR_VE);
      }
      for (int j = 0; ok && j < n; ++j) {
        const int j1 = j + 1;
        if (!mbar_wait_spin(sb + BAR_SC, j & 1, abort_flag, tmo, SITE_MMA)) break;
        if (j1 < n) {   // S(j) has been read: the next S may overwrite it
          const int ks1 = j1 % KS, vs1 = j1 % VS;
          if (!mbar_wait_spin(sb + BAR_KF + 8 * ks1, (j1 / KS) & 1, abort_flag, tmo, SITE_MMA)) break;
          tc_fence_after();
          issue_s(ks1);
          mma_commit(sb + BAR_S);
          // dP buffer j1 % 2 last held dS(j-1), consumed by dQ(j-1), issued
          // earlier on this thread: the tensor core reads it first.
          if (!mbar_wait_spin(sb + BAR_VF + 8 * vs1, (j1 / VS) & 1, abort_flag, tmo, SITE_MMA)) break;
          tc_fence_after();
          issue_dp(j1 & 1, vs1);
          mma_commit(sb + BAR_DP + 8 * (j1 & 1));
          mma_commit(sb + BAR_VE + 8 * vs1);
        }
        if (!mbar_wait_spin(sb + BAR_DS + 8 * (j & 1), (j >> 1) & 1, abort_flag, tmo, SITE_MMA)) break;
        tc_fence_after();
        issue_dq(j & 1, j % KS, j > 0);
        mma_commit(sb + BAR_KE + 8 * (j % KS));
      }
      if (n > 0) mma_commit(sb + BAR_DQ);
      mma_commit(sb + BAR_TAIL);
      mbar_wait(sb + BAR_TAIL, 0, 0u, tmo, SITE_TAIL);
    }
  } else {
    // ------------------------------------------------------------ row threads
    const int quad = warp & 3;                 // TMEM lane group of this warp
    const int half = (warp - 2) >> 2;          // which 64 keys of the walked tile
    const int col0 = half * 64;
    const int row = quad * 32 + lane;
    const int q_pos = q0 + row;
    const bool row_valid = row < q_rows;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + lane_base + col0;
    const uint32_t tDQ = tmem + lane_base + 256;
    const float c = p.scale_log2;
    const long long li = static_cast<long long>(U.b) * PB.lse_b + static_cast<long long>(U.h + PB.lse_h0) * PB.lse_h + q_pos;
    const long long di = (static_cast<long long>(U.b) * PB.H + U.h) * p.S + q_pos;
    const float lse2 = row_valid ? PB.lse[li] * 1.4426950408889634f : 0.f;
    const float delta = row_valid ? PB.delta[di] : 0.f;
    bool ok = true;
    for (int j = 0; ok && j < n; ++j) {
      // keys of tile j this row sees: all valid keys, cut at the row's own
      // position under the causal mask; none for rows past the sequence;
      // counted from this thread's first key
      int kvalid = min(128, kv_len - j * 128);
      if (p.causal) kvalid = min(kvalid, q_pos - j * 128 + 1);
      if (!row_valid) kvalid = 0;
      kvalid -= col0;
      bool w = mbar_wait(sb + BAR_S, j & 1, abort_flag, tmo, SITE_SOFTMAX);
      if (__any_sync(0xffffffffu, !w)) { ok = false; break; }
      __syncwarp();
      tc_fence_after();
      uint32_t s[64];
      tmem_ld64_wait(tS, s);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sb + BAR_SC);
      // P = 2^(S*c - lse2), kept in fp32 over the scores: the first 32 keys
      // before the dP wait (pinned there, so the compiler keeps them ahead of
      // it), the other 32 interleaved with dS of the first 32, so that the
      // dS arithmetic issues while the SFU works.
      auto p_of = [&](int k) {
        return __float_as_uint(k < kvalid ? ex2_approx(__uint_as_float(s[k]) * c - lse2) : 0.f);
      };
#pragma unroll
      for (int k = 0; k < 32; ++k) s[k] = p_of(k);
#pragma unroll
      for (int k = 0; k < 32; ++k) reg_pin(s[k]);
      w = mbar_wait(sb + BAR_DP + 8 * (j & 1), (j >> 1) & 1, abort_flag, tmo, SITE_SOFTMAX);
      if (__any_sync(0xffffffffu, !w)) { ok = false; break; }
      __syncwarp();
      tc_fence_after();
      const uint32_t tDP = tmem + lane_base + bwd_dq_dp_col(j & 1) + col0;
      // dS = P * (dP - delta), bf16 pairs over the dP columns already read
      auto ds_pair = [&](int k, const uint32_t *dp) {
        return pack_bf16x2(__uint_as_float(s[k]) * (__uint_as_float(dp[0]) - delta),
                           __uint_as_float(s[k + 1]) * (__uint_as_float(dp[1]) - delta));
      };
      {
        uint32_t dp[32], pk[16];
        tmem_ld32_wait(tDP, dp);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          s[32 + 2 * k] = p_of(32 + 2 * k);
          s[33 + 2 * k] = p_of(33 + 2 * k);
          pk[k] = ds_pair(2 * k, dp + 2 * k);
        }
        tmem_st16(tDP, pk);
        tmem_ld32_wait(tDP + 32, dp);
#pragma unroll
        for (int k = 0; k < 16; ++k) pk[k] = ds_pair(32 + 2 * k, dp + 2 * k);
        tmem_st16(tDP + 16, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sb + BAR_DS + 8 * (j & 1));
    }
    if (ok && n > 0) {
      const bool w = mbar_wait(sb + BAR_DQ, 0, abort_flag, tmo, SITE_EPILOGUE);
      if (__any_sync(0xffffffffu, !w)) ok = false;
      __syncwarp();
      tc_fence_after();
    }
    if (ok) {
      // each half of the row writes half of dQ's D columns
      const float scale = p.scale;
      const int d0 = half * (D / 2);
      __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(PB.dq) +
                           (row_valid ? bwd_out_elems<D>(PB, p.B, p.S, U.b, q_pos, U.h) : 0) + d0;
#pragma unroll
      for (int c0 = 0; c0 < D / 2; c0 += 32) {
        uint32_t o[32];
        if (n > 0) {
          tmem_ld32_wait(tDQ + d0 + c0, o);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = 0u;
        }
        if (row_valid) {
          uint4 *d4 = reinterpret_cast<uint4 *>(dst + c0);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            d4[k] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * k]) * scale, __uint_as_float(o[8 * k + 1]) * scale),
                               pack_bf16x2(__uint_as_float(o[8 * k + 2]) * scale, __uint_as_float(o[8 * k + 3]) * scale),
                               pack_bf16x2(__uint_as_float(o[8 * k + 4]) * scale, __uint_as_float(o[8 * k + 5]) * scale),
                               pack_bf16x2(__uint_as_float(o[8 * k + 6]) * scale, __uint_as_float(o[8 * k + 7]) * scale));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBwdTmemCols);
  }
}

// =================================================================== dK, dV
// kDs: also store dS for the dQ GEMM (every problem's ds set), through a
// shared-memory staging tile and asynchronous bulk stores.
template <int D, bool kDs>
__global__ void __launch_bounds__(kBwdThreads, 1) attn_bwd_dkv_kernel(const __grid_constant__ BwdParams p) {
  using L = BwdSmem<D, kDs ? 2 : 3, kDs>;
  constexpr uint32_t IDESC_SS = idesc_bf16_f32(128, 128, false);   // S^T = K Q^T, dP^T = V dO^T
  constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, D, true);     // dV += P^T dO, dK += dS^T Q
  extern __shared__ __align__(1024) uint8_t bwd_smem[];
  const uint32_t sb = smem_u32(bwd_smem);
  if (sb & 1023u) {
    if (threadIdx.x == 0) atomicOr(&g_device_status, SITE_LAYOUT);
    return;
  }
  constexpr int QS = L::kStagesC, OS = L::kStagesE;
  constexpr uint32_t BAR_KV = L::kOffBar;          // K and V loaded
  constexpr uint32_t BAR_QF = BAR_KV + 8;          // [QS]
  constexpr uint32_t BAR_QE = BAR_QF + 8 * QS;     // [QS]
  constexpr uint32_t BAR_OF = BAR_QE + 8 * QS;     // [OS] dO tile full
  constexpr uint32_t BAR_OE = BAR_OF + 8 * OS;     // [OS]
  constexpr uint32_t BAR_S = BAR_OE + 8 * OS;      // S^T(i) in TMEM
  constexpr uint32_t BAR_P = BAR_S + 8;            // P^T(i) written
  constexpr uint32_t BAR_DP = BAR_P + 8;           // dP^T(i) in TMEM
  constexpr uint32_t BAR_DS = BAR_DP + 8;          // dS^T(i) written
  constexpr uint32_t BAR_ACC = BAR_DS + 8;         // dV and dK complete
  constexpr uint32_t BAR_TAIL = BAR_ACC + 8;
  constexpr uint32_t BAR_VEC = BAR_TAIL + 8;       // this Q tile's LSE / Delta in smem (4 warps)
  constexpr uint32_t TMEM_SLOT = L::kOffMisc;
  constexpr uint32_t ABORT = L::kOffMisc + 4;
  static_assert(BAR_VEC + 8 <= L::kOffMisc, "barrier area");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t tmo = p.timeout_ns;
  const BwdUnit U = bwd_unit(p, false);        // causal: earlier K/V tiles see more queries and run first
  const BwdProblem &PB = p.prob[U.pi];
  const int nt = (p.S + 127) / 128;
  const int k0 = U.t * 128;
  const int k_rows = min(128, p.S - k0);
  const int qt0 = p.causal ? U.t : 0;         // Q tiles with a query at or after k0
  const int n = nt - qt0;
  const int row_base = U.b * p.S;

  if (threadIdx.x == 0) {
    mbar_init(sb + BAR_KV, 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(sb + BAR_QF + 8 * s, 1);
      mbar_init(sb + BAR_QE + 8 * s, 1);
    }
    for (int s = 0; s < OS; ++s) {
      mbar_init(sb + BAR_OF + 8 * s, 1);
      mbar_init(sb + BAR_OE + 8 * s, 1);
    }
    mbar_init(sb + BAR_S, 1);
    mbar_init(sb + BAR_P, kBwdRowWarps);
    mbar_init(sb + BAR_DP, 1);
    mbar_init(sb + BAR_DS, kBwdRowWarps);
    mbar_init(sb + BAR_ACC, 1);
    mbar_init(sb + BAR_TAIL, 1);
    mbar_init(sb + BAR_VEC, kBwdRowWarps);
    st_shared_volatile(sb + ABORT, 0u);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sb + TMEM_SLOT, kBwdTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ld_shared_volatile(sb + TMEM_SLOT);
  const uint32_t abort_flag = sb + ABORT;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&PB.tm_q);
      tma_prefetch_desc(&PB.tm_k);
      tma_prefetch_desc(&PB.tm_v);
      tma_prefetch_desc(&PB.tm_do);
      mbar_arrive_expect_tx(sb + BAR_KV, 2 * L::kTileBytes);
      for (int hf = 0; hf < L::kHalves; ++hf) {
        tma_load_3d(sb + L::kOffA + hf * L::kBoxBytes, &PB.tm_k, hf * 64, U.h, row_base + k0, sb + BAR_KV);
        tma_load_3d(sb + L::kOffB + hf * L::kBoxBytes, &PB.tm_v, hf * 64, U.h, row_base + k0, sb + BAR_KV);
      }
      for (int i = 0; i < n; ++i) {
        const int qs = i % QS, os = i % OS;
        const uint32_t qph = (i / QS) & 1, oph = (i / OS) & 1;
        const int qrow = row_base + (qt0 + i) * 128;
        if (!mbar_wait(sb + BAR_QE + 8 * qs, qph ^ 1, abort_flag, tmo, SITE_PRODUCER)) break;
        mbar_arrive_expect_tx(sb + BAR_QF + 8 * qs, L::kTileBytes);
        for (int hf = 0; hf < L::kHalves; ++hf)
          tma_load_3d(sb + L::kOffC + qs * L::kTileBytes + hf * L::kBoxBytes, &PB.tm_q, hf * 64, U.h, qrow,
                      sb + BAR_QF + 8 * qs);
        if (!mbar_wait(sb + BAR_OE + 8 * os, oph ^ 1, abort_flag, tmo, SITE_PRODUCER)) break;
        mbar_arrive_expect_tx(sb + BAR_OF + 8 * os, L::kTileBytes);
        for (int hf = 0; hf < L::kHalves; ++hf)
          tma_load_3d(sb + L::kOffE + os * L::kTileBytes + hf * L::kBoxBytes, &PB.tm_do, hf * 64, U.h, qrow,
                      sb + BAR_OF + 8 * os);
      }
      for (int st = 0; st < QS; ++st) {
        const int uses = n > st ? (n - 1 - st) / QS + 1 : 0;
        if (uses > 0) mbar_wait(sb + BAR_QE + 8 * st, (uses - 1) & 1, 0u, tmo, SITE_TAIL);
      }
      for (int st = 0; st < OS; ++st) {
        const int uses = n > st ? (n - 1 - st) / OS + 1 : 0;
        if (uses > 0) mbar_wait(sb + BAR_OE + 8 * st, (uses - 1) & 1, 0u, tmo, SITE_TAIL);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t dK = smem_desc_sw128(sb + L::kOffA, 16, 1024);
      const uint64_t dV = smem_desc_sw128(sb + L::kOffB, 16, 1024);
      const uint64_t dQk = smem_desc_sw128(sb + L::kOffC, 16, 1024);                 // K-major (S^T)
      const uint64_t dQmn = smem_desc_sw128(sb + L::kOffC, L::kBoxBytes, 1024);      // MN-major (dK)
      const uint64_t dOk = smem_desc_sw128(sb + L::kOffE, 16, 1024);                 // K-major (dP^T)
      const uint64_t dOmn = smem_desc_sw128(sb + L::kOffE, L::kBoxBytes, 1024);      // MN-major (dV)
      auto issue_ss = [&](uint32_t d, uint64_t a0, uint64_t b0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * L::kBoxBytes + (kk & 3) * 32) >> 4;
          mma_ss(d, a0 + off, b0 + off, IDESC_SS, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_acc = [&](uint32_t d, uint32_t a_tmem, uint64_t b0, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(d, a_tmem + bwd_packed_col(kk), b0 + ((kk * 2048) >> 4), IDESC_ACC, (acc || kk > 0) ? 1u : 0u);
      };
      auto stage_off = [&](int st) { return static_cast<uint64_t>((st * L::kTileBytes) >> 4); };
      bool ok = n > 0 && mbar_wait_spin(sb + BAR_KV, 0, abort_flag, tmo, SITE_MMA);
      if (ok) ok = mbar_wait_spin(sb + BAR_QF, 0, abort_flag, tmo, SITE_MMA);
      if (ok) {
        tc_fence_after();
        issue_ss(tmem, opaque_u64(dK), opaque_u64(dQk + stage_off(0)));
        mma_commit(sb + BAR_S);
      }
      if (ok) ok = mbar_wait_spin(sb + BAR_OF, 0, abort_flag, tmo, SITE_MMA);
      if (ok) {
        tc_fence_after();
        issue_ss(tmem + 128, opaque_u64(dV), opaque_u64(dOk + stage_off(0)));
        mma_commit(sb + BAR_DP);
      }
      for (int i = 0; ok && i < n; ++i) {
        const int i1 = i + 1;
        const bool more = i1 < n;
        // dV (+)= P^T dO: P^T (bf16 pairs) from TMEM over S^T, dO MN-major;
        // dO(i) has no later use, so its stage is released right behind it
        if (!mbar_wait_spin(sb + BAR_P, i & 1, abort_flag, tmo, SITE_MMA)) break;
        tc_fence_after();
        issue_acc(tmem + 256, tmem, opaque_u64(dOmn + stage_off(i % OS)), i > 0);
        mma_commit(sb + BAR_OE + 8 * (i % OS));
        if (more) {   // P^T(i) is consumed in order before S^T(i+1) overwrites it
          const int qs1 = i1 % QS;
          if (!mbar_wait_spin(sb + BAR_QF + 8 * qs1, (i1 / QS) & 1, abort_flag, tmo, SITE_MMA)) break;
          tc_fence_after();
          issue_ss(tmem, opaque_u64(dK), opaque_u64(dQk + stage_off(qs1)));
          mma_commit(sb + BAR_S);
        }
        // dK (+)= dS^T Q: dS^T (bf16 pairs) from TMEM over dP^T, Q MN-major
        if (!mbar_wait_spin(sb + BAR_DS, i & 1, abort_flag, tmo, SITE_MMA)) break;
        tc_fence_after();
        issue_acc(tmem + 256 + D, tmem + 128, opaque_u64(dQmn + stage_off(i % QS)), i > 0);
        mma_commit(sb + BAR_QE + 8 * (i % QS));
        if (more) {
          const int os1 = i1 % OS;
          if (!mbar_wait_spin(sb + BAR_OF + 8 * os1, (i1 / OS) & 1, abort_flag, tmo, SITE_MMA)) break;
          tc_fence_after();
          issue_ss(tmem + 128, opaque_u64(dV), opaque_u64(dOk + stage_off(os1)));
          mma_commit(sb + BAR_DP);
        }
      }
      if (n > 0) mma_commit(sb + BAR_ACC);
      mma_commit(sb + BAR_TAIL);
      mbar_wait(sb + BAR_TAIL, 0, 0u, tmo, SITE_TAIL);
    }
  } else {
    // ------------------------------------------------------------ row threads (two per key)
    const int quad = warp & 3;                 // TMEM lane group of this warp
    const int half = (warp - 2) >> 2;          // which 64 queries of the walked tile
    const int col0 = half * 64;
    const int row = quad * 32 + lane;
    const int k_pos = k0 + row;
    const bool row_valid = row < k_rows;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + lane_base + col0;
    const uint32_t tDP = tmem + lane_base + 128 + col0;
    const uint32_t tDV = tmem + lane_base + 256;
    const uint32_t tDK = tmem + lane_base + 256 + D;
    const float c = p.scale_log2;
    const long long lbase = static_cast<long long>(U.b) * PB.lse_b + static_cast<long long>(U.h + PB.lse_h0) * PB.lse_h;
    const long long dbase = (static_cast<long long>(U.b) * PB.H + U.h) * p.S;
    bool ok = true;
    // Each Q tile's log2-domain LSE and Delta are published in shared memory
    // by the first-half threads, one value per thread (queries past the
    // sequence get LSE = +inf, i.e. P = 0), loaded one tile ahead so that
    // their global-memory latency hides behind a tile.
    auto load_vec = [&](int i, float &l2, float &dl) {
      const int q = (qt0 + i) * 128 + row;
      l2 = q < p.S ? PB.lse[lbase + q] * 1.4426950408889634f : INFINITY;
      dl = q < p.S ? PB.delta[dbase + q] : 0.f;
    };
    float nl2 = 0.f, ndl = 0.f;
    if (n > 0 && half == 0) load_vec(0, nl2, ndl);
    for (int i = 0; ok && i < n; ++i) {
      const int q0 = (qt0 + i) * 128;
      const uint32_t vec = sb + L::kOffVec + (i & 1) * 1024;
      // this warp's 4 KB of the dS tile: keys [32 quad, 32 quad + 32), query
      // groups [8 half, 8 half + 8), in the tile layout (and in the staging
      // tile at the same offset)
      const uint32_t ds_part = static_cast<uint32_t>(quad * 8192 + half * 4096);
      unsigned char *const ds_dst =
          kDs ? PB.ds + bwd_ds_tile_index(U.b, U.hl, PB.nh, nt, qt0 + i, U.t, p.causal != 0) * kBwdDsTileBytes + ds_part
              : nullptr;
      const uint32_t ds_stage = sb + L::kOffStaging + ds_part;
      if (half == 0) {
        st_shared_f32(vec + 4 * row, nl2);
        st_shared_f32(vec + 512 + 4 * row, ndl);
        if (i + 1 < n) load_vec(i + 1, nl2, ndl);
      }
      // Every row warp has finished reading the previous use of this buffer
      // (tile i-2) before it is written for tile i -- its arrival for tile
      // i-1 came after those reads -- and the bounded barrier below
      // publishes the values; no unbounded named barrier.
      __syncwarp();
      if (lane == 0) mbar_arrive(sb + BAR_VEC);
      bool w = mbar_wait(sb + BAR_VEC, i & 1, abort_flag, tmo, SITE_SOFTMAX);
      if (__any_sync(0xffffffffu, !w)) { ok = false; break; }
      w = mbar_wait(sb + BAR_S, i & 1, abort_flag, tmo, SITE_SOFTMAX);
      if (__any_sync(0xffffffffu, !w)) { ok = false; break; }
      __syncwarp();
      tc_fence_after();
      uint32_t s[64];
      tmem_ld64_wait(tS, s);
      // P^T[k][q] = 2^(S^T*c - lse2[q]) for the queries that see key k.  The
      // per-query values are read as float4 through a plain shared-memory
      // pointer (the barrier waits above are compiler fences), so the loads
      // schedule freely around the exponentials.
      const float4 *lse4 = reinterpret_cast<const float4 *>(bwd_smem + (vec - sb)) + (col0 >> 2);
      const float4 *del4 = lse4 + 32;
      // queries q < qlim do not see this key; a key past the sequence (its K
      // and V rows are the next batch element's, or TMA fill) is seen by none,
      // so its P and dS are exactly 0 -- the stored dS meets real K rows of
      // that position in the dQ GEMM
      const int qlim = row_valid ? (p.causal ? k_pos - q0 : 0) - col0 : 64;
#pragma unroll
      for (int q4 = 0; q4 < 16; ++q4) {
        const float4 l = lse4[q4];
        const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int q = 4 * q4 + e;
          const float pv = ex2_approx(__uint_as_float(s[q]) * c - lv[e]);
          s[q] = __float_as_uint(q >= qlim ? pv : 0.f);
        }
      }
#pragma unroll
      for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) pk[k] = pack_bf16x2(__uint_as_float(s[c0 + 2 * k]), __uint_as_float(s[c0 + 2 * k + 1]));
        tmem_st16(tS + c0 / 2, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sb + BAR_P);
      w = mbar_wait(sb + BAR_DP, i & 1, abort_flag, tmo, SITE_SOFTMAX);
      if (__any_sync(0xffffffffu, !w)) { ok = false; break; }
      __syncwarp();
      tc_fence_after();
      // dS^T = P^T * (dP^T - delta[q]), bf16 pairs over the dP^T columns read
      if (kDs) {
        // the staging tile is free once the previous tile's bulk store has
        // read it (issued a whole tile ago)
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
      }
#pragma unroll
      for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t dp[32];
        tmem_ld32_wait(tDP + c0, dp);
        uint32_t pk[16];
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) {
          const float4 dl = del4[(c0 >> 2) + k4];
          const int q = c0 + 4 * k4;
          pk[2 * k4] = pack_bf16x2(__uint_as_float(s[q]) * (__uint_as_float(dp[4 * k4]) - dl.x),
                                   __uint_as_float(s[q + 1]) * (__uint_as_float(dp[4 * k4 + 1]) - dl.y));
          pk[2 * k4 + 1] = pack_bf16x2(__uint_as_float(s[q + 2]) * (__uint_as_float(dp[4 * k4 + 2]) - dl.z),
                                       __uint_as_float(s[q + 3]) * (__uint_as_float(dp[4 * k4 + 3]) - dl.w));
        }
        tmem_st16(tDP + c0 / 2, pk);
        if (kDs) {
          // the same bf16 values for the dQ GEMM: 8 queries (16 bytes) per
          // store, lanes on consecutive keys (512 contiguous bytes a warp)
#pragma unroll
          for (int g = 0; g < 4; ++g)
            st_shared_v4(ds_stage + ((c0 >> 3) + g) * 512 + lane * 16, pk[4 * g], pk[4 * g + 1], pk[4 * g + 2],
                         pk[4 * g + 3]);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sb + BAR_DS);
      if (kDs) {
        // After dS is published (the proxy fence waits for this thread's
        // shared-memory writes): the bulk store drains in the background
        // while the row threads go on, evicted first from L2, where the Q
        // and dO tiles that every CTA of the head walks should stay.
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) {
          bulk_store_hint(ds_dst, ds_stage, 4096, l2_evict_first_policy());
          bulk_commit();
        }
      }
    }
    if (kDs && lane == 0) bulk_wait_all();
    if (ok && n > 0) {
      const bool w = mbar_wait(sb + BAR_ACC, 0, abort_flag, tmo, SITE_EPILOGUE);
      if (__any_sync(0xffffffffu, !w)) ok = false;
      __syncwarp();
      tc_fence_after();
    }
    if (ok) {
      // each half of the row writes half of the D columns of dV and of dK
      const int d0 = half * (D / 2);
      const long long roff = (row_valid ? bwd_out_elems<D>(PB, p.B, p.S, U.b, k_pos, U.h) : 0) + d0;
      for (int which = 0; which < 2; ++which) {   // 0: dV, 1: dK (times the softmax scale)
        const float mul = which == 0 ? 1.0f : p.scale;
        __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(which == 0 ? PB.dv : PB.dk) + roff;
        const uint32_t tsrc = (which == 0 ? tDV : tDK) + d0;
#pragma unroll
        for (int c0 = 0; c0 < D / 2; c0 += 32) {
          uint32_t o[32];
          if (n > 0) {
            tmem_ld32_wait(tsrc + c0, o);
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = 0u;
          }
          if (row_valid) {
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + c0);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              d4[k] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * k]) * mul, __uint_as_float(o[8 * k + 1]) * mul),
                                 pack_bf16x2(__uint_as_float(o[8 * k + 2]) * mul, __uint_as_float(o[8 * k + 3]) * mul),
                                 pack_bf16x2(__uint_as_float(o[8 * k + 4]) * mul, __uint_as_float(o[8 * k + 5]) * mul),
                                 pack_bf16x2(__uint_as_float(o[8 * k + 6]) * mul, __uint_as_float(o[8 * k + 7]) * mul));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBwdTmemCols);
  }
}

// ============================================================== dQ GEMM
// dQ = dS K * scale over the dS tiles that the dK/dV kernel stored, so that S
// and dP are not computed a second time: per unit (b, h, Q tile) the products
// of the walked K tiles accumulate in TMEM.  A is the dS tile, MN-major
// (queries contiguous in groups of 8, the un-swizzled core-matrix layout) and
// loaded with one 32 KB bulk copy; B is the K tile, MN-major with the 128-byte
// swizzle (as in the dQ kernel).  The kernel is bound by the HBM reads of the
// dS tiles (32 KB per tile pair).  Persistent: one CTA per SM walks the units
// blockIdx.x, blockIdx.x + gridDim.x, ...; two TMEM accumulators, so that the
// epilogue of one unit overlaps the loads and MMAs of the next.  Units run
// head by head (the CTAs at work share a few heads' K tiles in L2); under the
// causal mask in pairs of equal total length (bwd_gemm_unit).
//   warp 0      producer: the dS tile (bulk copy) and the K tile (TMA) per stage
//   warp 1      TMEM allocator + single-thread MMA issuer
//   warps 2-5   epilogue: one dQ row per thread (TMEM lane), scaled, bf16
template <int D>
struct BwdGemmSmem {
  static constexpr int kATile = kBwdDsTileBytes;            // dS tile, 32 KB
  static constexpr int kBTile = BwdSmem<D>::kTileBytes;     // K tile
  static constexpr int kStage = kATile + kBTile;            // a multiple of 1024: the K tile stays swizzle-aligned
  static constexpr int kStages = D == 128 ? 3 : 4;
  static constexpr int kOffBar = kStages * kStage;
  static constexpr int kNumBars = 2 * kStages + 5;          // full[S], empty[S], acc_full[2], acc_empty[2], tail
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 16;
  static constexpr int kAllocBytes = kBytes;
};
static_assert(BwdGemmSmem<128>::kAllocBytes <= 232448 && BwdGemmSmem<64>::kAllocBytes <= 232448,
              "dQ GEMM shared memory exceeds the per-CTA limit");
constexpr int kBwdGemmThreads = 192;

// The k-th unit of this CTA's walk.  The CTA takes work items blockIdx.x,
// blockIdx.x + gridDim.x, ... in head order.  Without the causal mask an item
// is one Q tile.  Under it an item pairs Q tile nt - 1 - j with Q tile j of
// the same (b, h): together they walk nt + 1 K tiles, so that every item has
// the same length and the round-robin stays balanced.  Returns 0 when the walk
// is done, 1 for a unit, -1 for the second of a pair that is its first (the
// middle tile of an odd nt), which every role skips alike.
__device__ __forceinline__ int bwd_gemm_unit(const BwdParams &p, int k, bool causal, BwdUnit &u) {
  const int nt = (p.S + 127) / 128;
  const int per = causal ? (nt + 1) / 2 : nt;   // items per (b, h)
  const int sub = causal ? (k & 1) : 0;
  int item = static_cast<int>(blockIdx.x) + (causal ? (k >> 1) : k) * static_cast<int>(gridDim.x);
  int pi = 0;
  for (; pi < p.n_prob; ++pi) {
    const int items = p.B * p.prob[pi].nh * per;
    if (item < items) break;
    item -= items;
  }
  if (pi == p.n_prob) return 0;
  const int bh = item / per, j = item - bh * per;
  const int NH = p.prob[pi].nh;
  u.pi = pi;
  u.hl = bh % NH;
  u.h = p.prob[pi].h0 + u.hl;
  u.b = bh / NH;
  if (!causal) {
    u.t = j;
    return 1;
  }
  u.t = sub == 0 ? nt - 1 - j : j;
  return (sub == 1 && j == nt - 1 - j) ? -1 : 1;
}

template <int D>
__global__ void __launch_bounds__(kBwdGemmThreads, 1)
    attn_bwd_dq_gemm_kernel(const __grid_constant__ BwdParams p) {
  using L = BwdGemmSmem<D>;
  using T = BwdSmem<D>;
  constexpr uint32_t IDESC = idesc_bf16_f32(128, D, true, true);   // dS and K both MN-major
  constexpr uint32_t kAccCols = 2 * D;
  extern __shared__ __align__(1024) uint8_t bwd_smem[];
  const uint32_t sb = smem_u32(bwd_smem);
  if (sb & 1023u) {
    if (threadIdx.x == 0) atomicOr(&g_device_status, SITE_LAYOUT);
    return;
  }
  constexpr int ST = L::kStages;
  constexpr uint32_t BAR_FULL = L::kOffBar;                 // [ST] stage loaded
  constexpr uint32_t BAR_EMPTY = BAR_FULL + 8 * ST;         // [ST] stage consumed by the MMAs
  constexpr uint32_t BAR_AF = BAR_EMPTY + 8 * ST;           // [2] accumulator complete
  constexpr uint32_t BAR_AE = BAR_AF + 16;                  // [2] accumulator read out
  constexpr uint32_t BAR_TAIL = BAR_AE + 16;
  constexpr uint32_t TMEM_SLOT = L::kOffMisc;
  constexpr uint32_t ABORT = L::kOffMisc + 4;
  static_assert(BAR_TAIL + 8 <= L::kOffMisc, "barrier area");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t tmo = p.timeout_ns;
  const int nt = (p.S + 127) / 128;
  const bool causal = p.causal != 0;
  // K tiles a Q tile walks: the keys at or before its last query (causal).
  auto walked = [&](int t) {
    const int q0 = t * 128;
    const int kv_len = causal ? min(p.S, q0 + 128) : p.S;
    return (kv_len + 127) / 128;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(sb + BAR_FULL + 8 * s, 1);
      mbar_init(sb + BAR_EMPTY + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(sb + BAR_AF + 8 * a, 1);
      mbar_init(sb + BAR_AE + 8 * a, 4);   // one arrival per epilogue warp
    }
    mbar_init(sb + BAR_TAIL, 1);
    st_shared_volatile(sb + ABORT, 0u);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sb + TMEM_SLOT, kAccCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ld_shared_volatile(sb + TMEM_SLOT);
  const uint32_t abort_flag = sb + ABORT;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (int pi = 0; pi < p.n_prob; ++pi) tma_prefetch_desc(&p.prob[pi].tm_k);
      // the dS tiles are read once: evicted first, so that the K tiles, read
      // by every Q tile of their head, stay in L2
      const uint64_t once = l2_evict_first_policy();
      int it = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        BwdUnit U;
        const int got = bwd_gemm_unit(p, k, causal, U);
        if (got == 0) break;
        if (got < 0) continue;
        const BwdProblem &PB = p.prob[U.pi];
        const int n = walked(U.t);
        const unsigned char *a0 = PB.ds + bwd_ds_tile_index(U.b, U.hl, PB.nh, nt, U.t, 0, causal) * kBwdDsTileBytes;
        for (int j = 0; j < n; ++j, ++it) {
          const int st = it % ST;
          if (!mbar_wait(sb + BAR_EMPTY + 8 * st, ((it / ST) & 1) ^ 1, abort_flag, tmo, SITE_PRODUCER)) {
            ok = false;
            break;
          }
          const uint32_t full = sb + BAR_FULL + 8 * st;
          const uint32_t dst = sb + st * L::kStage;
          mbar_arrive_expect_tx(full, L::kStage);
          bulk_load_hint(dst, a0 + static_cast<long long>(j) * kBwdDsTileBytes, L::kATile, full, once);
          for (int hf = 0; hf < T::kHalves; ++hf)
            tma_load_3d(dst + L::kATile + hf * T::kBoxBytes, &PB.tm_k, hf * 64, U.h, U.b * p.S + j * 128, full);
        }
      }
      // Before the CTA exits, every stage's last use has been consumed by the
      // MMAs (so its loads landed) and its release arrived here (bounded).
      for (int j = 0; j < ST && j < it; ++j) {
        const int i = it - 1 - j;
        mbar_wait(sb + BAR_EMPTY + 8 * (i % ST), (i / ST) & 1, 0u, tmo, SITE_TAIL);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, local = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        BwdUnit U;
        const int got = bwd_gemm_unit(p, k, causal, U);
        if (got == 0) break;
        if (got < 0) continue;
        const int n = walked(U.t);
        const int a = local & 1;
        const uint32_t use = static_cast<uint32_t>(local >> 1);   // uses of accumulator a before this one
        ++local;
        if (!mbar_wait_spin(sb + BAR_AE + 8 * a, (use & 1) ^ 1, abort_flag, tmo, SITE_MMA)) break;
        tc_fence_after();
        const uint32_t d = tmem + a * D;
        for (int j = 0; j < n; ++j, ++it) {
          const int st = it % ST;
          if (!mbar_wait_spin(sb + BAR_FULL + 8 * st, (it / ST) & 1, abort_flag, tmo, SITE_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // dS: core matrices of 8 keys x 8 queries, 128 bytes apart along the
          // keys (LBO) and 512 bytes apart along the queries (SBO); the 16
          // keys of MMA kk start at quarter kk / 2 (8 KB each), half kk % 2.
          // K: rows of 128 bytes, 16 keys = 2048 bytes.
          const uint64_t da = opaque_u64(smem_desc_plain(sb + st * L::kStage, 128, 512));
          const uint64_t db = opaque_u64(smem_desc_sw128(sb + st * L::kStage + L::kATile, T::kBoxBytes, 1024));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(d, da + ((((kk >> 1) * 8192) + (kk & 1) * 256) >> 4), db + ((kk * 2048) >> 4), IDESC,
                   (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(sb + BAR_EMPTY + 8 * st);
        }
        if (ok) mma_commit(sb + BAR_AF + 8 * a);
      }
      // Drain: every issued MMA has completed before TMEM is released.
      mma_commit(sb + BAR_TAIL);
      mbar_wait(sb + BAR_TAIL, 0, 0u, tmo, SITE_TAIL);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;   // accumulator row = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    int local = 0;
    for (int k = 0;; ++k) {
      BwdUnit U;
      const int got = bwd_gemm_unit(p, k, causal, U);
      if (got == 0) break;
      if (got < 0) continue;
      const int a = local & 1;
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      ++local;
      const bool w = mbar_wait(sb + BAR_AF + 8 * a, use & 1, abort_flag, tmo, SITE_EPILOGUE);
      if (__any_sync(0xffffffffu, !w)) break;
      __syncwarp();
      tc_fence_after();
      const BwdProblem &PB = p.prob[U.pi];
      const int q = U.t * 128 + r;
      const bool row_ok = q < p.S;
      __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(PB.dq) + (row_ok ? bwd_out_elems<D>(PB, p.B, p.S, U.b, q, U.h) : 0);
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t v[32];
        __syncwarp();
        tmem_ld32_wait(tmem + lane_base + a * D + c, v);   // the whole warp, converged
        if (!row_ok) continue;
        uint4 *d4 = reinterpret_cast<uint4 *>(dst + c);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          d4[k] = make_uint4(
              pack_bf16x2(__uint_as_float(v[8 * k]) * p.scale, __uint_as_float(v[8 * k + 1]) * p.scale),
              pack_bf16x2(__uint_as_float(v[8 * k + 2]) * p.scale, __uint_as_float(v[8 * k + 3]) * p.scale),
              pack_bf16x2(__uint_as_float(v[8 * k + 4]) * p.scale, __uint_as_float(v[8 * k + 5]) * p.scale),
              pack_bf16x2(__uint_as_float(v[8 * k + 6]) * p.scale, __uint_as_float(v[8 * k + 7]) * p.scale));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sb + BAR_AE + 8 * a);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kAccCols);
  }
}

}  // namespace cpattn
