// attn_kernel.cuh -- blockwise non-causal softmax attention for sm_100a.
//
// What it computes (diffusers "Context parallelism", "Ring Attention": each
// GPU computes attention against the K/V block it holds, then passes it on;
// diffusers "parallel", convert_to_fp32: output and LSE kept in float32;
// SGLang "Sequence Parallelism", "Numerics across node boundaries": the
// partial results are combined by an online-softmax merge):
//   for a 128-row Q tile and the K/V row ranges of its segment, visited in the
//   order given (ring order for ring attention), one 128-key tile at a time:
//     S = Q K^T                      (tcgen05.mma, bf16 x bf16 -> f32 in TMEM)
//     m <- max(m, rowmax(S) * c)     (c = D**-0.5 * log2 e; the stored m is only
//                                     raised when it grows by more than 8, so
//                                     O and l are rescaled rarely -- exact either way)
//     P = 2^(S*c - m)                (registers, bf16 into TMEM over S)
//     O = O * 2^(m_old - m) + P V    (tcgen05.mma, P from TMEM, V from smem)
//     l = l * 2^(m_old - m) + rowsum(P)
//   out = O / l, LSE = (m + log2 l) * ln 2.
// The running (m, l, O) state *is* the LSE merge applied one chunk (and one
// tile) at a time, so ring attention is one launch with no partials in HBM.
//
// CTA organisation (one CTA per SM: 192 KB smem, 512 TMEM columns), two
// "slots" each with a 128-row Q tile, its S (scores / P) and O in TMEM:
//   warp 0      TMA producer: Q, then K and V tiles into 2-stage rings
//   warp 1      TMEM allocator + single-thread MMA issuer
//   warps 2-3   idle
//   warps 4-7   softmax + correction + epilogue for slot 0 (one row per thread)
//   warps 8-11  the same for slot 1
// A unit is either
//   * a pair: two consecutive Q tiles of a segment, one per slot, both walking
//     the segment's whole K/V tile list (each K/V tile serves both slots), or
//   * a split (a lone Q tile left over at the end of a segment): the same Q
//     tile in both slots, slot 0 walking the first half of the K/V tile list
//     and slot 1 the second half, each with its own K/V stage; the two partial
//     (m, l, O) states are merged with the LSE rule at the end.  This keeps
//     two softmax streams in flight for a lone tile instead of serialising
//     one tile's softmax and MMAs.
// TMEM columns: S0 [0,128)  S1 [128,256)  O0 [256, 256+D)  O1 [256+D, 256+2D);
// P_i (bf16 pairs) overwrites S_i columns [0, 64).
// MMA order per step j: PV0(j), QK0(j+1), PV1(j), QK1(j+1), so that the
// tensor core works on one slot while the other slot's softmax runs.  A
// commit after QK_i(j) also covers PV_i(j-1), so when softmax i sees S_i(j),
// O_i already holds every earlier tile and may be rescaled in place.  P is
// published in two halves so that PV starts on keys 0-63 while keys 64-127
// are still being exponentiated.
#pragma once

#include "cpattn_internal.h"
#include "cpattn_ptx.cuh"

namespace cpattn {

template <int D>
struct AttnSmem {
  static constexpr int kHalves = D / 64;             // 64-element (128-byte) column blocks
  static constexpr int kBoxBytes = 128 * 128;        // [128 rows][64 bf16], 128B-swizzled
  static constexpr int kTileBytes = kHalves * kBoxBytes;
  static constexpr int kStages = 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQTilesPerCTA * kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  // q, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_full[2], o_final[2], tail, p_half[2], ml
  static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 + 2 + 1 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffML = kOffMisc + 16;        // split units: slot 1's m[128], l[128]
  static constexpr int kBytes = kOffML + 2 * 128 * 4;
  static constexpr int kAllocBytes = kBytes + 1024;  // slack to align the base to 1024
};

constexpr int kAttnThreads = 384;
constexpr uint32_t kTmemCols = 512;
// Register split: launched at 168 per thread (384 x 168 = 64512); the
// producer/MMA warpgroup drops to 104 and the two softmax warpgroups rise to
// 200: 128 x 104 + 256 x 200 = 64512, exactly the launch allocation.  (The
// softmax row -- 128 fp32 scores -- lives in registers.)
constexpr int kRegsLaunch = 168;
constexpr int kRegsControl = 104;
constexpr int kRegsSoftmax = 200;
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= kAttnThreads * kRegsLaunch, "register split exceeds launch");
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale only if the max grows by > 2^8

// The work unit of this CTA: group -> head -> segment -> pair of Q tiles (or a
// split lone tile).  Recomputed inside every role (after its register budget
// is set) so that no decoded value stays live across the role split.
struct Unit {
  int gi, si, h, pair, q_row0, rows_left, n_tiles;
  int q_last;      // sequence position of the unit's last query row
  int n0, n1;      // K/V tiles walked by slot 0 / slot 1
  bool has_q1;     // pair with a second Q tile
  bool split;      // lone tile whose K/V list is split between the slots
};

// Rows of K/V range `kv` that a unit walks: all of them, or under the causal
// mask those at positions <= q_last (later rows are invisible to every query
// of the unit).
__device__ __forceinline__ int kv_rows_seen(const AttnParams &p, const AttnKV &kv, int q_last) {
  return p.causal ? max(0, min(kv.nrows, q_last - kv.s0 + 1)) : kv.nrows;
}

__device__ __forceinline__ Unit decode_unit(const AttnParams &p) {
  Unit u;
  const int unit = blockIdx.x;
  int gi = 0;
  while (gi + 1 < p.num_groups && p.group[gi + 1].unit_base <= unit) ++gi;
  const AttnGroup &G = p.group[gi];
  const int local = unit - G.unit_base;
  int t;
  if (!p.causal) {
    // Head-major: the CTAs running at once share one head's K/V through L2.
    u.h = local / G.tiles_per_head;
    t = local - u.h * G.tiles_per_head;
  } else {
    // Causal units differ in length: within a block of heads whose K/V fit
    // in L2 together, order them pair-major (the pair order below runs
    // heaviest first), so the launch order is close to longest first.
    const int H = p.prob[G.prob].H;
    const int block = local / (G.head_block * G.tiles_per_head);
    const int h0 = block * G.head_block;
    const int nb = min(G.head_block, H - h0);
    const int within = local - h0 * G.tiles_per_head;
    t = within / nb;
    u.h = h0 + (within - t * nb);
  }
  int si = G.seg_first;
  while (si + 1 < G.seg_first + G.seg_count && p.seg[si + 1].tile_base <= t) ++si;
  const AttnSeg &SG = p.seg[si];
  u.gi = gi;
  u.si = si;
  u.pair = t - SG.tile_base;
  // Under the causal mask a later pair walks more K/V tiles: launch a
  // segment's pairs last-first so the heaviest units start in the first wave.
  if (p.causal) u.pair = (SG.nrows + kQTilesPerCTA * kQTile - 1) / (kQTilesPerCTA * kQTile) - 1 - u.pair;
  u.q_row0 = SG.row0 + u.pair * (kQTilesPerCTA * kQTile);
  u.rows_left = SG.nrows - u.pair * (kQTilesPerCTA * kQTile);
  u.has_q1 = u.rows_left > kQTile || SG.q1_rows > 0;
  u.q_last = SG.s0 + u.pair * (kQTilesPerCTA * kQTile) + min(u.rows_left, kQTilesPerCTA * kQTile) - 1;
  int n = 0;
  for (int i = 0; i < SG.kv_count; ++i) n += (kv_rows_seen(p, p.kv[SG.kv_first + i], u.q_last) + kKVTile - 1) / kKVTile;
  u.n_tiles = n;
  u.split = SG.split != 0 && !u.has_q1 && n >= 2;
  if (u.split) {
    u.n0 = (n + 1) / 2;
    u.n1 = n - u.n0;
  } else {
    u.n0 = n;
    u.n1 = u.has_q1 ? n : 0;
    if (p.causal && u.has_q1) {
      // The first Q tile of a causal pair sees keys up to its own last row
      // only.  When the tiles it cannot see form a suffix of the walk (the
      // plan lists the chunk that the mask cuts last), slot 0 stops after the
      // prefix it sees; otherwise it walks every tile, fully masked ones too.
      const int q_last0 = SG.s0 + u.pair * (kQTilesPerCTA * kQTile) + kQTile - 1;
      int n0 = 0;
      bool cut = false, prefix = true;
      for (int i = 0; i < SG.kv_count; ++i) {
        const AttnKV kv = p.kv[SG.kv_first + i];
        const int t_all = (kv_rows_seen(p, kv, u.q_last) + kKVTile - 1) / kKVTile;
        const int t_own = (kv_rows_seen(p, kv, q_last0) + kKVTile - 1) / kKVTile;
        if (cut && t_all > 0) prefix = false;
        n0 += t_own;
        if (t_own < t_all) cut = true;
      }
      if (prefix && n0 >= 1) u.n0 = n0;
    }
  }
  return u;
}

// Row and number of valid keys of K/V tile `g` of a unit (tiles are numbered
// across the segment's K/V ranges in order, each range cut to the rows the
// unit walks).
__device__ __forceinline__ void kv_tile(const AttnParams &p, const AttnSeg &SG, int q_last, int g, int &row,
                                        int &valid) {
  for (int i = 0; i < SG.kv_count; ++i) {
    const AttnKV kv = p.kv[SG.kv_first + i];
    const int seen = kv_rows_seen(p, kv, q_last);
    const int nt = (seen + kKVTile - 1) / kKVTile;
    if (g < nt) {
      row = kv.row0 + g * kKVTile;
      valid = min(kKVTile, seen - g * kKVTile);
      return;
    }
    g -= nt;
  }
  row = 0;
  valid = 0;
}

// Element offset of output row (batch b, sequence position s, Q row grow)
// of head h, by the problem's output map (see AttnProblem).
template <int D>
__device__ __forceinline__ size_t out_row_elems(const AttnProblem &PB, int b, int s, int grow, int h) {
  if (PB.out_mode == 0) return (static_cast<size_t>(grow) * PB.H + h) * D;
  long long row;
  if (PB.out_mode == 1) {
    int lo = 0, hi = PB.out_nseq - 1;   // the sequence rank holding s (empty ranks skipped)
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (PB.out_seq_off[mid] <= s) lo = mid; else hi = mid - 1;
    }
    const int off = PB.out_seq_off[lo], len = PB.out_seq_off[lo + 1] - off;
    row = static_cast<long long>(PB.out_B) * off + static_cast<long long>(b) * len + (s - off);
  } else {
    row = static_cast<long long>(b) * PB.out_S + s;
  }
  return (static_cast<size_t>(row) * PB.out_H + PB.out_h0 + h) * D;
}

template <int D, bool OUT_F32>
__global__ void __launch_bounds__(kAttnThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  using L = AttnSmem<D>;
  constexpr int NST = L::kStages;
  constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, kKVTile, false);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);

  extern __shared__ uint8_t smem_raw[];
  // 32-bit shared-window addresses of everything (1024-aligned base).
  const uint32_t sb = (smem_u32(smem_raw) + 1023u) & ~1023u;
  constexpr uint32_t BAR_Q = L::kOffBar;
  constexpr uint32_t BAR_KF = BAR_Q + 8;               // [NST]
  constexpr uint32_t BAR_KE = BAR_KF + 8 * NST;        // [NST]
  constexpr uint32_t BAR_VF = BAR_KE + 8 * NST;        // [NST]
  constexpr uint32_t BAR_VE = BAR_VF + 8 * NST;        // [NST]
  constexpr uint32_t BAR_S = BAR_VE + 8 * NST;         // [2]
  constexpr uint32_t BAR_P = BAR_S + 16;               // [2]
  constexpr uint32_t BAR_O = BAR_P + 16;               // [2]
  constexpr uint32_t BAR_TAIL = BAR_O + 16;
  constexpr uint32_t BAR_PH = BAR_TAIL + 8;            // [2] first half of P written
  constexpr uint32_t BAR_ML = BAR_PH + 16;             // split: slot 1's (m, l) published
  constexpr uint32_t TMEM_SLOT = L::kOffMisc;
  constexpr uint32_t ABORT = L::kOffMisc + 4;
  static_assert(BAR_ML + 8 <= L::kOffMisc, "barrier area");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t tmo = p.timeout_ns;

  // ---- setup
  if (threadIdx.x == 0) {
    mbar_init(sb + BAR_Q, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(sb + BAR_KF + 8 * s, 1);
      mbar_init(sb + BAR_KE + 8 * s, 1);
      mbar_init(sb + BAR_VF + 8 * s, 1);
      mbar_init(sb + BAR_VE + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(sb + BAR_S + 8 * i, 1);
      mbar_init(sb + BAR_P + 8 * i, 4);  // one arrival per softmax warp
      mbar_init(sb + BAR_O + 8 * i, 1);
    }
    mbar_init(sb + BAR_TAIL, 1);
    mbar_init(sb + BAR_PH, 4);        // one arrival per softmax warp
    mbar_init(sb + BAR_PH + 8, 4);
    mbar_init(sb + BAR_ML, 4);        // one arrival per warp of softmax warpgroup 1
    st_shared_volatile(sb + ABORT, 0u);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sb + TMEM_SLOT, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ld_shared_volatile(sb + TMEM_SLOT);
  const uint32_t abort_flag = sb + ABORT;

  if (warp < 4) {
   setmaxnreg_dec<kRegsControl>();
   const Unit U = decode_unit(p);
   const AttnSeg &SG = p.seg[U.si];
   const AttnProblem &PB = p.prob[p.group[U.gi].prob];
   const int h = U.h, q_row0 = U.q_row0, n_tiles = U.n_tiles, n0 = U.n0, n1 = U.n1;
   const bool has_q1 = U.has_q1, split = U.split;
   if (warp == 0) {
    // =========================================================== producer
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&PB.tm_q);
      tma_prefetch_desc(&PB.tm_k);
      tma_prefetch_desc(&PB.tm_v);
      const uint32_t sQ = sb + L::kOffQ;
      mbar_arrive_expect_tx(sb + BAR_Q, (has_q1 ? 2 : 1) * L::kTileBytes);
      for (int hf = 0; hf < L::kHalves; ++hf)
        tma_load_3d(sQ + hf * L::kBoxBytes, &PB.tm_q, hf * 64, h, q_row0, sb + BAR_Q);
      if (has_q1) {
        const int q1_row = SG.q1_rows > 0 ? SG.q1_row0 : q_row0 + kQTile;   // a paired lone tile, or the next one
        for (int hf = 0; hf < L::kHalves; ++hf)
          tma_load_3d(sQ + L::kTileBytes + hf * L::kBoxBytes, &PB.tm_q, hf * 64, h, q1_row, sb + BAR_Q);
      }
      bool ok = true;
      auto load_kv = [&](int st, uint32_t ph, int row) -> bool {
        if (!mbar_wait(sb + BAR_KE + 8 * st, ph ^ 1, abort_flag, tmo, SITE_PRODUCER)) return false;
        mbar_arrive_expect_tx(sb + BAR_KF + 8 * st, L::kTileBytes);
        const uint32_t sK = sb + L::kOffK + st * L::kTileBytes;
        for (int hf = 0; hf < L::kHalves; ++hf)
          tma_load_3d(sK + hf * L::kBoxBytes, &PB.tm_k, hf * 64, h, row, sb + BAR_KF + 8 * st);
        if (!mbar_wait(sb + BAR_VE + 8 * st, ph ^ 1, abort_flag, tmo, SITE_PRODUCER)) return false;
        mbar_arrive_expect_tx(sb + BAR_VF + 8 * st, L::kTileBytes);
        const uint32_t sV = sb + L::kOffV + st * L::kTileBytes;
        for (int hf = 0; hf < L::kHalves; ++hf)
          tma_load_3d(sV + hf * L::kBoxBytes, &PB.tm_v, hf * 64, h, row, sb + BAR_VF + 8 * st);
        return true;
      };
      if (!split) {
        // Tiles in order through the NST-stage ring.
        int it = 0;
        for (int i = 0; ok && i < SG.kv_count; ++i) {
          const AttnKV kv = p.kv[SG.kv_first + i];
          const int seen = kv_rows_seen(p, kv, U.q_last);
          for (int r = 0; r < seen; r += kKVTile, ++it)
            if (!load_kv(it % NST, (it / NST) & 1, kv.row0 + r)) { ok = false; break; }
        }
      } else {
        // Slot 0's tile j and slot 1's tile j alternate; slot s uses stage s.
        for (int j = 0; ok && j < n0; ++j) {
          int row, valid;
          kv_tile(p, SG, U.q_last, j, row, valid);
          if (!load_kv(0, j & 1, row)) { ok = false; break; }
          if (j < n1) {
            kv_tile(p, SG, U.q_last, n0 + j, row, valid);
            if (!load_kv(1, j & 1, row)) { ok = false; break; }
          }
        }
      }
      // Tail: every stage's last use must be released by the MMA before the
      // CTA exits (the releases are asynchronous arrivals on our barriers).
      for (int st = 0; st < NST; ++st) {
        int uses;   // loads that went to stage st
        if (split) uses = st == 0 ? n0 : n1;
        else uses = n_tiles > st ? (n_tiles - 1 - st) / NST + 1 : 0;
        if (uses == 0) continue;
        const uint32_t ph = split ? ((uses - 1) & 1) : (((uses - 1) * NST + st) / NST) & 1;
        mbar_wait(sb + BAR_KE + 8 * st, ph, 0u, tmo, SITE_TAIL);
        mbar_wait(sb + BAR_VE + 8 * st, ph, 0u, tmo, SITE_TAIL);
      }
    }
   } else if (warp == 1) {
    // =========================================================== MMA issuer
    if (lane == 0 && n_tiles > 0) {
      const uint32_t sQ = sb + L::kOffQ;
      const uint32_t sK = sb + L::kOffK;
      const uint32_t sV = sb + L::kOffV;
      // S_s = Q K^T: K-major A and B, 128B swizzle, K advances 16 elements
      // (32 bytes) inside a 128-byte row, then jumps to the next column block.
      // Descriptors are built once; advancing the start address only
      // touches the low 14 bits (addresses stay below 256 KB, no carry).
      const uint64_t dQ = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dK = smem_desc_sw128(sK, 16, 1024);
      const uint64_t dV = smem_desc_sw128(sV, L::kBoxBytes, 1024);
      // slot s: S/P in TMEM columns s*128, O at 256 + s*D; its Q tile is
      // smem tile s for a pair, tile 0 (the same rows) for a split.
      auto issue_qk = [&](int s, int st) {
        const uint32_t d = tmem + s * 128;
        const uint64_t a0 = opaque_u64(dQ + (((split ? 0 : s) * L::kTileBytes) >> 4));
        const uint64_t b0 = opaque_u64(dK + ((st * L::kTileBytes) >> 4));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * L::kBoxBytes + (kk & 3) * 32) >> 4;
          mma_ss(d, a0 + off, b0 + off, IDESC_QK, kk > 0 ? 1u : 0u);
        }
      };
      // O_s (+)= P_s V: P (bf16 pairs) from TMEM over S_s, V MN-major
      // (keys are rows of 128 bytes): 16 keys = 2 groups of 8 rows = 2048
      // bytes per MMA, column blocks of 64 head-dim elements 16 KB apart.
      // Half h of the keys (kk = 4h .. 4h+3).
      auto issue_pv = [&](int s, int st, bool acc, int half) {
        const uint32_t d = tmem + 256 + s * D;
        const uint32_t a = tmem + s * 128;
        const uint64_t b0 = opaque_u64(dV + ((st * L::kTileBytes) >> 4));
#pragma unroll
        for (int k4 = 0; k4 < kKVTile / 32; ++k4) {
          const int kk = half * (kKVTile / 32) + k4;
          mma_ts(d, a + kk * 8, b0 + ((kk * 2048) >> 4), IDESC_PV, (acc || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait_spin(sb + BAR_Q, 0, abort_flag, tmo, SITE_MMA);
      if (!split) {
        // Pair (or a lone tile with one K/V tile): both slots read every K/V
        // stage; a stage is released after slot 1 (or slot 0 alone) read it.
        if (ok) ok = mbar_wait_spin(sb + BAR_KF, 0, abort_flag, tmo, SITE_MMA);
        if (ok) {
          tc_fence_after();
          issue_qk(0, 0);
          mma_commit(sb + BAR_S);
          if (has_q1) {
            issue_qk(1, 0);
            mma_commit(sb + BAR_S + 8);
          }
          mma_commit(sb + BAR_KE);
        }
        for (int j = 0; ok && j < n_tiles; ++j) {
          const int st = j % NST;
          const uint32_t ph = (j / NST) & 1;
          const int st1 = (j + 1) % NST;
          const uint32_t ph1 = ((j + 1) / NST) & 1;
          const bool more = j + 1 < n_tiles;
          if (!mbar_wait_spin(sb + BAR_VF + 8 * st, ph, abort_flag, tmo, SITE_MMA)) break;
          if (j < n0) {   // slot 0 may stop before slot 1 (causal pairs)
            if (!mbar_wait_spin(sb + BAR_PH, j & 1, abort_flag, tmo, SITE_MMA)) break;
            tc_fence_after();
            issue_pv(0, st, j > 0, 0);
            if (!mbar_wait_spin(sb + BAR_P, j & 1, abort_flag, tmo, SITE_MMA)) break;
            tc_fence_after();
            issue_pv(0, st, j > 0, 1);
            if (j == n0 - 1) mma_commit(sb + BAR_O);
          }
          if (more) {
            if (!mbar_wait_spin(sb + BAR_KF + 8 * st1, ph1, abort_flag, tmo, SITE_MMA)) break;
            tc_fence_after();
            if (j + 1 < n0) {
              issue_qk(0, st1);
              mma_commit(sb + BAR_S);
            }
          }
          if (has_q1) {
            if (!mbar_wait_spin(sb + BAR_PH + 8, j & 1, abort_flag, tmo, SITE_MMA)) break;
            tc_fence_after();
            issue_pv(1, st, j > 0, 0);
            if (!mbar_wait_spin(sb + BAR_P + 8, j & 1, abort_flag, tmo, SITE_MMA)) break;
            tc_fence_after();
            issue_pv(1, st, j > 0, 1);
            if (!more) mma_commit(sb + BAR_O + 8);
          }
          mma_commit(sb + BAR_VE + 8 * st);
          if (more) {
            if (has_q1) {
              issue_qk(1, st1);
              mma_commit(sb + BAR_S + 8);
            }
            mma_commit(sb + BAR_KE + 8 * st1);
          }
        }
      } else {
        // Split: slot s owns stage s; its j-th tile is that stage's j-th use.
        for (int s = 0; ok && s < 2; ++s) {
          if (!mbar_wait_spin(sb + BAR_KF + 8 * s, 0, abort_flag, tmo, SITE_MMA)) { ok = false; break; }
          tc_fence_after();
          issue_qk(s, s);
          mma_commit(sb + BAR_S + 8 * s);
          mma_commit(sb + BAR_KE + 8 * s);
        }
        for (int j = 0; ok && j < n0; ++j) {
          for (int s = 0; s < 2; ++s) {
            const int ns = s == 0 ? n0 : n1;
            if (j >= ns) continue;
            if (!mbar_wait_spin(sb + BAR_VF + 8 * s, j & 1, abort_flag, tmo, SITE_MMA)) { ok = false; break; }
            if (!mbar_wait_spin(sb + BAR_PH + 8 * s, j & 1, abort_flag, tmo, SITE_MMA)) { ok = false; break; }
            tc_fence_after();
            issue_pv(s, s, j > 0, 0);
            if (!mbar_wait_spin(sb + BAR_P + 8 * s, j & 1, abort_flag, tmo, SITE_MMA)) { ok = false; break; }
            tc_fence_after();
            issue_pv(s, s, j > 0, 1);
            if (j == ns - 1) mma_commit(sb + BAR_O + 8 * s);
            mma_commit(sb + BAR_VE + 8 * s);
            if (j + 1 < ns) {
              if (!mbar_wait_spin(sb + BAR_KF + 8 * s, (j + 1) & 1, abort_flag, tmo, SITE_MMA)) { ok = false; break; }
              tc_fence_after();
              issue_qk(s, s);
              mma_commit(sb + BAR_S + 8 * s);
              mma_commit(sb + BAR_KE + 8 * s);
            }
          }
        }
      }
      // Drain: everything issued has completed before TMEM is released.
      mma_commit(sb + BAR_TAIL);
      mbar_wait(sb + BAR_TAIL, 0, 0u, tmo, SITE_TAIL);
    }
   }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    const Unit U = decode_unit(p);
    const AttnSeg &SG = p.seg[U.si];
    const AttnGroup &G = p.group[U.gi];
    const AttnProblem &PB = p.prob[G.prob];
    const int h = U.h, q_row0 = U.q_row0, n_tiles = U.n_tiles, rows_left = U.rows_left, pair = U.pair;
    const int q_last = U.q_last;
    const bool has_q1 = U.has_q1, split = U.split;
    // =========================================================== softmax
    const int qt = (warp - 4) >> 2;            // slot
    const int row = ((warp & 3) << 5) + lane;  // TMEM lane == row of the Q tile
    const bool active = (qt == 0) || has_q1 || split;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) << 5) << 16;
    const uint32_t tS = tmem + lane_base + qt * 128;
    const uint32_t tO = tmem + lane_base + 256 + qt * D;
    const float c = p.scale_log2;
    // Sequence position of this thread's query row (both slots of a split
    // unit hold the same rows).
    const bool paired_lone = qt == 1 && SG.q1_rows > 0;   // slot 1 holds another shard's lone tile
    const int q_pos = paired_lone ? SG.q1_s0 + row
                                  : SG.s0 + pair * (kQTilesPerCTA * kQTile) + (split ? 0 : qt * kQTile) + row;
    const bool causal = p.causal != 0;
    // K/V tiles [g_lo, g_hi) of the segment belong to this slot.
    const int g_lo = (split && qt == 1) ? U.n0 : 0;
    const int g_hi = split ? (qt == 0 ? U.n0 : U.n0 + U.n1) : (qt == 0 ? U.n0 : n_tiles);
    float m = -INFINITY;  // running max, scaled (log2) domain
    float l = 0.f;        // running sum of 2^(x - m)
    bool ok = true;
    if (active && n_tiles > 0) {
      int g = 0;   // segment tile index; this slot handles g_lo <= g < g_hi
      for (int i = 0; ok && i < SG.kv_count && g < g_hi; ++i) {
        const AttnKV kv = p.kv[SG.kv_first + i];
        const int kv_n = kv_rows_seen(p, kv, q_last);
        for (int r = 0; r < kv_n && g < g_hi; r += kKVTile, ++g) {
          if (g < g_lo) continue;
          const int j = g - g_lo;
          // Keys of this tile visible to this row: the tile's valid keys, cut
          // under the causal mask at the row's own position (may be <= 0).
          int kvalid = min(kKVTile, kv_n - r);
          if (causal) kvalid = min(kvalid, q_pos - (kv.s0 + r) + 1);
          const bool w = mbar_wait(sb + BAR_S + 8 * qt, j & 1, abort_flag, tmo, SITE_SOFTMAX);
          if (__any_sync(0xffffffffu, !w)) { ok = false; break; }
          __syncwarp();
          tc_fence_after();
          uint32_t s[128];
          tmem_ld128_wait(tS, s);
          if (__any_sync(0xffffffffu, kvalid < kKVTile)) {
#pragma unroll
            for (int k = 0; k < 128; ++k)
              if (k >= kvalid) s[k] = __float_as_uint(-INFINITY);
          }
          // Row max: 8 independent chains of 3-input max.
          float mx[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = fmaxf(__uint_as_float(s[k]), __uint_as_float(s[k + 8]));
#pragma unroll
          for (int k = 16; k < 128; k += 16)
#pragma unroll
            for (int q = 0; q < 8; ++q) mx[q] = fmax3(mx[q], __uint_as_float(s[k + q]), __uint_as_float(s[k + 8 + q]));
          const float tmax = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * c;
          // Raise the stored max only when it grows by more than the
          // threshold; rows that keep a stale max see P <= 2^threshold.
          if (j == 0) {
            m = tmax;
          } else {
            const bool need = tmax > m + kRescaleThreshold;
            if (__any_sync(0xffffffffu, need)) {
              const float alpha = need ? ex2_approx(m - tmax) : 1.0f;
              if (need) {
                l *= alpha;
                m = tmax;
              }
              // O holds every earlier tile (the commit that published S
              // covered the previous PV): rescale it in place before this
              // tile's first PV.
#pragma unroll 1
              for (int c0 = 0; c0 < D; c0 += 16) {
                uint32_t o[16];
                tmem_ld16_wait(tO + c0, o);
#pragma unroll
                for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                tmem_st16(tO + c0, o);
              }
            }
          }
          // P = 2^(S*c - m), pairs of scores through packed f32x2 FMAs and
          // the exponentials on the SFU.  P is published in two halves (keys 0-63, 64-127) so that
          // the MMA warp starts PV on the first half while the second half
          // is computed.
          const uint64_t cc = f2_pack(c, c);
          // A row that has seen no key yet (only under the causal mask) keeps
          // m = -inf: exponentiate against 0 so its masked scores give P = 0.
          const float mb = m == -INFINITY ? 0.0f : m;
          const uint64_t mm = f2_pack(-mb, -mb);
          uint64_t lsum0 = 0, lsum1 = 0;   // packed partial row sums (0.0f bits)
#pragma unroll
          for (int c0 = 0; c0 < 128; c0 += 32) {
            uint32_t pk[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const uint64_t x = f2_fma(f2_pack(__uint_as_float(s[c0 + 2 * k]), __uint_as_float(s[c0 + 2 * k + 1])), cc, mm);
              float x0, x1;
              f2_unpack(x, x0, x1);
              const uint64_t pp = f2_pack(ex2_approx(x0), ex2_approx(x1));
              if (k & 1) lsum1 = f2_add(lsum1, pp); else lsum0 = f2_add(lsum0, pp);
              float p0, p1;
              f2_unpack(pp, p0, p1);
              pk[k] = pack_bf16x2(p0, p1);
            }
            tmem_st16(tS + c0 / 2, pk);
            if (c0 == 32) {
              tmem_st_wait();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(sb + BAR_PH + 8 * qt);
            }
          }
          {
            float a0, a1, b0, b1;
            f2_unpack(lsum0, a0, a1);
            f2_unpack(lsum1, b0, b1);
            l += (a0 + a1) + (b0 + b1);
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(sb + BAR_P + 8 * qt);
        }
      }
      if (ok) {
        const bool w = mbar_wait(sb + BAR_O + 8 * qt, 0, abort_flag, tmo, SITE_EPILOGUE);
        if (__any_sync(0xffffffffu, !w)) ok = false;
        __syncwarp();
        tc_fence_after();
      }
    }
    // =========================================================== epilogue
    if (split) {
      // Merge the two slots' partial states (same rows, disjoint keys) with
      // the LSE rule: slot 1 publishes (m, l) through shared memory, slot 0
      // combines O0 and O1 from TMEM and writes the rows.
      const uint32_t ml = sb + L::kOffML;
      if (qt == 1) {
        st_shared_f32(ml + 4 * row, m);            // published even after an abort,
        st_shared_f32(ml + 512 + 4 * row, l);      // so that slot 0 never waits in vain
        __syncwarp();
        if (lane == 0) mbar_arrive(sb + BAR_ML);
      } else {
        bool w = ok && mbar_wait(sb + BAR_ML, 0, abort_flag, tmo, SITE_EPILOGUE);
        w = w && mbar_wait(sb + BAR_O + 8, 0, abort_flag, tmo, SITE_EPILOGUE);
        if (__any_sync(0xffffffffu, !w)) ok = false;
        __syncwarp();
        tc_fence_after();
        if (ok) {
          const float m1 = ld_shared_f32(ml + 4 * row);
          const float l1 = ld_shared_f32(ml + 512 + 4 * row);
          const float mm = fmaxf(m, m1);
          const float a0 = ex2_approx(m - mm), a1 = ex2_approx(m1 - mm);
          const float lt = l * a0 + l1 * a1;
          const bool row_valid = row < rows_left;
          const int grow = q_row0 + row;
          const int sq = SG.s0 + pair * (kQTilesPerCTA * kQTile) + row;
          const size_t row_elems = out_row_elems<D>(PB, G.b, sq, grow, h);
          const long long lse_idx = static_cast<long long>(G.b) * PB.lse_b +
                                    static_cast<long long>(h + PB.lse_h0) * PB.lse_h + (sq - PB.lse_pos0);
          // This unit's own state (slots 0 and 1 merged), in log2 units, and
          // its merge with a previous partial state when the plan carries one.
          float own = lt > 0.0f ? mm + log2f(lt) : -INFINITY;
          float w0 = lt > 0.0f ? a0 / lt : 0.0f, w1 = lt > 0.0f ? a1 / lt : 0.0f, wp = 0.0f;
          const float *prev_row = nullptr;
          if (PB.prev != nullptr && row_valid) {
            const float lp = PB.lse[lse_idx] * 1.4426950408889634f;
            const float M = fmaxf(own, lp);
            if (M == -INFINITY) {
              w0 = w1 = 0.0f;
            } else {
              const float as = ex2_approx(own - M), ap = ex2_approx(lp - M);
              const float tot = as + ap;
              w0 *= as / tot;
              w1 *= as / tot;
              wp = ap / tot;
              own = M + log2f(tot);
              if (wp != 0.0f) prev_row = PB.prev + row_elems;
            }
          }
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o0[32], o1[32];
            tmem_ld32_wait(tO + c0, o0);
            tmem_ld32_wait(tO + D + c0, o1);
            float v[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(o0[k]) * w0 + __uint_as_float(o1[k]) * w1;
            if (prev_row != nullptr) {
              const float4 *src = reinterpret_cast<const float4 *>(prev_row + c0);
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const float4 pv = src[k];
                v[4 * k] += pv.x * wp;
                v[4 * k + 1] += pv.y * wp;
                v[4 * k + 2] += pv.z * wp;
                v[4 * k + 3] += pv.w * wp;
              }
            }
            if (row_valid) {
              if constexpr (OUT_F32) {
                float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(PB.out) + row_elems + c0);
#pragma unroll
                for (int k = 0; k < 8; ++k) dst[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
              } else {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(PB.out) + row_elems + c0);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  dst[k] = make_uint4(pack_bf16x2(v[8 * k], v[8 * k + 1]), pack_bf16x2(v[8 * k + 2], v[8 * k + 3]),
                                      pack_bf16x2(v[8 * k + 4], v[8 * k + 5]), pack_bf16x2(v[8 * k + 6], v[8 * k + 7]));
              }
            }
          }
          if (row_valid && PB.lse != nullptr) PB.lse[lse_idx] = own * 0.69314718055994531f;
        }
      }
    } else if (active && ok) {
      const int valid_rows = qt == 0 ? min(kQTile, rows_left) : (paired_lone ? SG.q1_rows : rows_left - kQTile);
      const bool row_valid = row < valid_rows;
      const int grow = paired_lone ? SG.q1_row0 + row : q_row0 + qt * kQTile + row;
      const int sq = paired_lone ? SG.q1_s0 + row : SG.s0 + pair * (kQTilesPerCTA * kQTile) + qt * kQTile + row;
      const size_t row_elems = out_row_elems<D>(PB, G.b, sq, grow, h);
      const long long lse_idx = static_cast<long long>(G.b) * PB.lse_b +
                                static_cast<long long>(h + PB.lse_h0) * PB.lse_h + (sq - PB.lse_pos0);
      // out = O * w_self + prev * w_prev: w_self = 1/l alone; with a previous
      // partial state (LSE read before it is overwritten) both are the LSE-rule
      // weights of the two states.
      float own = (n_tiles > 0 && l > 0.0f) ? m + log2f(l) : -INFINITY;   // log2 units
      float w_self = l > 0.0f ? 1.0f / l : 0.0f, wp = 0.0f;
      const float *prev_row = nullptr;
      if (PB.prev != nullptr && row_valid) {
        const float lp = PB.lse[lse_idx] * 1.4426950408889634f;
        const float M = fmaxf(own, lp);
        if (M == -INFINITY) {
          w_self = 0.0f;
        } else {
          const float as = ex2_approx(own - M), ap = ex2_approx(lp - M);
          const float tot = as + ap;
          w_self *= as / tot;
          wp = ap / tot;
          own = M + log2f(tot);
          if (wp != 0.0f) prev_row = PB.prev + row_elems;
        }
      }
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        if (n_tiles > 0) {
          tmem_ld32_wait(tO + c0, o);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = 0u;
        }
        float v[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(o[k]) * w_self;
        if (prev_row != nullptr) {
          const float4 *src = reinterpret_cast<const float4 *>(prev_row + c0);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float4 pv = src[k];
            v[4 * k] += pv.x * wp;
            v[4 * k + 1] += pv.y * wp;
            v[4 * k + 2] += pv.z * wp;
            v[4 * k + 3] += pv.w * wp;
          }
        }
        if (row_valid) {
          if constexpr (OUT_F32) {
            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(PB.out) + row_elems + c0);
#pragma unroll
            for (int k = 0; k < 8; ++k) dst[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
          } else {
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(PB.out) + row_elems + c0);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              dst[k] = make_uint4(pack_bf16x2(v[8 * k], v[8 * k + 1]), pack_bf16x2(v[8 * k + 2], v[8 * k + 3]),
                                  pack_bf16x2(v[8 * k + 4], v[8 * k + 5]), pack_bf16x2(v[8 * k + 6], v[8 * k + 7]));
          }
        }
      }
      if (row_valid && PB.lse != nullptr) PB.lse[lse_idx] = own * 0.69314718055994531f;
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if ((threadIdx.x >> 5) == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(ld_shared_volatile(((smem_u32(smem_raw) + 1023u) & ~1023u) + TMEM_SLOT), kTmemCols);
  }
}

}  // namespace cpattn
