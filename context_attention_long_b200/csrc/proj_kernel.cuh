// proj_kernel.cuh -- the Ulysses projections with the all-to-all fused in.
//
// The Ulysses flow (the Ulysses Sequence Parallelism article, section 4):
// each rank projects its own sequence chunk to Q, K and V, the first
// all-to-all regroups them by head, local attention runs, the second
// all-to-all regroups the output by token, and each rank applies the output
// projection to its own chunk.  Emulated on one GPU the all-to-alls are the
// permutations of permute_kernel.cuh; here they are folded into the two
// projection GEMMs instead:
//   QKV mode:  C = X W_qkv^T over the sequence-side token rows, and the
//              epilogue stores each (token, head) run of D outputs straight
//              into its head rank's buffer (the first all-to-all);
//   OUT mode:  C = O W_o^T over the tokens, whose A operand is loaded by TMA
//              from the head ranks' buffers (one tensor map per head rank,
//              chosen per 64-wide K block), and the epilogue stores each
//              token row into its sequence rank's buffer (the second
//              all-to-all).
// Layouts as in permute_kernel.cuh: the sequence side is the rank buffers
// (B, S_r, .) concatenated in rank order, the head side the rank buffers
// (B, S, H_u, D).  W is (N, K) row-major (the nn.Linear layout); the columns
// of W_qkv are [Q heads | K heads | V heads], head h at [h*D, (h+1)*D).
//
// Kernel: persistent, clusters of two CTAs on an SM pair.  Each cluster
// computes 256 x 256 output tiles with tcgen05.mma.cta_group::2 (M = 256,
// N = 256, bf16 in, f32 accumulate): each CTA holds 128 rows of the A tile
// and half of the W tile in shared memory, so every SM stages and reads only
// half of W.  (With one SM per 128 x 256 tile the TMA writes plus the MMA's
// operand reads need about 190 B/clk of shared-memory bandwidth against 128;
// the pair needs about 125.)  K in blocks of 64 (one 128-byte swizzle row),
// a 6-stage TMA ring per CTA, two 256-column TMEM accumulators per CTA so
// that the epilogue of tile i overlaps the main loop of tile i + 1:
//   warp 0      TMA producer (A 16 KB + half of W 16 KB per stage); both
//               CTAs' loads complete on the leader CTA's stage barrier
//   warp 1      TMEM allocator (both CTAs, one paired allocation) and, in
//               the leader CTA, the single-thread MMA issuer; its commits
//               reach the barriers of both CTAs
//   warps 2-5   epilogue: one accumulator row per thread (TMEM lane
//               (warp % 4) * 32 + lane), bf16 rounding, permuted stores;
//               accumulator releases go to the leader's barrier
// Every mbarrier wait is bounded as in attn_kernel.cuh.
#pragma once

#include "cpattn_internal.h"
#include "cpattn_ptx.cuh"

namespace cpattn {

constexpr int kProjThreads = 192;
constexpr int kProjBM = 128;          // rows per CTA (the cluster tile has 256)
constexpr int kProjBN = 256;          // columns per tile (each CTA stages half of W's rows)
constexpr int kProjBK = 64;
constexpr int kProjStages = 6;
constexpr int kProjMaxMaps = kMaxRanks;
constexpr uint32_t kProjTmemCols = 512;

struct ProjSmem {
  static constexpr int kABytes = kProjBM * kProjBK * 2;         // 16 KB
  static constexpr int kWBytes = (kProjBN / 2) * kProjBK * 2;   // 16 KB: this CTA's half of W
  static constexpr int kOffA = 0;
  static constexpr int kOffW = kOffA + kProjStages * kABytes;
  static constexpr int kOffBar = kOffW + kProjStages * kWBytes;
  // full[S], empty[S], acc_full[2], acc_empty[2], tail
  static constexpr int kNumBars = 2 * kProjStages + 5;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 16;
  static constexpr int kAllocBytes = kBytes + 1024;
};

struct alignas(64) ProjParams {
  CUtensorMap tm_a[kProjMaxMaps];   // QKV: [0] = X as 2-D [M, K]; OUT: head rank u as 3-D [B*S, H_u, D]
  CUtensorMap tm_w;                 // 2-D [N, K], box of 128 rows (half a tile)
  int out_mode;                     // 0: QKV (permuting stores), 1: OUT (gathering loads)
  int M, N, K;                      // token rows, output columns, reduction length
  int B, S, H, D;
  int n_seq, n_head;
  int seq_off[kMaxRanks + 1];       // token offsets of the sequence ranks
  int head_off[kMaxRanks + 1];      // head offsets of the head ranks
  unsigned short head_rank[kMaxHeads];
  void *y[3];                       // QKV: head-side Q, K, V; OUT: y[0] = sequence-side output
  unsigned long long timeout_ns;
};

// ------------------------------------------------ CTA-pair (cta_group::2) forms
__device__ __forceinline__ uint32_t proj_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Shared::cluster address of the same shared-memory offset in CTA `rank`.
__device__ __forceinline__ uint32_t proj_mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void proj_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void proj_arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}
// Tile loads into this CTA's shared memory whose completion is counted on the
// leader CTA's barrier (a shared::cluster address).  No multicast.
__device__ __forceinline__ void proj_tma_load_2d_pair(uint32_t smem_dst, const CUtensorMap *tm, int c0, int c1,
                                                      uint32_t cluster_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(cluster_bar)
      : "memory");
}
__device__ __forceinline__ void proj_tma_load_3d_pair(uint32_t smem_dst, const CUtensorMap *tm, int c0, int c1,
                                                      int c2, uint32_t cluster_bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(c2), "r"(cluster_bar)
      : "memory");
}
__device__ __forceinline__ void proj_tmem_alloc_pair(uint32_t smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_result), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void proj_tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void proj_tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D[tmem of both CTAs] (+)= A (128 rows in each CTA) * W^T (half of W's rows in each CTA).
__device__ __forceinline__ void proj_mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the barrier at offset `bar` of both CTAs of the pair when
// every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void proj_commit_pair_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}
// The same, on this CTA's barrier only.
__device__ __forceinline__ void proj_commit_pair_self(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// Tile order: groups of kProjGroupM row tiles, column tiles walked inside a
// group.  The CTAs running at once then share a few row tiles of A (kept in
// L2 while every column tile of the group passes) and a few column tiles of
// W, instead of streaming all of A from HBM once per column tile.
constexpr int kProjGroupM = 8;   // of 256-row cluster tiles
__device__ __forceinline__ void proj_tile(int tile, int mt, int nt, int &mi, int &ni) {
  const int group = tile / (kProjGroupM * nt);
  const int first = group * kProjGroupM;
  const int gm = min(kProjGroupM, mt - first);
  const int within = tile - group * kProjGroupM * nt;
  mi = first + within % gm;
  ni = within / gm;
}

__device__ __forceinline__ int proj_find(const int *off, int n, int x) {
  // largest i in [0, n) with off[i] <= x (empty ranges are skipped)
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Launched in clusters of 2 CTAs (cudaLaunchAttributeClusterDimension), grid
// even; CTA rank 0 of each cluster leads.
__global__ void __launch_bounds__(kProjThreads, 1) proj_gemm_kernel(const __grid_constant__ ProjParams p) {
  using L = ProjSmem;
  constexpr uint32_t IDESC = idesc_bf16_f32(2 * kProjBM, kProjBN, false);   // M = 256 over the pair
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sb = (smem_u32(smem_raw) + 1023u) & ~1023u;
  constexpr uint32_t BAR_FULL = L::kOffBar;                       // [S] leader: both CTAs' loads landed
  constexpr uint32_t BAR_EMPTY = BAR_FULL + 8 * kProjStages;      // [S] this CTA's stage consumed
  constexpr uint32_t BAR_AF = BAR_EMPTY + 8 * kProjStages;        // [2] accumulator written
  constexpr uint32_t BAR_AE = BAR_AF + 16;                        // [2] leader: accumulator read out by both
  constexpr uint32_t BAR_TAIL = BAR_AE + 16;
  constexpr uint32_t TMEM_SLOT = L::kOffMisc;
  constexpr uint32_t ABORT = L::kOffMisc + 4;
  static_assert(BAR_TAIL + 8 <= L::kOffMisc, "barrier area");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = proj_cluster_rank();       // 0: leader (issues the MMAs), 1: peer
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;
  const uint64_t tmo = p.timeout_ns;
  const int mt = (p.M + 2 * kProjBM - 1) / (2 * kProjBM);
  const int nt = (p.N + kProjBN - 1) / kProjBN;
  const int n_tiles = mt * nt;
  const int nkb = p.K / kProjBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kProjStages; ++s) {
      mbar_init(sb + BAR_FULL + 8 * s, 1);
      mbar_init(sb + BAR_EMPTY + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(sb + BAR_AF + 8 * a, 1);
      mbar_init(sb + BAR_AE + 8 * a, 8);   // one arrival per epilogue warp of both CTAs
    }
    mbar_init(sb + BAR_TAIL, 1);
    st_shared_volatile(sb + ABORT, 0u);
    fence_mbar_init();
  }
  if (warp == 1) {
    proj_tmem_alloc_pair(sb + TMEM_SLOT, kProjTmemCols);
    proj_tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  // Both CTAs' barriers are initialised before either signals the other's.
  proj_cluster_sync();
  tc_fence_after();
  const uint32_t tmem = ld_shared_volatile(sb + TMEM_SLOT);
  const uint32_t abort_flag = sb + ABORT;

  if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      if (p.out_mode) {
        for (int u = 0; u < p.n_head; ++u)
          if (p.head_off[u + 1] > p.head_off[u]) tma_prefetch_desc(&p.tm_a[u]);
      } else {
        tma_prefetch_desc(&p.tm_a[0]);
      }
      tma_prefetch_desc(&p.tm_w);
      int it = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < n_tiles; tile += n_clusters) {
        int mi, ni;
        proj_tile(tile, mt, nt, mi, ni);
        const int m0 = mi * 2 * kProjBM + static_cast<int>(rank) * kProjBM;   // this CTA's 128 rows
        const int w0 = ni * kProjBN + static_cast<int>(rank) * (kProjBN / 2);  // this CTA's half of W
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int st = it % kProjStages;
          const uint32_t ph = (it / kProjStages) & 1;
          if (!mbar_wait(sb + BAR_EMPTY + 8 * st, ph ^ 1, abort_flag, tmo, SITE_PRODUCER)) { ok = false; break; }
          const uint32_t full = proj_mapa(sb + BAR_FULL + 8 * st, 0);   // the leader's stage barrier
          if (leader) mbar_arrive_expect_tx(sb + BAR_FULL + 8 * st, 2 * (L::kABytes + L::kWBytes));
          const uint32_t sA = sb + L::kOffA + st * L::kABytes;
          if (p.out_mode) {
            const int k0 = kb * kProjBK;
            const int h = k0 / p.D;
            const int u = p.head_rank[h];
            proj_tma_load_3d_pair(sA, &p.tm_a[u], k0 - h * p.D, h - p.head_off[u], m0, full);
          } else {
            proj_tma_load_2d_pair(sA, &p.tm_a[0], kb * kProjBK, m0, full);
          }
          proj_tma_load_2d_pair(sb + L::kOffW + st * L::kWBytes, &p.tm_w, kb * kProjBK, w0, full);
        }
      }
      // Before the CTA exits, every stage's last use has been consumed by the
      // MMA (so its loads landed) and its release arrived here (bounded).
      for (int j = 0; j < kProjStages && j < it; ++j) {
        const int i = it - 1 - j;
        mbar_wait(sb + BAR_EMPTY + 8 * (i % kProjStages), (i / kProjStages) & 1, 0u, tmo, SITE_TAIL);
      }
    }
  } else if (warp == 1) {
    // ============================================================== MMA issuer
    if (lane == 0 && leader) {
      int it = 0, local = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < n_tiles; tile += n_clusters, ++local) {
        const int a = local & 1;
        if (!mbar_wait_spin(sb + BAR_AE + 8 * a, ((local >> 1) & 1) ^ 1, abort_flag, tmo, SITE_MMA)) break;
        tc_fence_after();
        const uint32_t d = tmem + a * kProjBN;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int st = it % kProjStages;
          const uint32_t ph = (it / kProjStages) & 1;
          if (!mbar_wait_spin(sb + BAR_FULL + 8 * st, ph, abort_flag, tmo, SITE_MMA)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = smem_desc_sw128(sb + L::kOffA + st * L::kABytes, 16, 1024);
          const uint64_t dw = smem_desc_sw128(sb + L::kOffW + st * L::kWBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kProjBK / 16; ++kk)
            proj_mma_pair(d, da + ((kk * 32) >> 4), dw + ((kk * 32) >> 4), IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
          proj_commit_pair_both(sb + BAR_EMPTY + 8 * st);
        }
        if (ok) proj_commit_pair_both(sb + BAR_AF + 8 * a);
      }
      // Drain: every issued MMA has completed before TMEM is released.
      proj_commit_pair_self(sb + BAR_TAIL);
      mbar_wait(sb + BAR_TAIL, 0, 0u, tmo, SITE_TAIL);
    }
  } else {
    // ================================================================ epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;   // accumulator row = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int HD = p.H * p.D;
    const uint32_t ae_leader = proj_mapa(sb + BAR_AE, 0);
    int local = 0;
    for (int tile = cluster; tile < n_tiles; tile += n_clusters, ++local) {
      const int a = local & 1;
      const bool w = mbar_wait(sb + BAR_AF + 8 * a, (local >> 1) & 1, abort_flag, tmo, SITE_EPILOGUE);
      if (__any_sync(0xffffffffu, !w)) break;
      __syncwarp();
      tc_fence_after();
      int mi, ni;
      proj_tile(tile, mt, nt, mi, ni);
      const int m = mi * 2 * kProjBM + static_cast<int>(rank) * kProjBM + r;
      const int n0 = ni * kProjBN;
      const bool row_ok = m < p.M;
      // Row-dependent part of the destination.
      long long row_elems = 0;   // OUT: element offset of the row; QKV: token index (b*S + s)
      if (row_ok) {
        if (p.out_mode) {
          const int b = m / p.S, s = m - (m / p.S) * p.S;
          const int rs = proj_find(p.seq_off, p.n_seq, s);
          const int len = p.seq_off[rs + 1] - p.seq_off[rs];
          row_elems = (static_cast<long long>(p.B) * p.seq_off[rs] + static_cast<long long>(b) * len +
                       (s - p.seq_off[rs])) * p.N;
        } else {
          // sequence-side order: rank rs, batch b, local position
          int lo = 0, hi = p.n_seq - 1;
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.B * p.seq_off[mid] <= m) lo = mid; else hi = mid - 1;
          }
          const int len = p.seq_off[lo + 1] - p.seq_off[lo];
          const int within = m - p.B * p.seq_off[lo];
          const int b = within / len;
          row_elems = static_cast<long long>(b) * p.S + p.seq_off[lo] + (within - b * len);
        }
      }
#pragma unroll 1
      for (int c = 0; c < kProjBN; c += 32) {
        uint32_t v[32];
        __syncwarp();
        tmem_ld32_wait(tmem + lane_base + a * kProjBN + c, v);   // the whole warp, converged
        const int n = n0 + c;
        if (!row_ok || n >= p.N) continue;                         // store skipped; lanes rejoin above
        __nv_bfloat16 *dst;
        if (p.out_mode) {
          dst = static_cast<__nv_bfloat16 *>(p.y[0]) + row_elems + n;
        } else {
          const int t = n / HD;
          const int h = (n - t * HD) / p.D;
          const int u = p.head_rank[h];
          const int Hu = p.head_off[u + 1] - p.head_off[u];
          const long long base = static_cast<long long>(p.B) * p.S * p.head_off[u] * p.D;
          dst = static_cast<__nv_bfloat16 *>(p.y[t]) + base +
                (row_elems * Hu + (h - p.head_off[u])) * p.D + (n - t * HD - h * p.D);
        }
        uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          d4[k] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * k]), __uint_as_float(v[8 * k + 1])),
                             pack_bf16x2(__uint_as_float(v[8 * k + 2]), __uint_as_float(v[8 * k + 3])),
                             pack_bf16x2(__uint_as_float(v[8 * k + 4]), __uint_as_float(v[8 * k + 5])),
                             pack_bf16x2(__uint_as_float(v[8 * k + 6]), __uint_as_float(v[8 * k + 7])));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) proj_arrive_remote(ae_leader + 8 * a);
    }
  }

  // Teardown: both CTAs finished every access to the pair's TMEM and to each
  // other's shared memory before the paired TMEM is released.
  tc_fence_before();
  __syncthreads();
  proj_cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    proj_tmem_dealloc_pair(tmem, kProjTmemCols);
  }
}

}  // namespace cpattn
