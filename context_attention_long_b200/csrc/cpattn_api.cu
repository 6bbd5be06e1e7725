// cpattn_api.cu -- the C ABI of libcpattn.so (declared in include/cpattn.h):
// argument validation, launch planning (row ranges for every shard / chunk),
// TMA descriptor encoding and kernel launches.  Single translation unit.
#include "cpattn.h"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <memory>
#include <mutex>
#include <vector>

#include "cpattn_internal.h"
#include "cpattn_ptx.cuh"
#include "attn_kernel.cuh"
#include "attn_bwd_kernel.cuh"
#include "merge_kernel.cuh"
#include "permute_kernel.cuh"
#include "proj_kernel.cuh"

namespace cpattn {

// ------------------------------------------------------------------ helpers

// A fused-ring unit walks one K/V range per chunk, and one launch holds at
// most kMaxKV ranges, so the ring degree is capped there; kv_gather walks a
// single range per shard and may use more shards.
constexpr int kMaxRingDegree = kMaxKV;
constexpr int kMaxGatherDegree = 1024;
constexpr int kMaxDevices = 64;

// Kernel parameters (the __grid_constant__ parameter blocks) are limited to
// 32764 bytes.
static_assert(sizeof(AttnParams) <= 32764, "AttnParams exceeds the kernel parameter limit");
static_assert(sizeof(BwdParams) <= 32764, "BwdParams exceeds the kernel parameter limit");
static_assert(sizeof(ProjParams) <= 32764, "ProjParams exceeds the kernel parameter limit");
static_assert(sizeof(PermuteParams) <= 32764 && sizeof(MergeParams) <= 32764, "kernel parameter limit");

static unsigned long long wait_timeout_ns() {
  static unsigned long long v = [] {
    const char *e = std::getenv("CPATTN_WAIT_TIMEOUT_MS");
    long long ms = e ? std::atoll(e) : 2000;
    if (ms < 1) ms = 1;
    return static_cast<unsigned long long>(ms) * 1000000ull;
  }();
  return v;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

static int check_attn_shape(int B, int H, int S, int D) {
  if (B < 1 || H < 1 || S < 1) return CPATTN_ERR_SHAPE;
  if (D != 64 && D != 128) return CPATTN_ERR_SHAPE;
  if (static_cast<long long>(B) * S > INT_MAX) return CPATTN_ERR_SHAPE;
  if (static_cast<long long>(B) * S * H * D > (1ll << 46)) return CPATTN_ERR_SHAPE;
  return CPATTN_OK;
}

// The backward also indexes its (token, head) rows in 32 bits: B*S*H < 2^31,
// which any [B, S, H, D] bf16 tensor that fits in a device's memory meets.
static int check_bwd_shape(int B, int H, int S, int D) {
  const int st = check_attn_shape(B, H, S, D);
  if (st != CPATTN_OK) return st;
  return static_cast<long long>(B) * S * H >= (1ll << 31) ? CPATTN_ERR_SHAPE : CPATTN_OK;
}

// Equal split (NULL: total % degree == 0 required, [CP] variants table) or
// explicit non-negative lengths summing to total ('anything' modes).
static int resolve_splits(int total, int degree, const int *splits, std::vector<int> &out) {
  if (degree < 1) return CPATTN_ERR_DEGREE;
  if (splits == nullptr) {
    if (degree > total) return CPATTN_ERR_DEGREE;
    if (total % degree != 0) return CPATTN_ERR_INDIVISIBLE;
    out.assign(degree, total / degree);
    return CPATTN_OK;
  }
  long long sum = 0;
  out.resize(degree);
  for (int i = 0; i < degree; ++i) {
    if (splits[i] < 0) return CPATTN_ERR_SPLITS;
    out[i] = splits[i];
    sum += splits[i];
  }
  return sum == total ? CPATTN_OK : CPATTN_ERR_SPLITS;
}

static std::vector<int> prefix(const std::vector<int> &lens) {
  std::vector<int> off(lens.size() + 1, 0);
  for (size_t i = 0; i < lens.size(); ++i) off[i + 1] = off[i] + lens[i];
  return off;
}

// The CUDA error behind the last CPATTN_ERR_CUDA this thread received, and
// the step that failed (cpattn_last_cuda_error reports them).
static thread_local cudaError_t t_last_cuda_error = cudaSuccess;
static thread_local const char *t_last_cuda_step = "";
static int cuda_fail(cudaError_t e, const char *step) {
  t_last_cuda_error = e == cudaSuccess ? cudaErrorUnknown : e;
  t_last_cuda_step = step;
  return CPATTN_ERR_CUDA;
}
static int cuda_result(cudaError_t e, const char *step) { return e == cudaSuccess ? CPATTN_OK : cuda_fail(e, step); }

// Is the current device an sm_100 part?
static int check_device(int *dev_out) {
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "device query");
  }
  if (dev < 0 || dev >= kMaxDevices) return CPATTN_ERR_UNSUPPORTED;
  // The tensor-map encoder is a driver call and needs a context current on
  // this thread; runtime calls bind the primary context lazily, so a thread
  // that has made none yet (torch's autograd engine thread, say) has none.
  // cudaSetDevice binds it; once per thread and device.
  static thread_local int t_bound_dev = -1;
  if (t_bound_dev != dev) {
    if (cudaError_t e = cudaSetDevice(dev); e != cudaSuccess) {
      cudaGetLastError();
      return cuda_fail(e, "binding the device's primary context");
    }
    t_bound_dev = dev;
  }
  static std::atomic<int> cc_major[kMaxDevices];   // 0 = not queried yet
  int major = cc_major[dev].load(std::memory_order_relaxed);
  if (major == 0) {
    if (cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev); e != cudaSuccess) {
      cudaGetLastError();
      return cuda_fail(e, "device query");
    }
    cc_major[dev].store(major, std::memory_order_relaxed);
  }
  if (major != 10) return CPATTN_ERR_UNSUPPORTED;
  if (dev_out) *dev_out = dev;
  return CPATTN_OK;
}

// What the last failed tensor-map encoding on this thread was given (the step
// text of the CPATTN_ERR_CUDA it causes).
static thread_local char t_encode_detail[256] = "tensor map encoding";

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      ptr = nullptr;
    }
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }();
  return fn;
}

// 3-D view [rows, H, D] of a bf16 tensor, box {64, 1, 128}, 128-byte swizzle.
static bool encode_rows_map(CUtensorMap *tm, const void *ptr, int D, int H, long long rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H) * D * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(kQTile)};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    std::snprintf(t_encode_detail, sizeof(t_encode_detail),
                  "tensor map encoding (driver result %d; address %p, dims %llu x %llu x %llu, strides %llu, %llu)",
                  static_cast<int>(r), ptr, static_cast<unsigned long long>(dims[0]),
                  static_cast<unsigned long long>(dims[1]), static_cast<unsigned long long>(dims[2]),
                  static_cast<unsigned long long>(strides[0]), static_cast<unsigned long long>(strides[1]));
  return r == CUDA_SUCCESS;
}

// 2-D view [rows, cols] of a bf16 row-major matrix, box {64, box_rows},
// 128-byte swizzle; rows past the end read as zero.
static bool encode_matrix_map(CUtensorMap *tm, const void *ptr, long long rows, long long cols, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    std::snprintf(t_encode_detail, sizeof(t_encode_detail),
                  "tensor map encoding (driver result %d; address %p, dims %llu x %llu, stride %llu)",
                  static_cast<int>(r), ptr, static_cast<unsigned long long>(dims[0]),
                  static_cast<unsigned long long>(dims[1]), static_cast<unsigned long long>(strides[0]));
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ launchers

template <int D, bool F32>
static cudaError_t launch_attn_t(const AttnParams &p, cudaStream_t stream) {
  static std::mutex mu;
  static bool configured[kMaxDevices] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured[dev]) {
      cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, F32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           AttnSmem<D>::kAllocBytes);
      if (e != cudaSuccess) return e;
      configured[dev] = true;
    }
  }
  attn_fwd_kernel<D, F32><<<p.total_units, kAttnThreads, AttnSmem<D>::kAllocBytes, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_attention(const AttnParams &p, int D, bool out_f32, cudaStream_t stream) {
  if (p.total_units <= 0) return cudaSuccess;
  if (D == 128) return out_f32 ? launch_attn_t<128, true>(p, stream) : launch_attn_t<128, false>(p, stream);
  return out_f32 ? launch_attn_t<64, true>(p, stream) : launch_attn_t<64, false>(p, stream);
}

// SMs of the current device (cached per device).
static int device_sm_count() {
  static std::mutex mu;
  static int sms[kMaxDevices] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < kMaxDevices && sms[dev] == 0 &&
      cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms[dev] = 0;
  return (dev >= 0 && dev < kMaxDevices && sms[dev] > 0) ? sms[dev] : 148;
}

static int grid_for(long long work_items, int items_per_block) {
  long long blocks = (work_items + items_per_block - 1) / items_per_block;
  blocks = std::max<long long>(1, std::min<long long>(blocks, 148ll * 16));
  return static_cast<int>(blocks);
}

template <int D>
static cudaError_t launch_merge_d(const MergeParams &p, cudaStream_t stream) {
  const long long nrows = static_cast<long long>(p.B) * p.H * p.S;
  const int rows_per_block = (kMergeThreads / 32) * (32 / (D / 4));
  const int grid = grid_for(nrows, rows_per_block);
  if (p.P <= 2) lse_merge_kernel<D, 2><<<grid, kMergeThreads, 0, stream>>>(p);
  else if (p.P <= 4) lse_merge_kernel<D, 4><<<grid, kMergeThreads, 0, stream>>>(p);
  else if (p.P <= 8) lse_merge_kernel<D, 8><<<grid, kMergeThreads, 0, stream>>>(p);
  else if (p.P <= 16) lse_merge_kernel<D, 16><<<grid, kMergeThreads, 0, stream>>>(p);
  else lse_merge_kernel_anyp<D><<<grid, kMergeThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_lse_merge(const MergeParams &p, cudaStream_t stream) {
  return p.D == 128 ? launch_merge_d<128>(p, stream) : launch_merge_d<64>(p, stream);
}

template <int D>
static cudaError_t launch_bwd_d(const BwdParams &p, int units, cudaStream_t stream) {
  static std::mutex mu;
  static bool configured[kMaxDevices] = {false};
  static int sms[kMaxDevices] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured[dev]) {
      cudaError_t e = cudaFuncSetAttribute(attn_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           BwdSmem<D>::kAllocBytes);
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(attn_bwd_dkv_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               BwdSmem<D>::kAllocBytes);
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(attn_bwd_dkv_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               BwdSmem<D, 2, true>::kAllocBytes);
      if (e != cudaSuccess) return e;
      e = cudaFuncSetAttribute(attn_bwd_dq_gemm_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               BwdGemmSmem<D>::kAllocBytes);
      if (e != cudaSuccess) return e;
      e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return e;
      configured[dev] = true;
    }
  }
  const bool with_ds = p.prob[0].ds != nullptr;
  if (!with_ds) {
    attn_bwd_dq_kernel<D><<<static_cast<unsigned>(units), kBwdThreads, BwdSmem<D>::kAllocBytes, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (with_ds)
    attn_bwd_dkv_kernel<D, true><<<static_cast<unsigned>(units), kBwdThreads, BwdSmem<D, 2, true>::kAllocBytes,
                                   stream>>>(p);
  else
    attn_bwd_dkv_kernel<D, false><<<static_cast<unsigned>(units), kBwdThreads, BwdSmem<D>::kAllocBytes, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !with_ds) return e;
  // one CTA per SM (its shared memory admits no second), each walking units
  const int grid = std::min(units, std::max(sms[dev], 1));
  attn_bwd_dq_gemm_kernel<D><<<static_cast<unsigned>(grid), kBwdGemmThreads, BwdGemmSmem<D>::kAllocBytes, stream>>>(
      p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_delta(const void *out, const void *dout, float *delta, int B, int S, int H, int D,
                             cudaStream_t stream) {
  const long long rows = static_cast<long long>(B) * S * H;
  if (rows == 0) return cudaSuccess;
  // as many CTAs as are resident at once (three per SM): every warp walks
  // several row groups instead of a new CTA starting for each
  const int grid = std::min(grid_for(rows, (256 / 32) * (32 / (D / 8)) * kDeltaPasses), 3 * device_sm_count());
  attn_bwd_delta_kernel<<<grid, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16 *>(out), static_cast<const __nv_bfloat16 *>(dout), delta, B, S, H, D);
  return cudaGetLastError();
}

cudaError_t launch_bwd_kernels(const BwdParams &p, int D, cudaStream_t stream) {
  const int nt = (p.S + 127) / 128;
  int units = 0;
  for (int i = 0; i < p.n_prob; ++i) units += p.B * p.prob[i].nh * nt;
  if (units == 0) return cudaSuccess;
  return D == 128 ? launch_bwd_d<128>(p, units, stream) : launch_bwd_d<64>(p, units, stream);
}

// Persistent projection GEMM in clusters of two CTAs: as many clusters as
// can be resident at once (or one per 256 x 256 tile, if fewer), so that
// every cluster runs from the start and the tile stride covers all tiles.
static cudaError_t launch_projection(const ProjParams &p, cudaStream_t stream) {
  static std::mutex mu;
  static int clusters[kMaxDevices] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kProjThreads, 1, 1);
  cfg.dynamicSmemBytes = ProjSmem::kAllocBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (clusters[dev] == 0) {
      cudaError_t e = cudaFuncSetAttribute(proj_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           ProjSmem::kAllocBytes);
      if (e != cudaSuccess) return e;
      int sms = 0;
      e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return e;
      cfg.gridDim = dim3(2 * std::max(1, sms / 2), 1, 1);
      int n = 0;
      e = cudaOccupancyMaxActiveClusters(&n, proj_gemm_kernel, &cfg);
      if (e != cudaSuccess) return e;
      if (n < 1) return cudaErrorInvalidConfiguration;
      clusters[dev] = n;
    }
  }
  const long long tiles = static_cast<long long>((p.M + 2 * kProjBM - 1) / (2 * kProjBM)) *
                          ((p.N + kProjBN - 1) / kProjBN);
  if (tiles <= 0) return cudaSuccess;
  cfg.gridDim = dim3(2 * static_cast<unsigned>(std::min<long long>(tiles, clusters[dev])), 1, 1);
  return cudaLaunchKernelEx(&cfg, proj_gemm_kernel, p);
}

cudaError_t launch_permute(const PermuteParams &p, cudaStream_t stream) {
  const long long ntok = static_cast<long long>(p.B) * p.S;
  const int grid = grid_for(ntok, kPermuteThreads / 32);
  permute_kernel<<<grid, kPermuteThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

__global__ void debug_wait_kernel(unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    st_shared_volatile(smem_u32(&abort_flag), 0u);
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
    // Nothing ever arrives: the wait must give up after timeout_ns.
    mbar_wait(smem_u32(&bar), 0, smem_u32(&abort_flag), timeout_ns, SITE_DEBUG);
  }
}

cudaError_t launch_debug_wait(unsigned long long timeout_ns, cudaStream_t stream) {
  debug_wait_kernel<<<1, 32, 0, stream>>>(timeout_ns);
  return cudaGetLastError();
}

cudaError_t read_and_clear_device_status(unsigned int *code, cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return e;
  }
  *code = v;
  return cudaSuccess;
}

// ------------------------------------------------------------ attention plans

struct ProblemSpec {
  const void *q, *k, *v;
  void *out;
  float *lse;
  long long lse_b, lse_h;
  int lse_h0;
  int H;
  long long rows;              // rows of Q and out (and of K and V unless rows_kv > 0)
  long long rows_kv = 0;       // rows of K and V when they are a separate buffer
  const float *prev = nullptr; // previous partial state merged into the output (see AttnProblem)
  int lse_pos0 = 0;            // sequence position of LSE column 0
  int out_mode = 0;            // output map (see AttnProblem)
  int out_H = 0, out_h0 = 0, out_B = 0, out_S = 0;
  std::vector<int> out_seq_off;   // out_mode 1: sequence offsets of the ranks (degree + 1 entries)
};
struct SegSpec {
  int row0, nrows, s0;
  std::vector<AttnKV> kv;
  int split = 0;   // a lone Q tile: split its K/V tiles between the two slots
  int q1_row0 = 0, q1_s0 = 0, q1_rows = 0;   // a lone tile paired with another shard's lone tile in slot 1
};
struct GroupSpec {
  int prob, b;
  std::vector<SegSpec> segs;
};

// Longest-first ordering of the CTAs: a segment whose row count leaves a
// lone 128-row Q tile (rows mod 256 in 1..128) is split into its full tile
// pairs and that lone tile.  The lone tile becomes a "split" unit (both slots
// hold its rows and divide its K/V tiles, merged with the LSE rule at the
// end), about half the work of a pair; those units are placed after every
// full pair, so they fill the gaps of the last wave instead of adding one.
// Without the causal mask, two lone tiles of one group whose K/V lists hold
// the same chunks (the shards of a fused ring: each walks every chunk, from
// its own) share one CTA as a pair: slot 1 takes the second tile's rows and
// both walk the first tile's list.  The second tile's keys are the same; only
// the order of its online-softmax steps (so its rounding) follows the other
// shard.  This replaces two split units, whose slots each stream their own
// K/V tiles and merge at the end, by one pair unit on one K/V stream.
static bool same_kv_set(std::vector<AttnKV> a, std::vector<AttnKV> b) {
  auto key = [](const AttnKV &x, const AttnKV &y) { return x.row0 < y.row0; };
  std::sort(a.begin(), a.end(), key);
  std::sort(b.begin(), b.end(), key);
  if (a.size() != b.size()) return false;
  for (size_t i = 0; i < a.size(); ++i)
    if (a[i].row0 != b[i].row0 || a[i].nrows != b[i].nrows || a[i].s0 != b[i].s0) return false;
  return true;
}
static void pair_lone_tiles(GroupSpec &g) {
  std::vector<SegSpec> out;
  std::vector<bool> used(g.segs.size(), false);
  for (size_t i = 0; i < g.segs.size(); ++i) {
    if (used[i]) continue;
    used[i] = true;
    SegSpec a = g.segs[i];
    for (size_t j = i + 1; j < g.segs.size(); ++j) {
      if (used[j] || g.segs[j].nrows <= 0 || a.nrows <= 0 || !same_kv_set(a.kv, g.segs[j].kv)) continue;
      used[j] = true;
      a.split = 0;
      a.q1_row0 = g.segs[j].row0;
      a.q1_s0 = g.segs[j].s0;
      a.q1_rows = g.segs[j].nrows;
      break;
    }
    out.push_back(std::move(a));
  }
  g.segs = std::move(out);
}


// Makespan, in half units, of the longest-first schedule over `sms` SMs of
// n2 units of length 2 followed by n1 of length 1.
static long long lpt_half_units(long long n2, long long n1, int sms) {
  std::vector<long long> load(static_cast<size_t>(std::max(1, sms)), 0);
  auto put = [&](long long w, long long n) {
    for (long long i = 0; i < n; ++i) {
      std::pop_heap(load.begin(), load.end(), std::greater<long long>());
      load.back() += w;
      std::push_heap(load.begin(), load.end(), std::greater<long long>());
    }
  };
  std::make_heap(load.begin(), load.end(), std::greater<long long>());
  put(2, n2);
  put(1, n1);
  return *std::max_element(load.begin(), load.end());
}

// heads[prob]: the head count of each problem (units run once per head).
static std::vector<GroupSpec> longest_first(const std::vector<GroupSpec> &groups, bool causal,
                                            const std::vector<int> &heads) {
  constexpr int kPairRows = kQTilesPerCTA * kQTile;
  std::vector<GroupSpec> head, tail, tail_paired;
  long long n_pairs = 0, n_lone = 0, n_cross = 0, n_single = 0;   // units, over all heads
  for (const GroupSpec &g : groups) {
    GroupSpec main_g{g.prob, g.b, {}}, tail_g{g.prob, g.b, {}};
    for (const SegSpec &s : g.segs) {
      const int rem = s.nrows % kPairRows;
      if (s.nrows <= kQTile) {          // the whole segment is one lone tile
        SegSpec t = s;
        t.split = 1;
        tail_g.segs.push_back(std::move(t));
        continue;
      }
      if (rem == 0 || rem > kQTile) {
        main_g.segs.push_back(s);
        continue;
      }
      SegSpec m = s, t = s;
      m.nrows = s.nrows - rem;
      t.row0 = s.row0 + m.nrows;
      t.s0 = s.s0 + m.nrows;
      t.nrows = rem;
      t.split = 1;
      main_g.segs.push_back(std::move(m));
      tail_g.segs.push_back(std::move(t));
    }
    const long long H = heads[g.prob];
    for (const SegSpec &s : main_g.segs) n_pairs += H * ((s.nrows + kPairRows - 1) / kPairRows);
    if (!main_g.segs.empty()) head.push_back(std::move(main_g));
    if (tail_g.segs.empty()) continue;
    GroupSpec paired = tail_g;
    if (!causal) pair_lone_tiles(paired);
    n_lone += H * static_cast<long long>(tail_g.segs.size());
    for (const SegSpec &s : paired.segs) (s.q1_rows > 0 ? n_cross : n_single) += H;
    tail.push_back(std::move(tail_g));
    tail_paired.push_back(std::move(paired));
  }
  // Paired lone tiles walk as long as a full pair; split units take about half
  // as long and fill the last wave.  Pair them unless that lengthens the
  // longest-first schedule (in half units: a pair 2, a split unit 1).
  if (n_cross > 0) {
    const int sms = device_sm_count();
    if (lpt_half_units(n_pairs + n_cross, n_single, sms) <= lpt_half_units(n_pairs, n_lone, sms))
      tail = std::move(tail_paired);
  }
  for (GroupSpec &g : tail) head.push_back(std::move(g));
  return head;
}

// Causal plans interleave the units of this many heads pair by pair: as many
// heads as have K and V (bf16, the distinct K/V rows of the group) within a
// 64 MiB share of the 126 MB L2, at least one.
static int causal_head_block(const GroupSpec &gs, int D, int H) {
  std::vector<std::pair<int, int>> ranges;
  for (const SegSpec &ss : gs.segs)
    for (const AttnKV &kv : ss.kv) ranges.emplace_back(kv.row0, kv.nrows);
  std::sort(ranges.begin(), ranges.end());
  ranges.erase(std::unique(ranges.begin(), ranges.end()), ranges.end());
  long long rows = 0;
  for (const auto &r : ranges) rows += r.second;
  const long long per_head = std::max(1LL, rows * D * 2 * 2);
  const long long fit = (64LL << 20) / per_head;
  return static_cast<int>(std::max(1LL, std::min<long long>(H, fit)));
}

// Packs the groups into as few launches as the parameter tables allow and
// launches them in order on `stream`.
static int run_attention(const std::vector<ProblemSpec> &probs, const std::vector<GroupSpec> &groups_in, int D,
                         bool out_f32, bool causal, cudaStream_t stream) {
  std::vector<int> heads(probs.size());
  for (size_t i = 0; i < probs.size(); ++i) heads[i] = probs[i].H;
  const std::vector<GroupSpec> groups = longest_first(groups_in, causal, heads);
  std::vector<AttnProblem> encoded(probs.size());
  for (size_t i = 0; i < probs.size(); ++i) {
    const ProblemSpec &ps = probs[i];
    AttnProblem &ap = encoded[i];
    std::memset(&ap, 0, sizeof(ap));
    const long long rows_kv = ps.rows_kv > 0 ? ps.rows_kv : ps.rows;
    if (!encode_rows_map(&ap.tm_q, ps.q, D, ps.H, ps.rows) || !encode_rows_map(&ap.tm_k, ps.k, D, ps.H, rows_kv) ||
        !encode_rows_map(&ap.tm_v, ps.v, D, ps.H, rows_kv))
      return cuda_fail(cudaErrorInvalidValue, t_encode_detail);
    ap.out = ps.out;
    ap.lse = ps.lse;
    ap.prev = ps.prev;
    ap.lse_b = ps.lse_b;
    ap.lse_h = ps.lse_h;
    ap.lse_h0 = ps.lse_h0;
    ap.lse_pos0 = ps.lse_pos0;
    ap.H = ps.H;
    ap.out_mode = ps.out_mode;
    ap.out_H = ps.out_H;
    ap.out_h0 = ps.out_h0;
    ap.out_B = ps.out_B;
    ap.out_S = ps.out_S;
    ap.out_nseq = static_cast<int>(ps.out_seq_off.size()) - 1;
    if (ap.out_nseq > kMaxRanks) return CPATTN_ERR_DEGREE;
    for (size_t r = 0; r < ps.out_seq_off.size(); ++r) ap.out_seq_off[r] = ps.out_seq_off[r];
  }
  const float scale_log2 = static_cast<float>((1.0 / std::sqrt(static_cast<double>(D))) * 1.4426950408889634);

  std::unique_ptr<AttnParams> P(new AttnParams);
  std::vector<int> prob_slot(probs.size(), -1);
  int n_prob = 0, n_seg = 0, n_kv = 0;
  int open_group = -1;  // index into P->group of the group being filled

  auto reset = [&] {
    std::memset(P.get(), 0, sizeof(AttnParams));
    std::fill(prob_slot.begin(), prob_slot.end(), -1);
    n_prob = n_seg = n_kv = 0;
    open_group = -1;
    P->scale_log2 = scale_log2;
    P->causal = causal ? 1 : 0;
    P->timeout_ns = wait_timeout_ns();
  };
  auto close_group = [&] {
    if (open_group >= 0) {
      AttnGroup &g = P->group[open_group];
      P->total_units += P->prob[g.prob].H * g.tiles_per_head;
      open_group = -1;
    }
  };
  auto flush = [&]() -> int {
    close_group();
    if (P->total_units > 0) {
      if (cudaError_t e = launch_attention(*P, D, out_f32, stream); e != cudaSuccess) return cuda_fail(e, "attention launch");
    }
    reset();
    return CPATTN_OK;
  };
  reset();

  for (const GroupSpec &gs : groups) {
    bool group_started_here = false;
    for (const SegSpec &ss : gs.segs) {
      if (ss.nrows <= 0) continue;
      const int need_kv = static_cast<int>(ss.kv.size());
      if (need_kv > kMaxKV) return CPATTN_ERR_DEGREE;
      const bool need_prob = prob_slot[gs.prob] < 0;
      const bool need_group = !group_started_here || open_group < 0;
      if ((need_prob && n_prob >= kMaxProblems) || (need_group && P->num_groups >= kMaxGroups) ||
          n_seg >= kMaxSegs || n_kv + need_kv > kMaxKV) {
        int st = flush();
        if (st != CPATTN_OK) return st;
        group_started_here = false;
      }
      if (prob_slot[gs.prob] < 0) {
        prob_slot[gs.prob] = n_prob;
        P->prob[n_prob++] = encoded[gs.prob];
      }
      if (!group_started_here || open_group < 0) {
        close_group();
        open_group = P->num_groups++;
        AttnGroup &g = P->group[open_group];
        g.prob = prob_slot[gs.prob];
        g.b = gs.b;
        g.seg_first = n_seg;
        g.seg_count = 0;
        g.tiles_per_head = 0;
        g.unit_base = P->total_units;
        g.head_block = causal_head_block(gs, D, probs[gs.prob].H);
        group_started_here = true;
      }
      AttnGroup &g = P->group[open_group];
      AttnSeg &sg = P->seg[n_seg++];
      sg.row0 = ss.row0;
      sg.nrows = ss.nrows;
      sg.s0 = ss.s0;
      sg.kv_first = n_kv;
      sg.kv_count = need_kv;
      sg.tile_base = g.tiles_per_head;
      sg.split = ss.split;
      sg.q1_row0 = ss.q1_row0;
      sg.q1_s0 = ss.q1_s0;
      sg.q1_rows = ss.q1_rows;
      for (const AttnKV &kv : ss.kv) P->kv[n_kv++] = kv;
      g.seg_count += 1;
      g.tiles_per_head += (ss.nrows + kQTilesPerCTA * kQTile - 1) / (kQTilesPerCTA * kQTile);
    }
    close_group();
  }
  return flush();
}

static ProblemSpec full_problem(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H,
                                int S) {
  ProblemSpec ps;
  ps.q = q;
  ps.k = k;
  ps.v = v;
  ps.out = out;
  ps.lse = lse;
  ps.lse_b = static_cast<long long>(H) * S;
  ps.lse_h = S;
  ps.lse_h0 = 0;
  ps.H = H;
  ps.rows = static_cast<long long>(B) * S;
  return ps;
}

// Ring plan over a [rows, H, D] tensor whose batch-b chunk c occupies rows
// row_of(b, c) .. + lens[c] at sequence positions off[c] ..; `step` < 0: all
// chunks (fused); otherwise only chunk (r - step) mod P.  Without the mask a
// fused shard walks the chunks in ring order from its own.  Under the causal
// mask a chunk after shard r is invisible to all of its queries and is left
// out (its ring-step partial is the empty one: out 0, lse -inf), and a fused
// shard walks the chunks it sees in sequence order, 0 .. r, its own chunk
// (the one the mask cuts) last -- so the keys that the first Q tile of a pair
// cannot see come last in the walk.  Every shard's causal walk is then a
// prefix of the next shard's: where a batch element's shards are contiguous
// rows, the fused causal plan is one segment over all of them with the chunks
// in sequence order, its Q tiles paired across shard boundaries (no lone tile
// per shard), and each row still walks chunks 0 .. r.
template <class RowOf>
static void ring_groups(std::vector<GroupSpec> &groups, int prob, int B, const std::vector<int> &lens,
                        const std::vector<int> &off, int step, bool causal, RowOf row_of) {
  const int P = static_cast<int>(lens.size());
  for (int b = 0; b < B; ++b) {
    GroupSpec g;
    g.prob = prob;
    g.b = b;
    bool contiguous = causal && step < 0;
    for (int c = 0; contiguous && c + 1 < P; ++c) contiguous = row_of(b, c + 1) == row_of(b, c) + lens[c];
    if (contiguous) {
      SegSpec s;
      s.row0 = row_of(b, 0);
      s.nrows = off[P];
      s.s0 = off[0];
      for (int c = 0; c < P; ++c)
        if (lens[c] > 0) s.kv.push_back(AttnKV{row_of(b, c), lens[c], off[c]});
      g.segs.push_back(std::move(s));
      groups.push_back(std::move(g));
      continue;
    }
    for (int i = 0; i < P; ++i) {
      const int r = causal ? P - 1 - i : i;   // causal: the shard that sees most chunks first
      SegSpec s;
      s.row0 = row_of(b, r);
      s.nrows = lens[r];
      s.s0 = off[r];
      if (causal && step < 0) {
        for (int c = 0; c <= r; ++c)
          if (lens[c] > 0) s.kv.push_back(AttnKV{row_of(b, c), lens[c], off[c]});
      } else {
        for (int t = 0; t < P; ++t) {
          if (step >= 0 && t != step) continue;
          const int c = ((r - t) % P + P) % P;  // chunk held by rank r after t hand-offs
          if (causal && c > r) continue;
          if (lens[c] > 0) s.kv.push_back(AttnKV{row_of(b, c), lens[c], off[c]});
        }
      }
      g.segs.push_back(std::move(s));
    }
    groups.push_back(std::move(g));
  }
}

// Q, K and V (same shape and splits) as the three tensors of one permute launch.
static void set_qkv(PermuteParams &pp, const void *q, const void *k, const void *v, void *yq, void *yk, void *yv) {
  const void *srcs[3] = {q, k, v};
  void *dsts[3] = {yq, yk, yv};
  for (int i = 0; i < 3; ++i) {
    pp.src[i] = static_cast<const unsigned char *>(srcs[i]);
    pp.dst[i] = static_cast<unsigned char *>(dsts[i]);
  }
  pp.n_tensors = 3;
}

static int permute_common(const void *src, void *dst, int B, int S, int H, int D, int elem_bytes, int degree,
                          const int *seq_splits, const int *head_splits, int direction, PermuteParams &pp) {
  if (src == nullptr || dst == nullptr) return CPATTN_ERR_NULL;
  if (B < 1 || S < 1 || H < 1 || D < 1) return CPATTN_ERR_SHAPE;
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8) return CPATTN_ERR_SHAPE;
  if ((static_cast<long long>(D) * elem_bytes) % 16 != 0 || static_cast<long long>(D) * elem_bytes > (1 << 20))
    return CPATTN_ERR_SHAPE;
  if (H > kMaxHeads || static_cast<long long>(B) * S > INT_MAX) return CPATTN_ERR_SHAPE;
  if (degree < 1 || degree > kMaxRanks) return CPATTN_ERR_DEGREE;
  std::vector<int> seq, heads;
  int st = resolve_splits(S, degree, seq_splits, seq);
  if (st != CPATTN_OK) return st;
  st = resolve_splits(H, degree, head_splits, heads);
  if (st != CPATTN_OK) return st;
  if (!aligned16(src) || !aligned16(dst)) return CPATTN_ERR_ALIGNMENT;
  std::memset(&pp, 0, sizeof(pp));
  pp.src[0] = static_cast<const unsigned char *>(src);
  pp.dst[0] = static_cast<unsigned char *>(dst);
  pp.n_tensors = 1;
  pp.B = B;
  pp.S = S;
  pp.H = H;
  pp.row_bytes = D * elem_bytes;
  pp.direction = direction;
  pp.seq_mode = 1;
  pp.n_seq = degree;
  std::vector<int> so = prefix(seq), ho = prefix(heads);
  for (int i = 0; i <= degree; ++i) {
    pp.seq_off[i] = so[i];
    pp.head_off[i] = ho[i];
  }
  pp.n_groups = 1;
  pp.group_off[0] = 0;
  pp.group_off[1] = S;
  pp.n_head = degree;
  return CPATTN_OK;
}

// Shared set-up of the two fused projections: shapes, splits, alignment and
// (with `fill` non-null, once the device is known to be usable) the rank
// tables and tensor maps.  QKV: M = B*S sequence-side token rows, N = 3*H*D, K = Dm;
// OUT: M = B*S tokens (head-side order), N = Dm, K = H*D.
static int projection_common(const void *a, const void *w, int B, int S, int H, int D, int Dm, int degree,
                             const int *seq_splits, const int *head_splits, bool out_mode, ProjParams *fill,
                             ProjParams &pp) {
  if (a == nullptr || w == nullptr) return CPATTN_ERR_NULL;
  if (B < 1 || S < 1 || H < 1 || (D != 64 && D != 128)) return CPATTN_ERR_SHAPE;
  if (Dm < kProjBK || Dm % kProjBK != 0 || Dm > (1 << 20)) return CPATTN_ERR_SHAPE;
  if (H > kMaxHeads || static_cast<long long>(B) * S > INT_MAX / 2) return CPATTN_ERR_SHAPE;
  if (3ll * H * D > INT_MAX / 2) return CPATTN_ERR_SHAPE;
  {
    // the kernel numbers its 256 x 256 tiles with int
    const long long rows = static_cast<long long>(B) * S, cols = out_mode ? Dm : 3ll * H * D;
    if (((rows + 2 * kProjBM - 1) / (2 * kProjBM)) * ((cols + kProjBN - 1) / kProjBN) > INT_MAX)
      return CPATTN_ERR_SHAPE;
  }
  if (degree < 1 || degree > kMaxRanks) return CPATTN_ERR_DEGREE;
  std::vector<int> seq, heads;
  int st = resolve_splits(S, degree, seq_splits, seq);
  if (st != CPATTN_OK) return st;
  st = resolve_splits(H, degree, head_splits, heads);
  if (st != CPATTN_OK) return st;
  if (!aligned16(a) || !aligned16(w)) return CPATTN_ERR_ALIGNMENT;
  if (fill == nullptr) return CPATTN_OK;   // arguments checked; nothing encoded yet
  std::memset(&pp, 0, sizeof(pp));
  pp.out_mode = out_mode ? 1 : 0;
  pp.B = B;
  pp.S = S;
  pp.H = H;
  pp.D = D;
  pp.M = B * S;
  pp.N = out_mode ? Dm : 3 * H * D;
  pp.K = out_mode ? H * D : Dm;
  pp.n_seq = degree;
  pp.n_head = degree;
  std::vector<int> so = prefix(seq), ho = prefix(heads);
  for (int i = 0; i <= degree; ++i) {
    pp.seq_off[i] = so[i];
    pp.head_off[i] = ho[i];
  }
  for (int u = 0; u < degree; ++u)
    for (int h = ho[u]; h < ho[u + 1]; ++h) pp.head_rank[h] = static_cast<unsigned short>(u);
  if (!encode_matrix_map(&pp.tm_w, w, pp.N, pp.K, kProjBN / 2)) return cuda_fail(cudaErrorInvalidValue, t_encode_detail);
  if (out_mode) {
    const char *base = static_cast<const char *>(a);
    for (int u = 0; u < degree; ++u) {
      const int Hu = ho[u + 1] - ho[u];
      if (Hu == 0) continue;
      const size_t off = static_cast<size_t>(B) * S * ho[u] * D * 2;
      if (!encode_rows_map(&pp.tm_a[u], base + off, D, Hu, static_cast<long long>(B) * S))
        return cuda_fail(cudaErrorInvalidValue, t_encode_detail);
    }
  } else if (!encode_matrix_map(&pp.tm_a[0], a, pp.M, pp.K, kProjBM)) {
    return cuda_fail(cudaErrorInvalidValue, t_encode_detail);
  }
  pp.timeout_ns = wait_timeout_ns();
  return CPATTN_OK;
}

}  // namespace cpattn

using namespace cpattn;

// =================================================================== C ABI

extern "C" {

const char *cpattn_status_string(int status) {
  switch (status) {
    case CPATTN_OK: return "CPATTN_OK";
    case CPATTN_ERR_NULL: return "CPATTN_ERR_NULL: a required pointer is NULL";
    case CPATTN_ERR_SHAPE: return "CPATTN_ERR_SHAPE: unsupported shape";
    case CPATTN_ERR_INDIVISIBLE: return "CPATTN_ERR_INDIVISIBLE: length not divisible by the degree (pass explicit splits)";
    case CPATTN_ERR_SPLITS: return "CPATTN_ERR_SPLITS: negative lengths or lengths not summing to the total";
    case CPATTN_ERR_DEGREE: return "CPATTN_ERR_DEGREE: degree or step out of range";
    case CPATTN_ERR_CUDA: return "CPATTN_ERR_CUDA: CUDA runtime/driver error";
    case CPATTN_ERR_DEVICE_TIMEOUT: return "CPATTN_ERR_DEVICE_TIMEOUT: a device-side bounded wait expired";
    case CPATTN_ERR_WORKSPACE: return "CPATTN_ERR_WORKSPACE: workspace missing or too small";
    case CPATTN_ERR_ALIGNMENT: return "CPATTN_ERR_ALIGNMENT: tensor pointer not 16-byte aligned";
    case CPATTN_ERR_UNSUPPORTED: return "CPATTN_ERR_UNSUPPORTED: current device is not sm_100";
    default: return "CPATTN: unknown status";
  }
}

int cpattn_version(void) { return 1 * 10000 + 2 * 100 + 0; }

int cpattn_front_loaded_splits(int total, int parts, int *out) {
  if (out == nullptr) return CPATTN_ERR_NULL;
  if (parts < 1) return CPATTN_ERR_DEGREE;
  if (total < 0) return CPATTN_ERR_SHAPE;
  const int base = total / parts, rem = total % parts;
  for (int i = 0; i < parts; ++i) out[i] = base + (i < rem ? 1 : 0);
  return CPATTN_OK;
}

static int ring_common(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H, int S, int D,
                       int ring_degree, const int *chunk_lens, int step, bool out_f32, bool causal,
                       cudaStream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return CPATTN_ERR_NULL;
  if (out_f32 && lse == nullptr) return CPATTN_ERR_NULL;
  int st = check_attn_shape(B, H, S, D);
  if (st != CPATTN_OK) return st;
  if (ring_degree < 1 || ring_degree > kMaxRingDegree) return CPATTN_ERR_DEGREE;
  if (step >= ring_degree) return CPATTN_ERR_DEGREE;
  std::vector<int> lens;
  st = resolve_splits(S, ring_degree, chunk_lens, lens);
  if (st != CPATTN_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (lse && !aligned4(lse)))
    return CPATTN_ERR_ALIGNMENT;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  const std::vector<int> off = prefix(lens);
  std::vector<ProblemSpec> probs{full_problem(q, k, v, out, lse, B, H, S)};
  std::vector<GroupSpec> groups;
  ring_groups(groups, 0, B, lens, off, step, causal,
              [&](int b, int c) { return b * S + off[c]; });
  return run_attention(probs, groups, D, out_f32, causal, stream);
}

int cpattn_ring_attention(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H, int S,
                          int D, int ring_degree, const int *chunk_lens, cpattn_stream_t stream) {
  return ring_common(q, k, v, out, lse, B, H, S, D, ring_degree, chunk_lens, -1, false, false, stream);
}

int cpattn_causal_ring_attention(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H,
                                 int S, int D, int ring_degree, const int *chunk_lens, cpattn_stream_t stream) {
  return ring_common(q, k, v, out, lse, B, H, S, D, ring_degree, chunk_lens, -1, false, true, stream);
}

int cpattn_ring_step(const void *q, const void *k, const void *v, float *part_out, float *part_lse, int B, int H,
                     int S, int D, int ring_degree, const int *chunk_lens, int step, cpattn_stream_t stream) {
  if (step < 0) return CPATTN_ERR_DEGREE;
  return ring_common(q, k, v, part_out, part_lse, B, H, S, D, ring_degree, chunk_lens, step, true, false, stream);
}

int cpattn_causal_ring_step(const void *q, const void *k, const void *v, float *part_out, float *part_lse, int B,
                            int H, int S, int D, int ring_degree, const int *chunk_lens, int step,
                            cpattn_stream_t stream) {
  if (step < 0) return CPATTN_ERR_DEGREE;
  return ring_common(q, k, v, part_out, part_lse, B, H, S, D, ring_degree, chunk_lens, step, true, true, stream);
}

int cpattn_lse_merge(const float *part_out, const float *part_lse, int P, int B, int H, int S, int D, float *out_f32,
                     void *out_bf16, float *lse_out, cpattn_stream_t stream) {
  if (part_out == nullptr || part_lse == nullptr) return CPATTN_ERR_NULL;
  if (out_f32 == nullptr && out_bf16 == nullptr) return CPATTN_ERR_NULL;
  if (P < 1) return CPATTN_ERR_SHAPE;
  int st = check_attn_shape(B, H, S, D);
  if (st != CPATTN_OK) return st;
  if (!aligned16(part_out) || !aligned4(part_lse) || (out_f32 && !aligned16(out_f32)) ||
      (out_bf16 && !aligned16(out_bf16)) || (lse_out && !aligned4(lse_out)))
    return CPATTN_ERR_ALIGNMENT;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  MergeParams mp;
  mp.part_out = part_out;
  mp.part_lse = part_lse;
  mp.out_f32 = out_f32;
  mp.out_bf16 = static_cast<__nv_bfloat16 *>(out_bf16);
  mp.lse_out = lse_out;
  mp.P = P;
  mp.B = B;
  mp.H = H;
  mp.S = S;
  mp.D = D;
  return cuda_result(launch_lse_merge(mp, stream), "merge launch");
}

int cpattn_kv_gather_attention(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H,
                               int S, int D, int degree, const int *q_lens, cpattn_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return CPATTN_ERR_NULL;
  int st = check_attn_shape(B, H, S, D);
  if (st != CPATTN_OK) return st;
  if (degree < 1 || degree > kMaxGatherDegree) return CPATTN_ERR_DEGREE;
  std::vector<int> lens;
  st = resolve_splits(S, degree, q_lens, lens);
  if (st != CPATTN_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (lse && !aligned4(lse)))
    return CPATTN_ERR_ALIGNMENT;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  const std::vector<int> off = prefix(lens);
  std::vector<ProblemSpec> probs{full_problem(q, k, v, out, lse, B, H, S)};
  std::vector<GroupSpec> groups;
  for (int b = 0; b < B; ++b) {
    GroupSpec g;
    g.prob = 0;
    g.b = b;
    for (int r = 0; r < degree; ++r) {
      SegSpec s;
      s.row0 = b * S + off[r];
      s.nrows = lens[r];
      s.s0 = off[r];
      s.kv.push_back(AttnKV{b * S, S, 0});   // the gathered, full K/V of batch b
      g.segs.push_back(std::move(s));
    }
    groups.push_back(std::move(g));
  }
  return run_attention(probs, groups, D, false, false, stream);
}

int cpattn_ulysses_permute(const void *x, void *y, int B, int S, int H, int D, int elem_bytes, int degree,
                           const int *seq_splits, const int *head_splits, cpattn_stream_t stream) {
  PermuteParams pp;
  int st = permute_common(x, y, B, S, H, D, elem_bytes, degree, seq_splits, head_splits, 0, pp);
  if (st != CPATTN_OK) return st;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  return cuda_result(launch_permute(pp, stream), "permute launch");
}

int cpattn_ulysses_permute_qkv(const void *q, const void *k, const void *v, void *yq, void *yk, void *yv, int B,
                               int S, int H, int D, int elem_bytes, int degree, const int *seq_splits,
                               const int *head_splits, cpattn_stream_t stream) {
  PermuteParams pp;
  int st = permute_common(q, yq, B, S, H, D, elem_bytes, degree, seq_splits, head_splits, 0, pp);
  if (st != CPATTN_OK) return st;
  if (k == nullptr || v == nullptr || yk == nullptr || yv == nullptr) return CPATTN_ERR_NULL;
  if (!aligned16(k) || !aligned16(v) || !aligned16(yk) || !aligned16(yv)) return CPATTN_ERR_ALIGNMENT;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  set_qkv(pp, q, k, v, yq, yk, yv);
  return cuda_result(launch_permute(pp, stream), "permute launch");
}

int cpattn_ulysses_unpermute(const void *y, void *x, int B, int S, int H, int D, int elem_bytes, int degree,
                             const int *seq_splits, const int *head_splits, cpattn_stream_t stream) {
  PermuteParams pp;
  int st = permute_common(y, x, B, S, H, D, elem_bytes, degree, seq_splits, head_splits, 1, pp);
  if (st != CPATTN_OK) return st;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  return cuda_result(launch_permute(pp, stream), "permute launch");
}

// Head-sharded problems: head rank u's buffers start at element B*S*hoff_u*D.
static void head_sharded_problems(std::vector<ProblemSpec> &probs, std::vector<int> &prob_rank, const void *yq,
                                  const void *yk, const void *yv, void *yo, float *lse, int B, int H, int S, int D,
                                  const std::vector<int> &heads) {
  const std::vector<int> ho = prefix(heads);
  for (size_t u = 0; u < heads.size(); ++u) {
    if (heads[u] == 0) continue;
    const size_t off_bytes = static_cast<size_t>(B) * S * ho[u] * D * 2;
    ProblemSpec ps;
    ps.q = static_cast<const char *>(yq) + off_bytes;
    ps.k = static_cast<const char *>(yk) + off_bytes;
    ps.v = static_cast<const char *>(yv) + off_bytes;
    ps.out = yo != nullptr ? static_cast<char *>(yo) + off_bytes : nullptr;
    ps.lse = lse;
    ps.lse_b = static_cast<long long>(H) * S;
    ps.lse_h = S;
    ps.lse_h0 = ho[u];
    ps.H = heads[u];
    ps.rows = static_cast<long long>(B) * S;
    probs.push_back(ps);
    prob_rank.push_back(static_cast<int>(u));
  }
}

// seq_out != nullptr: the output goes to the sequence-side rank buffers
// (offsets seq_off) instead of the head-side yo (the Ulysses flow's second
// all-to-all, fused into the epilogue).
static int head_sharded_attention_impl(const void *yq, const void *yk, const void *yv, void *yo, float *lse, int B,
                                       int H, int S, int D, const std::vector<int> &heads, bool causal,
                                       cudaStream_t stream, void *seq_out = nullptr,
                                       const std::vector<int> &seq_off = {}) {
  std::vector<ProblemSpec> probs;
  std::vector<int> prob_rank;
  head_sharded_problems(probs, prob_rank, yq, yk, yv, yo, lse, B, H, S, D, heads);
  if (seq_out != nullptr) {
    const std::vector<int> ho = prefix(heads);
    for (size_t pi = 0; pi < probs.size(); ++pi) {
      ProblemSpec &ps = probs[pi];
      ps.out = seq_out;
      ps.out_mode = 1;
      ps.out_H = H;
      ps.out_h0 = ho[prob_rank[pi]];
      ps.out_B = B;
      ps.out_S = S;
      ps.out_seq_off = seq_off;
    }
  }
  std::vector<GroupSpec> groups;
  for (size_t pi = 0; pi < probs.size(); ++pi) {
    for (int b = 0; b < B; ++b) {
      GroupSpec g;
      g.prob = static_cast<int>(pi);
      g.b = b;
      SegSpec s;
      s.row0 = b * S;
      s.nrows = S;
      s.s0 = 0;
      s.kv.push_back(AttnKV{b * S, S, 0});
      g.segs.push_back(std::move(s));
      groups.push_back(std::move(g));
    }
  }
  return run_attention(probs, groups, D, false, causal, stream);
}

static int head_sharded_common(const void *yq, const void *yk, const void *yv, void *yo, float *lse, int B, int H,
                               int S, int D, int degree, const int *head_splits, bool causal, cudaStream_t stream) {
  if (yq == nullptr || yk == nullptr || yv == nullptr || yo == nullptr) return CPATTN_ERR_NULL;
  int st = check_attn_shape(B, H, S, D);
  if (st != CPATTN_OK) return st;
  if (degree < 1 || degree > kMaxRanks) return CPATTN_ERR_DEGREE;
  std::vector<int> heads;
  st = resolve_splits(H, degree, head_splits, heads);
  if (st != CPATTN_OK) return st;
  if (!aligned16(yq) || !aligned16(yk) || !aligned16(yv) || !aligned16(yo) || (lse && !aligned4(lse)))
    return CPATTN_ERR_ALIGNMENT;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  return head_sharded_attention_impl(yq, yk, yv, yo, lse, B, H, S, D, heads, causal, stream);
}

int cpattn_head_sharded_attention(const void *yq, const void *yk, const void *yv, void *yo, float *lse, int B, int H,
                                  int S, int D, int degree, const int *head_splits, cpattn_stream_t stream) {
  return head_sharded_common(yq, yk, yv, yo, lse, B, H, S, D, degree, head_splits, false, stream);
}

int cpattn_causal_head_sharded_attention(const void *yq, const void *yk, const void *yv, void *yo, float *lse, int B,
                                         int H, int S, int D, int degree, const int *head_splits,
                                         cpattn_stream_t stream) {
  return head_sharded_common(yq, yk, yv, yo, lse, B, H, S, D, degree, head_splits, true, stream);
}

int cpattn_ulysses_qkv_projection(const void *x, const void *w_qkv, void *yq, void *yk, void *yv, int B, int S,
                                  int H, int D, int Dm, int degree, const int *seq_splits, const int *head_splits,
                                  cpattn_stream_t stream) {
  if (yq == nullptr || yk == nullptr || yv == nullptr) return CPATTN_ERR_NULL;
  ProjParams pp;
  int st = projection_common(x, w_qkv, B, S, H, D, Dm, degree, seq_splits, head_splits, false, nullptr, pp);
  if (st != CPATTN_OK) return st;
  if (!aligned16(yq) || !aligned16(yk) || !aligned16(yv)) return CPATTN_ERR_ALIGNMENT;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  st = projection_common(x, w_qkv, B, S, H, D, Dm, degree, seq_splits, head_splits, false, &pp, pp);
  if (st != CPATTN_OK) return st;
  pp.y[0] = yq;
  pp.y[1] = yk;
  pp.y[2] = yv;
  return cuda_result(launch_projection(pp, stream), "projection launch");
}

int cpattn_ulysses_output_projection(const void *yo, const void *w_o, void *out, int B, int S, int H, int D, int Dm,
                                     int degree, const int *seq_splits, const int *head_splits,
                                     cpattn_stream_t stream) {
  if (out == nullptr) return CPATTN_ERR_NULL;
  ProjParams pp;
  int st = projection_common(yo, w_o, B, S, H, D, Dm, degree, seq_splits, head_splits, true, nullptr, pp);
  if (st != CPATTN_OK) return st;
  if (!aligned16(out)) return CPATTN_ERR_ALIGNMENT;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  st = projection_common(yo, w_o, B, S, H, D, Dm, degree, seq_splits, head_splits, true, &pp, pp);
  if (st != CPATTN_OK) return st;
  pp.y[0] = out;
  return cuda_result(launch_projection(pp, stream), "projection launch");
}

size_t cpattn_ulysses_workspace_bytes(int B, int H, int S, int D) {
  if (B < 1 || H < 1 || S < 1 || D < 1) return 0;
  return static_cast<size_t>(4) * B * S * H * D * 2;
}

size_t cpattn_unified_workspace_bytes(int B, int H, int S, int D) { return cpattn_ulysses_workspace_bytes(B, H, S, D); }

static int ulysses_common(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H, int S,
                          int D, int degree, const int *seq_splits, const int *head_splits, void *workspace,
                          size_t workspace_bytes, bool causal, cudaStream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return CPATTN_ERR_NULL;
  int st = check_attn_shape(B, H, S, D);
  if (st != CPATTN_OK) return st;
  if (degree < 1 || degree > kMaxRanks) return CPATTN_ERR_DEGREE;
  std::vector<int> seq_chk, heads_chk;
  st = resolve_splits(S, degree, seq_splits, seq_chk);
  if (st != CPATTN_OK) return st;
  st = resolve_splits(H, degree, head_splits, heads_chk);
  if (st != CPATTN_OK) return st;
  if (workspace == nullptr || workspace_bytes < cpattn_ulysses_workspace_bytes(B, H, S, D)) return CPATTN_ERR_WORKSPACE;
  PermuteParams pq;
  st = permute_common(q, workspace, B, S, H, D, 2, degree, seq_splits, head_splits, 0, pq);
  if (st != CPATTN_OK) return st;
  if (!aligned16(k) || !aligned16(v) || !aligned16(out) || (lse && !aligned4(lse))) return CPATTN_ERR_ALIGNMENT;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  const size_t tensor_bytes = static_cast<size_t>(B) * S * H * D * 2;
  char *ws = static_cast<char *>(workspace);
  void *yq = ws, *yk = ws + tensor_bytes, *yv = ws + 2 * tensor_bytes;
  std::vector<int> heads;
  resolve_splits(H, degree, head_splits, heads);
  // first all-to-all: Q, K, V to the head-sharded layout, one launch
  {
    PermuteParams pp = pq;
    set_qkv(pp, q, k, v, yq, yk, yv);
    if (cudaError_t e = launch_permute(pp, stream); e != cudaSuccess) return cuda_fail(e, "permute launch");
  }
  // local attention of every head rank over all S tokens of its heads; the
  // second all-to-all is fused into its epilogue, which stores each output
  // row straight into the sequence-sharded rank buffers
  std::vector<int> seq;
  resolve_splits(S, degree, seq_splits, seq);
  return head_sharded_attention_impl(yq, yk, yv, nullptr, lse, B, H, S, D, heads, causal, stream, out, prefix(seq));
}

int cpattn_ulysses_attention(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H, int S,
                             int D, int degree, const int *seq_splits, const int *head_splits, void *workspace,
                             size_t workspace_bytes, cpattn_stream_t stream) {
  return ulysses_common(q, k, v, out, lse, B, H, S, D, degree, seq_splits, head_splits, workspace, workspace_bytes,
                        false, stream);
}

int cpattn_causal_ulysses_attention(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H,
                                    int S, int D, int degree, const int *seq_splits, const int *head_splits,
                                    void *workspace, size_t workspace_bytes, cpattn_stream_t stream) {
  return ulysses_common(q, k, v, out, lse, B, H, S, D, degree, seq_splits, head_splits, workspace, workspace_bytes,
                        true, stream);
}

static int unified_common(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H, int S,
                          int D, int ring_degree, int ulysses_degree, const int *ring_lens, const int *head_splits,
                          void *workspace, size_t workspace_bytes, bool causal, cudaStream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return CPATTN_ERR_NULL;
  int st = check_attn_shape(B, H, S, D);
  if (st != CPATTN_OK) return st;
  if (ring_degree < 1 || ring_degree > kMaxRanks || ulysses_degree < 1 || ulysses_degree > kMaxRanks)
    return CPATTN_ERR_DEGREE;
  std::vector<int> lens, heads;
  st = resolve_splits(S, ring_degree, ring_lens, lens);
  if (st != CPATTN_OK) return st;
  st = resolve_splits(H, ulysses_degree, head_splits, heads);
  if (st != CPATTN_OK) return st;
  if (H > kMaxHeads) return CPATTN_ERR_SHAPE;
  if (workspace == nullptr || workspace_bytes < cpattn_unified_workspace_bytes(B, H, S, D)) return CPATTN_ERR_WORKSPACE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(workspace) ||
      (lse && !aligned4(lse)))
    return CPATTN_ERR_ALIGNMENT;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  const std::vector<int> off = prefix(lens), ho = prefix(heads);
  const size_t tensor_bytes = static_cast<size_t>(B) * S * H * D * 2;
  char *ws = static_cast<char *>(workspace);
  void *yq = ws, *yk = ws + tensor_bytes, *yv = ws + 2 * tensor_bytes;

  // Permutation within every ring group (ring chunk i): full BSHD rows of the
  // chunk -> head group u buffer laid out [i][B, len_i, H_u, D].
  PermuteParams pp;
  std::memset(&pp, 0, sizeof(pp));
  pp.B = B;
  pp.S = S;
  pp.H = H;
  pp.row_bytes = D * 2;
  pp.seq_mode = 0;
  pp.n_seq = 1;
  pp.n_groups = ring_degree;
  for (int i = 0; i <= ring_degree; ++i) pp.group_off[i] = off[i];
  pp.n_head = ulysses_degree;
  for (int u = 0; u <= ulysses_degree; ++u) pp.head_off[u] = ho[u];
  {
    PermuteParams p1 = pp;
    set_qkv(p1, q, k, v, yq, yk, yv);
    p1.direction = 0;
    if (cudaError_t e = launch_permute(p1, stream); e != cudaSuccess) return cuda_fail(e, "permute launch");
  }
  // Ring attention per head group over the chunks (rows B*off_i + b*len_i).
  std::vector<ProblemSpec> probs;
  std::vector<int> prob_rank;
  head_sharded_problems(probs, prob_rank, yq, yk, yv, nullptr, lse, B, H, S, D, heads);
  // The inverse permutation is fused into the epilogue: each output row goes
  // straight to the full (B, S, H, D) tensor at its head's global index.
  for (size_t pi = 0; pi < probs.size(); ++pi) {
    ProblemSpec &ps = probs[pi];
    ps.out = out;
    ps.out_mode = 2;
    ps.out_H = H;
    ps.out_h0 = ho[prob_rank[pi]];
    ps.out_B = B;
    ps.out_S = S;
  }
  std::vector<GroupSpec> groups;
  for (size_t pi = 0; pi < probs.size(); ++pi)
    ring_groups(groups, static_cast<int>(pi), B, lens, off, -1, causal,
                [&](int b, int c) { return B * off[c] + b * lens[c]; });
  return run_attention(probs, groups, D, false, causal, stream);
}

int cpattn_unified_attention(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H, int S,
                             int D, int ring_degree, int ulysses_degree, const int *ring_lens,
                             const int *head_splits, void *workspace, size_t workspace_bytes,
                             cpattn_stream_t stream) {
  return unified_common(q, k, v, out, lse, B, H, S, D, ring_degree, ulysses_degree, ring_lens, head_splits, workspace,
                        workspace_bytes, false, stream);
}

int cpattn_causal_unified_attention(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H,
                                    int S, int D, int ring_degree, int ulysses_degree, const int *ring_lens,
                                    const int *head_splits, void *workspace, size_t workspace_bytes,
                                    cpattn_stream_t stream) {
  return unified_common(q, k, v, out, lse, B, H, S, D, ring_degree, ulysses_degree, ring_lens, head_splits, workspace,
                        workspace_bytes, true, stream);
}

// ------------------------------------------- building blocks of the exchanges

int cpattn_ring_chunk_attention(const void *q, const void *k, const void *v, void *out, float *lse,
                                const float *prev_out, int B, int H, int Sq, int Skv, int kv_batch_rows, int D,
                                int q_pos0, int kv_pos0, int causal, int out_f32, cpattn_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || lse == nullptr) return CPATTN_ERR_NULL;
  int st = check_attn_shape(B, H, Sq, D);
  if (st != CPATTN_OK) return st;
  if (Skv < 0 || kv_batch_rows < 1 || kv_batch_rows < Skv || q_pos0 < 0 || kv_pos0 < 0) return CPATTN_ERR_SHAPE;
  if (static_cast<long long>(B) * kv_batch_rows > INT_MAX ||
      static_cast<long long>(B) * kv_batch_rows * H * D > (1ll << 46) ||
      static_cast<long long>(q_pos0) + Sq > INT_MAX || static_cast<long long>(kv_pos0) + Skv > INT_MAX)
    return CPATTN_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned4(lse) ||
      (prev_out && !aligned16(prev_out)))
    return CPATTN_ERR_ALIGNMENT;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  ProblemSpec ps = full_problem(q, k, v, out, lse, B, H, Sq);
  ps.rows_kv = static_cast<long long>(B) * kv_batch_rows;
  ps.prev = prev_out;
  ps.lse_pos0 = q_pos0;
  std::vector<GroupSpec> groups;
  for (int b = 0; b < B; ++b) {
    GroupSpec g;
    g.prob = 0;
    g.b = b;
    SegSpec sg;
    sg.row0 = b * Sq;
    sg.nrows = Sq;
    sg.s0 = q_pos0;
    if (Skv > 0) sg.kv.push_back(AttnKV{b * kv_batch_rows, Skv, kv_pos0});
    g.segs.push_back(std::move(sg));
    groups.push_back(std::move(g));
  }
  return run_attention({ps}, groups, D, out_f32 != 0, causal != 0, stream);
}

int cpattn_gathered_kv_attention(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H,
                                 int D, int degree, const int *kv_lens, int kv_batch_rows, int rank, int causal,
                                 cpattn_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return CPATTN_ERR_NULL;
  if (degree < 1 || degree > kMaxRingDegree || rank < 0 || rank >= degree) return CPATTN_ERR_DEGREE;
  if (B < 1 || H < 1 || kv_batch_rows < 1) return CPATTN_ERR_SHAPE;
  std::vector<int> lens(degree, kv_batch_rows);
  if (kv_lens != nullptr)
    for (int c = 0; c < degree; ++c) {
      if (kv_lens[c] < 0 || kv_lens[c] > kv_batch_rows) return CPATTN_ERR_SPLITS;
      lens[c] = kv_lens[c];
    }
  const int Sq = lens[rank];
  long long total = 0;
  for (int c = 0; c < degree; ++c) total += lens[c];
  if (total > INT_MAX || Sq < 1) return CPATTN_ERR_SHAPE;
  int st = check_attn_shape(B, H, Sq, D);
  if (st != CPATTN_OK) return st;
  const long long rows_kv = static_cast<long long>(degree) * B * kv_batch_rows;
  if (rows_kv > INT_MAX || rows_kv * H * D > (1ll << 46)) return CPATTN_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (lse && !aligned4(lse)))
    return CPATTN_ERR_ALIGNMENT;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  const std::vector<int> off = prefix(lens);
  ProblemSpec ps = full_problem(q, k, v, out, lse, B, H, Sq);
  ps.rows_kv = rows_kv;
  ps.lse_pos0 = off[rank];
  std::vector<GroupSpec> groups;
  for (int b = 0; b < B; ++b) {
    GroupSpec g;
    g.prob = 0;
    g.b = b;
    SegSpec sg;
    sg.row0 = b * Sq;
    sg.nrows = Sq;
    sg.s0 = off[rank];
    for (int i_t = 0; i_t < degree; ++i_t) {
      // Ring order from this rank's own chunk (the order the chunks arrive
      // in); under the causal mask the chunks after the shard are invisible
      // and the own chunk, the one the mask cuts, is visited last, so that
      // the keys the first Q tile of a pair cannot see come last in the walk.
      const int t = causal ? (i_t + 1) % degree : i_t;
      const int c = ((rank - t) % degree + degree) % degree;
      if (causal && c > rank) continue;
      if (lens[c] > 0) sg.kv.push_back(AttnKV{(c * B + b) * kv_batch_rows, lens[c], off[c]});
    }
    g.segs.push_back(std::move(sg));
    groups.push_back(std::move(g));
  }
  return run_attention({ps}, groups, D, false, causal != 0, stream);
}

int cpattn_rank_buffer_attention(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H,
                                 int S, int D, int degree, const int *seq_splits, int causal,
                                 cpattn_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return CPATTN_ERR_NULL;
  int st = check_attn_shape(B, H, S, D);
  if (st != CPATTN_OK) return st;
  if (degree < 1 || degree > kMaxRanks) return CPATTN_ERR_DEGREE;
  std::vector<int> lens;
  st = resolve_splits(S, degree, seq_splits, lens);
  if (st != CPATTN_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (lse && !aligned4(lse)))
    return CPATTN_ERR_ALIGNMENT;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  const std::vector<int> off = prefix(lens);
  std::vector<ProblemSpec> probs{full_problem(q, k, v, out, lse, B, H, S)};
  std::vector<GroupSpec> groups;
  // Every rank buffer attends every rank buffer of its batch element: the
  // ring plan over the buffers, rows B*off_u + b*len_u.
  ring_groups(groups, 0, B, lens, off, -1, causal != 0, [&](int b, int c) { return B * off[c] + b * lens[c]; });
  return run_attention(probs, groups, D, false, causal != 0, stream);
}

size_t cpattn_attention_backward_workspace_bytes(int B, int H, int S) {
  if (B < 1 || H < 1 || S < 1) return 0;
  return static_cast<size_t>(B) * H * S * sizeof(float);
}

size_t cpattn_attention_backward_ds_bytes(int B, int S, int causal) {
  if (B < 1 || S < 1) return 0;
  const int nt = (S + 127) / 128;
  return static_cast<size_t>(B) * static_cast<size_t>(bwd_ds_tiles_per_head(nt, causal != 0)) * kBwdDsTileBytes;
}

// One backward problem over [B, S, H, D] tensors; LSE index b*lse_b + (h + lse_h0)*lse_h + s.
static bool backward_problem(BwdProblem &pb, const void *q, const void *k, const void *v, const void *dout,
                             const float *lse, long long lse_b, long long lse_h, int lse_h0, float *delta, void *dq,
                             void *dk, void *dv, int B, int S, int H, int D) {
  std::memset(&pb, 0, sizeof(pb));
  const long long rows = static_cast<long long>(B) * S;
  if (!encode_rows_map(&pb.tm_q, q, D, H, rows) || !encode_rows_map(&pb.tm_k, k, D, H, rows) ||
      !encode_rows_map(&pb.tm_v, v, D, H, rows) || !encode_rows_map(&pb.tm_do, dout, D, H, rows))
    return false;
  pb.lse = lse;
  pb.lse_b = lse_b;
  pb.lse_h = lse_h;
  pb.lse_h0 = lse_h0;
  pb.H = H;
  pb.h0 = 0;
  pb.nh = H;
  pb.delta = delta;
  pb.dq = dq;
  pb.dk = dk;
  pb.dv = dv;
  return true;
}

static void backward_common_params(BwdParams &P, int B, int S, int D, bool causal) {
  P.B = B;
  P.S = S;
  P.causal = causal ? 1 : 0;
  P.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  P.scale_log2 = static_cast<float>((1.0 / std::sqrt(static_cast<double>(D))) * 1.4426950408889634);
  P.timeout_ns = wait_timeout_ns();
}

// The part of a workspace past its first `used` bytes, from a 256-byte
// boundary, as dS scratch.
static void ds_scratch(void *workspace, size_t workspace_bytes, size_t used, unsigned char *&scratch,
                       size_t &scratch_bytes) {
  const size_t start = (used + 255) & ~static_cast<size_t>(255);
  const uintptr_t base = (reinterpret_cast<uintptr_t>(workspace) + start + 255) & ~static_cast<uintptr_t>(255);
  const size_t skip = base - reinterpret_cast<uintptr_t>(workspace);
  scratch = nullptr;
  scratch_bytes = 0;
  if (workspace_bytes > skip) {
    scratch = reinterpret_cast<unsigned char *>(base);
    scratch_bytes = workspace_bytes - skip;
  }
}

// The gradient kernels over `sets` (problems covering all their heads, Delta
// computed).  When the scratch holds the dS tiles of at least one head, the
// heads are cut into groups whose tiles fit the scratch together (up to
// kMaxProblems groups per launch): the dK/dV kernel stores dS and the dQ GEMM
// reads it.  The scratch is reused by the next launch, which the stream orders
// after the GEMM that read it.  Otherwise the dQ kernel recomputes S and dP.
static cudaError_t run_bwd_sets(const std::vector<BwdProblem> &sets, unsigned char *scratch, size_t scratch_bytes,
                                int B, int S, int D, bool causal, cudaStream_t stream) {
  const size_t per_head = cpattn_attention_backward_ds_bytes(B, S, causal ? 1 : 0);
  const long long cap = (scratch != nullptr && per_head > 0) ? static_cast<long long>(scratch_bytes / per_head) : 0;
  const int nt = (S + 127) / 128;
  std::unique_ptr<BwdParams> P(new BwdParams);
  std::memset(P.get(), 0, sizeof(BwdParams));
  int n_prob = 0, units = 0;
  long long used = 0;
  auto flush = [&]() -> cudaError_t {
    if (n_prob == 0) return cudaSuccess;
    P->n_prob = n_prob;
    backward_common_params(*P, B, S, D, causal);
    const cudaError_t e = launch_bwd_kernels(*P, D, stream);
    std::memset(P.get(), 0, sizeof(BwdParams));
    n_prob = 0;
    units = 0;
    used = 0;
    return e;
  };
  for (const BwdProblem &set : sets) {
    for (int h = 0; h < set.H;) {
      if (n_prob == kMaxProblems || (cap > 0 && used == cap))
        if (cudaError_t e = flush(); e != cudaSuccess) return e;
      BwdProblem &pb = P->prob[n_prob];
      pb = set;
      pb.h0 = h;
      pb.nh = cap > 0 ? static_cast<int>(std::min<long long>(set.H - h, cap - used)) : set.H;
      pb.ds = cap > 0 ? scratch + static_cast<size_t>(used) * per_head : nullptr;
      pb.unit_base = units;
      units += B * pb.nh * nt;
      used += cap > 0 ? pb.nh : 0;
      h += pb.nh;
      ++n_prob;
    }
  }
  return flush();
}

int cpattn_attention_backward(const void *q, const void *k, const void *v, const void *out, const float *lse,
                              const void *dout, void *dq, void *dk, void *dv, int B, int H, int S, int D,
                              int causal, void *workspace, size_t workspace_bytes, cpattn_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || lse == nullptr || dout == nullptr ||
      dq == nullptr || dk == nullptr || dv == nullptr)
    return CPATTN_ERR_NULL;
  int st = check_bwd_shape(B, H, S, D);
  if (st != CPATTN_OK) return st;
  const size_t delta_bytes = cpattn_attention_backward_workspace_bytes(B, H, S);
  if (workspace == nullptr || workspace_bytes < delta_bytes) return CPATTN_ERR_WORKSPACE;
  const void *ptrs[8] = {q, k, v, out, dout, dq, dk, dv};
  for (const void *ptr : ptrs)
    if (!aligned16(ptr)) return CPATTN_ERR_ALIGNMENT;
  if (!aligned4(lse) || !aligned4(workspace)) return CPATTN_ERR_ALIGNMENT;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  std::vector<BwdProblem> sets(1);
  float *delta = static_cast<float *>(workspace);
  if (!backward_problem(sets[0], q, k, v, dout, lse, static_cast<long long>(H) * S, S, 0, delta, dq, dk, dv, B, S,
                        H, D))
    return cuda_fail(cudaErrorInvalidValue, t_encode_detail);
  unsigned char *scratch;
  size_t scratch_bytes;
  ds_scratch(workspace, workspace_bytes, delta_bytes, scratch, scratch_bytes);
  if (cudaError_t e = launch_bwd_delta(out, dout, delta, B, S, H, D, stream); e != cudaSuccess)
    return cuda_fail(e, "backward launch");
  return cuda_result(run_bwd_sets(sets, scratch, scratch_bytes, B, S, D, causal != 0, stream), "backward launch");
}

size_t cpattn_ulysses_attention_backward_workspace_bytes(int B, int H, int S, int D) {
  if (B < 1 || H < 1 || S < 1 || D < 1) return 0;
  return static_cast<size_t>(5) * B * S * H * D * 2 + static_cast<size_t>(B) * H * S * sizeof(float);
}

int cpattn_ulysses_attention_backward(const void *q, const void *k, const void *v, const void *out,
                                      const float *lse, const void *dout, void *dq, void *dk, void *dv, int B,
                                      int H, int S, int D, int degree, const int *seq_splits,
                                      const int *head_splits, int causal, void *workspace, size_t workspace_bytes,
                                      cpattn_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || lse == nullptr || dout == nullptr ||
      dq == nullptr || dk == nullptr || dv == nullptr)
    return CPATTN_ERR_NULL;
  int st = check_bwd_shape(B, H, S, D);
  if (st != CPATTN_OK) return st;
  if (degree < 1 || degree > kMaxRanks) return CPATTN_ERR_DEGREE;
  std::vector<int> seq_chk, heads;
  st = resolve_splits(S, degree, seq_splits, seq_chk);
  if (st != CPATTN_OK) return st;
  st = resolve_splits(H, degree, head_splits, heads);
  if (st != CPATTN_OK) return st;
  const size_t base_bytes = cpattn_ulysses_attention_backward_workspace_bytes(B, H, S, D);
  if (workspace == nullptr || workspace_bytes < base_bytes) return CPATTN_ERR_WORKSPACE;
  PermuteParams pq;
  st = permute_common(q, workspace, B, S, H, D, 2, degree, seq_splits, head_splits, 0, pq);
  if (st != CPATTN_OK) return st;
  const void *ptrs[8] = {k, v, out, dout, dq, dk, dv, workspace};
  for (const void *ptr : ptrs)
    if (!aligned16(ptr)) return CPATTN_ERR_ALIGNMENT;
  if (!aligned4(lse)) return CPATTN_ERR_ALIGNMENT;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  // workspace: head-side yq, yk, yv, yo, ydo, then Delta per head rank, then
  // (optionally) dS scratch
  const size_t tb = static_cast<size_t>(B) * S * H * D * 2;
  char *ws = static_cast<char *>(workspace);
  void *y[5];
  for (int i = 0; i < 5; ++i) y[i] = ws + i * tb;
  float *delta = reinterpret_cast<float *>(ws + 5 * tb);
  unsigned char *scratch;
  size_t scratch_bytes;
  ds_scratch(workspace, workspace_bytes, base_bytes, scratch, scratch_bytes);
  // first all-to-all: Q, K, V, then O and dO, to the head-sharded layout
  {
    PermuteParams pp = pq;
    set_qkv(pp, q, k, v, y[0], y[1], y[2]);
    if (cudaError_t e = launch_permute(pp, stream); e != cudaSuccess) return cuda_fail(e, "permute launch");
    pp.src[0] = static_cast<const unsigned char *>(out);
    pp.dst[0] = static_cast<unsigned char *>(y[3]);
    pp.src[1] = static_cast<const unsigned char *>(dout);
    pp.dst[1] = static_cast<unsigned char *>(y[4]);
    pp.n_tensors = 2;
    if (cudaError_t e = launch_permute(pp, stream); e != cudaSuccess) return cuda_fail(e, "permute launch");
  }
  // the backward of every head rank's local attention: one problem per head
  // rank, its Delta first.  The kernels store dQ, dK and dV straight into the
  // sequence-sharded rank buffers (the second all-to-all, fused).
  const std::vector<int> ho = prefix(heads);
  const std::vector<int> so = prefix(seq_chk);
  // With equal head splits the head-side O and dO buffers of all ranks, and
  // their Delta slices, are one [degree * B, S, H / degree, D] tensor set:
  // one row-sum launch covers every rank.
  const bool even_heads = std::all_of(heads.begin(), heads.end(), [&](int x) { return x == heads[0]; });
  if (even_heads && heads[0] > 0) {
    if (cudaError_t e = launch_bwd_delta(y[3], y[4], delta, degree * B, S, heads[0], D, stream); e != cudaSuccess)
      return cuda_fail(e, "backward launch");
  }
  std::vector<BwdProblem> sets;
  sets.reserve(degree);
  for (int u = 0; u < degree; ++u) {
    if (heads[u] == 0) continue;
    const size_t off = static_cast<size_t>(B) * S * ho[u] * D * 2;
    auto at = [&](int i) { return static_cast<void *>(static_cast<char *>(y[i]) + off); };
    float *dl = delta + static_cast<size_t>(B) * ho[u] * S;
    sets.emplace_back();
    BwdProblem &pb = sets.back();
    if (!backward_problem(pb, at(0), at(1), at(2), at(4), lse, static_cast<long long>(H) * S, S, ho[u], dl, dq, dk,
                          dv, B, S, heads[u], D))
      return cuda_fail(cudaErrorInvalidValue, t_encode_detail);
    pb.out_mode = 1;
    pb.out_H = H;
    pb.out_h0 = ho[u];
    pb.out_nseq = degree;
    for (int r = 0; r <= degree; ++r) pb.out_seq_off[r] = so[r];
    if (!even_heads) {
      if (cudaError_t e = launch_bwd_delta(at(3), at(4), dl, B, S, heads[u], D, stream); e != cudaSuccess)
        return cuda_fail(e, "backward launch");
    }
  }
  return cuda_result(run_bwd_sets(sets, scratch, scratch_bytes, B, S, D, causal != 0, stream), "backward launch");
}

int cpattn_exchange_bytes(int mode, int B, int H, int S, int D, int elem_bytes, int degree, const int *seq_splits,
                          const int *head_splits, unsigned long long *send, unsigned long long *recv) {
  if (send == nullptr || recv == nullptr) return CPATTN_ERR_NULL;
  if (B < 1 || H < 1 || S < 1 || D < 1 || elem_bytes < 1 || mode < 0 || mode > 2) return CPATTN_ERR_SHAPE;
  std::vector<int> seq, heads;
  int st = resolve_splits(S, degree, seq_splits, seq);
  if (st != CPATTN_OK) return st;
  if (mode == 1) {
    st = resolve_splits(H, degree, head_splits, heads);
    if (st != CPATTN_OK) return st;
  }
  const unsigned long long row = static_cast<unsigned long long>(D) * elem_bytes;   // one (token, head)
  for (int r = 0; r < degree; ++r) {
    const unsigned long long sr = static_cast<unsigned long long>(seq[r]);
    const unsigned long long so = static_cast<unsigned long long>(S) - sr;
    if (mode == 1) {
      const unsigned long long hr = static_cast<unsigned long long>(heads[r]);
      const unsigned long long ho = static_cast<unsigned long long>(H) - hr;
      send[r] = (3ull * B * sr * ho + 1ull * B * so * hr) * row;
      recv[r] = (3ull * B * so * hr + 1ull * B * sr * ho) * row;
    } else {
      recv[r] = 2ull * B * so * static_cast<unsigned long long>(H) * row;
      send[r] = 2ull * static_cast<unsigned long long>(degree - 1) * B * sr * static_cast<unsigned long long>(H) * row;
    }
  }
  return CPATTN_OK;
}

// (query, key) pairs of queries at positions q0 .. q0+nq-1 and keys at
// k0 .. k0+nk-1 that attention sees: all of them, or under the causal mask
// those with key position <= query position.
static double visible_pairs(long long q0, long long nq, long long k0, long long nk, bool causal) {
  if (nq <= 0 || nk <= 0) return 0.0;
  if (!causal) return static_cast<double>(nq) * static_cast<double>(nk);
  // query i sees clamp(i - k0 + 1, 0, nk) keys; sum it in closed form over
  // the three stretches (none, a growing run, all nk)
  double total = 0.0;
  const long long q1 = q0 + nq;                       // exclusive
  const long long a = std::max(q0, k0);               // first query that sees a key
  const long long b = std::min(q1, k0 + nk - 1);      // first query that sees all nk
  if (a < b) {
    const double first = static_cast<double>(a - k0 + 1), last = static_cast<double>(b - 1 - k0 + 1);
    total += (first + last) * static_cast<double>(b - a) / 2.0;
  }
  const long long full_from = std::max(q0, k0 + nk - 1);
  if (q1 > full_from) total += static_cast<double>(q1 - full_from) * static_cast<double>(nk);
  return total;
}

int cpattn_plan_exchange(int B, int H, int S, int D, int elem_bytes, int degree, const int *seq_splits,
                         const int *head_splits, const cpattn_exchange_env *env, cpattn_exchange_plan *plan) {
  if (env == nullptr || plan == nullptr) return CPATTN_ERR_NULL;
  if (B < 1 || H < 1 || S < 1 || D < 1 || elem_bytes < 1) return CPATTN_ERR_SHAPE;
  if (!(env->link_gbs > 0.0) || !(env->attn_tflops > 0.0) || !(env->hbm_gbs > 0.0)) return CPATTN_ERR_SHAPE;
  if (degree < 1 || degree > kMaxRanks) return CPATTN_ERR_DEGREE;
  std::vector<int> seq, heads;
  int st = resolve_splits(S, degree, seq_splits, seq);
  if (st != CPATTN_OK) return st;
  const bool ulysses_ok = resolve_splits(H, degree, head_splits, heads) == CPATTN_OK;
  if (!ulysses_ok && head_splits != nullptr) return resolve_splits(H, degree, head_splits, heads);
  const bool causal = env->causal != 0;
  const std::vector<int> off = prefix(seq);
  std::vector<unsigned long long> snd(degree), rcv_ring(degree), rcv_uly(degree);
  st = cpattn_exchange_bytes(0, B, H, S, D, elem_bytes, degree, seq_splits, nullptr, snd.data(), rcv_ring.data());
  if (st != CPATTN_OK) return st;
  if (ulysses_ok) {
    st = cpattn_exchange_bytes(1, B, H, S, D, elem_bytes, degree, seq_splits, head_splits, snd.data(),
                               rcv_uly.data());
    if (st != CPATTN_OK) return st;
  }
  const double link = env->link_gbs * 1e9, flops_s = env->attn_tflops * 1e12, hbm = env->hbm_gbs * 1e9;
  const double row = static_cast<double>(D) * elem_bytes;          // bytes of one (token, head)
  const double pair_flops = 4.0 * D * B;                           // per (query, key, head)
  std::memset(plan, 0, sizeof(*plan));
  for (int m = 0; m < 3; ++m) plan->seconds[m] = 0.0;
  int max_chunk = 0;
  for (int c = 0; c < degree; ++c) max_chunk = std::max(max_chunk, seq[c]);
  for (int r = 0; r < degree; ++r) {
    // ring (and kv_gather, which attends to the same chunks)
    double t_ring = 0.0, f_all = 0.0;
    for (int t = 0; t < degree; ++t) {
      const int c = ((r - t) % degree + degree) % degree;
      const double f = pair_flops * H * visible_pairs(off[r], seq[r], off[c], seq[c], causal);
      const double a = f / flops_s;
      f_all += f;
      if (t == 0) t_ring += a;
      else t_ring += std::max(a, 2.0 * B * static_cast<double>(seq[c]) * H * row / link);
    }
    plan->seconds[0] = std::max(plan->seconds[0], t_ring);
    plan->flops[0] = std::max(plan->flops[0], f_all);
    plan->recv_bytes[0] = std::max(plan->recv_bytes[0], rcv_ring[r]);
    plan->resident_bytes[0] = std::max(plan->resident_bytes[0],
        static_cast<unsigned long long>((2.0 * seq[r] + 4.0 * max_chunk) * B * H * row));
    if (!causal) {
      plan->seconds[2] = std::max(plan->seconds[2], static_cast<double>(rcv_ring[r]) / link + f_all / flops_s);
      plan->flops[2] = std::max(plan->flops[2], f_all);
      plan->recv_bytes[2] = std::max(plan->recv_bytes[2], rcv_ring[r]);
      plan->resident_bytes[2] = std::max(plan->resident_bytes[2],
          static_cast<unsigned long long>((2.0 * seq[r] + 2.0 * S) * B * H * row));
    }
    if (ulysses_ok) {
      const double f = pair_flops * heads[r] * visible_pairs(0, S, 0, S, causal);
      const double t_u = static_cast<double>(rcv_uly[r]) / link + 8.0 * B * seq[r] * H * row / hbm + f / flops_s;
      plan->seconds[1] = std::max(plan->seconds[1], t_u);
      plan->flops[1] = std::max(plan->flops[1], f);
      plan->recv_bytes[1] = std::max(plan->recv_bytes[1], rcv_uly[r]);
      plan->resident_bytes[1] = std::max(plan->resident_bytes[1],
          static_cast<unsigned long long>(4.0 * B * S * heads[r] * row));
    }
  }
  if (!ulysses_ok) plan->seconds[1] = -1.0;
  if (causal) plan->seconds[2] = -1.0;
  plan->best = 0;
  for (int m = 1; m < 3; ++m)
    if (plan->seconds[m] >= 0.0 && plan->seconds[m] < plan->seconds[plan->best]) plan->best = m;
  return CPATTN_OK;
}

int cpattn_last_cuda_error(void) { return static_cast<int>(cpattn::t_last_cuda_error); }

const char *cpattn_last_cuda_error_string(void) {
  static thread_local char buf[256];
  const cudaError_t e = cpattn::t_last_cuda_error;
  if (e == cudaSuccess) return "no CUDA error recorded on this thread";
  std::snprintf(buf, sizeof(buf), "%s: %s (%s)", cpattn::t_last_cuda_step, cudaGetErrorName(e), cudaGetErrorString(e));
  return buf;
}

int cpattn_device_status(cpattn_stream_t stream, unsigned int *code) {
  if (code == nullptr) return CPATTN_ERR_NULL;
  int st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  unsigned int v = 0;
  if (cudaError_t e = read_and_clear_device_status(&v, stream); e != cudaSuccess) return cuda_fail(e, "status read");
  *code = v;
  return v == 0 ? CPATTN_OK : CPATTN_ERR_DEVICE_TIMEOUT;
}

int cpattn_debug_wait_timeout(unsigned int timeout_us, cpattn_stream_t stream) {
  if (timeout_us < 1 || timeout_us > 1000000) return CPATTN_ERR_SHAPE;
  int st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  return cuda_result(launch_debug_wait(static_cast<unsigned long long>(timeout_us) * 1000ull, stream),
                     "debug wait launch");
}

}  // extern "C"

// ======================================================= no-allocation variant
//
// Ulysses attention whose scratch is a file-scope device array instead of a
// caller-provided workspace (see cpattn_ulysses_attention_noalloc in
// cpattn.h).  In host code `g_noalloc_scratch` only names the symbol; its
// device address comes from cudaGetSymbolAddress, looked up once per device
// with that device current.

namespace cpattn {

static __device__ __align__(256) unsigned char g_noalloc_scratch[CPATTN_NOALLOC_SCRATCH_BYTES];

static int noalloc_scratch_address(void **out) {
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(e, "device query");
  }
  if (dev < 0 || dev >= kMaxDevices) return CPATTN_ERR_UNSUPPORTED;
  static std::mutex mu;
  static void *addr[kMaxDevices] = {nullptr};
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch); e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return cuda_fail(e, "scratch symbol lookup");
    }
    addr[dev] = p;
  }
  *out = addr[dev];
  return CPATTN_OK;
}

}  // namespace cpattn

extern "C" int cpattn_ulysses_attention_noalloc(const void *q, const void *k, const void *v, void *out, float *lse,
                                                int B, int H, int S, int D, int degree, const int *seq_splits,
                                                const int *head_splits, cpattn_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return CPATTN_ERR_NULL;
  int st = check_attn_shape(B, H, S, D);
  if (st != CPATTN_OK) return st;
  if (degree < 1 || degree > kMaxRanks) return CPATTN_ERR_DEGREE;
  std::vector<int> seq_chk, heads_chk;
  st = resolve_splits(S, degree, seq_splits, seq_chk);
  if (st != CPATTN_OK) return st;
  st = resolve_splits(H, degree, head_splits, heads_chk);
  if (st != CPATTN_OK) return st;
  if (cpattn_ulysses_workspace_bytes(B, H, S, D) > static_cast<size_t>(CPATTN_NOALLOC_SCRATCH_BYTES))
    return CPATTN_ERR_WORKSPACE;
  st = check_device(nullptr);
  if (st != CPATTN_OK) return st;
  void *scratch = nullptr;
  st = noalloc_scratch_address(&scratch);
  if (st != CPATTN_OK) return st;
  return cpattn_ulysses_attention(q, k, v, out, lse, B, H, S, D, degree, seq_splits, head_splits, scratch,
                                  static_cast<size_t>(CPATTN_NOALLOC_SCRATCH_BYTES), stream);
}
