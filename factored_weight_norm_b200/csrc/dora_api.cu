// dora_api.cu - the C ABI declared in include/dora.h: argument validation,
// launch planning, TMA descriptor encoding and kernel launches.
//
// The library never allocates device memory: every buffer, including the
// workspace, comes from the caller.  All work is enqueued on the caller's
// stream.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <atomic>
#include <chrono>
#include <mutex>

#include "../../include/dora.h"
#include "compose.cuh"
#include "linear_tc.cuh"
#include "norm_bwd.cuh"
#include "norm_simt.cuh"
#include "norm_tc.cuh"
#include "gram_cluster.cuh"
#include "norm_batched.cuh"

namespace dora {

// Device-side status word: kernels write DORA_ERR_TIMEOUT here when a bounded
// wait gives up.  One per device (a __device__ variable lives in every
// context that loads the library).
__device__ int g_status = 0;

namespace {

constexpr long long kWaitLimitCycles = 2000000000LL;  // ~1 s at B200 clocks

// linear_pair_kernel: as many 32 KB stages as fit, at most kLinStagesMax
int linear_pair_stages(int smem_optin) {
  return static_cast<int>(std::min<size_t>(kLinStagesMax, (smem_optin - 1024 - kLinBarrierBytes) / kPairStageBytes));
}
size_t linear_pair_smem(int smem_optin) {
  return static_cast<size_t>(linear_pair_stages(smem_optin)) * kPairStageBytes + 1024 + kLinBarrierBytes;
}
// Pair tile width along N for an output of N columns: the one of 256, 192,
// 128 that pads N least (the wider on a tie), e.g. r = 384 -> 2 x 192.
int pick_bn(long long N) {
  int best = 256;
  long long waste = (N + 255) / 256 * 256 - N;
  for (int bn : {192, 128}) {
    const long long w = (N + bn - 1) / bn * bn - N;
    if (w < waste) {
      waste = w;
      best = bn;
    }
  }
  return best;
}

template <typename K>
int pair_attrs(K kernel, int smem_optin) {
  return (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_optin) != cudaSuccess ||
          cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 0) != cudaSuccess)
             ? DORA_ERR_CUDA
             : DORA_OK;
}
constexpr int kMaxGrid = 1024;                         // bound on the persistent grid
constexpr int kMaxGramSplits = 32;
constexpr int kGramMinBlocks = 4;                      // fewest K blocks a Gram CTA of the norm takes
constexpr int kMaxBwdChunks = 64;
constexpr int kMaxDevices = 64;
constexpr int64_t kMaxRank = 4096;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  int smem_optin = 0;
  int* status = nullptr;
  int pair_clusters = 0;  // co-resident 2-CTA clusters of linear_pair_kernel
};

std::mutex g_mu;

// Kernels this library has launched in this process (every launch site
// counts itself once, before it launches).
std::atomic<unsigned long long> g_launches{0};
inline void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
DeviceInfo g_dev[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Per-device set-up, done once with that device current.
template <typename K>
int gram_cluster_attrs(K kernel) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kGcSmem)) !=
                 cudaSuccess ||
             cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                  cudaSharedmemCarveoutMaxShared) != cudaSuccess
             ? DORA_ERR_CUDA
             : DORA_OK;
}

int device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DORA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DORA_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return DORA_ERR_CUDA;
    d.status = static_cast<int*>(p);
    if (cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      return DORA_ERR_CUDA;
    if (cudaFuncSetAttribute(norm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, d.smem_optin) != cudaSuccess)
      return DORA_ERR_CUDA;
    if (cudaFuncSetAttribute(gram_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, d.smem_optin) != cudaSuccess)
      return DORA_ERR_CUDA;
    // Kernels that run beside the first CTAs of a GEMM launched behind them
    // ask for the largest shared-memory carveout: an SM configured for a
    // small one (the default for a kernel with little shared memory) takes no
    // GEMM CTA until it drains.
    if (cudaFuncSetAttribute(gram_reduce_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess ||
        cudaFuncSetAttribute(gram_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess ||
        cudaFuncSetAttribute(norm_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return DORA_ERR_CUDA;
    if (gram_cluster_attrs(gram_cluster_kernel<1>) || gram_cluster_attrs(gram_cluster_kernel<2>) ||
        gram_cluster_attrs(gram_cluster_kernel<4>) || gram_cluster_attrs(gram_cluster_kernel<8>))
      return DORA_ERR_CUDA;
    if (cudaFuncSetAttribute(norm_batched_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, d.smem_optin) !=
            cudaSuccess ||
        cudaFuncSetAttribute(gram_batched_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, d.smem_optin) !=
            cudaSuccess)
      return DORA_ERR_CUDA;
    if (pair_attrs(linear_pair_kernel<false, false>, d.smem_optin) ||
        pair_attrs(linear_pair_kernel<false, true>, d.smem_optin) ||
        pair_attrs(linear_pair_kernel<true, true>, d.smem_optin))
      return DORA_ERR_CUDA;
    {
      cudaLaunchConfig_t occ{};
      cudaLaunchAttribute cl[1];
      cl[0].id = cudaLaunchAttributeClusterDimension;
      cl[0].val.clusterDim.x = 2;
      cl[0].val.clusterDim.y = 1;
      cl[0].val.clusterDim.z = 1;
      occ.gridDim = dim3(2 * (d.num_sms / 2));
      occ.blockDim = dim3(kLinThreads);
      occ.dynamicSmemBytes = linear_pair_smem(d.smem_optin);
      occ.attrs = cl;
      occ.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&d.pair_clusters, linear_pair_kernel<false, false>, &occ) != cudaSuccess ||
          d.pair_clusters < 1)
        return DORA_ERR_CUDA;
    }
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return DORA_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    d.ready = true;
  }
  *out = &d;
  return DORA_OK;
}

// 2-D bf16 tensor map over a row-major [rows, cols] matrix, 64 x 128 boxes,
// 128-byte swizzle, zero fill outside the matrix.
int make_map(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows = kBoxRows) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DORA_OK : DORA_ERR_CUDA;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// One compose backward launch; the bias picks the instantiation.
// Tag of one compose-backward launch for its arrival counters (56 bits, new
// for every call in this process; the start mixes in the clock so that a
// buffer left by another process is unlikely to carry a live tag).
unsigned long long next_bwd_epoch() {
  static std::atomic<unsigned long long> counter{
      static_cast<unsigned long long>(std::chrono::steady_clock::now().time_since_epoch().count()) * 0x9E3779B97F4A7C15ull};
  return counter.fetch_add(1) & ((1ull << 56) - 1);
}

template <typename T, int VEC>
void launch_compose_bwd(dim3 grid, cudaStream_t st, const void* dy, const void* base_out, const void* lora_out,
                        const void* bias, const float* m, const float* n, float s, long long tokens, long long nvec,
                        long long d_out, void* d_base, void* d_lora, float* part, unsigned long long* cnt, float* d_m,
                        long long rows) {
  auto kernel = bias ? compose_bwd_kernel<T, VEC, true> : compose_bwd_kernel<T, VEC, false>;
  note_launch();
  kernel<<<grid, kBwdThreads, 0, st>>>(static_cast<const T*>(dy), static_cast<const T*>(base_out),
                                       static_cast<const T*>(lora_out), static_cast<const T*>(bias), m, n, s, tokens,
                                       nvec, d_out, static_cast<T*>(d_base), static_cast<T*>(d_lora), part, cnt, d_m,
                                       rows, next_bwd_epoch());
}

// ------------------------------------------------------------ norm planning
struct TcPlan {
  int m_tiles, n_chunks, chunk_n, kb_main, kb_ext, kb_total;
  long long units;
  size_t off_gs, off_part, off_cnt, total;
};

TcPlan plan_tc(int64_t d_out, int64_t d_in, int64_t r) {
  TcPlan p{};
  p.m_tiles = static_cast<int>(cdiv(d_out, kBM));
  p.n_chunks = static_cast<int>(cdiv(r, kMaxChunkN));
  p.chunk_n = static_cast<int>(align_up(static_cast<size_t>(cdiv(r, p.n_chunks)), 16));
  p.kb_main = static_cast<int>(cdiv(d_in, kBK));
  p.kb_ext = static_cast<int>(cdiv(r, kBK));
  p.kb_total = p.kb_main + p.kb_ext;
  p.units = static_cast<long long>(p.m_tiles) * p.n_chunks * p.kb_total;
  size_t off = 0;
  p.off_gs = off;
  off = align_up(off + static_cast<size_t>(r) * r * 2, 1024);
  // (the Gram clusters keep their K-split partials in shared memory)
  p.off_part = off;
  off = align_up(off + static_cast<size_t>(kMaxGrid + p.m_tiles * p.n_chunks) * kBM * 4, 256);
  p.off_cnt = off;
  off = align_up(off + static_cast<size_t>(p.m_tiles) * 4, 256);
  p.total = off;
  return p;
}

size_t f32_norm_ws(int64_t r) { return align_up(static_cast<size_t>(r) * r * 4, 256) + 256; }

int launch_error() { return cudaGetLastError() == cudaSuccess ? DORA_OK : DORA_ERR_CUDA; }

// Resident CTAs per SM of a kernel at the given block size (at least 1).
template <typename K>
int ctas_per_sm(K kernel, int threads) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return 1;
  }
  return n;
}

// Row chunks of the compose backward for `strips` column strips (at most
// k_max, at least one): as many as one wave of `slots` resident CTAs holds
// while that leaves each CTA at most kBwdWaveRows rows, else about two waves.
// Measured at d_out = 8192: one wave of longer CTAs beats two waves of
// shorter ones up to 8192 tokens (110.6 against 112.6 us; 57.3 against
// 59.4 us at 4096), since each CTA pays a ramp-up of its loads and a
// partial-sum write at its end; two waves win from 16384 tokens on (215.0
// against 218.9 us; 848.8 against 869.4 us at 65536).
constexpr long long kBwdWaveRows = 2048;
long long bwd_chunks(long long strips, long long slots, long long tokens, long long k_max) {
  long long k = std::max<long long>(1, slots / strips);
  if (cdiv(tokens, k) > kBwdWaveRows) k = std::max<long long>(1, 2 * slots / strips);
  return std::max<long long>(1, std::min<long long>(k, k_max));
}

int norm_bf16(const void* W, const void* A, const void* B, int64_t d_out, int64_t d_in, int64_t r, float s,
              float* n_out, void* ws, cudaStream_t st, DeviceInfo* dev, bool squared) {
  const TcPlan p = plan_tc(d_out, d_in, r);
  if (p.units > (1ll << 30)) return DORA_ERR_UNSUPPORTED;  // unit indices are 32-bit in the kernel
  uint8_t* w = static_cast<uint8_t*>(ws);
  __nv_bfloat16* Gs = reinterpret_cast<__nv_bfloat16*>(w + p.off_gs);
  float* part = reinterpret_cast<float*>(w + p.off_part);
  int* cnt = reinterpret_cast<int*>(w + p.off_cnt);

  CUtensorMap tmW, tmA, tmB, tmG;
  if (make_map(&tmW, W, d_out, d_in) || make_map(&tmA, A, r, d_in) || make_map(&tmB, B, d_out, r) ||
      make_map(&tmG, Gs, r, r))
    return DORA_ERR_CUDA;

  // 1) G' = (s/2) A A^T: one cluster of `splits` CTAs per tile on or above
  // the diagonal, each CTA a K split, summed inside the cluster; the launch
  // also zeroes the GEMM's tile counters.  2) The persistent GEMM behind it
  // with programmatic dependent launch: its CTAs start on the SMs the Gram
  // clusters leave free, meet G' only at the ends of their ranges and wait
  // for the Gram launch only there.
  const int nt = static_cast<int>(cdiv(r, kBoxRows));
  const int up_tiles = nt * (nt + 1) / 2;
  // as many K splits as a cluster holds (8), while each keeps at least
  // kGramMinBlocks K blocks and the clusters take at most a third of the
  // SMs: the Gram latency then stays well inside the GEMM's, small
  // problems included
  int splits = 1;
  while (splits < 8 && 2 * splits * kGramMinBlocks <= p.kb_main && up_tiles * 2 * splits <= std::max(1, dev->num_sms / 3))
    splits *= 2;
  {
    GramClusterArgs gca{};
    gca.r = static_cast<int>(r);
    gca.kb_main = p.kb_main;
    gca.nt = nt;
    gca.half_s = 0.5f * s;
    gca.Gs = Gs;
    gca.wait_limit = kWaitLimitCycles;
    gca.status = dev->status;
    gca.zero_cnt = cnt;
    gca.n_zero = p.m_tiles;
    cudaLaunchAttribute gat[1];
    gat[0].id = cudaLaunchAttributeClusterDimension;
    gat[0].val.clusterDim.x = static_cast<unsigned>(splits);
    gat[0].val.clusterDim.y = 1;
    gat[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t gcfg{};
    gcfg.stream = st;
    gcfg.attrs = gat;
    gcfg.numAttrs = 1;
    gcfg.gridDim = dim3(static_cast<unsigned>(up_tiles * splits));
    gcfg.blockDim = dim3(kGcThreads);
    gcfg.dynamicSmemBytes = kGcSmem;
    cudaError_t e = cudaSuccess;
    note_launch();
    switch (splits) {
      case 1: e = cudaLaunchKernelEx(&gcfg, gram_cluster_kernel<1>, tmA, gca); break;
      case 2: e = cudaLaunchKernelEx(&gcfg, gram_cluster_kernel<2>, tmA, gca); break;
      case 4: e = cudaLaunchKernelEx(&gcfg, gram_cluster_kernel<4>, tmA, gca); break;
      default: e = cudaLaunchKernelEx(&gcfg, gram_cluster_kernel<8>, tmA, gca); break;
    }
    if (e != cudaSuccess) return DORA_ERR_CUDA;
  }

  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;

  NormArgs na{};
  na.d_out = static_cast<int>(d_out);
  na.d_in = static_cast<int>(d_in);
  na.r = static_cast<int>(r);
  na.m_tiles = p.m_tiles;
  na.n_chunks = p.n_chunks;
  na.chunk_n = p.chunk_n;
  na.kb_main = p.kb_main;
  na.kb_total = p.kb_total;
  na.units = p.units;
  const int grid = static_cast<int>(std::min<long long>({static_cast<long long>(dev->num_sms), p.units, kMaxGrid}));
  const size_t smem_fixed = kNormTcSmemFixed + static_cast<size_t>(grid + 1) * 4;  // + the range-start table
  na.stage_bytes = static_cast<uint32_t>(kBoxBytes * (1 + cdiv(p.chunk_n, kBoxRows)));
  na.stages = static_cast<int>(std::min<size_t>(kMaxStages, (dev->smem_optin - smem_fixed) / (na.stage_bytes + 16)));
  if (na.stages < 2) return DORA_ERR_UNSUPPORTED;
  // a power of two of at least 64 columns: the epilogue reads V 64 columns at a time
  uint32_t cols = 64;
  while (cols < static_cast<uint32_t>(p.chunk_n)) cols <<= 1;
  na.tmem_cols = cols;
  na.two_s = 2.0f * s;
  na.wait_limit = kWaitLimitCycles;
  na.partials = part;
  na.counters = cnt;
  na.n_out = n_out;
  na.status = dev->status;
  na.squared = squared ? 1 : 0;
  {
    // The Gram CTAs hold one SM each (their shared memory): that many CTAs of
    // the GEMM start late and get that much less, so that all end together.
    // Start delay and GEMM unit time from traces of these kernels on B200
    // (8192 x 8192, r = 64 and 384): a Gram CTA takes about 3 us plus
    // 0.43 us per K block of its split, plus about 5 us to sum and mirror
    // off-diagonal tiles; a GEMM unit about 0.18 us plus 0.01 us per KB of its
    // ring stage.  A late CTA that ends early costs the grid a little; one
    // that ends late costs the whole gap, so the delay is taken 10% long,
    // 25% for Gram phases past 20 us, which the linear model underestimates
    // (r = 768 at 8192 x 8192: 111.7 against 115.7 us with 10%).
    const int gram_sms = std::min(dev->num_sms, up_tiles * splits);
    const int late = grid > gram_sms ? gram_sms : 0;
    const double gram_us = 3.0 + 0.43 * static_cast<double>(cdiv(p.kb_main, splits)) + (nt > 1 ? 5.0 : 1.0);
    const double unit_us = 0.18 + 0.01 * (static_cast<double>(na.stage_bytes) / 1024.0);
    const double delay = (gram_us > 20.0 ? 1.25 : 1.1) * gram_us / unit_us;
    const double f = (static_cast<double>(p.units) + late * delay) / grid;
    na.early = grid - late;
    na.w_early = std::max<long long>(1, std::llround(16.0 * f));
    na.w_late = late > 0 ? std::max<long long>(0, std::llround(16.0 * (f - delay))) : na.w_early;
  }
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kNormTcThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(na.stages) * (na.stage_bytes + 16) + smem_fixed;
  note_launch();
  if (cudaLaunchKernelEx(&cfg, norm_tc_kernel, tmW, tmA, tmB, tmG, na) != cudaSuccess) return DORA_ERR_CUDA;
  return launch_error();
}

// Argument checks of one factored norm, workspace aside.
int norm_arg_status(const void* W, const void* A, const void* B, int64_t d_out, int64_t d_in, int64_t r, dora_dtype dt,
                    const float* n_out) {
  if (dt != DORA_BF16 && dt != DORA_F32) return DORA_ERR_UNSUPPORTED;
  if (d_out < 0 || d_in < 0 || r < 0) return DORA_ERR_INVALID_ARG;
  if (d_out > INT32_MAX / 2 || d_in > INT32_MAX / 2 || r > kMaxRank) return DORA_ERR_UNSUPPORTED;
  if (d_out == 0) return DORA_OK;
  if (!n_out || (d_in > 0 && !W) || (r > 0 && d_in > 0 && (!A || !B))) return DORA_ERR_INVALID_ARG;
  if (!aligned(n_out, 4)) return DORA_ERR_UNSUPPORTED;
  if (dt == DORA_BF16) {
    if (d_in > 0 && (d_in % 8 != 0 || r % 16 != 0)) return DORA_ERR_UNSUPPORTED;
    if (!aligned(W, 16) || !aligned(A, 16) || !aligned(B, 16)) return DORA_ERR_UNSUPPORTED;
  } else {
    if (!aligned(W, 4) || !aligned(A, 4) || !aligned(B, 4)) return DORA_ERR_UNSUPPORTED;
  }
  return DORA_OK;
}

// ------------------------------------------------------- batched norms
// Modules that share the two batched launches: bf16, 16 <= r <= 512 (one
// TMEM chunk), something to compute.
bool batchable(const dora_norm_problem& q, dora_dtype dt) {
  return dt == DORA_BF16 && q.d_out > 0 && q.d_in > 0 && q.r >= 16 && q.r <= 512 && q.r % 16 == 0;
}

struct BatchLayout {
  std::vector<int> batched, single;  // problem indices on each path
  std::vector<size_t> off_gs;        // per batched problem: its G' in the workspace
  size_t off_items = 0, off_gitems = 0, off_single = 0, single_bytes = 0, total = 0;
  int n_items = 0, n_gitems = 0;
  uint32_t stage_bytes = 0;
};

int batch_layout(const dora_norm_problem* q, int count, dora_dtype dt, BatchLayout* L) {
  if (dt != DORA_BF16 && dt != DORA_F32) return DORA_ERR_UNSUPPORTED;
  if (count < 0 || (count > 0 && !q)) return DORA_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    if (q[i].d_out < 0 || q[i].d_in < 0 || q[i].r < 0) return DORA_ERR_INVALID_ARG;
    if (batchable(q[i], dt)) {
      L->batched.push_back(i);
      L->n_items += static_cast<int>(cdiv(q[i].d_out, kBM));
      const int nt = static_cast<int>(cdiv(q[i].r, kBoxRows));
      L->n_gitems += nt * nt;
      L->stage_bytes = std::max<uint32_t>(L->stage_bytes, kBoxBytes * (1 + nt));
    } else {
      L->single.push_back(i);
      L->single_bytes = std::max(L->single_bytes, dora_factored_norm_workspace_size(q[i].d_out, q[i].d_in, q[i].r, dt));
    }
  }
  size_t off = align_up(L->batched.size() * sizeof(BatchDesc), 256);
  L->off_items = off;
  off = align_up(off + static_cast<size_t>(L->n_items) * sizeof(BatchItem), 256);
  L->off_gitems = off;
  off = align_up(off + static_cast<size_t>(L->n_gitems) * sizeof(BatchItem), 256);
  for (int i : L->batched) {
    L->off_gs.push_back(off);
    off = align_up(off + static_cast<size_t>(q[i].r) * q[i].r * 2, 256);
  }
  L->off_single = off;
  L->total = off + L->single_bytes;
  return DORA_OK;
}

int norm_batched(const dora_norm_problem* q, const BatchLayout& L, uint8_t* ws, cudaStream_t st, DeviceInfo* dev) {
  const size_t nb = L.batched.size();
  // the descriptor table and both work lists, built here and copied in one go
  std::vector<uint8_t> host(L.off_gs.empty() ? L.off_gitems : L.off_gs[0]);
  BatchDesc* descs = reinterpret_cast<BatchDesc*>(host.data());
  BatchItem* items = reinterpret_cast<BatchItem*>(host.data() + L.off_items);
  BatchItem* gitems = reinterpret_cast<BatchItem*>(host.data() + L.off_gitems);
  int ni = 0, ng = 0;
  for (size_t j = 0; j < nb; ++j) {
    const dora_norm_problem& p = q[L.batched[j]];
    BatchDesc& d = descs[j];
    std::memset(&d, 0, sizeof(d));
    __nv_bfloat16* gs = reinterpret_cast<__nv_bfloat16*>(ws + L.off_gs[j]);
    if (make_map(&d.tmW, p.W, p.d_out, p.d_in) || make_map(&d.tmA, p.A, p.r, p.d_in) ||
        make_map(&d.tmB, p.B, p.d_out, p.r) || make_map(&d.tmG, gs, p.r, p.r))
      return DORA_ERR_CUDA;
    d.n_out = p.n_out;
    d.gs = gs;
    d.d_out = static_cast<int>(p.d_out);
    d.d_in = static_cast<int>(p.d_in);
    d.r = static_cast<int>(p.r);
    d.kb_main = static_cast<int>(cdiv(p.d_in, kBK));
    d.kb_total = d.kb_main + static_cast<int>(cdiv(p.r, kBK));
    d.two_s = 2.0f * p.s;
    d.half_s = 0.5f * p.s;
    for (int t = 0; t < cdiv(p.d_out, kBM); ++t) items[ni++] = BatchItem{static_cast<int>(j), t};
    const int nt = static_cast<int>(cdiv(p.r, kBoxRows));
    for (int t = 0; t < nt * nt; ++t) gitems[ng++] = BatchItem{static_cast<int>(j), t};
  }
  // longest items first, dealt round-robin over the persistent grid
  auto cost = [&](const BatchItem& it) {
    const BatchDesc& d = descs[it.prob];
    return static_cast<long long>(d.kb_total) * (1 + cdiv(d.r, kBoxRows));
  };
  std::stable_sort(items, items + ni, [&](const BatchItem& x, const BatchItem& y) { return cost(x) > cost(y); });
  if (cudaMemcpyAsync(ws, host.data(), host.size(), cudaMemcpyHostToDevice, st) != cudaSuccess) return DORA_ERR_CUDA;

  const BatchDesc* d_descs = reinterpret_cast<const BatchDesc*>(ws);
  const size_t gram_smem = kGramStages * kGramStageBytes + (2 * kGramStages + 1) * 8 + 16 + 1024;
  note_launch();
  gram_batched_kernel<<<ng, kNormThreads, gram_smem, st>>>(d_descs, reinterpret_cast<const BatchItem*>(ws + L.off_gitems),
                                                          kWaitLimitCycles, dev->status);
  if (launch_error()) return DORA_ERR_CUDA;

  BatchNormArgs a{};
  a.n_items = ni;
  a.stage_bytes = L.stage_bytes;
  const size_t fixed = 1024 + 64 + 16;
  a.stages = static_cast<int>(std::min<size_t>(kMaxStages, (dev->smem_optin - fixed) / (a.stage_bytes + 16)));
  if (a.stages < 2) return DORA_ERR_UNSUPPORTED;
  a.wait_limit = kWaitLimitCycles;
  a.status = dev->status;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(std::min<long long>({static_cast<long long>(dev->num_sms), ni, kMaxGrid})));
  cfg.blockDim = dim3(kNormThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(a.stages) * a.stage_bytes + (2 * a.stages + 3) * 8 + 16 + 1024;
  note_launch();
  if (cudaLaunchKernelEx(&cfg, norm_batched_kernel, d_descs, reinterpret_cast<const BatchItem*>(ws + L.off_items), a) !=
      cudaSuccess)
    return DORA_ERR_CUDA;
  return launch_error();
}

}  // namespace
}  // namespace dora

using namespace dora;

namespace dora {
namespace {
// The factored norm, n = sqrt(max(n^2, 0)) or, with `squared`, n^2 as summed.
int factored_norm(const void* W, const void* A, const void* B, int64_t d_out, int64_t d_in, int64_t r, float s,
                  dora_dtype dt, float* n_out, void* workspace, size_t workspace_bytes, void* stream, bool squared);
}  // namespace
}  // namespace dora

extern "C" {

const char* dora_status_string(int status) {
  switch (status) {
    case DORA_OK: return "DORA_OK";
    case DORA_ERR_INVALID_ARG: return "DORA_ERR_INVALID_ARG: invalid argument";
    case DORA_ERR_UNSUPPORTED: return "DORA_ERR_UNSUPPORTED: shape, alignment or dtype not supported";
    case DORA_ERR_WORKSPACE: return "DORA_ERR_WORKSPACE: workspace missing or too small";
    case DORA_ERR_CUDA: return "DORA_ERR_CUDA: a CUDA runtime call failed";
    case DORA_ERR_TIMEOUT: return "DORA_ERR_TIMEOUT: a bounded device-side wait gave up";
    default: return "unknown dora status";
  }
}

size_t dora_factored_norm_workspace_size(int64_t d_out, int64_t d_in, int64_t r, dora_dtype dt) {
  if (d_out < 0 || d_in < 0 || r < 0) return 0;
  if (dt == DORA_F32) return f32_norm_ws(r);
  if (dt != DORA_BF16) return 0;
  if (d_out == 0 || d_in == 0 || r == 0) return 256;
  return plan_tc(d_out, d_in, r).total;
}

int dora_factored_norm(const void* W, const void* A, const void* B, int64_t d_out, int64_t d_in, int64_t r, float s,
                       dora_dtype dt, float* n_out, void* workspace, size_t workspace_bytes, void* stream) {
  return factored_norm(W, A, B, d_out, d_in, r, s, dt, n_out, workspace, workspace_bytes, stream, false);
}

int dora_factored_norm_sq(const void* W, const void* A, const void* B, int64_t d_out, int64_t d_in, int64_t r,
                          float s, dora_dtype dt, float* n2_out, void* workspace, size_t workspace_bytes,
                          void* stream) {
  return factored_norm(W, A, B, d_out, d_in, r, s, dt, n2_out, workspace, workspace_bytes, stream, true);
}

int dora_norm_finish(float* n, int64_t d_out, void* stream) {
  if (d_out < 0) return DORA_ERR_INVALID_ARG;
  if (d_out == 0) return DORA_OK;
  if (!n) return DORA_ERR_INVALID_ARG;
  if (!aligned(n, 4)) return DORA_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  if (device_info(&dev)) return DORA_ERR_CUDA;
  note_launch();
  norm_finish_kernel<<<static_cast<unsigned>(cdiv(d_out, 256)), 256, 0, static_cast<cudaStream_t>(stream)>>>(n, d_out);
  return launch_error();
}

}  // extern "C"

namespace dora {
namespace {
int factored_norm(const void* W, const void* A, const void* B, int64_t d_out, int64_t d_in, int64_t r, float s,
                  dora_dtype dt, float* n_out, void* workspace, size_t workspace_bytes, void* stream, bool squared) {
  const int arg = norm_arg_status(W, A, B, d_out, d_in, r, dt, n_out);
  if (arg != DORA_OK || d_out == 0) return arg;
  const size_t need = dora_factored_norm_workspace_size(d_out, d_in, r, dt);
  const bool trivial = (d_in == 0);
  if (!trivial && (!workspace || workspace_bytes < need)) return DORA_ERR_WORKSPACE;
  if (!trivial && !aligned(workspace, 256)) return DORA_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  if (device_info(&dev)) return DORA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (trivial) {
    return cudaMemsetAsync(n_out, 0, static_cast<size_t>(d_out) * 4, st) == cudaSuccess ? DORA_OK : DORA_ERR_CUDA;
  }
  if (r == 0) {
    const int blocks = static_cast<int>(cdiv(d_out, 8));
    note_launch();
    if (dt == DORA_BF16)
      rownorm_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(W), static_cast<int>(d_out),
                                                            static_cast<int>(d_in), n_out, squared ? 1 : 0);
    else
      rownorm_kernel<float><<<blocks, 256, 0, st>>>(static_cast<const float*>(W), static_cast<int>(d_out),
                                                    static_cast<int>(d_in), n_out, squared ? 1 : 0);
    return launch_error();
  }
  if (dt == DORA_BF16) return norm_bf16(W, A, B, d_out, d_in, r, s, n_out, workspace, st, dev, squared);
  float* G = static_cast<float*>(workspace);
  const long long pairs = r * (r + 1) / 2;
  const int gblocks = static_cast<int>(std::min<long long>(cdiv(pairs, 8), 8LL * dev->num_sms));
  note_launch();
  gram_f32_kernel<<<gblocks, 256, 0, st>>>(static_cast<const float*>(A), static_cast<int>(r), static_cast<int>(d_in), G);
  if (launch_error()) return DORA_ERR_CUDA;
  note_launch();
  norm_f32_kernel<<<static_cast<unsigned>(d_out), 256, 0, st>>>(
      static_cast<const float*>(W), static_cast<const float*>(A), static_cast<const float*>(B), G,
      static_cast<int>(d_out), static_cast<int>(d_in), static_cast<int>(r), s, n_out, squared ? 1 : 0);
  return launch_error();
}
}  // namespace
}  // namespace dora

extern "C" {

int dora_compose_fwd(const void* base_out, const void* lora_out, const float* m, const float* n, float s,
                     int64_t tokens, int64_t d_out, dora_dtype dt, void* y, void* stream) {
  return dora_compose_fwd_bias(base_out, lora_out, nullptr, m, n, s, tokens, d_out, dt, y, stream);
}

int dora_compose_fwd_bias(const void* base_out, const void* lora_out, const void* bias, const float* m,
                          const float* n, float s, int64_t tokens, int64_t d_out, dora_dtype dt, void* y,
                          void* stream) {
  if (dt != DORA_BF16 && dt != DORA_F32) return DORA_ERR_UNSUPPORTED;
  if (tokens < 0 || d_out < 0) return DORA_ERR_INVALID_ARG;
  if (tokens == 0 || d_out == 0) return DORA_OK;
  if (!base_out || !lora_out || !m || !n || !y) return DORA_ERR_INVALID_ARG;
  const int vec_bf16 = 8;
  int vec = 1;
  if (dt == DORA_BF16) {
    if (d_out % vec_bf16 != 0) return DORA_ERR_UNSUPPORTED;
    if (!aligned(base_out, 16) || !aligned(lora_out, 16) || !aligned(y, 16)) return DORA_ERR_UNSUPPORTED;
    vec = vec_bf16;
  } else {
    if (!aligned(base_out, 4) || !aligned(lora_out, 4) || !aligned(y, 4)) return DORA_ERR_UNSUPPORTED;
    vec = (d_out % 4 == 0 && aligned(base_out, 16) && aligned(lora_out, 16) && aligned(y, 16)) ? 4 : 1;
  }
  if (!aligned(m, 4) || !aligned(n, 4) || !aligned(bias, dt == DORA_BF16 ? 16 : 4)) return DORA_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  if (device_info(&dev)) return DORA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long nvec = d_out / vec;
  const int threads = static_cast<int>(std::min<long long>(256, align_up(static_cast<size_t>(nvec), 32)));
  const long long gx = cdiv(nvec, threads);
  if (gx > INT32_MAX) return DORA_ERR_UNSUPPORTED;
  // Several short waves of small CTAs stream better than one wave of long
  // ones here: about 8 CTAs per SM in total, whatever the residency.
  const long long gy = std::max<long long>(1, std::min<long long>({8LL * dev->num_sms / gx, tokens, 65535}));
  const long long rows = cdiv(tokens, gy);
  const long long gy2 = cdiv(tokens, rows);
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy2));
  note_launch();
  if (dt == DORA_BF16)
    compose_fwd_kernel<__nv_bfloat16, 8><<<grid, threads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(base_out), static_cast<const __nv_bfloat16*>(lora_out),
        static_cast<const __nv_bfloat16*>(bias), m, n, s, tokens, nvec, d_out, static_cast<__nv_bfloat16*>(y), rows);
  else if (vec == 4)
    compose_fwd_kernel<float, 4><<<grid, threads, 0, st>>>(static_cast<const float*>(base_out),
                                                           static_cast<const float*>(lora_out),
                                                           static_cast<const float*>(bias), m, n, s, tokens, nvec,
                                                           d_out, static_cast<float*>(y), rows);
  else
    compose_fwd_kernel<float, 1><<<grid, threads, 0, st>>>(static_cast<const float*>(base_out),
                                                           static_cast<const float*>(lora_out),
                                                           static_cast<const float*>(bias), m, n, s, tokens, nvec,
                                                           d_out, static_cast<float*>(y), rows);
  return launch_error();
}

size_t dora_compose_bwd_workspace_size(int64_t tokens, int64_t d_out) {
  if (tokens < 0 || d_out < 0) return 0;
  const size_t strips = static_cast<size_t>(cdiv(std::max<int64_t>(d_out, 1), dora::kBwdVecs));
  return align_up(strips * 8, 256) + align_up(static_cast<size_t>(kMaxBwdChunks) * std::max<int64_t>(d_out, 1) * 4, 256);
}

int dora_compose_bwd(const void* dy, const void* base_out, const void* lora_out, const float* m, const float* n,
                     float s, int64_t tokens, int64_t d_out, dora_dtype dt, void* d_base, void* d_lora, float* d_m,
                     void* workspace, size_t workspace_bytes, void* stream) {
  return dora_compose_bwd_bias(dy, base_out, lora_out, nullptr, m, n, s, tokens, d_out, dt, d_base, d_lora, d_m,
                               workspace, workspace_bytes, stream);
}

int dora_compose_bwd_bias(const void* dy, const void* base_out, const void* lora_out, const void* bias,
                          const float* m, const float* n, float s, int64_t tokens, int64_t d_out, dora_dtype dt,
                          void* d_base, void* d_lora, float* d_m, void* workspace, size_t workspace_bytes,
                          void* stream) {
  if (dt != DORA_BF16 && dt != DORA_F32) return DORA_ERR_UNSUPPORTED;
  if (tokens < 0 || d_out < 0) return DORA_ERR_INVALID_ARG;
  if (d_out == 0) return DORA_OK;
  if (!m || !n || !d_m) return DORA_ERR_INVALID_ARG;
  if (tokens > 0 && (!dy || !base_out || !lora_out || !d_base || !d_lora)) return DORA_ERR_INVALID_ARG;
  int vec = 1;
  if (dt == DORA_BF16) {
    if (d_out % 8 != 0) return DORA_ERR_UNSUPPORTED;
    if (tokens > 0 && (!aligned(dy, 16) || !aligned(base_out, 16) || !aligned(lora_out, 16) ||
                       !aligned(d_base, 16) || !aligned(d_lora, 16)))
      return DORA_ERR_UNSUPPORTED;
    vec = 8;
  } else {
    const bool a16 = aligned(dy, 16) && aligned(base_out, 16) && aligned(lora_out, 16) && aligned(d_base, 16) &&
                     aligned(d_lora, 16) && aligned(bias, 16);
    if (!aligned(dy, 4) || !aligned(base_out, 4) || !aligned(lora_out, 4) || !aligned(d_base, 4) ||
        !aligned(d_lora, 4))
      return DORA_ERR_UNSUPPORTED;
    vec = (d_out % 4 == 0 && a16) ? 4 : 1;
  }
  if (!aligned(m, 4) || !aligned(n, 4) || !aligned(d_m, 4) || !aligned(bias, dt == DORA_BF16 ? 16 : 4))
    return DORA_ERR_UNSUPPORTED;
  const size_t need = dora_compose_bwd_workspace_size(tokens, d_out);
  if (!workspace || workspace_bytes < need) return DORA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return DORA_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  if (device_info(&dev)) return DORA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tokens == 0) return cudaMemsetAsync(d_m, 0, static_cast<size_t>(d_out) * 4, st) == cudaSuccess ? DORA_OK : DORA_ERR_CUDA;

  const long long nvec = d_out / vec;
  const long long strips = cdiv(nvec, kBwdVecs);
  if (strips > INT32_MAX) return DORA_ERR_UNSUPPORTED;
  int occ = 1;
  if (dt == DORA_BF16)
    occ = ctas_per_sm(compose_bwd_kernel<__nv_bfloat16, 8, false>, kBwdThreads);
  else if (vec == 4)
    occ = ctas_per_sm(compose_bwd_kernel<float, 4, false>, kBwdThreads);
  else
    occ = ctas_per_sm(compose_bwd_kernel<float, 1, false>, kBwdThreads);
  const long long chunks = bwd_chunks(strips, static_cast<long long>(dev->num_sms) * occ, tokens,
                                      std::min<long long>(kMaxBwdChunks, cdiv(tokens, kBwdSlots)));
  const long long rows = cdiv(tokens, chunks);
  const long long chunks2 = cdiv(tokens, rows);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  unsigned long long* cnt = reinterpret_cast<unsigned long long*>(w);  // tagged: no clearing needed
  const size_t strips_all = static_cast<size_t>(cdiv(d_out, kBwdVecs));
  float* part = reinterpret_cast<float*>(w + align_up(strips_all * 8, 256));
  dim3 grid(static_cast<unsigned>(strips), static_cast<unsigned>(chunks2));
  if (dt == DORA_BF16)
    launch_compose_bwd<__nv_bfloat16, 8>(grid, st, dy, base_out, lora_out, bias, m, n, s, tokens, nvec, d_out, d_base,
                                         d_lora, part, cnt, d_m, rows);
  else if (vec == 4)
    launch_compose_bwd<float, 4>(grid, st, dy, base_out, lora_out, bias, m, n, s, tokens, nvec, d_out, d_base, d_lora,
                                part, cnt, d_m, rows);
  else
    launch_compose_bwd<float, 1>(grid, st, dy, base_out, lora_out, bias, m, n, s, tokens, nvec, d_out, d_base, d_lora,
                                part, cnt, d_m, rows);
  return launch_error();
}

size_t dora_factored_norm_batched_workspace_size(const dora_norm_problem* problems, int count, dora_dtype dt) {
  BatchLayout L;
  if (batch_layout(problems, count, dt, &L) != DORA_OK) return 0;
  return std::max<size_t>(L.total, 256);
}

int dora_factored_norm_batched(const dora_norm_problem* problems, int count, dora_dtype dt, void* workspace,
                               size_t workspace_bytes, void* stream) {
  BatchLayout L;
  const int lay = batch_layout(problems, count, dt, &L);
  if (lay != DORA_OK) return lay;
  // every module's arguments are checked before anything is launched
  for (int i = 0; i < count; ++i) {
    const dora_norm_problem& q = problems[i];
    const int arg = norm_arg_status(q.W, q.A, q.B, q.d_out, q.d_in, q.r, dt, q.n_out);
    if (arg != DORA_OK) return arg;
  }
  if (count == 0) return DORA_OK;
  if (!workspace || workspace_bytes < L.total) return DORA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return DORA_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  if (device_info(&dev)) return DORA_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (!L.batched.empty()) {
    const int rc = norm_batched(problems, L, ws, static_cast<cudaStream_t>(stream), dev);
    if (rc != DORA_OK) return rc;
  }
  for (int i : L.single) {
    const dora_norm_problem& q = problems[i];
    const int rc = dora_factored_norm(q.W, q.A, q.B, q.d_out, q.d_in, q.r, q.s, dt, q.n_out, ws + L.off_single,
                                      L.single_bytes, stream);
    if (rc != DORA_OK) return rc;
  }
  return DORA_OK;
}

int dora_device_status(void* stream) {
  DeviceInfo* dev = nullptr;
  if (device_info(&dev)) return DORA_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DORA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return DORA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
  }
  return v;
}

int dora_selftest_timeout(int64_t limit_cycles, void* stream) {
  if (limit_cycles <= 0 || limit_cycles > kWaitLimitCycles) return DORA_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  if (device_info(&dev)) return DORA_ERR_CUDA;
  note_launch();
  timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles, dev->status);
  return launch_error();
}

uint64_t dora_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int dora_num_sms(void) {
  int n = 0;
  if (cudaGetDeviceCount(&n) != cudaSuccess || n == 0) {
    cudaGetLastError();
    return 0;
  }
  DeviceInfo* dev = nullptr;
  if (device_info(&dev)) return 0;
  return dev->num_sms;
}


size_t dora_fused_linear_fwd_workspace_size(int64_t tokens, int64_t r) {
  if (tokens < 0 || r < 0) return 0;
  return std::max<size_t>(256, align_up(static_cast<size_t>(tokens) * static_cast<size_t>(r) * 2, 256));
}

int dora_fused_linear_fwd(const void* x, const void* W, const void* A, const void* B, const void* bias, const float* m,
                          const float* n, float s, int64_t tokens, int64_t d_in, int64_t d_out, int64_t r,
                          dora_dtype dt, void* y, void* workspace, size_t workspace_bytes, void* stream) {
  if (dt != DORA_BF16) return DORA_ERR_UNSUPPORTED;
  if (tokens < 0 || d_in < 0 || d_out < 0 || r < 0) return DORA_ERR_INVALID_ARG;
  if (tokens == 0 || d_out == 0) return DORA_OK;
  if (d_in == 0) return DORA_ERR_UNSUPPORTED;
  if (tokens > INT32_MAX / 2 || d_in > INT32_MAX / 2 || d_out > INT32_MAX / 2 || r > INT32_MAX / 2)
    return DORA_ERR_UNSUPPORTED;
  if (!x || !W || !m || !n || !y || (r > 0 && (!A || !B))) return DORA_ERR_INVALID_ARG;
  if (d_in % 8 != 0 || d_out % 8 != 0 || r % 8 != 0) return DORA_ERR_UNSUPPORTED;
  if (!aligned(x, 16) || !aligned(W, 16) || !aligned(A, 16) || !aligned(B, 16) || !aligned(y, 16) ||
      !aligned(bias, 2) || !aligned(m, 4) || !aligned(n, 4))
    return DORA_ERR_UNSUPPORTED;
  if (cdiv(tokens, kPairBM) * cdiv(d_out, 128) > INT32_MAX) return DORA_ERR_UNSUPPORTED;
  const size_t need = dora_fused_linear_fwd_workspace_size(tokens, r);
  if (r > 0 && (!workspace || workspace_bytes < need)) return DORA_ERR_WORKSPACE;
  if (r > 0 && !aligned(workspace, 256)) return DORA_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  if (device_info(&dev)) return DORA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  __nv_bfloat16* P = static_cast<__nv_bfloat16*>(workspace);

  // B-side boxes hold the bn / 2 rows one CTA of a pair owns
  const int bn_p = r > 0 ? pick_bn(r) : 256, bn_y = pick_bn(d_out);
  CUtensorMap tmX, tmW, tmA, tmP, tmB;
  if (make_map(&tmX, x, tokens, d_in) || make_map(&tmW, W, d_out, d_in, bn_y / 2)) return DORA_ERR_CUDA;
  if (r > 0 && (make_map(&tmA, A, r, d_in, bn_p / 2) || make_map(&tmP, P, tokens, r) ||
                make_map(&tmB, B, d_out, r, bn_y / 2)))
    return DORA_ERR_CUDA;
  const int kb_main = static_cast<int>(cdiv(d_in, kLinBK));
  const int stages = linear_pair_stages(dev->smem_optin);
  if (stages < 2) return DORA_ERR_UNSUPPORTED;
  const long long tiles_m2 = cdiv(tokens, kPairBM);

  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = 2;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.stream = st;
  cfg.attrs = attrs;
  cfg.blockDim = dim3(kLinThreads);
  cfg.dynamicSmemBytes = linear_pair_smem(dev->smem_optin);
  auto pairs_for = [&](long long tiles) {
    return static_cast<unsigned>(2 * std::min<long long>(dev->pair_clusters, tiles));
  };

  // 1) P = bf16(s * x A^T) into the workspace
  if (r > 0) {
    LinearArgs pa{};
    pa.M = static_cast<int>(tokens);
    pa.N = static_cast<int>(r);
    pa.kb_main = pa.kb_total = kb_main;
    pa.tiles_m = static_cast<int>(tiles_m2);
    pa.bn = bn_p;
    pa.tiles_n = static_cast<int>(cdiv(r, bn_p));
    pa.stages = stages;
      pa.alpha = s;
    pa.out = P;
    pa.ldo = r;
    pa.wait_limit = kWaitLimitCycles;
    pa.status = dev->status;
    cfg.numAttrs = 1;  // cluster shape only: ordered after everything before it on the stream
    cfg.gridDim = dim3(pairs_for(static_cast<long long>(pa.tiles_m) * pa.tiles_n));
    note_launch();
    if (cudaLaunchKernelEx(&cfg, linear_pair_kernel<false, false>, tmX, tmA, tmX, tmA, pa) != cudaSuccess)
      return DORA_ERR_CUDA;
  }

  // 2) y = bf16(g * [x | P] [W | B]^T + b), dependent on 1) only for the extension blocks
  LinearArgs la{};
  la.M = static_cast<int>(tokens);
  la.N = static_cast<int>(d_out);
  la.kb_main = kb_main;
  la.kb_total = kb_main + static_cast<int>(cdiv(r, kLinBK));
  la.tiles_m = static_cast<int>(tiles_m2);
  la.bn = bn_y;
  la.tiles_n = static_cast<int>(cdiv(d_out, bn_y));
  la.stages = stages;
  la.alpha = 1.f;
  la.m = m;
  la.n = n;
  la.bias = static_cast<const __nv_bfloat16*>(bias);
  la.out = static_cast<__nv_bfloat16*>(y);
  la.ldo = d_out;
  la.ext_waits = r > 0 ? 1 : 0;
  la.wait_limit = kWaitLimitCycles;
  la.status = dev->status;
  cfg.numAttrs = r > 0 ? 2 : 1;
  cfg.gridDim = dim3(pairs_for(static_cast<long long>(la.tiles_m) * la.tiles_n));
  const CUtensorMap& tmA2 = r > 0 ? tmP : tmX;
  const CUtensorMap& tmB2 = r > 0 ? tmB : tmW;
  note_launch();
  if (cudaLaunchKernelEx(&cfg, linear_pair_kernel<false, false>, tmX, tmW, tmA2, tmB2, la) != cudaSuccess)
    return DORA_ERR_CUDA;
  return launch_error();
}


// ---------------------------------------------------- attached-norm backward
namespace {
struct BwdLayout {
  int nt, splits_max;  // K splits of each of the two Gram products (G and H) in one launch
  size_t off_part, off_part2, off_sg, off_h, off_bt, off_bct, total;
};
BwdLayout bwd_layout(int64_t d_out, int64_t r) {
  BwdLayout L{};
  L.nt = static_cast<int>(cdiv(r, kBoxRows));
  L.splits_max = std::max(1, std::min(kMaxGramSplits, 80 / (L.nt * L.nt)));
  const size_t part_bytes = static_cast<size_t>(L.splits_max) * L.nt * L.nt * kBoxRows * kBoxRows * 4;
  size_t off = 0;
  L.off_part = off;
  off = align_up(off + part_bytes, 256);
  L.off_part2 = off;
  off = align_up(off + part_bytes, 256);
  L.off_sg = off;
  off = align_up(off + static_cast<size_t>(r) * r * 2, 256);
  L.off_h = off;
  off = align_up(off + static_cast<size_t>(r) * r * 2, 256);
  L.off_bt = off;
  off = align_up(off + static_cast<size_t>(r) * d_out * 2, 256);
  L.off_bct = off;
  off = align_up(off + static_cast<size_t>(r) * d_out * 2, 256);
  L.total = std::max<size_t>(off, 256);
  return L;
}
}  // namespace

size_t dora_factored_norm_bwd_workspace_size(int64_t d_out, int64_t d_in, int64_t r) {
  if (d_out < 0 || d_in < 0 || r < 0) return 0;
  return bwd_layout(d_out, r).total;
}

int dora_factored_norm_bwd(const void* W, const void* A, const void* B, float s, const float* n, const float* d_n,
                           int64_t d_out, int64_t d_in, int64_t r, dora_dtype dt, float* dA, float* dB,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (dt != DORA_BF16) return DORA_ERR_UNSUPPORTED;
  if (d_out < 0 || d_in < 0 || r < 0) return DORA_ERR_INVALID_ARG;
  if (d_out > INT32_MAX / 2 || d_in > INT32_MAX / 2 || r > INT32_MAX / 2) return DORA_ERR_UNSUPPORTED;
  if (r == 0) return DORA_OK;  // dA and dB are empty
  if ((d_in > 0 && !dA) || (d_out > 0 && !dB)) return DORA_ERR_INVALID_ARG;
  if (!aligned(dA, 16) || !aligned(dB, 16)) return DORA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d_out == 0 || d_in == 0) {
    // no rows: dA = 0; no columns: V = 0 + s B A with A empty, so dB = 0
    float* z = d_out == 0 ? dA : dB;
    const size_t bytes = static_cast<size_t>(r) * (d_out == 0 ? d_in : d_out) * 4;
    if (bytes == 0) return DORA_OK;
    return cudaMemsetAsync(z, 0, bytes, st) == cudaSuccess ? DORA_OK : DORA_ERR_CUDA;
  }
  if (!W || !A || !B || !n || !d_n) return DORA_ERR_INVALID_ARG;
  if (d_in % 8 != 0 || d_out % 8 != 0 || r % 8 != 0) return DORA_ERR_UNSUPPORTED;
  if (!aligned(W, 16) || !aligned(A, 16) || !aligned(B, 16) || !aligned(n, 4) || !aligned(d_n, 4))
    return DORA_ERR_UNSUPPORTED;
  const BwdLayout L = bwd_layout(d_out, r);
  if (!workspace || workspace_bytes < L.total) return DORA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return DORA_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  if (device_info(&dev)) return DORA_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* part = reinterpret_cast<float*>(ws + L.off_part);
  float* part2 = reinterpret_cast<float*>(ws + L.off_part2);
  __nv_bfloat16* sG = reinterpret_cast<__nv_bfloat16*>(ws + L.off_sg);
  __nv_bfloat16* s2H = reinterpret_cast<__nv_bfloat16*>(ws + L.off_h);
  __nv_bfloat16* Bt = reinterpret_cast<__nv_bfloat16*>(ws + L.off_bt);
  __nv_bfloat16* Bct = reinterpret_cast<__nv_bfloat16*>(ws + L.off_bct);

  const int bn_b = pick_bn(r), bn_a = pick_bn(d_in);
  CUtensorMap tmW, tmA, tmAb, tmB, tmSG, tmBt, tmBct, tmH, tmWmn, tmAmn;
  if (make_map(&tmW, W, d_out, d_in) || make_map(&tmA, A, r, d_in) || make_map(&tmAb, A, r, d_in, bn_b / 2) ||
      make_map(&tmB, B, d_out, r) || make_map(&tmSG, sG, r, r, bn_b / 2) || make_map(&tmBt, Bt, r, d_out) ||
      make_map(&tmBct, Bct, r, d_out) || make_map(&tmH, s2H, r, r) || make_map(&tmWmn, W, d_out, d_in, 64) ||
      make_map(&tmAmn, A, r, d_in, 64))
    return DORA_ERR_CUDA;

  // 1) B^T and (s c B)^T
  note_launch();
  norm_bwd_prep_kernel<<<dim3(static_cast<unsigned>(cdiv(d_out, kPrepTile)), static_cast<unsigned>(cdiv(r, kPrepTile))),
                         256, 0, st>>>(static_cast<const __nv_bfloat16*>(B), d_n, n, s, static_cast<int>(d_out),
                               static_cast<int>(r), Bt, Bct);
  if (launch_error()) return DORA_ERR_CUDA;

  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;

  // 2) one Gram launch for both products: G = A A^T over d_in and
  //    s H = (s c B)^T B over d_out (split-K partial tiles), then one fixed-order
  //    reduction writing bf16 s G and s^2 H
  const int kb_g = static_cast<int>(cdiv(d_in, kBK)), kb_h = static_cast<int>(cdiv(d_out, kBK));
  GramArgs ga{};
  ga.r = static_cast<int>(r);
  ga.n_tiles = L.nt;
  ga.kb_main = kb_g;
  ga.splits = std::max(1, std::min({L.splits_max, (dev->num_sms / 2) / (L.nt * L.nt), kb_g}));
  ga.kb_main2 = kb_h;
  ga.splits2 = std::max(1, std::min({L.splits_max, (dev->num_sms / 2) / (L.nt * L.nt), kb_h}));
  ga.upper = 1;  // G = A A^T is symmetric: its tiles on or above the diagonal only
  ga.n_ctas1 = L.nt * (L.nt + 1) / 2 * ga.splits;
  ga.partial = part;
  ga.partial2 = part2;
  ga.wait_limit = kWaitLimitCycles;
  ga.status = dev->status;
  const size_t gram_smem = kGramStages * kGramStageBytes + (2 * kGramStages + 1) * 8 + 16 + 1024;
  note_launch();
  gram_tc_kernel<<<ga.n_ctas1 + L.nt * L.nt * ga.splits2, kNormThreads, gram_smem, st>>>(tmA, tmA, tmBct, tmBt, ga);
  if (launch_error()) return DORA_ERR_CUDA;
  {
    cudaLaunchConfig_t cfg{};
    cfg.stream = st;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    const long long rr = static_cast<long long>(r) * r;
    const int g1 = static_cast<int>(std::max<long long>(1, std::min<long long>(cdiv(rr, 1024), 2 * dev->num_sms)));
    cfg.gridDim = dim3(static_cast<unsigned>(2 * g1));
    cfg.blockDim = dim3(256);
    note_launch();
    if (cudaLaunchKernelEx(&cfg, gram_reduce_kernel, static_cast<const float*>(part), ga.splits, static_cast<int>(r), s,
                           sG, static_cast<int*>(nullptr), 0, g1, static_cast<const float*>(part2), ga.splits2, s,
                           s2H, 1) != cudaSuccess)
      return DORA_ERR_CUDA;
  }

  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = 2;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1] = pdl[0];
  cudaLaunchConfig_t pcfg{};
  pcfg.stream = st;
  pcfg.attrs = attrs;
  pcfg.numAttrs = 2;
  pcfg.blockDim = dim3(kLinThreads);
  pcfg.dynamicSmemBytes = linear_pair_smem(dev->smem_optin);
  const int stages = linear_pair_stages(dev->smem_optin);
  if (stages < 2) return DORA_ERR_UNSUPPORTED;
  auto pair_grid = [&](const LinearArgs& la) {
    return dim3(static_cast<unsigned>(2 * std::min<long long>(dev->pair_clusters,
                                                              static_cast<long long>(la.tiles_m) * la.tiles_n)));
  };

  // 3) dB = s c * ([W | B] [A | s G]^T), waiting for the reduction only
  //    before its K-extension blocks
  LinearArgs lb{};
  lb.M = static_cast<int>(d_out);
  lb.N = static_cast<int>(r);
  lb.kb_main = static_cast<int>(cdiv(d_in, kLinBK));
  lb.kb_total = lb.kb_main + static_cast<int>(cdiv(r, kLinBK));
  lb.tiles_m = static_cast<int>(cdiv(d_out, kPairBM));
  lb.bn = bn_b;
  lb.tiles_n = static_cast<int>(cdiv(r, bn_b));
  lb.stages = stages;
  lb.alpha = s;
  lb.rs_num = d_n;
  lb.rs_den = n;
  lb.out = dB;
  lb.ldo = r;
  lb.ext_waits = 1;
  lb.wait_limit = kWaitLimitCycles;
  lb.status = dev->status;
  pcfg.gridDim = pair_grid(lb);
  note_launch();
  if (cudaLaunchKernelEx(&pcfg, linear_pair_kernel<false, true>, tmW, tmAb, tmB, tmSG, lb) != cudaSuccess)
    return DORA_ERR_CUDA;

  // 4) dA = [(s c B)^T | s^2 H] [W ; A], dependent on dB through programmatic
  //    dependent launch: its CTAs take the SMs dB leaves free or finishes
  //    with; before its extension blocks it waits for dB's completion, which
  //    follows the reduction's
  LinearArgs la{};
  la.M = static_cast<int>(r);
  la.N = static_cast<int>(d_in);
  la.kb_main = static_cast<int>(cdiv(d_out, kLinBK));
  la.kb_total = la.kb_main + static_cast<int>(cdiv(r, kLinBK));
  la.tiles_m = static_cast<int>(cdiv(r, kPairBM));
  la.bn = bn_a;
  la.tiles_n = static_cast<int>(cdiv(d_in, bn_a));
  la.stages = stages;
  la.alpha = 1.f;
  la.out = dA;
  la.ldo = d_in;
  la.ext_waits = 1;
  la.wait_limit = kWaitLimitCycles;
  la.status = dev->status;
  pcfg.gridDim = pair_grid(la);
  note_launch();
  if (cudaLaunchKernelEx(&pcfg, linear_pair_kernel<true, true>, tmBct, tmWmn, tmH, tmAmn, la) != cudaSuccess)
    return DORA_ERR_CUDA;
  return launch_error();
}

}  // extern "C"

// ------------------------------------------------------------------------
// dora_compose_bwd_noalloc: the compose backward with library-owned scratch.
// The scratch is one file-scope device array; host code must not pass the
// array's name to a kernel (on the host it is only a stand-in symbol), so its
// device address is looked up once per device with that device current.
namespace dora {
namespace {

constexpr int kNoallocChunks = 16;     // row chunks of column partials
constexpr size_t kNoallocCounterBytes = 16384;
// 64-bit tagged arrival counters, one per 16-vector column strip; the most
// strips come with 1-element vectors at the largest d_out
static_assert((DORA_NOALLOC_MAX_D_OUT + kBwdVecs - 1) / kBwdVecs * 8 <= kNoallocCounterBytes,
              "counter area too small for the largest d_out");
static_assert(DORA_NOALLOC_SCRATCH_BYTES == kNoallocCounterBytes + kNoallocChunks * 4ull * DORA_NOALLOC_MAX_D_OUT,
              "scratch layout and the header's size disagree");

static __device__ __align__(256) unsigned char g_noalloc_scratch[DORA_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
unsigned char* g_noalloc_ptr[kMaxDevices] = {};
CUcontext g_noalloc_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn g_ctx_current = nullptr;

// The array's device address for the current device, looked up (with that
// device current) the first time this device's current context is seen.  A
// context torn down and created again (cudaDeviceReset) may load the module
// at another address, so the cached address is tied to the context it was
// looked up in.
int noalloc_scratch(unsigned char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DORA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_ctx_current) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return DORA_ERR_CUDA;
    g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(fn);
  }
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS) return DORA_ERR_CUDA;
  if (!g_noalloc_ptr[dev] || ctx == nullptr || ctx != g_noalloc_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return DORA_ERR_CUDA;
    }
    // the lookup makes the device's primary context current if none was
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return DORA_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<unsigned char*>(p);
    g_noalloc_ctx[dev] = ctx;
  }
  *out = g_noalloc_ptr[dev];
  return DORA_OK;
}

}  // namespace
}  // namespace dora

extern "C" int dora_compose_bwd_noalloc(const void* dy, const void* base_out, const void* lora_out, const float* m,
                                        const float* n, float s, int64_t tokens, int64_t d_out, dora_dtype dt,
                                        void* d_base, void* d_lora, float* d_m, void* stream) {
  return dora_compose_bwd_noalloc_bias(dy, base_out, lora_out, nullptr, m, n, s, tokens, d_out, dt, d_base, d_lora,
                                       d_m, stream);
}

extern "C" int dora_compose_bwd_noalloc_bias(const void* dy, const void* base_out, const void* lora_out,
                                             const void* bias, const float* m, const float* n, float s,
                                             int64_t tokens, int64_t d_out, dora_dtype dt, void* d_base,
                                             void* d_lora, float* d_m, void* stream) {
  if (dt != DORA_BF16 && dt != DORA_F32) return DORA_ERR_UNSUPPORTED;
  if (tokens < 0 || d_out < 0) return DORA_ERR_INVALID_ARG;
  if (d_out > DORA_NOALLOC_MAX_D_OUT) return DORA_ERR_UNSUPPORTED;
  if (d_out == 0) return DORA_OK;
  if (!m || !n || !d_m) return DORA_ERR_INVALID_ARG;
  if (tokens > 0 && (!dy || !base_out || !lora_out || !d_base || !d_lora)) return DORA_ERR_INVALID_ARG;
  int vec = 1;
  if (dt == DORA_BF16) {
    if (d_out % 8 != 0) return DORA_ERR_UNSUPPORTED;
    if (tokens > 0 && (!aligned(dy, 16) || !aligned(base_out, 16) || !aligned(lora_out, 16) ||
                       !aligned(d_base, 16) || !aligned(d_lora, 16)))
      return DORA_ERR_UNSUPPORTED;
    vec = 8;
  } else {
    const bool a16 = aligned(dy, 16) && aligned(base_out, 16) && aligned(lora_out, 16) && aligned(d_base, 16) &&
                     aligned(d_lora, 16) && aligned(bias, 16);
    if (!aligned(dy, 4) || !aligned(base_out, 4) || !aligned(lora_out, 4) || !aligned(d_base, 4) ||
        !aligned(d_lora, 4))
      return DORA_ERR_UNSUPPORTED;
    vec = (d_out % 4 == 0 && a16) ? 4 : 1;
  }
  if (!aligned(m, 4) || !aligned(n, 4) || !aligned(d_m, 4) || !aligned(bias, dt == DORA_BF16 ? 16 : 4))
    return DORA_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  if (device_info(&dev)) return DORA_ERR_CUDA;
  unsigned char* scratch = nullptr;
  if (noalloc_scratch(&scratch)) return DORA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tokens == 0) return cudaMemsetAsync(d_m, 0, static_cast<size_t>(d_out) * 4, st) == cudaSuccess ? DORA_OK : DORA_ERR_CUDA;

  const long long nvec = d_out / vec;
  const long long strips = cdiv(nvec, kBwdVecs);
  int occ = 1;
  if (dt == DORA_BF16)
    occ = ctas_per_sm(compose_bwd_kernel<__nv_bfloat16, 8, false>, kBwdThreads);
  else if (vec == 4)
    occ = ctas_per_sm(compose_bwd_kernel<float, 4, false>, kBwdThreads);
  else
    occ = ctas_per_sm(compose_bwd_kernel<float, 1, false>, kBwdThreads);
  const long long chunks = bwd_chunks(strips, static_cast<long long>(dev->num_sms) * occ, tokens,
                                      std::min<long long>(kNoallocChunks, cdiv(tokens, kBwdSlots)));
  const long long rows = cdiv(tokens, chunks);
  const long long chunks2 = cdiv(tokens, rows);
  // tagged strip counters (no clearing needed); the partials are written before read
  if (static_cast<size_t>(strips) * 8 > kNoallocCounterBytes) return DORA_ERR_UNSUPPORTED;
  unsigned long long* cnt = reinterpret_cast<unsigned long long*>(scratch);
  float* part = reinterpret_cast<float*>(scratch + kNoallocCounterBytes);
  dim3 grid(static_cast<unsigned>(strips), static_cast<unsigned>(chunks2));
  if (dt == DORA_BF16)
    launch_compose_bwd<__nv_bfloat16, 8>(grid, st, dy, base_out, lora_out, bias, m, n, s, tokens, nvec, d_out, d_base,
                                         d_lora, part, cnt, d_m, rows);
  else if (vec == 4)
    launch_compose_bwd<float, 4>(grid, st, dy, base_out, lora_out, bias, m, n, s, tokens, nvec, d_out, d_base, d_lora,
                                part, cnt, d_m, rows);
  else
    launch_compose_bwd<float, 1>(grid, st, dy, base_out, lora_out, bias, m, n, s, tokens, nvec, d_out, d_base, d_lora,
                                part, cnt, d_m, rows);
  return launch_error();
}
