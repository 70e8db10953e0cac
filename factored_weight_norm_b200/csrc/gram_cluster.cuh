// gram_cluster.cuh - G' = (s/2) A A^T as bf16 in one launch (tcgen05, sm_100a).
//
// "Scaling DoRA: High-Rank Adaptation via Factored Norms and Fused Kernels",
// Abstract: the Gram term of the factored norm needs G = A A^T (r x r), an
// O(r^2) intermediate.  The norm GEMM reads (s/2) G as the N-side operand of
// its K extension.
//
// One cluster of kSplit CTAs per 128 x 128 tile of G on or above the
// diagonal (G is symmetric): CTA k of the cluster accumulates the tile over
// its 1/kSplit of d_in in TMEM (tcgen05.mma, A's rows on both sides, fed by
// TMA), parks its fp32 partial in its own shared memory, and after a cluster
// barrier sums its share of the tile's rows over all CTAs' partials in CTA
// order (distributed shared memory), scales by s/2 and stores bf16, once for
// the tile and once transposed for its mirror below the diagonal.  No fp32
// partial ever goes to global memory, so a single launch of a few dozen CTAs
// replaces a split-K launch plus a reduction launch; it lets the kernel
// launched behind it (programmatic dependent launch) start as soon as it has
// begun.  The launch also zeroes that kernel's tile counters.
//
// Roles (192 threads): warp 0 TMA (lane 0 the M-side box, lane 1 the N-side
// box; a diagonal tile loads one box for both), warp 1 MMA issuer, warps 2..5
// TMEM epilogue (lane quarter = warp % 4).  Every mbarrier wait is bounded;
// every path reaches both cluster barriers.
#pragma once

#include "norm_tc.cuh"

namespace dora {

constexpr int kGcThreads = 192;
constexpr int kGcStages = 6;         // ring stages of one K block (two 16 KB boxes)
constexpr uint32_t kGcStageBytes = 2 * kBoxBytes;
constexpr int kGcPad = 132;          // fp32 row pitch of the parked partial (bank spread)
constexpr size_t kGcSmem = 1024 + kGcStages * kGcStageBytes + (2 * kGcStages + 2) * 8 + 16;
static_assert(static_cast<size_t>(kBM) * kGcPad * 4 <= kGcStages * kGcStageBytes, "partial fits in the ring");

struct GramClusterArgs {
  int r, kb_main, nt;  // rank, K blocks over d_in, 128-row tiles of r
  float half_s;
  __nv_bfloat16* Gs;   // [r][r]
  long long wait_limit;
  int* status;
  int* zero_cnt;       // [n_zero] ints zeroed by this launch
  int n_zero;
};

// kSplit: CTAs per cluster (K splits of a tile), a power of two up to 8.
template <int kSplit>
__global__ void __launch_bounds__(kGcThreads, 1)
    gram_cluster_kernel(const __grid_constant__ CUtensorMap tmA, const GramClusterArgs a) {
  static_assert(kSplit >= 1 && kSplit <= 8 && (kSplit & (kSplit - 1)) == 0, "cluster of 1, 2, 4 or 8 CTAs");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base_s - raw_s);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGcStages * kGcStageBytes);
  uint64_t* empty = full + kGcStages;
  uint64_t* tmem_full = empty + kGcStages;
  uint64_t* drain = tmem_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* park = reinterpret_cast<float*>(smem);  // [128][kGcPad], after the MMAs are done with the ring

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int k = static_cast<int>(cluster_ctarank());
  const long long limit = a.wait_limit;
  for (int i = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x); i < a.n_zero;
       i += static_cast<int>(gridDim.x * blockDim.x))
    a.zero_cnt[i] = 0;
  // tile (mi, ni), mi <= ni, from the cluster index (row-major upper triangle)
  int t = static_cast<int>(blockIdx.x) / kSplit;
  int mi = 0;
  while (t >= a.nt - mi) {
    t -= a.nt - mi;
    ++mi;
  }
  const int ni = mi + t;
  const bool diag = mi == ni;
  const int m_rows = min(kBM, a.r - mi * kBM);
  const int n_this = min(kBM, a.r - ni * kBM);
  const int kb_lo = static_cast<int>(static_cast<long long>(k) * a.kb_main / kSplit);
  const int kb_hi = static_cast<int>(static_cast<long long>(k + 1) * a.kb_main / kSplit);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGcStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmA);
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_launch();  // the GEMM behind this launch may take the SMs this one leaves free

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint32_t bytes = diag ? kBoxBytes : 2 * kBoxBytes;
    int stage = 0;
    uint32_t phase = 0, parity_bits = 0, filled_mask = 0;
    for (int kb = kb_lo; kb < kb_hi; ++kb) {
      bool got = true;
      if (lane == 0) {
        got = mbar_wait(&empty[stage], phase ^ 1u, limit);
        if (got) mbar_arrive_expect_tx(&full[stage], bytes);
        else record_timeout(a.status, abort_flag);
      }
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
      __syncwarp();
      const uint32_t dst = base_s + stage * kGcStageBytes;
      if (lane == 0) tma_load_2d(dst, &tmA, &full[stage], kb * kBK, mi * kBM);
      else if (lane == 1 && !diag) tma_load_2d(dst + kBoxBytes, &tmA, &full[stage], kb * kBK, ni * kBM);
      parity_bits = (parity_bits & ~(1u << stage)) | (phase << stage);
      filled_mask |= 1u << stage;
      if (++stage == kGcStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (lane == 0)
      for (int s2 = 0; s2 < kGcStages; ++s2)
        if ((filled_mask >> s2) & 1u) mbar_wait(&full[s2], (parity_bits >> s2) & 1u, limit);
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, n_this);
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        if (!mbar_wait(&full[stage], phase, limit)) {
          record_timeout(a.status, abort_flag);
          break;
        }
        tc_fence_after();
        const uint64_t ad = sw128_kmajor_desc(base_s + stage * kGcStageBytes);
        const uint64_t bd = diag ? ad : ad + (kBoxBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          mma_bf16(tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb == kb_lo && kk == 0) ? 0u : 1u);
        mma_commit(&empty[stage]);
        if (++stage == kGcStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      mma_commit(tmem_full);
      mma_commit(drain);
      mbar_wait(drain, 0, limit);
    }
  } else {
    // ------------------------------------------ park this split's partial
    const int q = warp & 3;
    const int row = q * 32 + lane;
    float* dst = park + static_cast<size_t>(row) * kGcPad;
    const bool ok = mbar_wait_warp(tmem_full, 0, limit);
    if (!ok && lane == 0) record_timeout(a.status, abort_flag);
    tc_fence_after();
    for (int j0 = 0; j0 < kBM; j0 += 32) {
      float v[32];
      if (ok && kb_hi > kb_lo) {
        tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + j0, v);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0.f;  // no K blocks (d_in < the split count): a zero partial
      }
#pragma unroll
      for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(dst + j0 + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
    }
  }

  // every CTA's partial is parked
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();

  // ---- this CTA's rows of the tile: sum the splits in CTA order, scale, store
  // (four columns per load; two groups in flight per thread; r is a multiple
  // of 16, so a group is all in or all out of the tile)
  {
    constexpr int kRowsPer = kBM / kSplit;
    constexpr int kGroups = kRowsPer * (kBM / 4);
    const uint32_t park_s = smem_u32(park);
    uint32_t peer[kSplit];
#pragma unroll
    for (int c = 0; c < kSplit; ++c) peer[c] = mapa_shared(park_s, static_cast<uint32_t>(c));
    for (int e0 = threadIdx.x; e0 < kGroups; e0 += 2 * kGcThreads) {
      float4 v[2][kSplit];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int e = min(e0 + h * kGcThreads, kGroups - 1);
        const int rr = k * kRowsPer + e / (kBM / 4), cc = (e % (kBM / 4)) * 4;
        const uint32_t off = static_cast<uint32_t>((rr * kGcPad + cc) * 4);
#pragma unroll
        for (int c = 0; c < kSplit; ++c)
          asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(v[h][c].x), "=f"(v[h][c].y), "=f"(v[h][c].z), "=f"(v[h][c].w)
                       : "r"(peer[c] + off)
                       : "memory");
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int e = e0 + h * kGcThreads;
        const int rr = k * kRowsPer + e / (kBM / 4), cc = (e % (kBM / 4)) * 4;
        if (e >= kGroups || rr >= m_rows || cc >= n_this) continue;
        float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < kSplit; ++c) {
          sum[0] += v[h][c].x;
          sum[1] += v[h][c].y;
          sum[2] += v[h][c].z;
          sum[3] += v[h][c].w;
        }
        __nv_bfloat16 g[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) g[t] = __float2bfloat16_rn(a.half_s * sum[t]);
        const int gi = mi * kBM + rr, gj = ni * kBM + cc;
        __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(a.Gs + static_cast<size_t>(gi) * a.r + gj);
        dst[0] = __halves2bfloat162(g[0], g[1]);
        dst[1] = __halves2bfloat162(g[2], g[3]);
        if (!diag)
#pragma unroll
          for (int t = 0; t < 4; ++t) a.Gs[static_cast<size_t>(gj + t) * a.r + gi] = g[t];
      }
    }
  }

  // no CTA leaves (or frees the shared memory others read) before all have read
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 128);
}

}  // namespace dora
