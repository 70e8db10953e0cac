// norm_tc.cuh - bf16 factored row norm on tcgen05 tensor cores (sm_100a).
//
// "Scaling DoRA: High-Rank Adaptation via Factored Norms and Fused Kernels",
// Abstract: the squared row norm of W + sBA splits into base, cross and Gram
// terms that need only O(d_out r + r^2) intermediates:
//
//   n_i^2 = ||W_i||^2 + 2s <B_i, U_i> + s^2 B_i G B_i^T,  U = W A^T, G = A A^T.
//
// Folding the Gram term into the same contraction: with G' = (s/2) G,
//   V = [W | B] [A | G']^T = W A^T + (s/2) B G     (K extended by r)
//   n_i^2 = ||W_i||^2 + 2s <B_i, V_i>.
// So one tensor-core GEMM (M = d_out, N = r, K = d_in + r) with a row-dot
// epilogue gives every term; W is streamed from HBM exactly once and the
// [d_out, r] product V never leaves TMEM.
//
// Kernels (one stream, chained with programmatic dependent launch):
//   gram_cluster_kernel (gram_cluster.cuh) G' = (s/2) A A^T from clusters of
//                      K splits on a few SMs; also zeroes the tile counters
//   norm_tc_kernel     persistent stream-K GEMM over (M tile, N chunk, K
//                      block) units in weighted contiguous ranges (shorter
//                      for the CTAs that start behind the Gram clusters); a
//                      range that crosses a tile boundary is walked from that
//                      boundary on, so its K-extension blocks (the only reads
//                      of G') come last and the GEMM seldom waits for the
//                      Gram launch.  Two warps sum ||W_i||^2 from the
//                      shared-memory W stages; at each segment end B's rows
//                      arrive through the same TMA ring and four epilogue
//                      warps dot them with V_i read from TMEM; one fp32
//                      partial per (row, segment); the last warp to finish an
//                      M tile sums its partials in fixed order and writes
//                      n = sqrt(max(., 0)).
// gram_tc_kernel and gram_reduce_kernel below (split-K Gram tiles and their
// fixed-order reduction) serve the attached-norm backward's two Gram
// products.
#pragma once

#include "sm100_ptx.cuh"

namespace dora {

constexpr int kBM = 128;              // rows per M tile (TMEM lanes)
constexpr int kBK = 64;               // bf16 along K per 128-byte swizzled row
constexpr int kBoxRows = 128;         // rows per TMA box
constexpr int kBoxBytes = kBoxRows * 128;
constexpr int kNormThreads = 192;     // Gram and batched kernels: warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
// norm_tc_kernel: warp 0 TMA, warp 1 MMA, warps 2..5 TMEM epilogue at segment
// ends, warps 6 and 7 ||W_i||^2 over every W stage.  A warp runs on the SM
// sub-partition (warp index mod 4) whose TMEM lane quarter it may read, so one
// epilogue warp always shares the MMA thread's sub-partition; the per-stage
// work goes to warps 6 and 7 (sub-partitions 2 and 3) so that it does not
// compete with the MMA thread for issue slots.
constexpr int kNormTcThreads = 256;
// shared memory besides the stages: 1024-byte alignment slack, five single
// mbarriers, the TMEM address and abort flag (16 bytes), the W^2 hand-off
// (kBM floats); each stage adds its two mbarriers
// (plus the table of the grid's G + 1 range starts, 4 bytes each)
constexpr int kNormTcSmemFixed = 1024 + 5 * 8 + 16 + kBM * 4;
constexpr int kMaxChunkN = 512;       // TMEM columns
constexpr int kMaxStages = 8;
constexpr int kStatusTimeout = 5;     // == DORA_ERR_TIMEOUT
constexpr int kFinOwners = 4;         // partial owners the finalizing warp loads together
constexpr int kBAhead = 8;            // units before a segment's end at which its B rows are prefetched to L2

struct NormArgs {
  int d_out, d_in, r;
  int m_tiles, n_chunks, chunk_n, kb_main, kb_total;
  long long units;
  // CTA c's unit range is [unit_start(c), unit_start(c + 1)): lengths in
  // proportion to w_early for the first `early` CTAs and to w_late after (the
  // CTAs that wait for the SMs the Gram launch holds)
  int early;
  long long w_early, w_late;
  int stages;
  uint32_t stage_bytes;   // W-side tile + N-side tiles (a multiple of kBoxBytes)
  uint32_t tmem_cols;
  float two_s;
  long long wait_limit;
  float* partials;        // [(gridDim.x + m_tiles * n_chunks) * 128]
  int* counters;          // [m_tiles], zeroed by the Gram launch ahead of this one
  float* n_out;           // [d_out]
  int* status;
  int squared;            // 1: write n^2 as summed (a shard's partial), 0: sqrt(max(n^2, 0))
};

// Weighted stream-K ranges: CTA c owns [unit_start(c), unit_start(c + 1)),
// the cumulative weight of the CTAs before c scaled to the unit count.  The
// kernel tabulates the starts in shared memory once; the lookups below run
// on that table.
__host__ __device__ __forceinline__ long long unit_cum(const NormArgs& a, int c) {
  return a.w_early * (c < a.early ? c : a.early) + a.w_late * (c > a.early ? c - a.early : 0);
}
__host__ __device__ __forceinline__ long long unit_start(const NormArgs& a, int c, int G) {
  return a.units * unit_cum(a, c) / unit_cum(a, G);
}
// Owner of unit u in the table `st` of G + 1 starts: the largest c with
// st[c] <= u (an empty range never owns a unit, since the next range starts
// where it does).
__device__ __forceinline__ int unit_owner(const int* st, int u, int G) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (st[mid] <= u) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}
__device__ __forceinline__ bool unit_range_nonempty(const int* st, int c) { return st[c + 1] > st[c]; }

__device__ __forceinline__ void record_timeout(int* status, volatile int* abort_flag) {
  atomicExch(status, kStatusTimeout);
  *abort_flag = 1;
}

__device__ __forceinline__ float sumsq_bf16x8(uint4 v) {
  float a = bf16_lo(v.x), b = bf16_hi(v.x), c = bf16_lo(v.y), d = bf16_hi(v.y);
  float e = bf16_lo(v.z), f = bf16_hi(v.z), g = bf16_lo(v.w), h = bf16_hi(v.w);
  float s0 = a * a, s1 = b * b;
  s0 = fmaf(c, c, s0);
  s1 = fmaf(d, d, s1);
  s0 = fmaf(e, e, s0);
  s1 = fmaf(f, f, s1);
  s0 = fmaf(g, g, s0);
  s1 = fmaf(h, h, s1);
  return s0 + s1;
}

__device__ __forceinline__ float dot_bf16x8(uint4 w, const float* x) {
  float s0 = bf16_lo(w.x) * x[0];
  float s1 = bf16_hi(w.x) * x[1];
  s0 = fmaf(bf16_lo(w.y), x[2], s0);
  s1 = fmaf(bf16_hi(w.y), x[3], s1);
  s0 = fmaf(bf16_lo(w.z), x[4], s0);
  s1 = fmaf(bf16_hi(w.z), x[5], s1);
  s0 = fmaf(bf16_lo(w.w), x[6], s0);
  s1 = fmaf(bf16_hi(w.w), x[7], s1);
  return s0 + s1;
}

// Byte offset of 16-byte chunk `c` of row `row` inside a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_chunk(int row, int c) {
  return static_cast<uint32_t>(row * 128 + ((c ^ (row & 7)) << 4));
}

// Walks a CTA's range of (M tile, N chunk, K block) units.  A range [u0, u1)
// that crosses a tile boundary is walked from its first boundary tb on,
// [tb, u1), then [u0, tb): the part that ends with a tile's K-extension
// blocks (the only reads of the Gram launch's G') comes last, so a CTA
// seldom waits for that launch.  Only the starts need a division; stepping
// is compare-and-increment, so the single-thread producer and MMA loops
// spend a few instructions per unit.
struct UnitIter {
  int tc, kb, mt, ch, c0, n_this, left;
  int len2;               // units of the part walked second (0: no wrap)
  long long wrap_to;      // its first unit
  bool seg_first;

  __device__ __forceinline__ void seek(const NormArgs& a, long long u) {
    tc = static_cast<int>(u / a.kb_total);
    kb = static_cast<int>(u - static_cast<long long>(tc) * a.kb_total);
    mt = tc / a.n_chunks;
    ch = tc - mt * a.n_chunks;
    c0 = ch * a.chunk_n;
    n_this = min(a.chunk_n, a.r - c0);
    seg_first = true;
  }
  __device__ __forceinline__ void start(const NormArgs& a, long long u_begin, long long u_end) {
    const long long tb = min(u_end, (u_begin + a.kb_total - 1) / a.kb_total * a.kb_total);
    left = static_cast<int>(u_end - u_begin);
    if (tb > u_begin && tb < u_end) {
      len2 = static_cast<int>(tb - u_begin);
      wrap_to = u_begin;
      seek(a, tb);
    } else {
      len2 = 0;
      wrap_to = 0;
      seek(a, u_begin);
    }
  }
  __device__ __forceinline__ bool valid() const { return left > 0; }
  __device__ __forceinline__ bool seg_last(const NormArgs& a) const {
    return left == 1 || kb == a.kb_total - 1 || (len2 > 0 && left == len2 + 1);
  }
  // Units of this segment after the current one.
  __device__ __forceinline__ int seg_rem(const NormArgs& a) const {
    const int to_range_end = (len2 > 0 && left > len2) ? left - len2 - 1 : left - 1;
    return min(a.kb_total - 1 - kb, to_range_end);
  }
  __device__ __forceinline__ void next(const NormArgs& a) {
    --left;
    if (len2 > 0 && left == len2) {
      seek(a, wrap_to);
      return;
    }
    if (++kb == a.kb_total) {
      kb = 0;
      ++tc;
      if (++ch == a.n_chunks) {
        ch = 0;
        ++mt;
      }
      c0 = ch * a.chunk_n;
      n_this = min(a.chunk_n, a.r - c0);
      seg_first = true;
    } else {
      seg_first = false;
    }
  }
};

// Ring slots that carry B's rows for a segment epilogue.
__device__ __forceinline__ int b_stages(const NormArgs& a, int n_this) {
  const int nbox = (n_this + kBK - 1) / kBK;
  const int slots = static_cast<int>(a.stage_bytes / kBoxBytes);
  return (nbox + slots - 1) / slots;
}

// ===================================================================== norm
__global__ void __launch_bounds__(kNormTcThreads, 1)
    norm_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmA,
                   const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmG,
                   const NormArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base_s - raw_s);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.stages * a.stage_bytes);
  uint64_t* empty = full + a.stages;
  uint64_t* tmem_full = empty + a.stages;
  uint64_t* tmem_empty = tmem_full + 1;
  uint64_t* drain = tmem_empty + 1;
  uint64_t* w2_full = drain + 1;   // the W^2 warps' row sums of a segment are in w2
  uint64_t* w2_empty = w2_full + 1;  // the epilogue warps have read them
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(w2_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* w2 = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(w2_empty + 1) + 16);
  int* starts = reinterpret_cast<int*>(w2 + kBM);  // [gridDim.x + 1] unit range starts

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const long long u_begin = unit_start(a, blockIdx.x, G);
  const long long u_end = unit_start(a, blockIdx.x + 1, G);
  for (int c = threadIdx.x; c <= G; c += blockDim.x) starts[c] = static_cast<int>(unit_start(a, c, G));
  const long long limit = a.wait_limit;
  const int slots = static_cast<int>(a.stage_bytes / kBoxBytes);

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&full[s], 1);
      // W stages: the MMA commit + 3 from each W^2 warp; segment-end B
      // stages: the MMA warp + one arrive per epilogue and per W^2 warp.
      // Every warp that waits on a stage's fills also arrives on its
      // releases, so no fill can complete twice before a waiter sees it
      // (a parity wait cannot tell phase k from phase k + 2).
      mbar_init(&empty[s], 1 + 4 + 2);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 4);
    mbar_init(drain, 1);
    mbar_init(w2_full, 2);
    mbar_init(w2_empty, 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmG);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, a.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop; lane 0 owns the ring bookkeeping and each
    // lane issues at most one TMA box per stage (lane 0 the W-side box, lanes
    // 1.. the N-side boxes), so the issue latency of one thread is not paid
    // once per box.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t parity_bits = 0;  // bit s: parity of the latest fill of stage s
    uint32_t filled_mask = 0;
    bool gram_ready = false;
    bool ok = true;
    auto acquire = [&](uint32_t bytes) -> bool {
      bool got = true;
      if (lane == 0) {
        got = mbar_wait(&empty[stage], phase ^ 1u, limit);
        if (got) mbar_arrive_expect_tx(&full[stage], bytes);
        else record_timeout(a.status, abort_flag);
      }
      got = __shfl_sync(0xffffffffu, got, 0);
      __syncwarp();
      return got;
    };
    auto advance = [&]() {
      parity_bits = (parity_bits & ~(1u << stage)) | (phase << stage);
      filled_mask |= 1u << stage;
      if (++stage == a.stages) {
        stage = 0;
        phase ^= 1u;
      }
    };
    UnitIter x;
    for (x.start(a, u_begin, u_end); x.valid() && ok; x.next(a)) {
      const int nboxes = (x.n_this + kBoxRows - 1) / kBoxRows;
      const bool ext = x.kb >= a.kb_main;
      {
        // B's rows for this segment's epilogue: into L2 kBAhead units before
        // the segment ends, so that the ring loads of them at its end do not
        // wait for HBM (and the W stream has no time to evict them first)
        const int rem = x.seg_rem(a);
        if (rem == kBAhead || (x.seg_first && rem < kBAhead)) {
          const int nbox = (x.n_this + kBK - 1) / kBK;
          for (int b = lane; b < nbox; b += 32) tma_prefetch_l2_2d(&tmB, x.c0 + b * kBK, x.mt * kBM);
        }
      }
      if (ext && !gram_ready) {
        grid_dep_wait();  // G' is written by the Gram kernels
        gram_ready = true;
      }
      if (!(ok = acquire(static_cast<uint32_t>(kBoxBytes * (1 + nboxes))))) break;
      if (lane <= nboxes) {
        const CUtensorMap* map = lane == 0 ? (ext ? &tmB : &tmW) : (ext ? &tmG : &tmA);
        const int xk = (ext ? x.kb - a.kb_main : x.kb) * kBK;
        const int y = lane == 0 ? x.mt * kBM : x.c0 + (lane - 1) * kBoxRows;
        tma_load_2d(base_s + stage * a.stage_bytes + lane * kBoxBytes, map, &full[stage], xk, y);
      }
      advance();
      if (x.seg_last(a)) {
        // B[m tile rows, chunk columns] for the segment epilogue, 64 columns per box
        const int nbox = (x.n_this + kBK - 1) / kBK;
        for (int b0 = 0; b0 < nbox; b0 += slots) {
          const int nb = min(slots, nbox - b0);
          if (!(ok = acquire(static_cast<uint32_t>(kBoxBytes * nb)))) break;
          if (lane < nb)
            tma_load_2d(base_s + stage * a.stage_bytes + lane * kBoxBytes, &tmB, &full[stage],
                        x.c0 + (b0 + lane) * kBK, x.mt * kBM);
          advance();
        }
      }
    }
    // Never leave a TMA copy in flight: wait for the latest fill of every stage.
    if (lane == 0)
      for (int s2 = 0; s2 < a.stages; ++s2)
        if ((filled_mask >> s2) & 1u) mbar_wait(&full[s2], (parity_bits >> s2) & 1u, limit);
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int seg = 0;
      bool ok = true;
      auto advance = [&]() {
        if (++stage == a.stages) {
          stage = 0;
          phase ^= 1u;
        }
      };
      auto fail = [&]() {
        record_timeout(a.status, abort_flag);
        ok = false;
      };
      const uint64_t desc0 = sw128_kmajor_desc(base_s);
      const uint64_t desc_step = a.stage_bytes >> 4;
      UnitIter x;
      int n_cur = -1;
      uint32_t idesc0 = 0, idesc1 = 0;
      for (x.start(a, u_begin, u_end); x.valid() && ok; x.next(a)) {
        if (x.n_this != n_cur) {  // MMA pieces of N <= 256 for this chunk width
          n_cur = x.n_this;
          idesc0 = idesc_bf16_f32(kBM, min(256, n_cur));
          idesc1 = n_cur > 256 ? idesc_bf16_f32(kBM, n_cur - 256) : 0u;
        }
        if (x.seg_first && seg > 0) {
          if (!mbar_wait(tmem_empty, static_cast<uint32_t>((seg - 1) & 1), limit)) {
            fail();
            break;
          }
          tc_fence_after();
        }
        if (!mbar_wait(&full[stage], phase, limit)) {
          fail();
          break;
        }
        tc_fence_after();
        // the stage's descriptors differ from stage 0's only in the start
        // address field; +32 bytes along K inside the swizzled row is +2
        const uint64_t adesc = desc0 + static_cast<uint64_t>(stage) * desc_step;
        const uint64_t bdesc = adesc + (kBoxBytes >> 4);
        const uint32_t acc0 = x.seg_first ? 0u : 1u;
        if (idesc1) {
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint32_t acc = k == 0 ? acc0 : 1u;
            mma_bf16(tmem, adesc + 2 * k, bdesc + 2 * k, idesc0, acc);
            mma_bf16(tmem + 256, adesc + 2 * k, bdesc + (256 * 128 >> 4) + 2 * k, idesc1, acc);
          }
        } else {
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) mma_bf16(tmem, adesc + 2 * k, bdesc + 2 * k, idesc0, k == 0 ? acc0 : 1u);
        }
        mma_commit(&empty[stage]);
        advance();
        if (x.seg_last(a)) {
          mma_commit(tmem_full);
          ++seg;
          // the B stages feed the epilogue only: release them on arrival
          const int nbst = b_stages(a, x.n_this);
          for (int i = 0; i < nbst; ++i) {
            if (!mbar_wait(&full[stage], phase, limit)) {
              fail();
              break;
            }
            mbar_arrive(&empty[stage]);
            advance();
          }
        }
      }
      if (u_end > u_begin) {  // (an empty range issued no MMA to wait for)
        mma_commit(drain);
        mbar_wait(drain, 0, limit);
      }
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------- ||W_i||^2 warps
    // Warp 6 sums rows 0..63 of every W stage, warp 7 rows 64..127 (lane l:
    // rows l and l + 32 of its half), and releases the stage with a triple
    // arrival; at each segment end the row sums go to the epilogue warps
    // through shared memory.  The sum ignores the chunk order, and visiting
    // chunk (j ^ row % 8) keeps the eight rows of a quarter-warp on distinct
    // banks.
    const int r0 = (warp - 6) * 64 + lane;
    int stage = 0;
    uint32_t phase = 0;
    int seg = 0;
    float acc0 = 0.f, acc1 = 0.f;
    auto step = [&]() {
      if (++stage == a.stages) {
        stage = 0;
        phase ^= 1u;
      }
    };
    UnitIter x;
    for (x.start(a, u_begin, u_end); x.valid(); x.next(a)) {
      if (__any_sync(0xffffffffu, !mbar_wait(&full[stage], phase, limit))) {
        if (lane == 0) record_timeout(a.status, abort_flag);
        break;
      }
      if (x.ch == 0 && x.kb < a.kb_main) {
        const uint8_t* tile = smem + stage * a.stage_bytes;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          acc0 += sumsq_bf16x8(*reinterpret_cast<const uint4*>(tile + sw128_chunk(r0, j)));
          acc1 += sumsq_bf16x8(*reinterpret_cast<const uint4*>(tile + sw128_chunk(r0 + 32, j)));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_cnt(&empty[stage], 3);
      step();
      if (!x.seg_last(a)) continue;
      // the segment-end B stages: the epilogue warps read them; these warps
      // only keep their place in the ring
      const int nbst = b_stages(a, x.n_this);
      bool ok = true;
      for (int i = 0; i < nbst; ++i) {
        if (__any_sync(0xffffffffu, !mbar_wait(&full[stage], phase, limit))) {
          if (lane == 0) record_timeout(a.status, abort_flag);
          ok = false;
          break;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
        step();
      }
      if (!ok) break;
      if (seg > 0 && !mbar_wait_warp(w2_empty, static_cast<uint32_t>((seg - 1) & 1), limit)) {
        if (lane == 0) record_timeout(a.status, abort_flag);
        break;
      }
      w2[r0] = acc0;
      w2[r0 + 32] = acc1;
      acc0 = acc1 = 0.f;
      __threadfence_block();
      __syncwarp();
      if (lane == 0) mbar_arrive(w2_full);
      ++seg;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row_local = q * 32 + lane;
    const uint32_t tmem_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
    int stage = 0;
    uint32_t phase = 0;
    int seg = 0;
    bool deps_ready = false;
    auto step = [&]() {
      if (++stage == a.stages) {
        stage = 0;
        phase ^= 1u;
      }
    };
    auto release = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      step();
    };
    UnitIter x;
    for (x.start(a, u_begin, u_end); x.valid(); x.next(a)) {
      step();  // the W stages are the MMA thread's and the W^2 warps'
      if (!x.seg_last(a)) continue;

      // segments of this M tile: the nonempty ranges meeting each of its chunks
      // (counted while the segment's MMAs still run)
      int expected = 0;
      for (int c2 = 0; c2 < a.n_chunks; ++c2) {
        const int s0 = (x.mt * a.n_chunks + c2) * a.kb_total;
        const int o1 = unit_owner(starts, s0 + a.kb_total - 1, G);
        for (int o = unit_owner(starts, s0, G); o <= o1; ++o) expected += unit_range_nonempty(starts, o) ? 1 : 0;
      }

      // ---- segment epilogue: <B_i, V_i> over this chunk's columns
      if (!mbar_wait_warp(tmem_full, static_cast<uint32_t>(seg & 1), limit)) {
        if (lane == 0) record_timeout(a.status, abort_flag);
        break;
      }
      tc_fence_after();
      float dot = 0.f;
      const int nbox = (x.n_this + kBK - 1) / kBK;
      bool ok = true;
      for (int b0 = 0; b0 < nbox; b0 += slots) {
        if (!mbar_wait_warp(&full[stage], phase, limit)) {
          if (lane == 0) record_timeout(a.status, abort_flag);
          ok = false;
          break;
        }
        const uint8_t* sb = smem + stage * a.stage_bytes;
        const int nb = min(slots, nbox - b0);
        for (int b = 0; b < nb; ++b) {
          const uint8_t* tile = sb + b * kBoxBytes;
          const int j0 = (b0 + b) * kBK;
          // the box's 64 columns of V in one TMEM round trip (the accumulator
          // is allocated in a power of two of at least 64 columns)
          float acc[64];
          tmem_ld64(tmem_lane + j0, acc);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            if (j0 + 8 * v < x.n_this)
              dot += dot_bf16x8(*reinterpret_cast<const uint4*>(tile + sw128_chunk(row_local, v)), acc + 8 * v);
        }
        release();
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tmem_empty);
      ++seg;

      // this segment's ||W_i||^2 from the W^2 warps
      if (!mbar_wait_warp(w2_full, static_cast<uint32_t>((seg - 1) & 1), limit)) {
        if (lane == 0) record_timeout(a.status, abort_flag);
        break;
      }
      const float base_acc = w2[row_local];
      __syncwarp();
      if (lane == 0) mbar_arrive(w2_empty);
      const float partial = base_acc + a.two_s * dot;
      if (!deps_ready) {
        grid_dep_wait();  // counters are zeroed by the Gram launch
        deps_ready = true;
      }
      a.partials[static_cast<size_t>(blockIdx.x + x.tc) * kBM + row_local] = partial;

      // ---- the last of the M tile's segment-warps to arrive finishes the tile
      __threadfence();
      __syncwarp();
      int last = 0;
      if (lane == 0) last = (atomicAdd(&a.counters[x.mt], 1) == 4 * expected - 1);
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        __threadfence();
        // lane l owns rows l, l + 32, l + 64, l + 96; the partials of up to
        // kFinOwners owners are loaded together, then added in owner order
        constexpr int kRows = kBM / 32;
        float total[kRows];
#pragma unroll
        for (int j = 0; j < kRows; ++j) total[j] = 0.f;
        for (int c2 = 0; c2 < a.n_chunks; ++c2) {
          const int tc2 = x.mt * a.n_chunks + c2;
          const int s0 = tc2 * a.kb_total;
          const int o0 = unit_owner(starts, s0, G);
          const int o1 = unit_owner(starts, s0 + a.kb_total - 1, G);
          for (int ob = o0; ob <= o1; ob += kFinOwners) {
            float v[kFinOwners][kRows];
            bool use[kFinOwners];
#pragma unroll
            for (int k = 0; k < kFinOwners; ++k) use[k] = ob + k <= o1 && unit_range_nonempty(starts, ob + k);
#pragma unroll
            for (int k = 0; k < kFinOwners; ++k)
#pragma unroll
              for (int j = 0; j < kRows; ++j)
                v[k][j] = use[k] ? ld_cg_f32(&a.partials[static_cast<size_t>(ob + k + tc2) * kBM + lane + 32 * j])
                                 : 0.f;
#pragma unroll
            for (int k = 0; k < kFinOwners; ++k)
#pragma unroll
              for (int j = 0; j < kRows; ++j)
                if (use[k]) total[j] += v[k][j];
          }
        }
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
          const int row2 = x.mt * kBM + lane + 32 * j;
          if (row2 < a.d_out) a.n_out[row2] = a.squared ? total[j] : sqrtf(fmaxf(total[j], 0.f));
        }
        if (lane == 0) a.counters[x.mt] = 0;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, a.tmem_cols);
}

// ============================================================== self-test
// One warp waits, bounded by `limit` cycles, on an mbarrier phase that nothing
// completes, and takes the same exit as every other bounded wait here: the
// timeout status is recorded and the kernel returns.  Exercises the failure
// path (status word, host read-back, context still usable) without a fault.
__global__ void timeout_probe_kernel(long long limit, int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (!mbar_wait_warp(&bar, 0, limit) && threadIdx.x == 0) record_timeout(status, &abort_flag);
}

// ===================================================================== Gram
struct GramArgs {
  int r, kb_main, splits, n_tiles;
  // 1: the first product is symmetric (A A^T) and only its tiles on or above
  // the diagonal are computed, row-major over the upper triangle
  int upper;
  long long wait_limit;
  float* partial;  // [splits][tiles][128][128] fp32; tiles = n_tiles^2, or n_tiles (n_tiles + 1) / 2 when upper
  int* status;
  // optional second product of the same r x r shape in the same launch:
  // CTAs from n_ctas1 on compute it from the second pair of maps
  int n_ctas1;     // CTAs of the first product (= the grid when there is no second)
  int kb_main2, splits2;
  float* partial2;
};

constexpr int kGramKPerStage = 2;  // K blocks per ring stage: 4 boxes, one per producer lane
constexpr int kGramStages = 3;
constexpr uint32_t kGramStageBytes = 2 * kGramKPerStage * kBoxBytes;

__global__ void __launch_bounds__(kNormThreads, 1)
    gram_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2, const GramArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base_s - raw_s);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGramStages * kGramStageBytes);
  uint64_t* empty = full + kGramStages;
  uint64_t* tmem_full = empty + kGramStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tmem_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long limit = a.wait_limit;

  // which product, then (tile, K split) of this CTA; every tile of the
  // n_tiles x n_tiles grid is computed so the reduction reads each output
  // element contiguously
  const bool second = static_cast<int>(blockIdx.x) >= a.n_ctas1;
  const int bid = second ? static_cast<int>(blockIdx.x) - a.n_ctas1 : static_cast<int>(blockIdx.x);
  const int splits = second ? a.splits2 : a.splits;
  const int kb_main = second ? a.kb_main2 : a.kb_main;
  float* const partial = second ? a.partial2 : a.partial;
  const CUtensorMap* const mapM = second ? &tmA2 : &tmA;
  const CUtensorMap* const mapN = second ? &tmB2 : &tmB;
  const int split = bid % splits;
  const int tile = bid / splits;
  const bool upper = a.upper && !second;
  const int n_stored = upper ? a.n_tiles * (a.n_tiles + 1) / 2 : a.n_tiles * a.n_tiles;
  int mi = tile / a.n_tiles;
  int ni = tile % a.n_tiles;
  if (upper) {
    int t = tile;
    mi = 0;
    while (t >= a.n_tiles - mi) {
      t -= a.n_tiles - mi;
      ++mi;
    }
    ni = mi + t;
  }
  // a tile on the diagonal of A A^T has the same rows on both sides: one box per K block
  const bool same = upper && mi == ni;
  const int n_this = min(kBoxRows, a.r - ni * kBoxRows);
  const int kb_lo = static_cast<int>(static_cast<long long>(split) * kb_main / splits);
  const int kb_hi = static_cast<int>(static_cast<long long>(split + 1) * kb_main / splits);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGramStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(mapM);
    tma_prefetch_desc(mapN);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_launch();  // the reduction kernel may be scheduled now; it waits for us

  if (warp == 0) {
    // lane 2i loads the M-side rows, lane 2i+1 the N-side rows, of K block kb0 + i
    int stage = 0;
    uint32_t phase = 0;
    uint32_t parity_bits = 0, filled_mask = 0;
    for (int kb0 = kb_lo; kb0 < kb_hi; kb0 += kGramKPerStage) {
      const int nk = min(kGramKPerStage, kb_hi - kb0);
      bool got = true;
      if (lane == 0) {
        got = mbar_wait(&empty[stage], phase ^ 1u, limit);
        if (got) mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>((same ? 1 : 2) * nk * kBoxBytes));
        else record_timeout(a.status, abort_flag);
      }
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
      __syncwarp();
      if (lane < 2 * nk && !(same && (lane & 1)))
        tma_load_2d(base_s + stage * kGramStageBytes + lane * kBoxBytes, (lane & 1) ? mapN : mapM, &full[stage],
                    (kb0 + (lane >> 1)) * kBK, ((lane & 1) ? ni : mi) * kBoxRows);
      parity_bits = (parity_bits & ~(1u << stage)) | (phase << stage);
      filled_mask |= 1u << stage;
      if (++stage == kGramStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (lane == 0)
      for (int s2 = 0; s2 < kGramStages; ++s2)
        if ((filled_mask >> s2) & 1u) mbar_wait(&full[s2], (parity_bits >> s2) & 1u, limit);
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t idesc = idesc_bf16_f32(kBM, n_this);
      for (int kb0 = kb_lo; kb0 < kb_hi; kb0 += kGramKPerStage) {
        const int nk = min(kGramKPerStage, kb_hi - kb0);
        if (!mbar_wait(&full[stage], phase, limit)) {
          record_timeout(a.status, abort_flag);
          break;
        }
        tc_fence_after();
        const uint64_t d0 = sw128_kmajor_desc(base_s + stage * kGramStageBytes);
        for (int i = 0; i < nk; ++i)
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            mma_bf16(tmem, d0 + (2 * i) * (kBoxBytes >> 4) + 2 * k, d0 + (2 * i + (same ? 0 : 1)) * (kBoxBytes >> 4) + 2 * k,
                     idesc, (kb0 == kb_lo && i == 0 && k == 0) ? 0u : 1u);
        mma_commit(&empty[stage]);
        if (++stage == kGramStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      mma_commit(tmem_full);
      mbar_wait(tmem_full, 0, limit);
    }
  } else {
    const int q = warp & 3;
    const int row_local = q * 32 + lane;
    const bool ok = mbar_wait_warp(tmem_full, 0, limit);
    if (ok && !__any_sync(0xffffffffu, *abort_flag != 0)) {
      tc_fence_after();
      float* dst = partial + (static_cast<size_t>(split) * n_stored + tile) * (kBoxRows * kBoxRows) +
                   static_cast<size_t>(row_local) * kBoxRows;
      for (int j0 = 0; j0 < n_this; j0 += 32) {
        float acc[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + j0, acc);
        const int nv = min(8, (n_this - j0) >> 2);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          if (v < nv)
            reinterpret_cast<float4*>(dst + j0)[v] =
                make_float4(acc[4 * v], acc[4 * v + 1], acc[4 * v + 2], acc[4 * v + 3]);
      }
    } else if (!ok && lane == 0) {
      record_timeout(a.status, abort_flag);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 128);
}

// Sums the K splits of G = A A^T in fixed order, scales by s/2 and writes the
// bf16 G' the norm kernel's K extension reads; also zeroes the norm kernel's
// tile counters.  With `upper`, the first product's partials hold only the
// tiles on or above the diagonal, and an element below it is read from its
// mirror.  CTAs from `g1` on reduce a second product the same way
// (`partial2`, `splits2`, `scale2`, `Gs2`; a Gram launch of two products).
// 64 registers a thread at most (__launch_bounds__(256, 4)): a CTA of it then
// fits beside a CTA of the norm kernel launched behind it, which can stream
// W while the reduction still runs.
__global__ void __launch_bounds__(256, 4)
    gram_reduce_kernel(const float* __restrict__ partial, int splits, int r, float half_s,
                       __nv_bfloat16* __restrict__ Gs, int* counters, int n_counters, int g1,
                       const float* __restrict__ partial2, int splits2, float scale2,
                       __nv_bfloat16* __restrict__ Gs2, int upper) {
  grid_dep_launch();
  grid_dep_wait();  // the Gram partial tiles are complete
  if (static_cast<int>(blockIdx.x) >= g1) {
    partial = partial2;
    splits = splits2;
    half_s = scale2;
    Gs = Gs2;
    n_counters = 0;
    upper = 0;
  }
  const int bx = static_cast<int>(blockIdx.x) >= g1 ? static_cast<int>(blockIdx.x) - g1 : static_cast<int>(blockIdx.x);
  const int gx = static_cast<int>(blockIdx.x) >= g1 ? static_cast<int>(gridDim.x) - g1 : g1;
  const long long total = static_cast<long long>(r) * r;
  const int nt = (r + kBoxRows - 1) / kBoxRows;
  const long long split_stride =
      static_cast<long long>(upper ? nt * (nt + 1) / 2 : nt * nt) * kBoxRows * kBoxRows;
  // four elements per thread and four splits per round: 16 independent loads
  // in flight; each element still adds its splits in increasing order
  constexpr int kE = 4, kS = 4;
  const long long step = static_cast<long long>(gx) * blockDim.x;
  for (long long base = bx * static_cast<long long>(blockDim.x) + threadIdx.x; base < total;
       base += kE * step) {
    long long src[kE];
    float sum[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) {
      const long long idx = min(base + e * step, total - 1);
      int j = static_cast<int>(idx / r);
      int k = static_cast<int>(idx - static_cast<long long>(j) * r);
      int ti = j / kBoxRows, tk = k / kBoxRows;
      long long tile;
      if (upper) {
        if (ti > tk) {  // below the diagonal: G[j][k] = G[k][j]
          const int t = j;
          j = k;
          k = t;
          const int tt = ti;
          ti = tk;
          tk = tt;
        }
        tile = static_cast<long long>(ti) * nt - static_cast<long long>(ti) * (ti - 1) / 2 + (tk - ti);
      } else {
        tile = static_cast<long long>(ti) * nt + tk;
      }
      src[e] = tile * kBoxRows * kBoxRows + static_cast<long long>(j % kBoxRows) * kBoxRows + (k % kBoxRows);
      sum[e] = 0.f;
    }
    for (int s0 = 0; s0 < splits; s0 += kS) {
      float v[kE][kS];
#pragma unroll
      for (int e = 0; e < kE; ++e)
#pragma unroll
        for (int t = 0; t < kS; ++t) v[e][t] = (s0 + t < splits) ? __ldg(partial + (s0 + t) * split_stride + src[e]) : 0.f;
#pragma unroll
      for (int e = 0; e < kE; ++e)
#pragma unroll
        for (int t = 0; t < kS; ++t) sum[e] += v[e][t];
    }
#pragma unroll
    for (int e = 0; e < kE; ++e)
      if (base + e * step < total) Gs[base + e * step] = __float2bfloat16_rn(half_s * sum[e]);
  }
  const int tid = bx * static_cast<int>(blockDim.x) + static_cast<int>(threadIdx.x);
  if (tid < n_counters) counters[tid] = 0;
}

}  // namespace dora
