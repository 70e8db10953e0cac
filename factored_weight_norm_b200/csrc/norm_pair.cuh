// norm_pair.cuh - bf16 factored row norm on CTA pairs (tcgen05 cta_group::2).
//
// "Scaling DoRA: High-Rank Adaptation via Factored Norms and Fused Kernels",
// Abstract: the squared row norm of W + sBA splits into base, cross and Gram
// terms computable from O(d_out r + r^2) intermediates:
//
//   n_i^2 = ||W_i||^2 + 2s <B_i, U_i> + s^2 B_i G B_i^T,  U = W A^T, G = A A^T.
//
// The Gram term rides along as a K extension of the same contraction,
// V = [W | B] [A | G']^T with G' = (s/2) G (computed by gram_tc_kernel and
// gram_reduce_kernel before this launch), so that
// n_i^2 = ||W_i||^2 + 2s <B_i, V_i>, and W streams from HBM exactly once.
//
// Operand traffic.  The contraction has N = r (a few hundred) and K = d_in, so
// every 64-deep K block of a 128-row W tile needs all r rows of A too: A, not
// W, dominates the bytes moved from L2 into shared memory, and that L2 -> SM
// traffic summed over all SMs is what such a kernel waits on.  Two SMs share
// one 256-row tile here (a cluster of two CTAs, tcgen05.mma.cta_group::2,
// M = 256): each SM loads its own 128 rows of W and HALF of the chunk's rows
// of A per K block, and the pair MMA reads both halves (16 KB + r x 64 B per
// SM and K block instead of 16 KB + r x 128 B: 40 instead of 64 KB at
// r = 384).
//
// The row dot at each segment end needs B_i over the chunk's columns.  With
// the ring streaming, any global load or TMA copy waits microseconds in the
// memory system's queues, so B's rows come through the ring as "B items"
// (ring slots holding 64-column boxes of this CTA's rows of B) placed
// kPnBAhead K blocks before the segment's end; as soon as one lands, the
// epilogue warps copy it into the TMEM columns the accumulator leaves free
// (384..511: B's first 256 columns, packed bf16) and registers (the rest, at
// most 128 columns) and free the slot.  At the segment end nothing is
// fetched.  (Measured: B_i fetched at the segment end cost ~16 us of idle
// tensor cores read from global memory, ~5 us through ring slots; fetched
// with plain loads early in the segment it slowed every ring's start; a
// separate shared-memory buffer for B cost two of five ring stages.)
//
// Roles (352 threads per CTA, the same in both CTAs of a pair):
//   warps 0..3  TMEM epilogue (lane quarter = warp index): fetch the next
//               segment's B_i, then at its end <B_i, V_i>, the segment's
//               ||W_i||^2, one fp32 partial per (row, segment); the last warp
//               to finish a tile's half sums its partials in fixed order and
//               writes n
//   warp 4      MMA issuer (the even CTA's lane 0 issues for the pair)
//   warps 5, 6  ||W_i||^2 from this CTA's W rows of every stage, read once the
//               pair's MMAs on that stage have completed
//   warps 7..10 TMA producers; ring stage s belongs to warp 7 + s % 4, so one
//               warp's copies never queue behind another's
// Barriers: full[s] lives in the even CTA and counts both CTAs' copies; the
// even MMA thread's multicast commit signals done[s] (both CTAs) once the
// MMAs of a K block in stage s have completed, b_landed[s] once a B item in
// stage s has landed; empty[s] (each CTA) takes four arrivals: two from each
// ||W_i||^2 warp for a K block, one from each epilogue warp for a B item.
// Each waiter waits on every phase of the barriers it waits on, in order,
// and releases the slots it waits for (the ||W_i||^2 warps the K blocks, the
// epilogue the B items), so the ring can neither lap it nor let it run ahead:
// a parity wait cannot tell a phase from the one two phases later.
// tmem_full (both CTAs) and tmem_empty (even CTA, eight epilogue warps) hand
// the accumulator over.
// Ranges of (tile, K block) units go to pairs in the order they start (a
// ticket taken from a counter): the Gram clusters launched just before hold
// some SMs for a while, and the pairs that start late get shorter ranges.
// Each pair walks its contiguous range rotated so that the part ending at a
// tile's end (with that tile's extension blocks, which need G') comes last.
// Every wait is bounded.
#pragma once

#include "norm_tc.cuh"

namespace dora {

constexpr int kPnThreads = 352;
constexpr int kPnMmaWarp = 4;
constexpr int kPnW2Warp0 = 5;
constexpr int kPnProdWarp0 = 7;
constexpr int kPnProdWarps = 4;
constexpr int kPnMaxStages = 8;
constexpr int kPnTileRows = 256;                 // rows of W per pair tile
constexpr int kPnMaxChunk = 384;                 // accumulator columns per chunk of r
constexpr int kPnBAhead = 10;                    // K blocks of a segment after its B items
constexpr int kPnBTmemCol = 384;                 // TMEM column of B's packed first 256 columns
constexpr int kPnBTmem = 256;                    // B columns kept in TMEM; the rest of a chunk in registers
constexpr uint32_t kPnWBytes = kBM * 128;        // one CTA's 128 W rows x 64 bf16
// fixed shared memory: alignment slack, barriers (4 per stage + 5), TMEM
// address, abort flag, start rank, the ||W_i||^2 hand-off
constexpr int kPnSmemFixed = 1024 + (4 * kPnMaxStages + 5) * 8 + 16 + kBM * 4;
static_assert(kPnBTmemCol + kPnBTmem / 2 <= 512 && kPnMaxChunk <= kPnBTmemCol, "TMEM columns");
constexpr int kPnTagShift = 24;                  // counter word: (tag << 24) | count

struct PairNormArgs {
  int d_out, d_in, r;
  int n_chunks, chunk_n;   // chunks of <= kPnMaxChunk columns of r (equal widths, zero rows past r)
  int kb_main, kb_total;   // K blocks over d_in; plus the K extension over r
  int pm_tiles, tiles;     // pair M tiles; tiles = pm_tiles * n_chunks
  int units;               // tiles * kb_total
  int early;               // pairs expected to start at once; later ones get w_late
  long long w_early, w_late;  // relative range lengths by start order
  int stages;
  uint32_t stage_bytes;    // per CTA: 16 KB of W-side rows + (h0 + h1) x 128 B
  int h0, h1;              // rows per CTA of the two MMA pieces (N = 2 h0 and 2 h1; h1 = 0: one piece)
  int b_boxes;             // 64-column boxes of B per segment (the chunk's columns)
  int b_per_item;          // B boxes per ring slot
  int b_items;             // B items per segment
  float two_s;
  const __nv_bfloat16* B;  // [d_out, r]
  long long wait_limit;
  unsigned long long tag;  // this call's tag, already shifted by kPnTagShift
  float* partials;         // [(pairs + tiles) * 256]
  unsigned long long* counters;  // [pm_tiles * 2] tagged arrival counts per tile half, then ticket, exit
  float* n_out;
  int* status;
  int squared;
};

// ------------------------------------------------------- tagged counters
// A counter word holds (tag << kPnTagShift) | count; a word with another tag
// (an earlier call, or whatever the workspace held) counts as zero, so the
// counters need no clearing before a launch.
__device__ __forceinline__ int tagged_arrive(unsigned long long* c, unsigned long long tag) {
  unsigned long long v = *reinterpret_cast<volatile unsigned long long*>(c);
  while (true) {
    const int seen = (v >> kPnTagShift) == (tag >> kPnTagShift) ? static_cast<int>(v & ((1ull << kPnTagShift) - 1)) : 0;
    const unsigned long long prev = atomicCAS(c, v, tag | static_cast<unsigned long long>(seen + 1));
    if (prev == v) return seen;
    v = prev;
  }
}

// One arrival under `tag` by a single atomic add (for counters many pairs hit
// at once, where a compare-and-swap loop would serialize them): a word still
// carrying another tag is first reset to count 0 under this one, by a
// compare-and-swap that succeeds only if the word is unchanged.  Returns the
// count before this arrival.
__device__ __forceinline__ int tagged_ticket(unsigned long long* c, unsigned long long tag) {
  const unsigned long long v = *reinterpret_cast<volatile unsigned long long*>(c);
  if ((v >> kPnTagShift) != (tag >> kPnTagShift)) atomicCAS(c, v, tag);
  const unsigned long long old = atomicAdd(c, 1ull);
  return static_cast<int>(old & ((1ull << kPnTagShift) - 1));
}

// The range of start rank c is [pn_start(c), pn_start(c + 1)): lengths in
// proportion to w_early for the first `early` ranks, w_late after.
__device__ __forceinline__ long long pn_cum(const PairNormArgs& a, int c) {
  return a.w_early * min(c, a.early) + a.w_late * max(0, c - a.early);
}
__device__ __forceinline__ int pn_start(const PairNormArgs& a, int c, int P) {
  return static_cast<int>(static_cast<long long>(a.units) * pn_cum(a, c) / pn_cum(a, P));
}
// Start rank whose range holds unit u: the largest c with pn_start(c) <= u.
__device__ __forceinline__ int pn_owner(const PairNormArgs& a, int u, int P) {
  int lo = 0, hi = P - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pn_start(a, mid, P) <= u) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}
__device__ __forceinline__ bool pn_nonempty(const PairNormArgs& a, int c, int P) {
  return pn_start(a, c + 1, P) > pn_start(a, c, P);
}

// A pair's range [m0, m1), walked from its first tile boundary tb on, then
// [m0, tb) (which lies within one tile and ends with that tile's extension
// blocks) last.
struct PnWork {
  int m0, m1, tb, n;
  __device__ __forceinline__ void init(const PairNormArgs& a, int rk, int P) {
    m0 = pn_start(a, rk, P);
    m1 = pn_start(a, rk + 1, P);
    tb = min(m1, (m0 + a.kb_total - 1) / a.kb_total * a.kb_total);
    n = m1 - m0;
  }
  // unit i -> (tile, K block, first and last index of its segment)
  __device__ __forceinline__ void at(const PairNormArgs& a, int i, int& tile, int& kb, int& sf, int& sl) const {
    const int len1 = m1 - tb;
    if (i < len1) {
      const int u = tb + i;
      tile = u / a.kb_total;
      kb = u - tile * a.kb_total;
      sf = i - kb;  // this part starts at a tile boundary
      sl = min(i - kb + a.kb_total - 1, len1 - 1);
    } else {
      const int u = m0 + (i - len1);
      tile = u / a.kb_total;
      kb = u - tile * a.kb_total;
      sf = len1;
      sl = n - 1;
    }
  }
};

// Walks a pair's ring items in order: each segment's K blocks, with its B
// items inserted before the last kPnBAhead of them.  `item` is the item's
// index (ring slot item % S, phase (item / S) & 1); for a B item, b >= 0 and
// i, kb already name the K block that follows it.  The decode (divisions)
// happens only when a segment starts, so the per-item cost of the loops that
// must keep pace with the tensor cores stays a few instructions.
struct PnItems {
  int item, i, sf, sl, tile, kb, seg, b, cut;
  __device__ __forceinline__ void enter(const PairNormArgs& a, const PnWork& w) {
    w.at(a, i, tile, kb, sf, sl);
    cut = max(sf, sl - kPnBAhead + 1);
    b = (i == cut && a.b_items > 0) ? 0 : -1;
  }
  __device__ __forceinline__ void start(const PairNormArgs& a, const PnWork& w) {
    item = i = seg = 0;
    b = -1;
    if (w.n > 0) enter(a, w);
  }
  __device__ __forceinline__ bool valid(const PnWork& w) const { return i < w.n; }
  __device__ __forceinline__ void next(const PairNormArgs& a, const PnWork& w) {
    ++item;
    if (b >= 0) {
      if (++b == a.b_items) b = -1;
      return;
    }
    if (i == sl) {
      ++seg;
      if (++i < w.n) enter(a, w);
      return;
    }
    ++i;
    ++kb;
    if (i == cut && a.b_items > 0) b = 0;
  }
};

__global__ void __launch_bounds__(kPnThreads, 1)
    norm_pair_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                     const __grid_constant__ CUtensorMap tmG0, const __grid_constant__ CUtensorMap tmG1,
                     const PairNormArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base_s - raw_s);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.stages * a.stage_bytes);
  uint64_t* done = full + kPnMaxStages;
  uint64_t* empty = done + kPnMaxStages;
  uint64_t* b_landed = empty + kPnMaxStages;
  uint64_t* tmem_full = b_landed + kPnMaxStages;
  uint64_t* tmem_empty = tmem_full + 1;
  uint64_t* drain = tmem_empty + 1;
  uint64_t* w2_full = drain + 1;
  uint64_t* w2_empty = w2_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(w2_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* rank_slot = const_cast<int*>(reinterpret_cast<volatile int*>(tmem_slot + 2));
  float* w2 = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(w2_empty + 1) + 16);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int P = static_cast<int>(gridDim.x >> 1);
  const long long limit = a.wait_limit;
  const int S = a.stages;
  const int w_row = static_cast<int>(rank) * kBM;  // this CTA's rows within a pair tile
  unsigned long long* const cnt_ticket = a.counters + 2 * a.pm_tiles;
  unsigned long long* const cnt_exit = cnt_ticket + 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);   // the even producer's arrive; bytes of both CTAs' copies
      mbar_init(&done[s], 1);   // the even MMA thread's multicast commit
      mbar_init(&empty[s], 4);  // two from each ||W_i||^2 warp (a K block) or one per epilogue warp (a B item)
      mbar_init(&b_landed[s], 1);  // the even MMA thread's multicast commit (a B item)
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 8);   // four epilogue warps in each CTA
    mbar_init(drain, 1);
    mbar_init(w2_full, 2);
    mbar_init(w2_empty, 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 0 && leader) *rank_slot = tagged_ticket(cnt_ticket, a.tag);  // this pair's start rank
  if (warp == kPnProdWarp0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmG0);
    tma_prefetch_desc(&tmG1);
  }
  if (warp == kPnMmaWarp) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any copy, commit or arrive reaches them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
  const uint32_t tmem_empty_leader = mapa_shared(smem_u32(tmem_empty), 0);
  // start rank (the pair's range and partial slots): the odd CTA reads the
  // even CTA's copy, only now that the cluster barrier has shown both running
  int cid;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(cid) : "r"(mapa_shared(smem_u32(rank_slot), 0)) : "memory");
  PnWork wk;
  wk.init(a, cid, P);

  if (warp >= kPnProdWarp0) {
    // ------------------------------------------------------------ producers
    const int p = warp - kPnProdWarp0;
    bool gram_ready = false;
    int last_item[kPnMaxStages / kPnProdWarps];  // the last item filled into each of this warp's stages
#pragma unroll
    for (int j = 0; j < kPnMaxStages / kPnProdWarps; ++j) last_item[j] = -1;
    PnItems it;
    for (it.start(a, wk); it.valid(wk); it.next(a, wk)) {
      const int stage = it.item % S;
      if (stage % kPnProdWarps != p) continue;  // warp-uniform
      const uint32_t phase = static_cast<uint32_t>((it.item / S) & 1);
      const int mt = it.tile / a.n_chunks;
      const int c0 = (it.tile - mt * a.n_chunks) * a.chunk_n;
      const bool ext = it.b < 0 && it.kb >= a.kb_main;
      if (ext && !gram_ready) {
        grid_dep_wait();          // G' is written by the Gram kernel
        fence_proxy_async_all();  // ... through the generic proxy; TMA reads it
        gram_ready = true;
      }
      const int nb = it.b < 0 ? 0 : min(a.b_per_item, a.b_boxes - it.b * a.b_per_item);
      const uint32_t bytes = it.b < 0 ? a.stage_bytes : static_cast<uint32_t>(nb) * kBoxBytes;
      bool got = true;
      if (lane == 0) {
        got = mbar_wait(&empty[stage], phase ^ 1u, limit);
        if (got && leader) mbar_arrive_expect_tx(&full[stage], 2u * bytes);
        if (!got) record_timeout(a.status, abort_flag);
      }
      got = __shfl_sync(0xffffffffu, got, 0);
      __syncwarp();
      if (!got) break;
      const uint32_t dst = base_s + static_cast<uint32_t>(stage) * a.stage_bytes;
      const uint32_t bar = full_leader + static_cast<uint32_t>(stage) * 8u;
      if (it.b >= 0) {
        // B item: this CTA's rows of B, boxes b * per_item .. of the chunk
        if (lane < nb)
          tma_load_2d_pair(dst + lane * kBoxBytes, &tmB, bar, c0 + (it.b * a.b_per_item + lane) * kBK,
                           mt * kPnTileRows + w_row);
      } else {
        const int xk = (ext ? it.kb - a.kb_main : it.kb) * kBK;
        if (lane == 0) {
          tma_load_2d_pair(dst, ext ? &tmB : &tmW, bar, xk, mt * kPnTileRows + w_row);
        } else if (lane == 1) {
          tma_load_2d_pair(dst + kPnWBytes, ext ? &tmG0 : &tmA0, bar, xk, c0 + static_cast<int>(rank) * a.h0);
        } else if (lane == 2 && a.h1 > 0) {
          tma_load_2d_pair(dst + kPnWBytes + a.h0 * 128, ext ? &tmG1 : &tmA1, bar, xk,
                           c0 + 2 * a.h0 + static_cast<int>(rank) * a.h1);
        }
      }
      last_item[stage / kPnProdWarps] = it.item;
    }
    // never leave a copy in flight: the even CTA waits for the last fill of
    // each stage this warp owns (its full barrier counts both CTAs' bytes;
    // the odd CTA's copies are also covered by the cluster barrier at the end)
    if (lane == 0 && leader) {
#pragma unroll
      for (int j = 0; j < kPnMaxStages / kPnProdWarps; ++j)
        if (last_item[j] >= 0)
          mbar_wait(&full[last_item[j] % S], static_cast<uint32_t>((last_item[j] / S) & 1), limit);
    }
  } else if (warp == kPnMmaWarp) {
    // ---------------------------------------------- MMA issuer (even CTA)
    if (leader && lane == 0) {
      const uint32_t idesc0 = idesc_bf16_f32(kPnTileRows, 2 * a.h0);
      const uint32_t idesc1 = a.h1 > 0 ? idesc_bf16_f32(kPnTileRows, 2 * a.h1) : 0u;
      const uint64_t desc0 = sw128_kmajor_desc(base_s);
      const uint64_t step = a.stage_bytes >> 4;
      const uint64_t off0 = kPnWBytes >> 4;
      const uint64_t off1 = (kPnWBytes + a.h0 * 128) >> 4;
      int stage = 0;
      uint32_t phase = 0;
      PnItems it;
      for (it.start(a, wk); it.valid(wk); it.next(a, wk)) {
        const bool unit = it.b < 0;
        const bool seg_first = unit && it.i == it.sf;
        if (seg_first && it.seg > 0) {
          if (!mbar_wait(tmem_empty, static_cast<uint32_t>((it.seg - 1) & 1), limit)) {
            record_timeout(a.status, abort_flag);
            break;
          }
          tc_fence_after();
        }
        if (!mbar_wait(&full[stage], phase, limit)) {
          record_timeout(a.status, abort_flag);
          break;
        }
        if (unit) {
          tc_fence_after();
          const uint64_t ad = desc0 + static_cast<uint64_t>(stage) * step;
          if (idesc1) {
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k) {
              const uint32_t acc = (seg_first && k == 0) ? 0u : 1u;
              mma_bf16_pair(tmem, ad + 2 * k, ad + off0 + 2 * k, idesc0, acc);
              mma_bf16_pair(tmem + 256, ad + 2 * k, ad + off1 + 2 * k, idesc1, acc);
            }
          } else {
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
              mma_bf16_pair(tmem, ad + 2 * k, ad + off0 + 2 * k, idesc0, (seg_first && k == 0) ? 0u : 1u);
          }
        }
        // a K block: its MMAs have completed; a B item: its copies have landed
        mma_commit_pair(unit ? &done[stage] : &b_landed[stage], 0x3);
        if (unit && it.i == it.sl) mma_commit_pair(tmem_full, 0x3);
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      mma_commit_pair(drain, 0x1);
      mbar_wait(drain, 0, limit);
    }
  } else if (warp >= kPnW2Warp0) {
    // ------------------------------------------------------ ||W_i||^2 warps
    // Warp 5 sums rows 0..63 of this CTA's W rows, warp 6 rows 64..127 (lane
    // l: rows l and l + 32 of its half).  The chunk order does not matter for
    // the sum; visiting chunk (j ^ row % 8) keeps a quarter-warp's eight rows
    // on distinct banks.  These warps release every slot.
    const int r0 = (warp - kPnW2Warp0) * 64 + lane;
    int stage = 0;
    uint32_t uphase = 0;  // bit s: parity of the next K-block use of stage s
    float acc0 = 0.f, acc1 = 0.f;
    PnItems it;
    for (it.start(a, wk); it.valid(wk); it.next(a, wk)) {
      if (it.b >= 0) {  // a B item: the epilogue's
        if (++stage == S) stage = 0;
        continue;
      }
      if (__any_sync(0xffffffffu, !mbar_wait(&done[stage], (uphase >> stage) & 1u, limit))) {
        if (lane == 0) record_timeout(a.status, abort_flag);
        break;
      }
      uphase ^= 1u << stage;
      if (it.kb < a.kb_main && it.tile % a.n_chunks == 0) {
        const uint8_t* t = smem + stage * a.stage_bytes;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          acc0 += sumsq_bf16x8(*reinterpret_cast<const uint4*>(t + sw128_chunk(r0, j)));
          acc1 += sumsq_bf16x8(*reinterpret_cast<const uint4*>(t + sw128_chunk(r0 + 32, j)));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_cnt(&empty[stage], 2);
      if (++stage == S) stage = 0;
      if (it.i != it.sl) continue;
      // the segment's ||W_i||^2 to the epilogue
      if (it.seg > 0 && !mbar_wait_warp(w2_empty, static_cast<uint32_t>((it.seg - 1) & 1), limit)) {
        if (lane == 0) record_timeout(a.status, abort_flag);
        break;
      }
      w2[r0] = acc0;
      w2[r0 + 32] = acc1;
      acc0 = acc1 = 0.f;
      __threadfence_block();
      __syncwarp();
      if (lane == 0) mbar_arrive(w2_full);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp;  // TMEM lane quarter
    const int row_local = q * 32 + lane;
    const uint32_t tmem_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
    int stage = 0;
    uint32_t bphase = 0;  // bit s: parity of the next B-item use of stage s
    uint4 breg[(kPnMaxChunk - kPnBTmem) / 8];  // B_i's columns past kPnBTmem
#pragma unroll
    for (int j = 0; j < (kPnMaxChunk - kPnBTmem) / 8; ++j) breg[j] = make_uint4(0, 0, 0, 0);
    PnItems it;
    for (it.start(a, wk); it.valid(wk); it.next(a, wk)) {
      const int cur_stage = stage;
      if (++stage == S) stage = 0;
      if (it.b >= 0) {
        // ---- a B item: copy its boxes (this row's 64 columns each) out of
        // the slot, into TMEM or registers, and free the slot
        if (!mbar_wait_warp(&b_landed[cur_stage], (bphase >> cur_stage) & 1u, limit)) {
          if (lane == 0) record_timeout(a.status, abort_flag);
          break;
        }
        bphase ^= 1u << cur_stage;
        const uint8_t* slot = smem + cur_stage * a.stage_bytes;
        const int box0 = it.b * a.b_per_item;
#pragma unroll
        for (int bx = 0; bx < kPnMaxChunk / 64; ++bx) {
          if (bx < box0 || bx >= box0 + a.b_per_item || bx >= a.b_boxes) continue;  // warp-uniform
          const uint8_t* box = slot + (bx - box0) * kBoxBytes;
          uint4 t[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) t[j] = *reinterpret_cast<const uint4*>(box + sw128_chunk(row_local, j));
          if (bx * 64 < kPnBTmem) {
            uint32_t w[32];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              w[4 * j] = t[j].x;
              w[4 * j + 1] = t[j].y;
              w[4 * j + 2] = t[j].z;
              w[4 * j + 3] = t[j].w;
            }
            tmem_st32(tmem_lane + kPnBTmemCol + 32 * bx, w);
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) breg[(bx * 64 - kPnBTmem) / 8 + j] = t[j];
          }
        }
        tmem_st_wait();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[cur_stage]);  // one of the slot's four releases
        continue;
      }
      if (it.i != it.sl) continue;
      const int tile = it.tile;
      const int seg = it.seg;
      const int mt = tile / a.n_chunks;
      const int c0 = (tile - mt * a.n_chunks) * a.chunk_n;
      const int n_valid = min(a.chunk_n, a.r - c0);

      // ---- <B_i, V_i> over the chunk's columns, 64 at a time
      if (!mbar_wait_warp(tmem_full, static_cast<uint32_t>(seg & 1), limit)) {
        if (lane == 0) record_timeout(a.status, abort_flag);
        break;
      }
      tc_fence_after();
      float dot = 0.f;
#pragma unroll
      for (int b = 0; b < kPnMaxChunk / 64; ++b) {
        if (b * 64 < a.chunk_n) {  // warp-uniform
          uint4 bv[8];  // B_i's 64 columns of this block, 8 per vector
          if (b * 64 < kPnBTmem) {
            float wf[32];
            tmem_ld32(tmem_lane + kPnBTmemCol + 32 * b, wf);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              bv[j] = make_uint4(__float_as_uint(wf[4 * j]), __float_as_uint(wf[4 * j + 1]), __float_as_uint(wf[4 * j + 2]),
                                 __float_as_uint(wf[4 * j + 3]));
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) bv[j] = breg[(b * 64 - kPnBTmem) / 8 + j];
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float v[32];
            tmem_ld32(tmem_lane + static_cast<uint32_t>(b * 64 + 32 * h), v);
            // columns past the chunk's valid width hold no product of this
            // segment: never let them into the sum
#pragma unroll
            for (int j = 0; j < 4; ++j)
              if (b * 64 + 32 * h + 8 * j < n_valid) dot += dot_bf16x8(bv[4 * h + j], v + 8 * j);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tmem_empty_leader);

      // ---- this segment's ||W_i||^2
      if (!mbar_wait_warp(w2_full, static_cast<uint32_t>(seg & 1), limit)) {
        if (lane == 0) record_timeout(a.status, abort_flag);
        break;
      }
      const float base_acc = w2[row_local];
      __syncwarp();
      if (lane == 0) mbar_arrive(w2_empty);
      const float partial = base_acc + a.two_s * dot;
      a.partials[static_cast<size_t>(cid + tile) * kPnTileRows + rank * kBM + row_local] = partial;

      // ---- the last of this half-tile's epilogue warps finishes its 128 rows
      __threadfence();
      __syncwarp();
      int expected = 0;
      for (int c2 = 0; c2 < a.n_chunks; ++c2) {
        const int s0 = (mt * a.n_chunks + c2) * a.kb_total;
        const int o1 = pn_owner(a, s0 + a.kb_total - 1, P);
        for (int o = pn_owner(a, s0, P); o <= o1; ++o) expected += pn_nonempty(a, o, P) ? 1 : 0;
      }
      int last = 0;
      unsigned long long* cnt = a.counters + mt * 2 + static_cast<int>(rank);
      if (lane == 0) last = tagged_arrive(cnt, a.tag) == 4 * expected - 1;
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        __threadfence();
        constexpr int kRows = kBM / 32;  // lane l: rows l, l + 32, l + 64, l + 96 of the half
        float total[kRows];
#pragma unroll
        for (int j = 0; j < kRows; ++j) total[j] = 0.f;
        for (int c2 = 0; c2 < a.n_chunks; ++c2) {
          const int tc2 = mt * a.n_chunks + c2;
          const int s0 = tc2 * a.kb_total;
          const int o0 = pn_owner(a, s0, P);
          const int o1 = pn_owner(a, s0 + a.kb_total - 1, P);
          for (int ob = o0; ob <= o1; ob += kFinOwners) {
            float vv[kFinOwners][kRows];
            bool use[kFinOwners];
#pragma unroll
            for (int k = 0; k < kFinOwners; ++k) use[k] = ob + k <= o1 && pn_nonempty(a, ob + k, P);
#pragma unroll
            for (int k = 0; k < kFinOwners; ++k)
#pragma unroll
              for (int j = 0; j < kRows; ++j)
                vv[k][j] = use[k] ? ld_cg_f32(&a.partials[static_cast<size_t>(ob + k + tc2) * kPnTileRows +
                                                          rank * kBM + lane + 32 * j])
                                  : 0.f;
#pragma unroll
            for (int k = 0; k < kFinOwners; ++k)
#pragma unroll
              for (int j = 0; j < kRows; ++j)
                if (use[k]) total[j] += vv[k][j];
          }
        }
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
          const int row2 = mt * kPnTileRows + static_cast<int>(rank) * kBM + lane + 32 * j;
          if (row2 < a.d_out) a.n_out[row2] = a.squared ? total[j] : sqrtf(fmaxf(total[j], 0.f));
        }
        if (lane == 0) *cnt = a.tag;  // count 0 under this call's tag (a graph replay starts clean)
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA frees TMEM or exits while the pair still uses it
  tc_fence_after();
  if (warp == kPnMmaWarp) tmem_dealloc_pair(tmem, 512);
  // the last pair to leave sets the ticket back to zero under this call's tag
  // (a replay of the same launch in a CUDA graph starts clean)
  if (threadIdx.x == 0 && leader && tagged_ticket(cnt_exit, a.tag) == P - 1) {
    *cnt_ticket = a.tag;
    *cnt_exit = a.tag;
  }
}

}  // namespace dora
