// norm_batched.cuh - factored row norms of many adapted modules in two launches.
//
// "Scaling DoRA: High-Rank Adaptation via Factored Norms and Fused Kernels",
// Abstract: a model carries hundreds of adapted modules, each needing
//   n_i^2 = ||W_i||^2 + 2s <B_i, U_i> + s^2 B_i G B_i^T   (U = W A^T, G = A A^T)
// every step.  Computed one module at a time, small modules leave the GPU idle
// between launches.  Here every module with bf16 weights and 16 <= r <= 512
// (so that its N = r fits one TMEM chunk) is handled by two launches:
//   gram_batched_kernel  one CTA per (module, 128 x 128 tile of G): the tile
//                        over all of d_in, written as bf16 (s/2) G;
//   norm_batched_kernel  a persistent grid over a work list of (module,
//                        128-row M tile) items, sorted longest first and dealt
//                        round-robin; an item is the whole K range of its tile
//                        (d_in blocks of W A^T, then the K-extension blocks of
//                        B (s/2) G), so every row's norm is finished by one
//                        CTA: no partials, no counters.
// The per-unit machinery (TMA ring, tcgen05 MMAs into TMEM, epilogue reading
// W for ||W_i||^2 and B for <B_i, V_i>) is that of norm_tc_kernel before its
// ||W_i||^2 reads moved to warps of their own; here that move measured no
// faster (2.89-2.94 ms for 112 modules either way), so the four epilogue
// warps keep reading every W stage.
#pragma once

#include "norm_tc.cuh"

namespace dora {

// One module, as the kernels see it (in device memory, written by the host).
struct alignas(64) BatchDesc {
  CUtensorMap tmW, tmA, tmB, tmG;  // W [d_out, d_in], A [r, d_in], B [d_out, r], G' [r, r]
  float* n_out;                     // [d_out]
  __nv_bfloat16* gs;                // G' = (s/2) G, [r, r]
  int d_out, d_in, r, kb_main, kb_total;
  float two_s, half_s;
};

// (module, tile) of a work list entry
struct BatchItem {
  int prob, tile;
};

// ---------------------------------------------------------------- Gram
// G tile (mi, ni) of module `prob` over all of d_in, scaled by s/2 and
// written as bf16.  Ring and roles as in gram_tc_kernel.
__global__ void __launch_bounds__(kNormThreads, 1)
    gram_batched_kernel(const BatchDesc* __restrict__ probs, const BatchItem* __restrict__ items, long long limit,
                        int* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + (base_s - raw_s) + kGramStages * kGramStageBytes);
  uint64_t* empty = full + kGramStages;
  uint64_t* tmem_full = empty + kGramStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tmem_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const BatchItem it = items[blockIdx.x];
  const BatchDesc* d = probs + it.prob;
  const int r = d->r;
  const int nt = (r + kBoxRows - 1) / kBoxRows;
  const int mi = it.tile / nt;
  const int ni = it.tile - mi * nt;
  const int n_this = min(kBoxRows, r - ni * kBoxRows);
  const int kb_end = d->kb_main;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGramStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tensormap_acquire(&d->tmA);  // the table was written by a copy before this launch
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_launch();  // the norm kernel may be scheduled now; it waits for us before reading G'

  if (warp == 0) {
    // lane 2i loads the M-side rows, lane 2i+1 the N-side rows, of K block kb0 + i
    int stage = 0;
    uint32_t phase = 0;
    uint32_t parity_bits = 0, filled_mask = 0;
    for (int kb0 = 0; kb0 < kb_end; kb0 += kGramKPerStage) {
      const int nk = min(kGramKPerStage, kb_end - kb0);
      bool got = true;
      if (lane == 0) {
        got = mbar_wait(&empty[stage], phase ^ 1u, limit);
        if (got) mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(2 * nk * kBoxBytes));
        else record_timeout(status, abort_flag);
      }
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
      __syncwarp();
      if (lane < 2 * nk)
        tma_load_2d(base_s + stage * kGramStageBytes + lane * kBoxBytes, &d->tmA, &full[stage],
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
      for (int kb0 = 0; kb0 < kb_end; kb0 += kGramKPerStage) {
        const int nk = min(kGramKPerStage, kb_end - kb0);
        if (!mbar_wait(&full[stage], phase, limit)) {
          record_timeout(status, abort_flag);
          break;
        }
        tc_fence_after();
        const uint64_t d0 = sw128_kmajor_desc(base_s + stage * kGramStageBytes);
        for (int i = 0; i < nk; ++i)
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            mma_bf16(tmem, d0 + (2 * i) * (kBoxBytes >> 4) + 2 * k, d0 + (2 * i + 1) * (kBoxBytes >> 4) + 2 * k, idesc,
                     (kb0 == 0 && i == 0 && k == 0) ? 0u : 1u);
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
    // row mi*128 + q*32 + lane of G, columns ni*128 .. + n_this, as bf16 (s/2) G
    const int q = warp & 3;
    const int row = mi * kBoxRows + q * 32 + lane;
    const bool ok = mbar_wait_warp(tmem_full, 0, limit);
    if (ok && !__any_sync(0xffffffffu, *abort_flag != 0)) {
      tc_fence_after();
      for (int j0 = 0; j0 < n_this; j0 += 32) {
        float acc[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + j0, acc);
        if (row < r) {
          __nv_bfloat16* dst = d->gs + static_cast<size_t>(row) * r + ni * kBoxRows + j0;
          const int nv = min(32, n_this - j0);  // a multiple of 16
#pragma unroll
          for (int v = 0; v < 32; v += 8) {
            if (v >= nv) break;
            uint4 pk;
            pk.x = pack_bf16x2(d->half_s * acc[v], d->half_s * acc[v + 1]);
            pk.y = pack_bf16x2(d->half_s * acc[v + 2], d->half_s * acc[v + 3]);
            pk.z = pack_bf16x2(d->half_s * acc[v + 4], d->half_s * acc[v + 5]);
            pk.w = pack_bf16x2(d->half_s * acc[v + 6], d->half_s * acc[v + 7]);
            *reinterpret_cast<uint4*>(dst + v) = pk;
          }
        }
      }
    } else if (!ok && lane == 0) {
      record_timeout(status, abort_flag);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 128);
}

// ---------------------------------------------------------------- norm
struct BatchNormArgs {
  int n_items;
  int stages;
  uint32_t stage_bytes;  // the largest module's W-side tile + N-side tiles
  long long wait_limit;
  int* status;
};

// Walks this CTA's items (blockIdx.x, blockIdx.x + gridDim.x, ...) and the K
// blocks of each; loads a module's fields when its item starts.
struct BatchIter {
  int item, kb, kb_main, kb_total, n_this, m0;
  const BatchDesc* d;
  __device__ __forceinline__ void load(const BatchDesc* probs, const BatchItem* items) {
    const BatchItem it = items[item];
    d = probs + it.prob;
    kb = 0;
    kb_main = d->kb_main;
    kb_total = d->kb_total;
    n_this = d->r;
    m0 = it.tile * kBM;
  }
  __device__ __forceinline__ bool last_unit() const { return kb == kb_total - 1; }
};

__global__ void __launch_bounds__(kNormThreads, 1)
    norm_batched_kernel(const BatchDesc* __restrict__ probs, const BatchItem* __restrict__ items, const BatchNormArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base_s - raw_s);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.stages * a.stage_bytes);
  uint64_t* empty = full + a.stages;
  uint64_t* tmem_full = empty + a.stages;
  uint64_t* tmem_empty = tmem_full + 1;
  uint64_t* drain = tmem_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long limit = a.wait_limit;
  const int slots = static_cast<int>(a.stage_bytes / kBoxBytes);

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 4);  // MMA warp + one arrive per epilogue warp
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 4);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t parity_bits = 0, filled_mask = 0;
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
    BatchIter x;
    for (x.item = blockIdx.x; x.item < a.n_items && ok; x.item += gridDim.x) {
      x.load(probs, items);
      // the table was written by a copy before this launch
      tensormap_acquire(&x.d->tmW);
      tensormap_acquire(&x.d->tmA);
      tensormap_acquire(&x.d->tmB);
      tensormap_acquire(&x.d->tmG);
      const int nboxes = (x.n_this + kBoxRows - 1) / kBoxRows;
      {
        // B's rows for the item's epilogue: into L2 now
        const int nbox = (x.n_this + kBK - 1) / kBK;
        for (int b = lane; b < nbox; b += 32) tma_prefetch_l2_2d(&x.d->tmB, b * kBK, x.m0);
      }
      for (; x.kb < x.kb_total; ++x.kb) {
        const bool ext = x.kb >= x.kb_main;
        if (ext && !gram_ready) {
          grid_dep_wait();  // G' is written by gram_batched_kernel
          gram_ready = true;
        }
        if (!(ok = acquire(static_cast<uint32_t>(kBoxBytes * (1 + nboxes))))) break;
        if (lane <= nboxes) {
          const CUtensorMap* map = lane == 0 ? (ext ? &x.d->tmB : &x.d->tmW) : (ext ? &x.d->tmG : &x.d->tmA);
          const int xk = (ext ? x.kb - x.kb_main : x.kb) * kBK;
          const int y = lane == 0 ? x.m0 : (lane - 1) * kBoxRows;
          tma_load_2d(base_s + stage * a.stage_bytes + lane * kBoxBytes, map, &full[stage], xk, y);
        }
        advance();
      }
      if (!ok) break;
      // B[item rows, all r columns] for the epilogue, 64 columns per box
      const int nbox = (x.n_this + kBK - 1) / kBK;
      for (int b0 = 0; b0 < nbox; b0 += slots) {
        const int nb = min(slots, nbox - b0);
        if (!(ok = acquire(static_cast<uint32_t>(kBoxBytes * nb)))) break;
        if (lane < nb)
          tma_load_2d(base_s + stage * a.stage_bytes + lane * kBoxBytes, &x.d->tmB, &full[stage], (b0 + lane) * kBK,
                      x.m0);
        advance();
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
      int done_items = 0;
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
      BatchIter x;
      for (x.item = blockIdx.x; x.item < a.n_items && ok; x.item += gridDim.x) {
        x.load(probs, items);
        const uint32_t idesc0 = idesc_bf16_f32(kBM, min(256, x.n_this));
        const uint32_t idesc1 = x.n_this > 256 ? idesc_bf16_f32(kBM, x.n_this - 256) : 0u;
        if (done_items > 0) {  // the epilogue has drained the previous item's accumulator
          if (!mbar_wait(tmem_empty, static_cast<uint32_t>((done_items - 1) & 1), limit)) {
            fail();
            break;
          }
          tc_fence_after();
        }
        for (; x.kb < x.kb_total; ++x.kb) {
          if (!mbar_wait(&full[stage], phase, limit)) {
            fail();
            break;
          }
          tc_fence_after();
          const uint64_t adesc = desc0 + static_cast<uint64_t>(stage) * desc_step;
          const uint64_t bdesc = adesc + (kBoxBytes >> 4);
          const uint32_t acc0 = x.kb == 0 ? 0u : 1u;
          if (idesc1) {
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k) {
              const uint32_t acc = k == 0 ? acc0 : 1u;
              mma_bf16(tmem, adesc + 2 * k, bdesc + 2 * k, idesc0, acc);
              mma_bf16(tmem + 256, adesc + 2 * k, bdesc + (256 * 128 >> 4) + 2 * k, idesc1, acc);
            }
          } else {
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
              mma_bf16(tmem, adesc + 2 * k, bdesc + 2 * k, idesc0, k == 0 ? acc0 : 1u);
          }
          mma_commit(&empty[stage]);
          advance();
        }
        if (!ok) break;
        mma_commit(tmem_full);
        ++done_items;
        // the B stages feed the epilogue only: release them on arrival
        const int nbst = ((x.n_this + kBK - 1) / kBK + slots - 1) / slots;
        for (int i = 0; i < nbst; ++i) {
          if (!mbar_wait(&full[stage], phase, limit)) {
            fail();
            break;
          }
          mbar_arrive(&empty[stage]);
          advance();
        }
      }
      mma_commit(drain);
      mbar_wait(drain, 0, limit);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row_local = q * 32 + lane;
    const uint32_t tmem_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
    int stage = 0;
    uint32_t phase = 0;
    int done_items = 0;
    bool ok = true;
    auto release = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (++stage == a.stages) {
        stage = 0;
        phase ^= 1u;
      }
    };
    BatchIter x;
    for (x.item = blockIdx.x; x.item < a.n_items && ok; x.item += gridDim.x) {
      x.load(probs, items);
      float base_acc = 0.f;
      for (; x.kb < x.kb_total; ++x.kb) {
        if (__any_sync(0xffffffffu, !mbar_wait(&full[stage], phase, limit))) {
          if (lane == 0) record_timeout(a.status, abort_flag);
          ok = false;
          break;
        }
        if (x.kb < x.kb_main) {
          // ||W_i||^2 from the swizzled W stage (chunk j ^ row % 8: distinct banks)
          const uint8_t* tile = smem + stage * a.stage_bytes;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            base_acc += sumsq_bf16x8(*reinterpret_cast<const uint4*>(tile + sw128_chunk(row_local, j)));
        }
        release();
      }
      if (!ok) break;
      if (!mbar_wait_warp(tmem_full, static_cast<uint32_t>(done_items & 1), limit)) {
        if (lane == 0) record_timeout(a.status, abort_flag);
        break;
      }
      tc_fence_after();
      float dot = 0.f;
      const int nbox = (x.n_this + kBK - 1) / kBK;
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
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int j0 = (b0 + b) * kBK + h * 32;
            if (j0 >= x.n_this) break;
            float acc[32];
            tmem_ld32(tmem_lane + j0, acc);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              if (j0 + 8 * v < x.n_this)  // TMEM columns past r hold stale values
                dot += dot_bf16x8(*reinterpret_cast<const uint4*>(tile + sw128_chunk(row_local, h * 4 + v)),
                                  acc + 8 * v);
          }
        }
        release();
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tmem_empty);
      ++done_items;
      const int row = x.m0 + row_local;
      if (row < x.d->d_out) x.d->n_out[row] = sqrtf(fmaxf(base_acc + x.d->two_s * dot, 0.f));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace dora
