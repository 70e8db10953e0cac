// linear_tc.cuh - DoRA linear forward with the compose fused into the GEMM
// epilogue, on tcgen05 tensor cores (sm_100a).
//
// "Scaling DoRA: High-Rank Adaptation via Factored Norms and Fused Kernels",
// Abstract: the DoRA composition is fused so that the activations make as few
// trips through memory as possible.  Here the compose moves into the GEMMs
// that produce its inputs:
//
//   y = b + g * ((x W^T) + s * (x A^T) B^T),   g = m / n   (per output column)
//     = b + g * ([x | P] [W | B]^T),           P = s * (x A^T)   [T, r]
//
// so base_out and lora_out never exist in memory.  Two launches of one
// persistent GEMM kernel on CTA pairs:
//   1) P = bf16(s * x A^T)                 (M = T, N = r, K = d_in)
//   2) y = bf16(g * [x | P] [W | B]^T + b) (M = T, N = d_out, K = d_in, then r
//      more K from the extension pair), launched with programmatic dependent
//      launch: its CTAs take SMs as launch 1's leave and wait for P only
//      before their first extension block, which comes last in each tile.
// The product accumulates in fp32 in TMEM and the epilogue applies g and b in
// fp32, with one rounding to bf16: nothing near unity is ever rounded to bf16
// on its own.
//
// A cluster of two CTAs (tcgen05 cta_group::2) owns a 256 x 256 output tile.
// Roles per CTA (192 threads): warp 0 the TMA producer, warp 1 the MMA issuer
// (the even CTA's lane 0 issues the pair MMAs for both), warps 2..5 the
// epilogue (TMEM lane quarter = warp % 4).  Two TMEM accumulators of 256
// columns let the epilogue of one tile overlap the main loop of the next.
// Each ring stage holds two 64-deep K blocks: the MMA issuer's fixed cost per
// stage (barrier wait, fence, commit) is then paid once per 1024 tensor-core
// cycles; measured, one K block per stage ran at 0.83 of the two-block speed
// and three (two stages only) at 0.87.  Tiles are walked in groups of
// kLinGroupM M tiles along N so that the x and W rows in use at once stay in
// L2.  Every wait is bounded.
#pragma once

#include "sm100_ptx.cuh"

namespace dora {

constexpr int kLinThreads = 192;
constexpr int kLinBM = 128;
constexpr int kLinBK = 64;
constexpr int kLinStagesMax = 8;
constexpr int kLinGroupM = 16;
constexpr uint32_t kLinABytes = kLinBM * 128;  // one 128-row x 64-column bf16 box
// full/empty per stage, two acc_full, two acc_empty, drain (8 bytes each), the
// TMEM address slot and the abort flag
constexpr size_t kLinBarrierBytes = (2 * kLinStagesMax + 5) * 8 + 8;
static_assert(kLinBarrierBytes <= 256, "barrier area");

struct LinearArgs {
  int M, N;                // output rows and columns
  int kb_main, kb_total;   // K blocks from the first operand pair; total with the extension pair
  int tiles_m, tiles_n;
  int bn;                  // pair tile width along N: 128, 192 or 256 (each CTA holds bn / 2)
  int stages;             // ring stages of kPairStageBytes
  float alpha;             // uniform scale of the product
  const float* m;          // per-column g = m / n, or null (g = 1)
  const float* n;
  const float* rs_num;     // per-row scale rs_num / rs_den, or null (1)
  const float* rs_den;
  const __nv_bfloat16* bias;  // per-column bias, or null
  void* out;               // [M, ldo] row-major, bf16 or fp32 (kernel template)
  long long ldo;
  int ext_waits;           // 1: the extension operands come from the preceding grid
  long long wait_limit;
  int* status;
};

__device__ __forceinline__ void lin_tile(const LinearArgs& a, int t, int& tm, int& tn) {
  const int per_group = kLinGroupM * a.tiles_n;
  const int g = t / per_group;
  const int first = g * kLinGroupM;
  const int gm = min(kLinGroupM, a.tiles_m - first);
  const int rem = t - g * per_group;
  tm = first + rem % gm;
  tn = rem / gm;
}

__device__ __forceinline__ void lin_timeout(int* status, volatile int* abort_flag) {
  atomicExch(status, 5);  // DORA_ERR_TIMEOUT
  *abort_flag = 1;
}

// ===================================================== CTA-pair version
// The same GEMM on CTA pairs (cluster of 2, tcgen05 cta_group::2): a pair owns
// a 256 x 256 output tile; CTA r of the pair loads rows r*128.. of the A-side
// tile and rows r*128.. of the B-side tile, one pair MMA (M = 256, N = 256)
// reads both CTAs' halves, and CTA r's TMEM receives output rows r*128...  Per
// SM a 64-deep K block is then 32 KB of shared memory for 512 tensor-core
// cycles instead of 48 KB, so more stages fit and each covers more of the
// load latency.
//
// Barriers: full[s] lives in the even CTA and counts both CTAs' bytes (the
// even producer announces them); empty[s] and acc_full[b] live in both CTAs
// and are signalled by the even MMA thread's multicast commit; acc_empty[b]
// lives in the even CTA and counts the eight epilogue warps of the pair.
constexpr int kPairBM = 256;
constexpr int kPairBN = 256;
constexpr int kPairKps = 2;  // 64-deep K blocks per ring stage (one barrier round trip per 1024 MMA cycles)
// per stage: kPairKps boxes of 128 A-side rows, then kPairKps boxes of 128 B-side rows
constexpr uint32_t kPairStageBytes = 2 * kPairKps * kLinABytes;

// B_MN: the B-side operand is stored N-contiguous (its rows run along K), as
// W is for a contraction over d_out; it is loaded as two 64-column boxes per
// K block and read through MN-major descriptors.  OUT_F32: fp32 output.
template <bool B_MN, bool OUT_F32>
__global__ void __launch_bounds__(kLinThreads, 1)
    linear_pair_kernel(const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                       const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                       const LinearArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base_s - raw_s);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.stages * kPairStageBytes);
  uint64_t* empty = full + a.stages;
  uint64_t* acc_full = empty + a.stages;  // [2]
  uint64_t* acc_empty = acc_full + 2;     // [2], the even CTA's are used
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const long long limit = a.wait_limit;
  const int n_tiles = a.tiles_m * a.tiles_n;
  const int half_bn = a.bn / 2;
  // MN-major B: 64-column boxes per K block covering this CTA's bn / 2 columns
  const int mn_boxes = (half_bn + 63) / 64;
  // bytes one CTA's copies bring per stage
  const uint32_t stage_tx =
      kPairKps * (kLinABytes + (B_MN ? static_cast<uint32_t>(mn_boxes) * (kLinABytes / 2) : half_bn * 128u));

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&full[s], 1);   // the even producer's arrive; transaction bytes of both CTAs
      mbar_init(&empty[s], 1);  // the even MMA thread's multicast commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 8);  // four epilogue warps in each CTA of the pair
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB1);
    tma_prefetch_desc(&tmA2);
    tma_prefetch_desc(&tmB2);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 2 * kPairBN);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any copy or arrive reaches them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
  const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
  grid_dep_launch();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t parity_bits = 0;
    uint32_t filled_mask = 0;
    bool ext_ready = a.ext_waits == 0;
    bool ok = true;
    for (int t = cid; t < n_tiles && ok; t += n_pairs) {
      int tm, tn;
      lin_tile(a, t, tm, tn);
      const int ya = tm * kPairBM + static_cast<int>(rank) * kLinBM;
      const int yb = tn * a.bn + static_cast<int>(rank) * (a.bn / 2);
      for (int kb0 = 0; kb0 < a.kb_total; kb0 += kPairKps) {
        // K blocks past kb_total load boxes that lie wholly outside the
        // tensor: zero-filled, they add nothing
        if (kb0 + kPairKps > a.kb_main && !ext_ready) {
          grid_dep_wait();
          fence_proxy_async_all();
          ext_ready = true;
        }
        bool got = true;
        if (lane == 0) {
          got = mbar_wait(&empty[stage], phase ^ 1u, limit);
          if (got && leader) mbar_arrive_expect_tx(&full[stage], 2 * stage_tx);
          if (!got) lin_timeout(a.status, abort_flag);
        }
        got = __shfl_sync(0xffffffffu, got, 0);
        __syncwarp();
        if (!got) {
          ok = false;
          break;
        }
        const uint32_t dst = base_s + stage * kPairStageBytes;
        const uint32_t bar = full_leader + static_cast<uint32_t>(stage) * 8u;
        if (lane < kPairKps) {
          const int kb = kb0 + lane;
          const bool ext = kb >= a.kb_main && a.kb_total > a.kb_main;
          const int xk = (ext ? kb - a.kb_main : kb) * kLinBK;
          tma_load_2d_pair(dst + lane * kLinABytes, ext ? &tmA2 : &tmA1, bar, xk, ya);
        } else if (!B_MN && lane < 2 * kPairKps) {
          const int i = lane - kPairKps;
          const int kb = kb0 + i;
          const bool ext = kb >= a.kb_main && a.kb_total > a.kb_main;
          const int xk = (ext ? kb - a.kb_main : kb) * kLinBK;
          tma_load_2d_pair(dst + (kPairKps + i) * kLinABytes, ext ? &tmB2 : &tmB1, bar, xk, yb);
        } else if (B_MN && lane < kPairKps + kPairKps * mn_boxes) {
          // K block i: columns yb + 64 h .. of rows (K) kb * 64 .., 8 KB boxes
          const int i = (lane - kPairKps) / mn_boxes, h = (lane - kPairKps) % mn_boxes;
          const int kb = kb0 + i;
          const bool ext = kb >= a.kb_main && a.kb_total > a.kb_main;
          const int yk = (ext ? kb - a.kb_main : kb) * kLinBK;
          tma_load_2d_pair(dst + (kPairKps + i) * kLinABytes + h * (kLinABytes / 2), ext ? &tmB2 : &tmB1, bar,
                           yb + 64 * h, yk);
        }
        parity_bits = (parity_bits & ~(1u << stage)) | (phase << stage);
        filled_mask |= 1u << stage;
        if (++stage == a.stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    // never leave a TMA copy in flight: the even CTA's full barriers count the
    // bytes of both CTAs' copies
    if (lane == 0 && leader)
      for (int s2 = 0; s2 < a.stages; ++s2)
        if ((filled_mask >> s2) & 1u) mbar_wait(&full[s2], (parity_bits >> s2) & 1u, limit);
  } else if (warp == 1) {
    // ------------------------------------------- MMA issuer (even CTA only)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint32_t idesc = idesc_bf16_f32(kPairBM, a.bn) | (B_MN ? kIdescBMnMajor : 0u);
      const uint64_t desc0 = sw128_kmajor_desc(base_s);
      const uint64_t desc_step = kPairStageBytes >> 4;
      // MN-major B: the two 64-column boxes of a K block are 8 KB apart (the
      // leading byte offset); 8-row K groups are 1024 B apart; 16 K rows per MMA
      const uint64_t bdesc_mn0 = sw128_mn_desc(base_s + kPairKps * kLinABytes, kLinABytes / 2);
      int it = 0;
      for (int t = cid; t < n_tiles && ok; t += n_pairs, ++it) {
        const int ab = it & 1;
        if (!mbar_wait(&acc_empty[ab], static_cast<uint32_t>((it >> 1) & 1) ^ 1u, limit)) {
          lin_timeout(a.status, abort_flag);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(ab * kPairBN);
        for (int kb0 = 0; kb0 < a.kb_total; kb0 += kPairKps) {
          if (!mbar_wait(&full[stage], phase, limit)) {
            lin_timeout(a.status, abort_flag);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = desc0 + static_cast<uint64_t>(stage) * desc_step;
          const uint64_t bdesc = B_MN ? bdesc_mn0 + static_cast<uint64_t>(stage) * desc_step
                                      : adesc + ((kPairKps * kLinABytes) >> 4);
          // K-major: +32 B along K inside the swizzled row; MN-major: +16 rows of 128 B
          constexpr uint64_t kb_step = B_MN ? (16 * 128) >> 4 : 2;
#pragma unroll
          for (int i = 0; i < kPairKps; ++i)
#pragma unroll
            for (int k = 0; k < kLinBK / 16; ++k)
              mma_bf16_pair(d, adesc + i * (kLinABytes >> 4) + 2 * k, bdesc + i * (kLinABytes >> 4) + kb_step * k,
                            idesc, (kb0 > 0 || i > 0 || k > 0) ? 1u : 0u);
          mma_commit_pair(&empty[stage], 0x3);
          if (++stage == a.stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) mma_commit_pair(&acc_full[ab], 0x3);
      }
      mma_commit_pair(drain, 0x1);
      mbar_wait(drain, 0, limit);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint32_t tmem_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
    int it = 0;
    for (int t = cid; t < n_tiles; t += n_pairs, ++it) {
      int tm, tn;
      lin_tile(a, t, tm, tn);
      const int ab = it & 1;
      if (!mbar_wait_warp(&acc_full[ab], static_cast<uint32_t>((it >> 1) & 1), limit)) {
        if (lane == 0) lin_timeout(a.status, abort_flag);
        break;
      }
      tc_fence_after();
      const long long row = static_cast<long long>(tm) * kPairBM + rank * kLinBM + q * 32 + lane;
      const bool row_ok = row < a.M;
      const float rscale = (row_ok && a.rs_num) ? __ldg(a.rs_num + row) / __ldg(a.rs_den + row) : 1.f;
#pragma unroll 1
      for (int c = 0; c < a.bn / 32; ++c) {
        const int col0 = tn * a.bn + c * 32;
        if (col0 >= a.N) break;  // warp-uniform
        float v[32];
        tmem_ld32(tmem_lane + static_cast<uint32_t>(ab * kPairBN + c * 32), v);
        const int my_col = col0 + lane;
        float gl = 0.f, bl = 0.f;
        if (my_col < a.N) {
          gl = a.m ? a.alpha * (__ldg(a.m + my_col) / __ldg(a.n + my_col)) : a.alpha;
          if (a.bias) bl = __bfloat162float(a.bias[my_col]);
        }
#pragma unroll
        for (int e = 0; e < 32; ++e)
          v[e] = fmaf(v[e] * rscale, __shfl_sync(0xffffffffu, gl, e), __shfl_sync(0xffffffffu, bl, e));
        if (row_ok) {
          if (OUT_F32) {
            float* dst_row = static_cast<float*>(a.out) + row * a.ldo;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (col0 + 4 * j < a.N)
                *reinterpret_cast<float4*>(dst_row + col0 + 4 * j) =
                    make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          } else {
            __nv_bfloat16* dst_row = static_cast<__nv_bfloat16*>(a.out) + row * a.ldo;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              if (col0 + 8 * j < a.N) {
                uint4 pk;
                pk.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
                pk.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
                pk.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
                pk.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
                *reinterpret_cast<uint4*>(dst_row + col0 + 8 * j) = pk;
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader + static_cast<uint32_t>(ab) * 8u);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA frees TMEM or exits while the pair still uses it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, 2 * kPairBN);
}

}  // namespace dora
