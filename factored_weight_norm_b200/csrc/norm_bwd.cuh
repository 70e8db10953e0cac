// norm_bwd.cuh - pieces of the attached-norm backward (gradients of the row
// norms n_i = ||W_i + s B_i A|| into A and B) that are not GEMMs.
//
// "Scaling DoRA: High-Rank Adaptation via Factored Norms and Fused Kernels",
// Abstract: the factored norm never forms B A; its gradients keep to the same
// factors.  With c = d_n / n (d_n the upstream gradient of n), G = A A^T and
// H = (c * B)^T B:
//
//   dB = s c * (W A^T + s B G)                 = s c * ([W | B] [A | s G]^T)
//   dA = s (c * B)^T W + s^2 H A               = [s (c*B)^T | s^2 H] [W ; A]
//
// Both are GEMMs on tensor cores (the second contracts over d_out, so W is
// read N-contiguous).  This file holds the prep pass: B^T and (s c * B)^T as
// K-major [r, d_out] bf16 copies (6 MB at d_out = 8192, r = 384), the operands
// of H and of dA's first term.
#pragma once

#include "sm100_ptx.cuh"

namespace dora {

// Bt[m][k] = B[k][m],  Bct[m][k] = bf16(s * d_n[k] / n[k] * B[k][m]).
// One 64 (k) x 64 (m) tile per CTA through shared memory (rows padded to 66
// bf16, so the column reads meet at most two-way bank conflicts); 16-byte
// loads of B's rows and 16-byte stores of the transposed rows.  d_out and r
// are multiples of 8, so every 8-element vector is wholly in or out.
constexpr int kPrepTile = 64;
constexpr int kPrepPad = 66;

__global__ void __launch_bounds__(256) norm_bwd_prep_kernel(const __nv_bfloat16* __restrict__ B,
                                                            const float* __restrict__ d_n,
                                                            const float* __restrict__ n, float s, int d_out, int r,
                                                            __nv_bfloat16* __restrict__ Bt,
                                                            __nv_bfloat16* __restrict__ Bct) {
  __shared__ __nv_bfloat16 tile[kPrepTile][kPrepPad];
  __shared__ float cs[kPrepTile];
  const int k0 = blockIdx.x * kPrepTile, m0 = blockIdx.y * kPrepTile;
  const int t = threadIdx.x;
  if (t < kPrepTile) {
    const int k = k0 + t;
    cs[t] = (k < d_out) ? s * (__ldg(d_n + k) / __ldg(n + k)) : 0.f;
  }
  // load: 64 rows of B x 8 vectors of 8 bf16
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = (t >> 3) + 32 * h, vec = t & 7;
    const int k = k0 + row, m = m0 + vec * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (k < d_out && m < r) v = __ldg(reinterpret_cast<const uint4*>(B + static_cast<size_t>(k) * r + m));
    const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
    for (int i = 0; i < 8; ++i) tile[row][vec * 8 + i] = e[i];
  }
  __syncthreads();
  // store: 64 output rows (m) x 8 vectors of 8 consecutive k
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int col = (t >> 3) + 32 * h, vk = t & 7;
    const int m = m0 + col, k = k0 + vk * 8;
    if (m >= r || k >= d_out) continue;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __bfloat162float(tile[vk * 8 + i][col]);
    uint4 raw, scaled;
    raw.x = pack_bf16x2(v[0], v[1]);
    raw.y = pack_bf16x2(v[2], v[3]);
    raw.z = pack_bf16x2(v[4], v[5]);
    raw.w = pack_bf16x2(v[6], v[7]);
    scaled.x = pack_bf16x2(cs[vk * 8 + 0] * v[0], cs[vk * 8 + 1] * v[1]);
    scaled.y = pack_bf16x2(cs[vk * 8 + 2] * v[2], cs[vk * 8 + 3] * v[3]);
    scaled.z = pack_bf16x2(cs[vk * 8 + 4] * v[4], cs[vk * 8 + 5] * v[5]);
    scaled.w = pack_bf16x2(cs[vk * 8 + 6] * v[6], cs[vk * 8 + 7] * v[7]);
    *reinterpret_cast<uint4*>(Bt + static_cast<size_t>(m) * d_out + k) = raw;
    *reinterpret_cast<uint4*>(Bct + static_cast<size_t>(m) * d_out + k) = scaled;
  }
}

}  // namespace dora
