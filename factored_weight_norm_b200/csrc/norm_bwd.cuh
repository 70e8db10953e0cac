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

// Bt[m][k] = B[k][m],  Bct[m][k] = bf16(s * d_n[k] / n[k] * B[k][m]);
// 32 x 32 tiles through shared memory, both sides coalesced.
__global__ void __launch_bounds__(256) norm_bwd_prep_kernel(const __nv_bfloat16* __restrict__ B,
                                                            const float* __restrict__ d_n,
                                                            const float* __restrict__ n, float s, int d_out, int r,
                                                            __nv_bfloat16* __restrict__ Bt,
                                                            __nv_bfloat16* __restrict__ Bct) {
  __shared__ float tile[32][33];
  const int k0 = blockIdx.x * 32, m0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int k = k0 + ty + 8 * j, m = m0 + tx;
    tile[ty + 8 * j][tx] = (k < d_out && m < r) ? __bfloat162float(B[static_cast<size_t>(k) * r + m]) : 0.f;
  }
  __syncthreads();
  const int k = k0 + tx;
  const float c = (k < d_out) ? s * (__ldg(d_n + k) / __ldg(n + k)) : 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int m = m0 + ty + 8 * j;
    if (m < r && k < d_out) {
      const float v = tile[tx][ty + 8 * j];
      Bt[static_cast<size_t>(m) * d_out + k] = __float2bfloat16_rn(v);
      Bct[static_cast<size_t>(m) * d_out + k] = __float2bfloat16_rn(c * v);
    }
  }
}

}  // namespace dora
