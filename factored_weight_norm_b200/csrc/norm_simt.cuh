// norm_simt.cuh - fp32 factored row norm on CUDA cores, and the plain row norm
// used when the adapter has rank 0.
//
// Same decomposition as the tensor-core path ("Scaling DoRA: High-Rank
// Adaptation via Factored Norms and Fused Kernels", Abstract: base, cross and
// Gram terms), evaluated in fp32 FMA arithmetic so fp32 inputs keep fp32
// accuracy (no TF32 anywhere):
//   n_i^2 = ||W_i||^2 + 2s <B_i, W_i A^T> + s^2 B_i G B_i^T,  G = A A^T.
#pragma once

#include "sm100_ptx.cuh"

namespace dora {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// G = A A^T, fp32 [r][r]; one warp per (j, k) pair with j <= k.
__global__ void gram_f32_kernel(const float* __restrict__ A, int r, int d_in, float* __restrict__ G) {
  const long long pairs = static_cast<long long>(r) * (r + 1) / 2;
  const int lane = threadIdx.x & 31;
  const long long warps_total = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long p = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5); p < pairs;
       p += warps_total) {
    // p -> (j, k), j <= k, row-major over the upper triangle
    long long rem = p;
    int j = 0;
    while (rem >= r - j) {
      rem -= r - j;
      ++j;
    }
    const int k = j + static_cast<int>(rem);
    const float* aj = A + static_cast<size_t>(j) * d_in;
    const float* ak = A + static_cast<size_t>(k) * d_in;
    float acc = 0.f;
    for (int c = lane; c < d_in; c += 32) acc = fmaf(aj[c], ak[c], acc);
    acc = warp_sum(acc);
    if (lane == 0) {
      G[static_cast<size_t>(j) * r + k] = acc;
      G[static_cast<size_t>(k) * r + j] = acc;
    }
  }
}

// One CTA of 256 threads per output row.
__global__ void __launch_bounds__(256) norm_f32_kernel(const float* __restrict__ W, const float* __restrict__ A,
                                                       const float* __restrict__ B, const float* __restrict__ G,
                                                       int d_out, int d_in, int r, float s,
                                                       float* __restrict__ n_out, int squared) {
  __shared__ float red[3][8];
  const int i = blockIdx.x;
  if (i >= d_out) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* wi = W + static_cast<size_t>(i) * d_in;
  const float* bi = B + static_cast<size_t>(i) * r;

  float base = 0.f;
  for (int c = threadIdx.x; c < d_in; c += blockDim.x) base = fmaf(wi[c], wi[c], base);

  float cross = 0.f;  // sum_j B_ij (W_i . A_j), one warp per j
  for (int j = warp; j < r; j += 8) {
    const float* aj = A + static_cast<size_t>(j) * d_in;
    float u = 0.f;
    for (int c = lane; c < d_in; c += 32) u = fmaf(wi[c], aj[c], u);
    u = warp_sum(u);
    if (lane == 0) cross = fmaf(bi[j], u, cross);
  }

  float gram = 0.f;  // sum_{j,l} B_ij G_jl B_il
  const long long rr = static_cast<long long>(r) * r;
  for (long long p = threadIdx.x; p < rr; p += blockDim.x) {
    const int j = static_cast<int>(p / r), l = static_cast<int>(p % r);
    gram = fmaf(bi[j] * G[p], bi[l], gram);
  }

  base = warp_sum(base);
  cross = warp_sum(cross);
  gram = warp_sum(gram);
  if (lane == 0) {
    red[0][warp] = base;
    red[1][warp] = cross;
    red[2][warp] = gram;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.f, x = 0.f, g = 0.f;
    for (int w = 0; w < 8; ++w) {
      b += red[0][w];
      x += red[1][w];
      g += red[2][w];
    }
    const float n2 = b + 2.f * s * x + s * s * g;
    n_out[i] = squared ? n2 : sqrtf(fmaxf(n2, 0.f));
  }
}

// Plain row norm ||W_i|| (rank-0 adapter, or s*BA == 0 by construction).
template <typename T>
__global__ void rownorm_kernel(const T* __restrict__ W, int d_out, int d_in, float* __restrict__ n_out, int squared) {
  const int warps = blockDim.x >> 5;
  const int i = blockIdx.x * warps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= d_out) return;
  const T* wi = W + static_cast<size_t>(i) * d_in;
  float acc = 0.f;
  for (int c = lane; c < d_in; c += 32) {
    const float v = static_cast<float>(wi[c]);
    acc = fmaf(v, v, acc);
  }
  acc = warp_sum(acc);
  if (lane == 0) n_out[i] = squared ? acc : sqrtf(acc);
}

// n = sqrt(max(n^2, 0)) in place: the last step of a norm whose squared
// partials were summed across d_in shards.
__global__ void norm_finish_kernel(float* __restrict__ n, long long d_out) {
  const long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (i < d_out) n[i] = sqrtf(fmaxf(n[i], 0.f));
}

}  // namespace dora
