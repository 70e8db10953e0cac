// compose.cuh - fused DoRA compose forward / backward (memory-bound).
//
// "Scaling DoRA: High-Rank Adaptation via Factored Norms and Fused Kernels",
// Abstract: the DoRA composition runs as one pass over the activations, in a
// form that stays accurate when the magnitude rescaling g = m / n is close to 1.
//
// Forward, per output channel i (fp32, never rounded to the activation type):
//   g = m / n,  delta = (m - n) / n   (m - n is exact when m / n is in [1/2, 2])
//   y = base + (delta * (base - b) + g * s * lora)  one final rounding
// where b is the base layer's bias (0 without one): base = x W^T + b, and the
// rescaling acts on the weight's product only, b + g * ((base - b) + s * lora).
// Backward with n constant and b frozen:
//   d_base = g * dy,  d_lora = s * (g * dy),
//   d_m    = (sum_t dy * ((base - b) + s * lora)) / n
//
// Both kernels stream 16-byte vectors (8 bf16 or 4 fp32), coalesced along the
// contiguous d_out axis; each thread keeps its channels' g / delta in
// registers for all the rows it visits.  The backward carries the token sum
// in fp32 registers, folds the two half-warps with a shuffle and the eight
// warps through shared memory, writes one partial per (row chunk, channel),
// and the last CTA of each column strip adds the chunks in fixed order.
#pragma once

#include "sm100_ptx.cuh"

namespace dora {

template <typename T, int VEC>
struct VecIO;

// load() widens at once; raw() / unpack() keep a vector packed (fewer
// registers while several rows are in flight) and widen it at its use.
template <>
struct VecIO<__nv_bfloat16, 8> {
  using Raw = uint4;
  static __device__ __forceinline__ Raw raw(const __nv_bfloat16* p) { return ld_stream_u4(p); }
  static __device__ __forceinline__ Raw raw_param(const __nv_bfloat16* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
  static __device__ __forceinline__ void unpack(const Raw& u, float (&v)[8]) {
    v[0] = bf16_lo(u.x);
    v[1] = bf16_hi(u.x);
    v[2] = bf16_lo(u.y);
    v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z);
    v[5] = bf16_hi(u.z);
    v[6] = bf16_lo(u.w);
    v[7] = bf16_hi(u.w);
  }
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 u = ld_stream_u4(p);
    v[0] = bf16_lo(u.x);
    v[1] = bf16_hi(u.x);
    v[2] = bf16_lo(u.y);
    v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z);
    v[5] = bf16_hi(u.z);
    v[6] = bf16_lo(u.w);
    v[7] = bf16_hi(u.w);
  }
  static __device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[8]) {
    uint4 u;
    u.x = pack2(v[0], v[1]);
    u.y = pack2(v[2], v[3]);
    u.z = pack2(v[4], v[5]);
    u.w = pack2(v[6], v[7]);
    st_stream_u4(p, u);
  }
};

template <>
struct VecIO<float, 4> {
  using Raw = uint4;
  static __device__ __forceinline__ Raw raw(const float* p) { return ld_stream_u4(p); }
  static __device__ __forceinline__ Raw raw_param(const float* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
  static __device__ __forceinline__ void unpack(const Raw& u, float (&v)[4]) {
    v[0] = __uint_as_float(u.x);
    v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z);
    v[3] = __uint_as_float(u.w);
  }
  static __device__ __forceinline__ void load(const float* p, float (&v)[4]) {
    const uint4 u = ld_stream_u4(p);
    v[0] = __uint_as_float(u.x);
    v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z);
    v[3] = __uint_as_float(u.w);
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[4]) {
    st_stream_u4(p, make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                               __float_as_uint(v[3])));
  }
};

template <>
struct VecIO<float, 1> {
  using Raw = float;
  static __device__ __forceinline__ Raw raw(const float* p) { return __ldg(p); }
  static __device__ __forceinline__ Raw raw_param(const float* p) { return __ldg(p); }
  static __device__ __forceinline__ void unpack(const Raw& u, float (&v)[1]) { v[0] = u; }
  static __device__ __forceinline__ void load(const float* p, float (&v)[1]) { v[0] = __ldg(p); }
  static __device__ __forceinline__ void store(float* p, const float (&v)[1]) { p[0] = v[0]; }
};

// One per-channel parameter of the activation type, widened to fp32.
__device__ __forceinline__ float ld_param(const __nv_bfloat16* p) { return __bfloat162float(p[0]); }
__device__ __forceinline__ float ld_param(const float* p) { return __ldg(p); }

// ------------------------------------------------------------------ forward
template <typename T, int VEC>
__global__ void __launch_bounds__(256, 3) compose_fwd_kernel(const T* __restrict__ base, const T* __restrict__ lora,
                                                          const T* __restrict__ bias, const float* __restrict__ m,
                                                          const float* __restrict__ n, float s,
                                                          long long tokens, long long nvec, long long d_out,
                                                          T* __restrict__ y, long long rows_per_cta) {
  const long long v = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (v >= nvec) return;
  const long long col = v * VEC;
  float delta[VEC], gs[VEC], bb[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    const float mm = __ldg(m + col + e), nn = __ldg(n + col + e);
    delta[e] = (mm - nn) / nn;
    gs[e] = (mm / nn) * s;
    bb[e] = bias ? ld_param(bias + col + e) : 0.f;
  }
  const long long row0 = blockIdx.y * rows_per_cta;
  const long long row1 = min(tokens, row0 + rows_per_cta);
  constexpr int U = 4;
  // U rows per pass, their loads issued together; the last pass predicates
  // the rows past row1 (one memory round trip for the leftover rows too)
  using Raw = typename VecIO<T, VEC>::Raw;
  for (long long row = row0; row < row1; row += U) {
    Raw rb[U], rl[U];  // packed until used: fewer registers with U rows in flight
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if (row + k < row1) {
        rb[k] = VecIO<T, VEC>::raw(base + (row + k) * d_out + col);
        rl[k] = VecIO<T, VEC>::raw(lora + (row + k) * d_out + col);
      }
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if (row + k < row1) {
        float b[VEC], l[VEC], o[VEC];
        VecIO<T, VEC>::unpack(rb[k], b);
        VecIO<T, VEC>::unpack(rl[k], l);
#pragma unroll
        for (int e = 0; e < VEC; ++e) o[e] = b[e] + fmaf(delta[e], b[e] - bb[e], gs[e] * l[e]);
        VecIO<T, VEC>::store(y + (row + k) * d_out + col, o);
      }
    }
  }
}

// ----------------------------------------------------------------- backward
constexpr int kBwdThreads = 256;  // 8 warps; a half-warp spans 16 vectors of one row
constexpr int kBwdVecs = 16;      // vectors (column groups) per CTA strip
constexpr int kBwdSlots = 16;     // rows visited concurrently by one CTA
constexpr int kBwdRows = 4;       // rows in flight per thread

// HAS_BIAS: a separate instantiation, so that the bias registers cost the
// no-bias kernel nothing
template <typename T, int VEC, bool HAS_BIAS>
__global__ void __launch_bounds__(kBwdThreads, 2) compose_bwd_kernel(
    const T* __restrict__ dy, const T* __restrict__ base, const T* __restrict__ lora, const T* __restrict__ bias,
    const float* __restrict__ m,
    const float* __restrict__ n, float s, long long tokens, long long nvec, long long d_out, T* __restrict__ d_base,
    T* __restrict__ d_lora, float* __restrict__ partial, unsigned long long* __restrict__ counters,
    float* __restrict__ d_m, long long rows_per_chunk, unsigned long long epoch) {
  __shared__ float red[kBwdThreads / 32][kBwdVecs][VEC];
  __shared__ int is_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = lane >> 4, vi = lane & 15;
  const int slot = warp * 2 + half;
  const long long v = blockIdx.x * static_cast<long long>(kBwdVecs) + vi;
  const bool valid = v < nvec;
  const long long col = v * VEC;

  // d_lora is formed as s * d_base (fp32) rather than from a second per-channel
  // factor g * s: the registers go to the bias instead
  // the bias stays packed in the activation type (half the registers for
  // bf16) and is widened where it is used
  using Raw = typename VecIO<T, VEC>::Raw;
  float g[VEC], acc[VEC];
  Raw bias_raw{};
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    acc[e] = 0.f;
    g[e] = 0.f;
  }
  if (valid) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) g[e] = __ldg(m + col + e) / __ldg(n + col + e);
    if (HAS_BIAS) bias_raw = VecIO<T, VEC>::raw_param(bias + col);
    const long long row0 = blockIdx.y * rows_per_chunk;
    const long long row1 = min(tokens, row0 + rows_per_chunk);
    long long row = row0 + slot;
    // kBwdRows rows of this thread in flight: their three loads are issued
    // before any is used
    for (; row + (kBwdRows - 1) * kBwdSlots < row1; row += kBwdRows * kBwdSlots) {
      Raw ra[kBwdRows], rb[kBwdRows], rl[kBwdRows];
#pragma unroll
      for (int u = 0; u < kBwdRows; ++u) {
        const long long o = (row + u * kBwdSlots) * d_out + col;
        ra[u] = VecIO<T, VEC>::raw(dy + o);
        rb[u] = VecIO<T, VEC>::raw(base + o);
        rl[u] = VecIO<T, VEC>::raw(lora + o);
      }
#pragma unroll
      for (int u = 0; u < kBwdRows; ++u) {
        const long long o = (row + u * kBwdSlots) * d_out + col;
        float a[VEC], b[VEC], l[VEC], db[VEC], dl[VEC];
        VecIO<T, VEC>::unpack(ra[u], a);
        VecIO<T, VEC>::unpack(rb[u], b);
        VecIO<T, VEC>::unpack(rl[u], l);
        if (HAS_BIAS) {
          float bb[VEC];
          VecIO<T, VEC>::unpack(bias_raw, bb);
#pragma unroll
          for (int e = 0; e < VEC; ++e) b[e] -= bb[e];
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          db[e] = g[e] * a[e];
          dl[e] = s * db[e];
          acc[e] = fmaf(a[e], fmaf(s, l[e], b[e]), acc[e]);
        }
        VecIO<T, VEC>::store(d_base + o, db);
        VecIO<T, VEC>::store(d_lora + o, dl);
      }
    }
    for (; row < row1; row += kBwdSlots) {
      float a0[VEC], b0[VEC], l0[VEC], db[VEC], dl[VEC];
      const long long o0 = row * d_out + col;
      VecIO<T, VEC>::load(dy + o0, a0);
      VecIO<T, VEC>::load(base + o0, b0);
      VecIO<T, VEC>::load(lora + o0, l0);
      if (HAS_BIAS) {
        float bb[VEC];
        VecIO<T, VEC>::unpack(bias_raw, bb);
#pragma unroll
        for (int e = 0; e < VEC; ++e) b0[e] -= bb[e];
      }
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        db[e] = g[e] * a0[e];
        dl[e] = s * db[e];
        acc[e] = fmaf(a0[e], fmaf(s, l0[e], b0[e]), acc[e]);
      }
      VecIO<T, VEC>::store(d_base + o0, db);
      VecIO<T, VEC>::store(d_lora + o0, dl);
    }
  }

  // fold the two half-warps (same columns, different rows), then the 8 warps
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
  if (half == 0) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) red[warp][vi][e] = acc[e];
  }
  __syncthreads();
  const int t = threadIdx.x;
  const long long tcol = blockIdx.x * static_cast<long long>(kBwdVecs) * VEC + t;
  const bool t_ok = t < kBwdVecs * VEC && tcol < d_out;
  if (t_ok) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kBwdThreads / 32; ++w) sum += red[w][t / VEC][t % VEC];
    partial[blockIdx.y * d_out + tcol] = sum;
  }
  __threadfence();
  __syncthreads();
  // arrivals per column strip in a word tagged with this call's epoch,
  // (epoch << 8) | count: a word with any other tag (an earlier call, or
  // whatever the caller's buffer held) counts as zero, so the counters need
  // no clearing before the launch
  const unsigned long long tag = epoch << 8;
  if (t == 0) {
    unsigned long long* c = counters + blockIdx.x;
    unsigned long long v = *reinterpret_cast<volatile unsigned long long*>(c);
    int seen = 0;
    while (true) {
      seen = (v & ~0xffull) == tag ? static_cast<int>(v & 0xffull) : 0;
      const unsigned long long prev = atomicCAS(c, v, tag | static_cast<unsigned long long>(seen + 1));
      if (prev == v) break;
      v = prev;
    }
    is_last = (seen == static_cast<int>(gridDim.y) - 1);
  }
  __syncthreads();
  if (is_last) {
    __threadfence();
    if (t_ok) {
      float total = 0.f;
      for (unsigned c = 0; c < gridDim.y; ++c) total += ld_cg_f32(&partial[c * d_out + tcol]);
      d_m[tcol] = total / __ldg(n + tcol);
    }
    if (t == 0) counters[blockIdx.x] = tag;  // count 0 under this tag: a replay of the same launch starts clean
  }
}

}  // namespace dora
