// Device helpers shared by the kernels: element loads/stores and RoPE angles.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "la_internal.h"

namespace la {

// Eight consecutive elements of a row as float (16 B of bf16 or 32 B of f32).
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&x)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ void load8(const float* p, float (&x)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // round to nearest even
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int kCount>
__device__ __forceinline__ void store_row(__nv_bfloat16* p, const float* x) {
  static_assert(kCount % 8 == 0, "16-byte stores");
#pragma unroll
  for (int i = 0; i < kCount; i += 8) {
    uint4 u;
    u.x = pack_bf16x2(x[i + 0], x[i + 1]);
    u.y = pack_bf16x2(x[i + 2], x[i + 3]);
    u.z = pack_bf16x2(x[i + 4], x[i + 5]);
    u.w = pack_bf16x2(x[i + 6], x[i + 7]);
    *reinterpret_cast<uint4*>(p + i) = u;
  }
}
template <int kCount>
__device__ __forceinline__ void store_row(float* p, const float* x) {
  static_assert(kCount % 4 == 0, "16-byte stores");
#pragma unroll
  for (int i = 0; i < kCount; i += 4)
    *reinterpret_cast<float4*>(p + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
}

// Position of token n along axis a (0 = t global, 1 = h, 2 = w).
__device__ __forceinline__ int rope_pos(const Rope& r, int n, int axis) {
  const int w = n % r.W;
  const int hw = n / r.W;
  if (axis == 2) return w;
  if (axis == 1) return hw % r.Hh;
  return hw / r.Hh + r.t_offset;
}

// cos and sin of pos * inv_freq: the angle is formed and reduced to
// [-pi, pi] in double, then evaluated in float.
__device__ __forceinline__ void rope_cos_sin(int pos, double inv_freq, float& c, float& s) {
  const double kTwoPi = 6.283185307179586476925286766559;
  const double a = static_cast<double>(pos) * inv_freq;
  const double r = a - kTwoPi * rint(a * (1.0 / kTwoPi));
  sincosf(static_cast<float>(r), &s, &c);
}

// Second phase of the state reduce, run by every thread of a CTA once it has
// written its split's partials for heads [h0, h0 + nh) of batch b. The CTA
// that arrives last for (b, h0) sums all splits' partials in split order,
// adds the carry when given, writes the outputs and re-zeroes the counter.
// No thread waits on another CTA: the others just return.
__device__ __forceinline__ void finish_reduce(const Problem& p, int b, int h0, int nh,
                                              const float* partials, unsigned* counters,
                                              const StateOut& out) {
  __shared__ int s_last;
  __threadfence();  // this thread's partial stores, visible device-wide
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(&counters[static_cast<size_t>(b) * p.H + h0], 1u);
    s_last = prev == static_cast<unsigned>(p.splits - 1);
  }
  __syncthreads();
  if (!s_last) return;
  if (out.out1_S == nullptr && out.out1_z == nullptr && out.out2_S == nullptr &&
      out.out2_z == nullptr) {  // partials only (the token-causal pass reads them)
    if (threadIdx.x == 0) counters[static_cast<size_t>(b) * p.H + h0] = 0u;
    return;
  }
  __threadfence();
  // Each thread sums float4 columns of the partials; the loads of up to 8
  // splits are issued together and then added in split order.
  constexpr int kVec = kStateFloats / 4;
  const int heads = min(nh, p.H - h0);
  for (int v = threadIdx.x; v < heads * kVec; v += blockDim.x) {
    const int hh = v / kVec, i = (v - hh * kVec) * 4;
    const size_t bh = static_cast<size_t>(b) * p.H + h0 + hh;
    const float* src = partials + bh * p.splits * kStateFloats + i;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int s0 = 0; s0 < p.splits; s0 += 8) {
      float4 t[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (s0 + k < p.splits)
          t[k] = __ldcg(reinterpret_cast<const float4*>(src + static_cast<size_t>(s0 + k) * kStateFloats));
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (s0 + k < p.splits) {
          acc.x += t[k].x;
          acc.y += t[k].y;
          acc.z += t[k].z;
          acc.w += t[k].w;
        }
    }
    const bool is_s = i < kD * kD;
    const size_t o = is_s ? bh * kD * kD + i : bh * kD + (i - kD * kD);
    const float* c = is_s ? out.carry_S : out.carry_z;
    if (c != nullptr) {
      const float4 cv = *reinterpret_cast<const float4*>(c + o);
      acc = make_float4(cv.x + acc.x, cv.y + acc.y, cv.z + acc.z, cv.w + acc.w);
    }
    float* d1 = is_s ? out.out1_S : out.out1_z;
    float* d2 = is_s ? out.out2_S : out.out2_z;
    if (d1 != nullptr) *reinterpret_cast<float4*>(d1 + o) = acc;
    if (d2 != nullptr) *reinterpret_cast<float4*>(d2 + o) = acc;
  }
  if (threadIdx.x == 0) counters[static_cast<size_t>(b) * p.H + h0] = 0u;
}

}  // namespace la
