// Backward pass of the non-causal layer on CUDA cores (the float32-I/O path;
// bf16 I/O runs on the tensor cores, la_backward_tc.cu).
//
// "Sana: Efficient High-Resolution Image Synthesis with Linear Diffusion
// Transformers", section Infra, runs the linear attention with a fused forward
// and backward. With den_i = ReLU(q_i).z + eps and O_i = phi(q_i) S / den_i:
//
//   dnum_i = dO_i / den_i,            dden_i = -(dO_i . O_i) / den_i
//   dS = sum_i phi(q_i)^T dnum_i,     dz = sum_i dden_i ReLU(q_i)
//   dq_i = [R_i^T (dnum_i S^T) + dden_i z] * [q_i > 0]
//   dk_j = [R_j^T (dS v_j) + dz] * [k_j > 0],   dv_j = phi(k_j) dS
//
// (R = the 3D RoPE rotation of the token, the identity without RoPE.) The
// forward output is not an input: dO_i . O_i = phi(q_i) . (S dnum_i^T), and
// S dnum_i^T is the term dq_i needs anyway. Two launches: the query side produces dQ and reduces dS, dz (split-N partials,
// last CTA of each head combines them in split order); the key side then
// produces dK and dV.
#include "la_common.cuh"

namespace la {
namespace {

constexpr int kBT = 64;  // token rows per tile of the query-side kernel
constexpr int kBThreads = 256;

// Rotate the 4 pairs of dims [d0, d0 + 8) of token n by +theta (sign = 1) or
// -theta (sign = -1).
__device__ __forceinline__ void rotate8(const Problem& p, int n, int d0, float sign,
                                        float (&x)[8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = d0 / 2 + i;
    float c, s;
    rope_cos_sin(rope_pos(p.rope, n, p.rope.axis[j]), p.rope.inv_freq[j], c, s);
    s *= sign;
    const float x0 = x[2 * i], x1 = x[2 * i + 1];
    x[2 * i] = fmaf(x0, c, -x1 * s);
    x[2 * i + 1] = fmaf(x0, s, x1 * c);
  }
}

// Query side: one CTA per (split, head, batch). Thread t stages dims
// [(t%4)*8, +8) of row t/4 of each 64-token tile, forms the row's
// denominator with shuffles over the 4 threads of the row, computes
// t = S dnum for its 8 dims, then dO . O = phi(q) . t / den (so O itself is
// not read), the row's dq, and the running dz of those dims; for dS it owns a
// 4x4 block over a quarter of the tile's rows.
template <typename T>
__global__ void __launch_bounds__(kBThreads)
bwd_q_simt(const Problem p, const T* __restrict__ Q, const T* __restrict__ dO,
           const float* __restrict__ S, const float* __restrict__ z, T* __restrict__ dQ,
           float* partials, unsigned* counters, const StateOut out) {
  __shared__ float Ss[kD][kD + 1];  // +1: the 4 row groups of a warp hit 4 banks
  __shared__ float zs[kD];
  __shared__ __align__(16) float phq[kBT][kD + 4];
  __shared__ __align__(16) float dnum[kBT][kD + 4];
  __shared__ __align__(16) float red[4][kD * kD];
  __shared__ float zred[kBThreads / 4][kD / 8][8];

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const size_t bh = static_cast<size_t>(b) * p.H + h;
  for (int i = tid; i < kD * kD; i += kBThreads) Ss[i / kD][i % kD] = S[bh * kD * kD + i];
  if (tid < kD) zs[tid] = z[bh * kD + tid];
  __syncthreads();

  const int n_begin = split * p.chunk;
  const int n_end = min(p.N, n_begin + p.chunk);
  const int lr = tid >> 2, ld = (tid & 3) * 8;
  const int tg = tid >> 6, blk = tid & 63;
  const int d0 = (blk >> 3) * 4, e0 = (blk & 7) * 4;
  float acc[4][4] = {};
  float zacc[8] = {};

  for (int n0 = n_begin; n0 < n_end; n0 += kBT) {
    const int n = n0 + lr;
    const bool row = n < n_end;
    const size_t off = ((static_cast<size_t>(b) * p.N + (row ? n : 0)) * p.H + h) * kD + ld;
    float q[8], g[8];
    if (row) {
      load8(Q + off, q);
      load8(dO + off, g);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = g[i] = 0.0f;
    }
    float qp[8], ph[8];
    float den = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      qp[i] = fmaxf(q[i], 0.0f);
      ph[i] = qp[i];
      den = fmaf(qp[i], zs[ld + i], den);
    }
    if (p.rope.enabled && row) rotate8(p, n, ld, 1.0f, ph);
    den += __shfl_xor_sync(0xffffffffu, den, 1);
    den += __shfl_xor_sync(0xffffffffu, den, 2);
    den += p.eps;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      phq[lr][ld + i] = ph[i];
      dnum[lr][ld + i] = row ? g[i] / den : 0.0f;
    }
    __syncthreads();
    // dS block of this thread over a quarter of the rows
#pragma unroll 4
    for (int r = tg; r < kBT; r += 4) {
      const float4 a = *reinterpret_cast<const float4*>(&phq[r][d0]);
      const float4 c = *reinterpret_cast<const float4*>(&dnum[r][e0]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], cv[j], acc[i][j]);
    }
    // t = S dnum for this row's 8 dims; dO . O = phi(q) . t / den
    float t[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) t[i] = 0.0f;
#pragma unroll 8
    for (int e = 0; e < kD; ++e) {
      const float de = dnum[lr][e];
#pragma unroll
      for (int i = 0; i < 8; ++i) t[i] = fmaf(de, Ss[ld + i][e], t[i]);
    }
    float dot = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) dot = fmaf(ph[i], t[i], dot);
    dot += __shfl_xor_sync(0xffffffffu, dot, 1);
    dot += __shfl_xor_sync(0xffffffffu, dot, 2);
    const float dden = row ? -dot / den : 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) zacc[i] = fmaf(dden, qp[i], zacc[i]);
    if (row) {
      if (p.rope.enabled) rotate8(p, n, ld, -1.0f, t);
#pragma unroll
      for (int i = 0; i < 8; ++i) t[i] = q[i] > 0.0f ? fmaf(dden, zs[ld + i], t[i]) : 0.0f;
      store_row<8>(dQ + off, t);
    }
    __syncthreads();
  }

  // fixed-order reduction of the partial dS and dz, then the split combine
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) red[tg][(d0 + i) * kD + e0 + j] = acc[i][j];
#pragma unroll
  for (int i = 0; i < 8; ++i) zred[lr][ld / 8][i] = zacc[i];
  __syncthreads();
  float* part = partials + (bh * p.splits + split) * kStateFloats;
  for (int i = tid; i < kD * kD; i += kBThreads)
    part[i] = ((red[0][i] + red[1][i]) + red[2][i]) + red[3][i];
  if (tid < kD) {
    float s = 0.0f;
    for (int r = 0; r < kBThreads / 4; ++r) s += zred[r][tid / 8][tid % 8];
    part[kD * kD + tid] = s;
  }
  finish_reduce(p, b, h, 1, partials, counters, out);
}

constexpr int kKT = 128;  // token rows per CTA of the key-side kernel

// Key side: one CTA per (128-token tile, head, batch). Thread t stages and
// computes dims [(t%4)*8, +8) of rows t/4 and t/4 + 64.
template <typename T>
__global__ void __launch_bounds__(kBThreads)
bwd_kv_simt(const Problem p, const T* __restrict__ K, const T* __restrict__ V,
            const float* __restrict__ dS, const float* __restrict__ dz, T* __restrict__ dK,
            T* __restrict__ dV) {
  __shared__ float dSs[kD][kD + 1];
  __shared__ float dzs[kD];
  __shared__ __align__(16) float phk[kKT][kD + 4];
  __shared__ __align__(16) float vs[kKT][kD + 4];

  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const size_t bh = static_cast<size_t>(b) * p.H + h;
  for (int i = tid; i < kD * kD; i += kBThreads) dSs[i / kD][i % kD] = dS[bh * kD * kD + i];
  if (tid < kD) dzs[tid] = dz[bh * kD + tid];

  const int ld = (tid & 3) * 8;
  float kr[2][8];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int lr = (tid >> 2) + half * 64;
    const int n = tile * kKT + lr;
    float v[8];
    if (n < p.N) {
      const size_t off = ((static_cast<size_t>(b) * p.N + n) * p.H + h) * kD + ld;
      load8(K + off, kr[half]);
      load8(V + off, v);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) kr[half][i] = v[i] = 0.0f;
    }
    float ph[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) ph[i] = fmaxf(kr[half][i], 0.0f);
    if (p.rope.enabled && n < p.N) rotate8(p, n, ld, 1.0f, ph);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      phk[lr][ld + i] = ph[i];
      vs[lr][ld + i] = v[i];
    }
  }
  __syncthreads();

#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int lr = (tid >> 2) + half * 64;
    const int n = tile * kKT + lr;
    if (n >= p.N) continue;
    float dk[8], dv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) dk[i] = dv[i] = 0.0f;
#pragma unroll 4
    for (int e = 0; e < kD; ++e) {
      const float ve = vs[lr][e];   // dphi(k)[d] = sum_e dS[d][e] v[e]
      const float pe = phk[lr][e];  // dv[e'] = sum_d phi(k)[d] dS[d][e']
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        dk[i] = fmaf(dSs[ld + i][e], ve, dk[i]);
        dv[i] = fmaf(pe, dSs[e][ld + i], dv[i]);
      }
    }
    if (p.rope.enabled) rotate8(p, n, ld, -1.0f, dk);
#pragma unroll
    for (int i = 0; i < 8; ++i) dk[i] = kr[half][i] > 0.0f ? dk[i] + dzs[ld + i] : 0.0f;
    const size_t off = ((static_cast<size_t>(b) * p.N + n) * p.H + h) * kD + ld;
    store_row<8>(dK + off, dk);
    store_row<8>(dV + off, dv);
  }
}

}  // namespace

cudaError_t launch_backward_q_simt(const Problem& p, const void* Q, const void* dO, const float* S,
                                   const float* z, void* dQ, float* partials,
                                   unsigned* counters, const StateOut& out, cudaStream_t s) {
  const dim3 grid(p.splits, p.H, p.B);
  if (p.io == 0)
    bwd_q_simt<__nv_bfloat16><<<grid, kBThreads, 0, s>>>(
        p, static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(dO),
        S, z, static_cast<__nv_bfloat16*>(dQ), partials, counters, out);
  else
    bwd_q_simt<float><<<grid, kBThreads, 0, s>>>(
        p, static_cast<const float*>(Q), static_cast<const float*>(dO),
        S, z, static_cast<float*>(dQ), partials, counters, out);
  return cudaGetLastError();
}

cudaError_t launch_backward_kv_simt(const Problem& p, const void* K, const void* V, const float* dS,
                                    const float* dz, void* dK, void* dV, cudaStream_t s) {
  const dim3 grid((p.N + kKT - 1) / kKT, p.H, p.B);
  if (p.io == 0)
    bwd_kv_simt<__nv_bfloat16><<<grid, kBThreads, 0, s>>>(
        p, static_cast<const __nv_bfloat16*>(K), static_cast<const __nv_bfloat16*>(V), dS, dz,
        static_cast<__nv_bfloat16*>(dK), static_cast<__nv_bfloat16*>(dV));
  else
    bwd_kv_simt<float><<<grid, kBThreads, 0, s>>>(p, static_cast<const float*>(K),
                                                  static_cast<const float*>(V), dS, dz,
                                                  static_cast<float*>(dK), static_cast<float*>(dV));
  return cudaGetLastError();
}

}  // namespace la
