// CUDA-core kernels: the split-N state reduce, the fixed-order combine and
// the apply. They serve the float32-I/O mode (whose 1e-4 tolerance rules out
// 16-bit tensor-core operands) and every shape the tensor-core path does not
// take.
//
// State reduce and apply follow "SANA-Video: Efficient Video Generation with
// Block Linear Diffusion Transformer", sections 2.1 and 2.2, and the Sana
// Linear DiT ("Sana: Efficient High-Resolution Image Synthesis with Linear
// Diffusion Transformers", section 模型架构 item 2).
#include "la_common.cuh"

namespace la {
namespace {

constexpr int kRedTile = 64;     // tokens staged per iteration of the reduce
constexpr int kRedThreads = 256;

// Load 8 consecutive dims [d0, d0+8) of one (token, head) row, return
// ReLU(x) in `plus` and phi(x) (rotated when RoPE is on) in `phi`.
template <typename T>
__device__ __forceinline__ void feature8(const Problem& p, const T* row, int n, int d0,
                                         float (&plus)[8], float (&phi)[8]) {
  float x[8];
  load8(row + d0, x);
#pragma unroll
  for (int i = 0; i < 8; ++i) plus[i] = fmaxf(x[i], 0.0f);
  if (!p.rope.enabled) {
#pragma unroll
    for (int i = 0; i < 8; ++i) phi[i] = plus[i];
    return;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = d0 / 2 + i;  // pair index
    float c, s;
    rope_cos_sin(rope_pos(p.rope, n, p.rope.axis[j]), p.rope.inv_freq[j], c, s);
    const float x0 = plus[2 * i], x1 = plus[2 * i + 1];
    phi[2 * i] = fmaf(x0, c, -x1 * s);
    phi[2 * i + 1] = fmaf(x0, s, x1 * c);
  }
}

// One CTA per (split, head, batch). Thread t stages dims [(t%4)*8, +8) of
// token row t/4 of each 64-token tile and keeps the running key sum of those
// dims; for the contraction it owns a 4x4 block of S over a quarter of the
// tile's tokens.
template <typename T>
__global__ void __launch_bounds__(kRedThreads)
reduce_simt(const Problem p, const T* __restrict__ K, const T* __restrict__ V,
            float* partials, unsigned* counters, const StateOut out) {
  // float4 reads below: the staging arrays must be 16-byte aligned.
  __shared__ __align__(16) float ks[kRedTile][kD + 4];
  __shared__ __align__(16) float vs[kRedTile][kD + 4];
  __shared__ __align__(16) float red[4][kD * kD];
  __shared__ float zred[kRedThreads / 4][kD / 8][8];

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int n_begin = split * p.chunk;
  const int n_end = min(p.N, n_begin + p.chunk);

  const int lr = tid >> 2;        // staged row in the tile
  const int ld = (tid & 3) * 8;   // staged dims
  const int tg = tid >> 6;        // token group of the contraction
  const int blk = tid & 63;
  const int d0 = (blk >> 3) * 4, e0 = (blk & 7) * 4;

  float acc[4][4] = {};
  float zacc[8] = {};

  for (int n0 = n_begin; n0 < n_end; n0 += kRedTile) {
    const int n = n0 + lr;
    float plus[8], phi[8], v[8];
    if (n < n_end) {
      const size_t off = ((static_cast<size_t>(b) * p.N + n) * p.H + h) * kD;
      feature8(p, K + off, n, ld, plus, phi);
      load8(V + off + ld, v);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) plus[i] = phi[i] = v[i] = 0.0f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      zacc[i] += plus[i];
      ks[lr][ld + i] = phi[i];
      vs[lr][ld + i] = v[i];
    }
    __syncthreads();
#pragma unroll 4
    for (int r = tg; r < kRedTile; r += 4) {
      const float4 a = *reinterpret_cast<const float4*>(&ks[r][d0]);
      const float4 c = *reinterpret_cast<const float4*>(&vs[r][e0]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], cv[j], acc[i][j]);
    }
    __syncthreads();
  }

  // Fixed-order reduction of the four token groups and of the key sums.
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) red[tg][(d0 + i) * kD + e0 + j] = acc[i][j];
#pragma unroll
  for (int i = 0; i < 8; ++i) zred[lr][ld / 8][i] = zacc[i];
  __syncthreads();

  float* part = partials + ((static_cast<size_t>(b) * p.H + h) * p.splits + split) * kStateFloats;
  for (int i = tid; i < kD * kD; i += kRedThreads)
    part[i] = ((red[0][i] + red[1][i]) + red[2][i]) + red[3][i];
  if (tid < kD) {
    float s = 0.0f;
    for (int r = 0; r < kRedThreads / 4; ++r) s += zred[r][tid / 8][tid % 8];
    part[kD * kD + tid] = s;
  }
  finish_reduce(p, b, h, 1, partials, counters, out);
}

constexpr int kApplyTile = 128;  // tokens per CTA
constexpr int kApplyThreads = 256;

// One CTA per (128-token tile, head, batch). Staging: thread t handles dims
// [(t%4)*8, +8) of rows t/4 and t/4 + 64 and forms their share of the
// denominator, summed over the 4 threads of a row with shuffles. Contraction:
// thread t computes 16 outputs of token t/2.
template <typename T>
__global__ void __launch_bounds__(kApplyThreads)
apply_simt(const Problem p, const T* __restrict__ Q, const float* __restrict__ S,
           const float* __restrict__ z, T* __restrict__ O) {
  __shared__ __align__(16) float Ss[kD][kD];
  __shared__ float zs[kD];
  __shared__ __align__(16) float qs[kApplyTile][kD + 4];
  __shared__ float den[kApplyTile];

  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const size_t bh = static_cast<size_t>(b) * p.H + h;
  for (int i = tid; i < kD * kD; i += kApplyThreads) Ss[i / kD][i % kD] = S[bh * kD * kD + i];
  if (tid < kD) zs[tid] = z[bh * kD + tid];
  __syncthreads();

  const int n_tile = tile * kApplyTile;
  const int ld = (tid & 3) * 8;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int lr = (tid >> 2) + half * 64;
    const int n = n_tile + lr;
    float plus[8], phi[8];
    if (n < p.N) {
      const size_t off = ((static_cast<size_t>(b) * p.N + n) * p.H + h) * kD;
      feature8(p, Q + off, n, ld, plus, phi);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) plus[i] = phi[i] = 0.0f;
    }
    float dpart = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      dpart = fmaf(plus[i], zs[ld + i], dpart);
      qs[lr][ld + i] = phi[i];
    }
    dpart += __shfl_xor_sync(0xffffffffu, dpart, 1);
    dpart += __shfl_xor_sync(0xffffffffu, dpart, 2);
    if ((tid & 3) == 0) den[lr] = dpart + p.eps;
  }
  __syncthreads();

  const int r = tid >> 1;
  const int e0 = (tid & 1) * 16;
  const int n = n_tile + r;
  if (n >= p.N) return;
  float num[16] = {};
#pragma unroll 8
  for (int d = 0; d < kD; ++d) {
    const float a = qs[r][d];
#pragma unroll
    for (int j = 0; j < 16; j += 4) {
      const float4 s4 = *reinterpret_cast<const float4*>(&Ss[d][e0 + j]);
      num[j] = fmaf(a, s4.x, num[j]);
      num[j + 1] = fmaf(a, s4.y, num[j + 1]);
      num[j + 2] = fmaf(a, s4.z, num[j + 2]);
      num[j + 3] = fmaf(a, s4.w, num[j + 3]);
    }
  }
  const float dn = den[r];
  float o[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) o[j] = num[j] / dn;
  const size_t off = ((static_cast<size_t>(b) * p.N + n) * p.H + h) * kD + e0;
  store_row<16>(O + off, o);
}

}  // namespace

cudaError_t launch_reduce_simt(const Problem& p, const void* K, const void* V, float* partials,
                               unsigned* counters, const StateOut& out, cudaStream_t s) {
  const dim3 grid(p.splits, p.H, p.B);
  if (p.io == 0)
    reduce_simt<__nv_bfloat16><<<grid, kRedThreads, 0, s>>>(
        p, static_cast<const __nv_bfloat16*>(K), static_cast<const __nv_bfloat16*>(V), partials,
        counters, out);
  else
    reduce_simt<float><<<grid, kRedThreads, 0, s>>>(p, static_cast<const float*>(K),
                                                    static_cast<const float*>(V), partials,
                                                    counters, out);
  return cudaGetLastError();
}

cudaError_t launch_apply_simt(const Problem& p, const void* Q, const float* S, const float* z,
                              void* O, cudaStream_t s) {
  const dim3 grid((p.N + kApplyTile - 1) / kApplyTile, p.H, p.B);
  if (p.io == 0)
    apply_simt<__nv_bfloat16><<<grid, kApplyThreads, 0, s>>>(
        p, static_cast<const __nv_bfloat16*>(Q), S, z, static_cast<__nv_bfloat16*>(O));
  else
    apply_simt<float><<<grid, kApplyThreads, 0, s>>>(p, static_cast<const float*>(Q), S, z,
                                                     static_cast<float*>(O));
  return cudaGetLastError();
}

}  // namespace la
