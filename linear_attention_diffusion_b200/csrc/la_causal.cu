// Token-causal linear attention: query n sees keys 0..n (SANA-Video: Efficient
// Video Generation with Block Linear Diffusion Transformer, section 2.3, with
// the sum over earlier j read at token granularity; a block of one token in
// the block-causal mode is the same thing). With a carried state (S0, z0):
//
//   S_n = S0 + sum_{j<=n} phi(k_j)^T v_j,   z_n = z0 + sum_{j<=n} ReLU(k_j)
//   O_n = phi(q_n) S_n / (ReLU(q_n) . z_n + eps)
//
// Two launches. The state reduce leaves each token split's partial state in
// the workspace (its combine is skipped). This kernel then runs one CTA per
// (split, head, batch): it starts from S0 plus the partials of the earlier
// splits, summed in split order, and walks its tokens in chunks of 32:
//
//   num_i = phi(q_i) R_S + sum_{j<=i in chunk} (phi(q_i) . phi(k_j)) v_j
//   den_i = ReLU(q_i) . (R_z + sum_{j<=i in chunk} ReLU(k_j)) + eps
//   R    += the chunk's own state
//
// so the work per token is O(D^2 + chunk D) instead of the quadratic form's
// O(N D). The last CTA of each head to read the carry folds the whole
// sequence into it when asked (update = 1). CUDA cores, float32 arithmetic,
// bf16 or float32 I/O.
#include "la_common.cuh"

namespace la {
namespace {

constexpr int kCT = 32;         // tokens per chunk
constexpr int kCThreads = 256;  // thread t: row t / 8 of a chunk, dims [(t % 8) * 4, +4)

__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&x)[4]) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  x[0] = __uint_as_float(u.x << 16);
  x[1] = __uint_as_float(u.x & 0xffff0000u);
  x[2] = __uint_as_float(u.y << 16);
  x[3] = __uint_as_float(u.y & 0xffff0000u);
}
__device__ __forceinline__ void load4(const float* p, float (&x)[4]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, const float (&x)[4]) {
  uint2 u;
  u.x = pack_bf16x2(x[0], x[1]);
  u.y = pack_bf16x2(x[2], x[3]);
  *reinterpret_cast<uint2*>(p) = u;
}
__device__ __forceinline__ void store4(float* p, const float (&x)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
}

template <typename T>
__device__ __forceinline__ void load_row4(const Problem& p, const T* Q, const T* K, const T* V,
                                          int b, int h, int n, bool row, int d0, float (&q)[4],
                                          float (&k)[4], float (&v)[4]) {
  if (row) {
    const size_t off = ((static_cast<size_t>(b) * p.N + n) * p.H + h) * kD + d0;
    load4(Q + off, q);
    load4(K + off, k);
    load4(V + off, v);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = k[i] = v[i] = 0.0f;
  }
}

// Shared-memory layout: every product below reads one 16-byte vector per
// four FMAs (rows padded to 36 floats keep the vectors aligned and spread
// the rows of a warp over the banks).
template <typename T>
__global__ void __launch_bounds__(kCThreads)
causal_simt(const Problem p, const T* __restrict__ Q, const T* __restrict__ K,
            const T* __restrict__ V, const float* __restrict__ partials, float* S_carry,
            float* z_carry, int update, unsigned* counters, T* __restrict__ O) {
  __shared__ __align__(16) float Rs[kD][kD + 4];      // running state S[d][e]
  __shared__ __align__(16) float Rz[kD];              // running key sum
  __shared__ __align__(16) float phq[kCT][kD + 4];    // phi(q)[i][d]
  __shared__ __align__(16) float phkT[kD][kCT + 4];   // phi(k)[j][d], transposed: [d][j]
  __shared__ __align__(16) float kcum[kCT][kD + 4];   // ReLU(k), then its prefix over rows
  __shared__ __align__(16) float vs[kCT][kD + 4];     // v[j][e]
  __shared__ __align__(16) float A[kCT][kCT + 4];     // phi(q_i) . phi(k_j) for j <= i, else 0
  __shared__ int s_last;

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const size_t bh = static_cast<size_t>(b) * p.H + h;

  // ---- starting state: carry + the earlier splits' partials, in split order
  for (int i = tid; i < kStateFloats; i += kCThreads) {
    float acc = 0.0f;
    if (S_carry != nullptr) acc = i < kD * kD ? S_carry[bh * kD * kD + i] : z_carry[bh * kD + i - kD * kD];
    const float* src = partials + bh * p.splits * kStateFloats + i;
    for (int s = 0; s < split; ++s) acc += __ldcg(src + static_cast<size_t>(s) * kStateFloats);
    if (i < kD * kD) Rs[i / kD][i % kD] = acc;
    else Rz[i - kD * kD] = acc;
  }
  __syncthreads();

  // ---- the last CTA of the head to have read the carry folds the sequence in
  if (update) {
    if (tid == 0) {
      __threadfence();
      const unsigned prev = atomicAdd(&counters[bh], 1u);
      s_last = prev == static_cast<unsigned>(p.splits - 1);
      if (s_last) __threadfence();
    }
    __syncthreads();
    if (s_last) {
      for (int i = tid; i < kStateFloats; i += kCThreads) {
        float* dst = i < kD * kD ? S_carry + bh * kD * kD + i : z_carry + bh * kD + i - kD * kD;
        float acc = *dst;
        const float* src = partials + bh * p.splits * kStateFloats + i;
        for (int s = 0; s < p.splits; ++s) acc += __ldcg(src + static_cast<size_t>(s) * kStateFloats);
        *dst = acc;
      }
      if (tid == 0) counters[bh] = 0u;
    }
  }

  const int n_begin = split * p.chunk;
  const int n_end = min(p.N, n_begin + p.chunk);
  const int r = tid >> 3, d0 = (tid & 7) * 4;  // token row, first of 4 dims (also e0, j0)
  const int warp = tid >> 5, lane = tid & 31;

  float q[4], k[4], v[4];
  if (n_begin < n_end) load_row4(p, Q, K, V, b, h, n_begin + r, n_begin + r < n_end, d0, q, k, v);
  for (int n0 = n_begin; n0 < n_end; n0 += kCT) {
    const int n = n0 + r;
    const bool row = n < n_end;
    float qp[4], pq[4], pk[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      qp[i] = fmaxf(q[i], 0.0f);
      pq[i] = qp[i];
      k[i] = fmaxf(k[i], 0.0f);
      pk[i] = k[i];
    }
    if (p.rope.enabled && row) {
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        const int j = d0 / 2 + pr;
        float c, s;
        rope_cos_sin(rope_pos(p.rope, n, p.rope.axis[j]), p.rope.inv_freq[j], c, s);
        const float a0 = pq[2 * pr], a1 = pq[2 * pr + 1];
        pq[2 * pr] = fmaf(a0, c, -a1 * s);
        pq[2 * pr + 1] = fmaf(a0, s, a1 * c);
        const float b0 = pk[2 * pr], b1 = pk[2 * pr + 1];
        pk[2 * pr] = fmaf(b0, c, -b1 * s);
        pk[2 * pr + 1] = fmaf(b0, s, b1 * c);
      }
    }
    *reinterpret_cast<float4*>(&phq[r][d0]) = make_float4(pq[0], pq[1], pq[2], pq[3]);
    *reinterpret_cast<float4*>(&kcum[r][d0]) = make_float4(k[0], k[1], k[2], k[3]);
    *reinterpret_cast<float4*>(&vs[r][d0]) = make_float4(v[0], v[1], v[2], v[3]);
#pragma unroll
    for (int i = 0; i < 4; ++i) phkT[d0 + i][r] = pk[i];
    __syncthreads();
    // the next chunk's loads are in flight during this chunk's arithmetic
    if (n0 + kCT < n_end) load_row4(p, Q, K, V, b, h, n + kCT, n + kCT < n_end, d0, q, k, v);

    // ---- A[r][j0 .. j0+4), masked to j <= r
    {
      float a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      if (d0 <= r) {
#pragma unroll
        for (int d = 0; d < kD; d += 4) {
          const float4 x = *reinterpret_cast<const float4*>(&phq[r][d]);
          const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int dd = 0; dd < 4; ++dd) {
            const float4 y = *reinterpret_cast<const float4*>(&phkT[d + dd][d0]);
            a[0] = fmaf(xs[dd], y.x, a[0]);
            a[1] = fmaf(xs[dd], y.y, a[1]);
            a[2] = fmaf(xs[dd], y.z, a[2]);
            a[3] = fmaf(xs[dd], y.w, a[3]);
          }
        }
      }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) a[jj] = d0 + jj <= r ? a[jj] : 0.0f;
      *reinterpret_cast<float4*>(&A[r][d0]) = make_float4(a[0], a[1], a[2], a[3]);
    }
    // ---- inclusive prefix of ReLU(k) over the rows: warp w scans dims 4w..4w+3
    {
      float4 c = *reinterpret_cast<const float4*>(&kcum[lane][warp * 4]);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float4 u = make_float4(__shfl_up_sync(0xffffffffu, c.x, o),
                                     __shfl_up_sync(0xffffffffu, c.y, o),
                                     __shfl_up_sync(0xffffffffu, c.z, o),
                                     __shfl_up_sync(0xffffffffu, c.w, o));
        if (lane >= o) c = make_float4(c.x + u.x, c.y + u.y, c.z + u.z, c.w + u.w);
      }
      __syncwarp();
      *reinterpret_cast<float4*>(&kcum[lane][warp * 4]) = c;
    }
    __syncthreads();

    // ---- output of row r, dims [d0, d0 + 4)
    {
      float num[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int d = 0; d < kD; d += 4) {
        const float4 x = *reinterpret_cast<const float4*>(&phq[r][d]);
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int dd = 0; dd < 4; ++dd) {
          const float4 y = *reinterpret_cast<const float4*>(&Rs[d + dd][d0]);
          num[0] = fmaf(xs[dd], y.x, num[0]);
          num[1] = fmaf(xs[dd], y.y, num[1]);
          num[2] = fmaf(xs[dd], y.z, num[2]);
          num[3] = fmaf(xs[dd], y.w, num[3]);
        }
      }
      for (int j = 0; j <= r; j += 4) {
        const float4 x = *reinterpret_cast<const float4*>(&A[r][j]);  // zero beyond r
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float4 y = *reinterpret_cast<const float4*>(&vs[j + jj][d0]);
          num[0] = fmaf(xs[jj], y.x, num[0]);
          num[1] = fmaf(xs[jj], y.y, num[1]);
          num[2] = fmaf(xs[jj], y.z, num[2]);
          num[3] = fmaf(xs[jj], y.w, num[3]);
        }
      }
      const float4 rz = *reinterpret_cast<const float4*>(&Rz[d0]);
      const float4 kc = *reinterpret_cast<const float4*>(&kcum[r][d0]);
      float den = qp[0] * (rz.x + kc.x);
      den = fmaf(qp[1], rz.y + kc.y, den);
      den = fmaf(qp[2], rz.z + kc.z, den);
      den = fmaf(qp[3], rz.w + kc.w, den);
      den += __shfl_xor_sync(0xffffffffu, den, 1);
      den += __shfl_xor_sync(0xffffffffu, den, 2);
      den += __shfl_xor_sync(0xffffffffu, den, 4);
      den += p.eps;
      if (row) {
        float o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] = num[e] / den;
        store4(O + ((static_cast<size_t>(b) * p.N + n) * p.H + h) * kD + d0, o);
      }
    }
    __syncthreads();

    // ---- R += the chunk's state (rows beyond the split are zero)
    {
      const int d = r;  // state row d, columns [d0, d0 + 4)
      float4 acc = *reinterpret_cast<const float4*>(&Rs[d][d0]);
#pragma unroll
      for (int j = 0; j < kCT; j += 4) {
        const float4 x = *reinterpret_cast<const float4*>(&phkT[d][j]);
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float4 y = *reinterpret_cast<const float4*>(&vs[j + jj][d0]);
          acc.x = fmaf(xs[jj], y.x, acc.x);
          acc.y = fmaf(xs[jj], y.y, acc.y);
          acc.z = fmaf(xs[jj], y.z, acc.z);
          acc.w = fmaf(xs[jj], y.w, acc.w);
        }
      }
      *reinterpret_cast<float4*>(&Rs[d][d0]) = acc;
      if (tid < kD) Rz[tid] += kcum[kCT - 1][tid];
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_causal(const Problem& p, const void* Q, const void* K, const void* V,
                          const float* partials, float* S_carry, float* z_carry, int update,
                          unsigned* counters, void* O, cudaStream_t s) {
  const dim3 grid(p.splits, p.H, p.B);
  if (p.io == LA_IO_BF16)
    causal_simt<__nv_bfloat16><<<grid, kCThreads, 0, s>>>(
        p, static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K),
        static_cast<const __nv_bfloat16*>(V), partials, S_carry, z_carry, update, counters,
        static_cast<__nv_bfloat16*>(O));
  else
    causal_simt<float><<<grid, kCThreads, 0, s>>>(
        p, static_cast<const float*>(Q), static_cast<const float*>(K),
        static_cast<const float*>(V), partials, S_carry, z_carry, update, counters,
        static_cast<float*>(O));
  return cudaGetLastError();
}

}  // namespace la
