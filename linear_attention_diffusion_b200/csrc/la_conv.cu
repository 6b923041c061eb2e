// Temporal depth-wise convolution of the spatial-temporal Mix-FFN with the
// block-causal conv cache ("SANA-Video: Efficient Video Generation with Block
// Linear Diffusion Transformer", Stage 2: a 1D temporal convolution joins the
// Mix-FFN through a shortcut; section 4: the conv cache f, the last frame of
// the temporal convolution, is the third part of the KV cache):
//
//   y[t] = x[t] + b + w[c,0] x[t-1] + w[c,1] x[t] + w[c,2] x[t+1]
//
// per channel c, with x[-1] = f (the previous block's last frame, zero when
// absent) and x[T] = 0 (later blocks are never seen); the next cache is
// x[T-1]. x, y [B][T][Hh*W][C] channels last; f [B][Hh*W][C].
//
// The operation streams x once and writes y once. A CTA owns 256 columns
// (pixel, 8 channels) of one batch element; their part of a frame is one
// contiguous slab of x, which a ring of kSlots one-dimensional bulk copies
// (cp.async.bulk, completing on mbarriers) keeps in flight ahead of the
// threads. Each thread slides a three-frame window of its column down the
// time axis in registers and stores y with 16-byte coalesced stores. Each
// column belongs to one thread and every frame is copied in before any of
// it is overwritten, so y may be x and f_out may be f_in.
#include "la_common.cuh"
#include "la_sm100.cuh"

namespace la {

// Device error word of the convolution (a bounded wait that gave up).
__device__ unsigned g_conv_error;

namespace {

using namespace sm100;

constexpr int kConvThreads = 256;  // columns per CTA
constexpr int kSlots = 8;          // frames in flight per CTA
enum : unsigned { kConvErrWait = 1u };

template <typename T>
__global__ void __launch_bounds__(kConvThreads)
temporal_conv_kernel(ConvProblem cp, const T* x, const float* __restrict__ w,
                     const float* __restrict__ bias, const T* f_in, T* f_out, T* y) {
  constexpr int kColBytes = 8 * sizeof(T);
  extern __shared__ __align__(128) uint8_t ring[];   // [kSlots][kConvThreads * kColBytes]
  __shared__ uint64_t full[kSlots];
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int cvecs = cp.C / 8;
  const long long cols_b = static_cast<long long>(cp.HW) * cvecs;  // columns per batch element
  const long long col0 = static_cast<long long>(blockIdx.x) * kConvThreads;
  const int b = blockIdx.y;
  const int ncols = static_cast<int>(min(static_cast<long long>(kConvThreads), cols_b - col0));
  const uint32_t slab = static_cast<uint32_t>(ncols) * kColBytes;  // multiple of 16
  const size_t frame = static_cast<size_t>(cp.HW) * cp.C;          // elements per frame
  const T* xb = x + static_cast<size_t>(b) * cp.T * frame + col0 * 8;
  const int nT = cp.T;

  if (tid == 0) {
    for (int i = 0; i < kSlots; ++i) mbar_init(&full[i], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int t) {  // thread 0: copy frame t into its slot
    uint64_t* bar = &full[t % kSlots];
    mbar_arrive_expect_tx(bar, slab);
    bulk_load(ring + (t % kSlots) * kConvThreads * kColBytes, xb + static_cast<size_t>(t) * frame,
              slab, bar);
  };
  if (tid == 0)
    for (int t = 0; t < min(kSlots, nT); ++t) issue(t);

  const bool own = tid < ncols;
  const long long col = col0 + tid;
  const int c0 = static_cast<int>(col % cvecs) * 8;
  float w0[8], w1[8], w2[8], bb[8], prev[8], cur[8], nxt[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) prev[i] = cur[i] = nxt[i] = w0[i] = w1[i] = w2[i] = bb[i] = 0.0f;
  const size_t fofs = (static_cast<size_t>(b) * cp.HW * cvecs + col) * 8;
  if (own) {
    const float4* wp = reinterpret_cast<const float4*>(w + static_cast<size_t>(c0) * 3);
    float t24[24];
#pragma unroll
    for (int i = 0; i < 6; ++i) {
      const float4 v = __ldg(wp + i);
      t24[4 * i] = v.x; t24[4 * i + 1] = v.y; t24[4 * i + 2] = v.z; t24[4 * i + 3] = v.w;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w0[i] = t24[3 * i];
      w1[i] = t24[3 * i + 1];
      w2[i] = t24[3 * i + 2];
      bb[i] = bias != nullptr ? __ldg(bias + c0 + i) : 0.0f;
    }
    if (f_in != nullptr) {  // plain load: f_out may be f_in
      if (sizeof(T) == 2) {
        const uint4 u = *reinterpret_cast<const uint4*>(f_in + fofs);
        const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          prev[2 * i] = __uint_as_float(q[i] << 16);
          prev[2 * i + 1] = __uint_as_float(q[i] & 0xffff0000u);
        }
      } else {
        const float4 a = reinterpret_cast<const float4*>(f_in + fofs)[0];
        const float4 c = reinterpret_cast<const float4*>(f_in + fofs)[1];
        prev[0] = a.x; prev[1] = a.y; prev[2] = a.z; prev[3] = a.w;
        prev[4] = c.x; prev[5] = c.y; prev[6] = c.z; prev[7] = c.w;
      }
    }
  }
  auto read_slot = [&](int t, float (&v)[8]) {
    const uint8_t* src = ring + (t % kSlots) * kConvThreads * kColBytes + tid * kColBytes;
    if (sizeof(T) == 2) {
      const uint4 u = *reinterpret_cast<const uint4*>(src);
      const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(q[i] << 16);
        v[2 * i + 1] = __uint_as_float(q[i] & 0xffff0000u);
      }
    } else {
      const float4 a = reinterpret_cast<const float4*>(src)[0];
      const float4 c = reinterpret_cast<const float4*>(src)[1];
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
    }
  };

  // frame 0 into `cur`; then its slot takes frame kSlots
  bool ok = mbar_wait(&full[0], 0, &abort_flag, &g_conv_error, kConvErrWait);
  if (ok && own) read_slot(0, cur);
  int issued = min(kSlots, nT);
  for (int t = 0; t < nT; ++t) {
    // every thread is done with frame t (the slot of frame t + kSlots)
    ok = !__syncthreads_or(!ok || abort_flag);
    if (!ok) break;
    if (tid == 0 && t + kSlots < nT) {
      fence_proxy_async_smem();
      issue(t + kSlots);
      issued = t + kSlots + 1;
    }
    if (t + 1 < nT) {
      ok = mbar_wait(&full[(t + 1) % kSlots], ((t + 1) / kSlots) & 1, &abort_flag, &g_conv_error,
                     kConvErrWait);
      if (ok && own) read_slot(t + 1, nxt);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) nxt[i] = 0.0f;
    }
    if (ok && own) {
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        o[i] = fmaf(w2[i], nxt[i], fmaf(w1[i], cur[i], fmaf(w0[i], prev[i], cur[i] + bb[i])));
      store_row<8>(y + (static_cast<size_t>(b) * nT + t) * frame + col * 8, o);
      if (t == nT - 1 && f_out != nullptr) store_row<8>(f_out + fofs, cur);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      prev[i] = cur[i];
      cur[i] = nxt[i];
    }
  }
  // copies still in flight land before the CTA leaves (bounded)
  if (tid == 0)
    for (int t = max(0, issued - kSlots); t < issued; ++t)  // the latest copy of each slot
      mbar_drain(&full[t % kSlots], (t / kSlots) & 1, &g_conv_error, kConvErrWait);
}

}  // namespace

cudaError_t launch_temporal_conv(const ConvProblem& cp, const void* x, const float* w,
                                 const float* bias, const void* f_in, void* f_out, void* y,
                                 cudaStream_t s) {
  const long long cols_b = static_cast<long long>(cp.HW) * (cp.C / 8);
  const long long bx = (cols_b + kConvThreads - 1) / kConvThreads;
  if (bx > 0x7fffffffLL || cp.B > 65535) return cudaErrorInvalidConfiguration;
  if (bx == 0 || cp.B == 0 || cp.T == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(bx), static_cast<unsigned>(cp.B));
  if (cp.io == LA_IO_BF16) {
    const int smem = kSlots * kConvThreads * 16;
    temporal_conv_kernel<__nv_bfloat16><<<grid, kConvThreads, smem, s>>>(
        cp, static_cast<const __nv_bfloat16*>(x), w, bias,
        static_cast<const __nv_bfloat16*>(f_in), static_cast<__nv_bfloat16*>(f_out),
        static_cast<__nv_bfloat16*>(y));
  } else {
    const int smem = kSlots * kConvThreads * 32;
    cudaError_t e = cudaFuncSetAttribute(temporal_conv_kernel<float>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    temporal_conv_kernel<float><<<grid, kConvThreads, smem, s>>>(
        cp, static_cast<const float*>(x), w, bias, static_cast<const float*>(f_in),
        static_cast<float*>(f_out), static_cast<float*>(y));
  }
  return cudaGetLastError();
}

cudaError_t read_device_error_conv(unsigned* code, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(code, g_conv_error, sizeof(unsigned));
  if (e == cudaSuccess && reset) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_conv_error, &zero, sizeof(unsigned));
  }
  return e;
}

}  // namespace la
