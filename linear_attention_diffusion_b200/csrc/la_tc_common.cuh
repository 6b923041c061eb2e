// Helpers shared by the tensor-core kernels (la_tc.cu, la_backward_tc.cu):
// the per-CTA RoPE table and token positions, packed bf16 conversions,
// shared-memory vector access, bounded flag waits, the split combine of the
// state partials, and the TMA tensor maps of [B][N][H*32] bf16 tensors.
// Everything has internal linkage: each translation unit gets its own copy.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "la_common.cuh"
#include "la_sm100.cuh"

namespace la {
namespace {

using namespace sm100;

constexpr int kGroupHeads = 4;
constexpr int kRopeTableMax = 768;  // float2 entries of the per-CTA RoPE table

enum : unsigned { kErrWait = 1u };

// ------------------------------------------------------------------ RoPE

// Per-CTA table of (cos, sin) for every position of the block: T frames x 4
// pairs (time), then Hh rows of 6 pairs (height) and W rows of 6 pairs
// (width), each of these rows padded to 8 entries so that every row starts on
// a 16-byte boundary and two pairs load as one 16-byte vector. Angles are
// formed and reduced to [-pi, pi] in double, then evaluated in float. When the
// table does not fit in shared memory the angles are evaluated per token
// instead.
struct RopeTable {
  int enabled;
  int on_the_fly;
};

__host__ __device__ inline int rope_table_entries(const Rope& r) {
  return 4 * r.T + 8 * r.Hh + 8 * r.W;
}

__device__ void build_rope_table(const Rope& r, float2* tab, int tid, int nthreads) {
  const int total = rope_table_entries(r);
  for (int i = tid; i < total; i += nthreads) {
    int pos, j;
    if (i < 4 * r.T) {
      pos = r.t_offset + i / 4;
      j = i % 4;
    } else if (i < 4 * r.T + 8 * r.Hh) {
      const int k = i - 4 * r.T;
      pos = k / 8;
      j = k % 8 < 6 ? 4 + k % 8 : -1;
    } else {
      const int k = i - 4 * r.T - 8 * r.Hh;
      pos = k / 8;
      j = k % 8 < 6 ? 10 + k % 8 : -1;
    }
    if (j < 0) {  // padding
      tab[i] = make_float2(0.0f, 0.0f);
      continue;
    }
    float cs, sn;
    rope_cos_sin(pos, r.inv_freq[j], cs, sn);
    tab[i] = make_float2(cs, sn);
  }
}

struct TokPos {
  int t, h, w;  // local frame, row, column of a token
};

__device__ __forceinline__ TokPos token_pos(const Rope& r, int n) {
  const int hw = n / r.W;
  const int t = hw / r.Hh;
  return {t, hw - t * r.Hh, n - hw * r.W};
}

// Position of token n + step from that of token n (raster order, step >= 0).
__device__ __forceinline__ void token_pos_advance(const Rope& r, TokPos& tp, int step) {
  tp.w += step;
  while (tp.w >= r.W) {
    tp.w -= r.W;
    if (++tp.h == r.Hh) {
      tp.h = 0;
      ++tp.t;
    }
  }
}

// RoPE feature-map variants a kernel is compiled for.
enum RopeMode : int { kNoRope = 0, kRopeTable = 1, kRopeOnTheFly = 2 };

// Segment (0 = time, 1 = height, 2 = width) and index inside it of pair j.
__host__ __device__ constexpr int pair_axis(int j) { return j < 4 ? 0 : (j < 10 ? 1 : 2); }
__host__ __device__ constexpr int pair_off(int j) { return j < 4 ? j : (j < 10 ? j - 4 : j - 10); }

// Table offsets of the three segments' rows for token position tp.
struct RopeBases {
  int t, h, w;
};
__device__ __forceinline__ RopeBases rope_bases(const Rope& r, const TokPos& tp) {
  return {tp.t * 4, 4 * r.T + tp.h * 8, 4 * r.T + 8 * r.Hh + tp.w * 8};
}

// (cos, sin) of the 8 pairs [8 kHalf, 8 kHalf + 8) of one token (16 dims of a
// head): from the table, four 16-byte loads (every row base is even).
template <int kHalf>
__device__ __forceinline__ void rope_table8(const float2* tab, const RopeBases& rb,
                                            float2 (&cs)[8]) {
  const float4* t4 = reinterpret_cast<const float4*>(tab);
  float4 v[4];
  if (kHalf == 0) {  // pairs 0-3: time; 4-7: height 0-3
    v[0] = t4[rb.t / 2];
    v[1] = t4[rb.t / 2 + 1];
    v[2] = t4[rb.h / 2];
    v[3] = t4[rb.h / 2 + 1];
  } else {           // pairs 8-9: height 4-5; 10-15: width 0-5
    v[0] = t4[rb.h / 2 + 2];
    v[1] = t4[rb.w / 2];
    v[2] = t4[rb.w / 2 + 1];
    v[3] = t4[rb.w / 2 + 2];
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    cs[2 * k] = make_float2(v[k].x, v[k].y);
    cs[2 * k + 1] = make_float2(v[k].z, v[k].w);
  }
}

// The same 8 pairs evaluated from the token's position (no table).
template <int kHalf>
__device__ __forceinline__ void rope_fly8(const Rope& r, const TokPos& tp, float2 (&cs)[8]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int j = 8 * kHalf + q;
    const int ax = j < 4 ? 0 : (j < 10 ? 1 : 2);
    const int pos = ax == 0 ? r.t_offset + tp.t : (ax == 1 ? tp.h : tp.w);
    rope_cos_sin(pos, r.inv_freq[j], cs[q].x, cs[q].y);
  }
}

// Rotate 8 interleaved pairs of x by (cos, sin): (x0, x1) -> (x0 c - x1 s, x0 s + x1 c).
__device__ __forceinline__ void rotate8(float (&x)[16], const float2 (&cs)[8]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float2 t = __fmul2_rn(make_float2(x[2 * q + 1], x[2 * q + 1]),
                                make_float2(-cs[q].y, cs[q].x));
    const float2 y = __ffma2_rn(make_float2(x[2 * q], x[2 * q]), cs[q], t);
    x[2 * q] = y.x;
    x[2 * q + 1] = y.y;
  }
}

// Barrier over `threads` threads of named barrier `id` that also ORs `pred`
// across them: every participant gets the same answer.
__device__ __forceinline__ bool bar_any(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&x)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
  uint4 u;
  u.x = pack_bf16x2(x[0], x[1]);
  u.y = pack_bf16x2(x[2], x[3]);
  u.z = pack_bf16x2(x[4], x[5]);
  u.w = pack_bf16x2(x[6], x[7]);
  return u;
}

// max(x, 0) on packed bf16 pairs: exact.
__device__ __forceinline__ uint32_t relu_bf16x2(uint32_t v) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(0u));
  return r;
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// Wait until *flag != 0, for at most kWaitLimitNs; on timeout raise the abort
// flag and `err` and return false.
__device__ __forceinline__ bool spin_flag(const unsigned* flag, volatile int* abort_flag,
                                          unsigned* err) {
  if (ld_acquire_gpu(flag) != 0u) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (ld_acquire_gpu(flag) != 0u) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(err, kErrWait);
      return false;
    }
    __nanosleep(64);
  }
}

// Sum of the head group's split partials in split order (+ carry), written to
// StateOut, by the kThreads math threads (thread index mt) of the CTA that
// arrived last. Each thread owns
// at most kPerThread float4 columns and issues the loads of all of them for 4
// splits at once before adding, so the combine costs one L2 round trip per 4
// splits.
template <int kThreads, int kHeads = kGroupHeads>
__device__ __forceinline__ void combine_from_global(const Problem& p, int b, int h0, int mt,
                                                    const float* partials, const StateOut& out,
                                                    float* s_smem = nullptr,
                                                    float* z_smem = nullptr) {
  constexpr int kVec = kStateFloats / 4;                     // 264 float4 per head
  constexpr int kPerThread = (kHeads * kVec + kThreads - 1) / kThreads;
  const int heads = min(kHeads, p.H - h0);
  const size_t cidx = static_cast<size_t>(b) * p.H + h0;
  float4 acc[kPerThread];
  const float* src[kPerThread];
  bool own[kPerThread];
#pragma unroll
  for (int u = 0; u < kPerThread; ++u) {
    const int v = mt + u * kThreads;
    own[u] = v < heads * kVec;
    const int hh = own[u] ? v / kVec : 0, i = own[u] ? (v - hh * kVec) * 4 : 0;
    src[u] = partials + (cidx + hh) * p.splits * kStateFloats + i;
    acc[u] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  }
  for (int s0 = 0; s0 < p.splits; s0 += 4) {
    float4 t[kPerThread][4];
#pragma unroll
    for (int u = 0; u < kPerThread; ++u)
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (own[u] && s0 + k < p.splits)
          t[u][k] = __ldcg(reinterpret_cast<const float4*>(src[u] + static_cast<size_t>(s0 + k) * kStateFloats));
#pragma unroll
    for (int u = 0; u < kPerThread; ++u)
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (own[u] && s0 + k < p.splits) {
          acc[u].x += t[u][k].x;
          acc[u].y += t[u][k].y;
          acc[u].z += t[u][k].z;
          acc[u].w += t[u][k].w;
        }
  }
#pragma unroll
  for (int u = 0; u < kPerThread; ++u) {
    if (!own[u]) continue;
    const int v = mt + u * kThreads;
    const int hh = v / kVec, i = (v - hh * kVec) * 4;
    const size_t bh = cidx + hh;
    const bool is_s = i < kD * kD;
    const size_t o = is_s ? bh * kD * kD + i : bh * kD + (i - kD * kD);
    const float* c = is_s ? out.carry_S : out.carry_z;
    float4 r = acc[u];
    if (c != nullptr) {
      const float4 cv = *reinterpret_cast<const float4*>(c + o);
      r = make_float4(cv.x + r.x, cv.y + r.y, cv.z + r.z, cv.w + r.w);
    }
    float* d1 = is_s ? out.out1_S : out.out1_z;
    float* d2 = is_s ? out.out2_S : out.out2_z;
    if (d1 != nullptr) *reinterpret_cast<float4*>(d1 + o) = r;
    if (d2 != nullptr) *reinterpret_cast<float4*>(d2 + o) = r;
    // shared-memory copy: S as [head][32][32], z as [head][32]
    if (is_s && s_smem != nullptr) *reinterpret_cast<float4*>(s_smem + hh * kD * kD + i) = r;
    if (!is_s && z_smem != nullptr) *reinterpret_cast<float4*>(z_smem + hh * kD + i - kD * kD) = r;
  }
}

// Wait until *counter >= target (acquire), for at most kWaitLimitNs; on
// timeout raise the abort flag and `err` and return false.
__device__ __forceinline__ bool spin_count(const unsigned* counter, unsigned target,
                                           volatile int* abort_flag, unsigned* err) {
  const uint64_t t0 = globaltimer_ns();
  while (ld_acquire_gpu(counter) < target) {
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(err, kErrWait);
      return false;
    }
    __nanosleep(32);
  }
  return true;
}

// ------------------------------------------------------------------ host

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_err = cudaSuccess;

cudaError_t get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    g_encode_err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (g_encode_err == cudaSuccess && (q != cudaDriverEntryPointSuccess || fn == nullptr))
      g_encode_err = cudaErrorNotSupported;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode_err;
}

// [B][N][H*32] bf16 viewed as a 3D tensor; box = 64 dims x rows tokens x 1.
cudaError_t make_map(CUtensorMap* m, const void* base, const Problem& p, int rows) {
  cudaError_t e = get_encoder();
  if (e != cudaSuccess) return e;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(p.H) * kD, static_cast<cuuint64_t>(p.N),
                              static_cast<cuuint64_t>(p.B)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(p.H) * kD * 2,
                                 static_cast<cuuint64_t>(p.N) * p.H * kD * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

RopeTable rope_table_for(const Problem& p) {
  RopeTable rt{};
  rt.enabled = p.rope.enabled;
  if (rt.enabled) rt.on_the_fly = rope_table_entries(p.rope) > kRopeTableMax;
  return rt;
}

constexpr int kMaxDev = 64;
bool g_attr_set[16][kMaxDev] = {};  // [kernel variant][device]
std::mutex g_attr_mu;

// Opt-in to `bytes` of dynamic shared memory for kernel variant `which` (< 16)
// on the current device, once per (variant, device).
cudaError_t ensure_smem_attr(int which, const void* fn, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_attr_mu);
  if (!g_attr_set[which][dev]) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    g_attr_set[which][dev] = true;
  }
  return cudaSuccess;
}

int rope_mode(const RopeTable& rt) {
  return !rt.enabled ? kNoRope : (rt.on_the_fly ? kRopeOnTheFly : kRopeTable);
}

}  // namespace
}  // namespace la
