// Tensor-core (tcgen05) kernels of the bf16 path: the state reduce and the
// apply. Both stream their operands HBM -> shared memory with TMA, run the
// element-wise feature map (ReLU, 3D RoPE) and the key sum / denominator on
// CUDA cores in shared memory, and leave the 32x32 contractions to tcgen05.mma
// with fp32 accumulators in tensor memory.
//
// What is computed follows "SANA-Video: Efficient Video Generation with Block
// Linear Diffusion Transformer", sections 2.1-2.2 (state computed once, RoPE
// after ReLU, unrotated denominator), and the Sana Linear DiT ("Sana: Efficient
// High-Resolution Image Synthesis with Linear Diffusion Transformers", section
// 模型架构 item 2).
//
// Layout of the work: a CTA owns a group of 4 heads (128 feature dims, 256
// bytes of a token row) of one batch element and a contiguous token range.
//
//   reduce: per 64-token stage, A = phi(K)^T (M = 128 dims, MN-major) and
//           B = V (N = 128 dims, MN-major), K = tokens; one 128x128 fp32
//           accumulator whose four 32x32 diagonal blocks are the heads'
//           states (the off-diagonal blocks are discarded; the tensor pipe has
//           ample headroom at this arithmetic intensity).
//   apply:  per 128-token tile and head, A = phi(Q) (M = 128 tokens, K = 32
//           dims, K-major, straight from the TMA tile) and B = S^T (bf16,
//           K-major); D = 128 x 32 fp32 per head in tensor memory.
//
// Warp roles (320 threads): warp 0 issues TMA loads, warp 1 allocates tensor
// memory and issues the MMAs (one elected lane), warps 2..9 transform tiles
// in shared memory and run the epilogue. Every mbarrier wait is bounded; a
// wait that gives up raises the library's device error word and the CTA
// drains its copies and MMAs and frees its tensor memory before returning.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <utility>

#include "la_common.cuh"
#include "la_sm100.cuh"

namespace la {

// Device-wide error word: bit 0 = a bounded wait of a tensor-core kernel gave
// up. Read (and cleared) by la_device_error().
__device__ unsigned g_tc_error;

namespace {

using namespace sm100;

constexpr int kApWG = 3;            // apply: math warpgroups, one tile each in turn
constexpr int kThreads = 64 + 128 * kApWG;  // apply: TMA warp, MMA warp, math warpgroups
constexpr int kMathThreads = 128 * kApWG;
constexpr int kRedMath = 512;       // reduce: 16 math warps
constexpr int kRedThreads = 64 + kRedMath;
constexpr int kGroupHeads = 4;
constexpr int kRopeTableMax = 1536;  // float2 entries of the per-CTA RoPE table

enum : unsigned { kErrWait = 1u };

// ------------------------------------------------------------------ RoPE

// Per-CTA table of (cos, sin) for every position of the block: T frames x 4
// pairs (time), then Hh x 6 pairs (height), then W x 6 pairs (width). Angles
// are formed and reduced to [-pi, pi] in double, then evaluated in float. When
// the table does not fit in shared memory the angles are evaluated per token
// instead.
struct RopeTable {
  int enabled;
  int on_the_fly;
};

__host__ __device__ inline int rope_table_entries(const Rope& r) {
  return 4 * r.T + 6 * r.Hh + 6 * r.W;
}

__device__ void build_rope_table(const Rope& r, float2* tab, int tid, int nthreads) {
  const int total = rope_table_entries(r);
  for (int i = tid; i < total; i += nthreads) {
    int pos, j;
    if (i < 4 * r.T) {
      pos = r.t_offset + i / 4;
      j = i % 4;
    } else if (i < 4 * r.T + 6 * r.Hh) {
      const int k = i - 4 * r.T;
      pos = k / 6;
      j = 4 + k % 6;
    } else {
      const int k = i - 4 * r.T - 6 * r.Hh;
      pos = k / 6;
      j = 10 + k % 6;
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
  return {tp.t * 4, 4 * r.T + tp.h * 6, 4 * r.T + 6 * r.Hh + tp.w * 6};
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

// ================================================================ reduce

constexpr int kRedT = 64;                          // tokens per stage
constexpr int kRedStages = 5;
constexpr int kRedBox = kRedT * 128;               // bytes of one [64 tokens][64 dims] box
constexpr int kRedStageBytes = 4 * kRedBox;        // K box 0, K box 1, V box 0, V box 1
constexpr int kRedTmemCols = 128;

struct RedSmem {
  // offsets from the 1024-aligned base
  static constexpr int stages = 0;
  static constexpr int zred = stages + kRedStages * kRedStageBytes;    // [512][8] float
  static constexpr int rope = zred + kRedMath * 8 * 4;                 // float2[kRopeTableMax]
  static constexpr int bars = rope + kRopeTableMax * 8;                // mbarriers
  static constexpr int nbars = 3 * kRedStages + 3;
  static constexpr int misc = bars + nbars * 8;                        // tmem base, abort
  static constexpr int bytes = misc + 16;
};
constexpr int kRedSmemBytes = RedSmem::bytes + 1024;

// Second phase of the reduce for a group of 4 heads: the CTA that arrives
// last for the group copies the group's partials (contiguous: heads x splits
// x 1056 floats) into shared memory with bulk copies, sums them in split
// order, adds the carry when given, writes the outputs and re-zeroes the
// counter. Falls back to the register version when they do not fit.
__device__ __forceinline__ void finish_reduce_bulk(const Problem& p, int b, int h0,
                                                   const float* partials, unsigned* counters,
                                                   const StateOut& out, uint8_t* smem,
                                                   uint64_t* comb_full, volatile int* abort_flag) {
  const int heads = min(kGroupHeads, p.H - h0);
  const uint32_t per_head = static_cast<uint32_t>(p.splits) * kStateFloats * 4;
  if (static_cast<size_t>(heads) * per_head > static_cast<size_t>(kRedStages) * kRedStageBytes) {
    finish_reduce(p, b, h0, kGroupHeads, partials, counters, out);
    return;
  }
  __shared__ int s_last;
  // The CTA barrier orders every thread's partial stores before thread 0's
  // release fence; the CTA that arrives last acquires all groups' stores.
  __syncthreads();
  const size_t cidx = static_cast<size_t>(b) * p.H + h0;
  if (threadIdx.x == 0) {
    fence_acq_rel_gpu();
    const unsigned prev = atomicAdd(&counters[cidx], 1u);
    s_last = prev == static_cast<unsigned>(p.splits - 1);
    if (s_last) fence_acq_rel_gpu();
  }
  __syncthreads();
  if (!s_last) return;
  const float* src = partials + cidx * p.splits * kStateFloats;
  float* buf = reinterpret_cast<float*>(smem + RedSmem::stages);
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(comb_full, heads * per_head);
    for (int hh = 0; hh < heads; ++hh)
      bulk_load(reinterpret_cast<uint8_t*>(buf) + hh * per_head,
                reinterpret_cast<const uint8_t*>(src) + hh * per_head, per_head, comb_full);
  }
  const bool ok = mbar_wait(comb_full, 0, abort_flag, &g_tc_error, kErrWait);
  if (!ok) return;  // the counter stays raised: the device error word reports it
  constexpr int kVec = kStateFloats / 4;
  for (int v = threadIdx.x; v < heads * kVec; v += blockDim.x) {
    const int hh = v / kVec, i = (v - hh * kVec) * 4;
    const float4* col = reinterpret_cast<const float4*>(buf + hh * p.splits * kStateFloats + i);
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int sp = 0; sp < p.splits; ++sp) {
      const float4 t = col[sp * (kStateFloats / 4)];
      acc.x += t.x;
      acc.y += t.y;
      acc.z += t.z;
      acc.w += t.w;
    }
    const size_t bh = cidx + hh;
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
  if (threadIdx.x == 0) counters[cidx] = 0u;
}

template <int kRope>
__global__ void __launch_bounds__(kRedThreads, 1)
reduce_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
          const Problem p, const RopeTable rt, float* partials, unsigned* counters,
          const StateOut out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + RedSmem::bars);
  uint64_t* ready = full + kRedStages;
  uint64_t* empty = ready + kRedStages;
  uint64_t* acc_full = empty + kRedStages;
  uint64_t* mma_done = acc_full + 1;
  uint64_t* comb_full = mma_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + RedSmem::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + RedSmem::misc + 4);
  float* zred = reinterpret_cast<float*>(smem + RedSmem::zred);
  float2* rope_tab = reinterpret_cast<float2*>(smem + RedSmem::rope);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, group = blockIdx.y, b = blockIdx.z;
  const int h0 = group * kGroupHeads;
  const int n_begin = split * p.chunk;
  const int n_end = min(p.N, n_begin + p.chunk);
  const int ntiles = n_end > n_begin ? (n_end - n_begin + kRedT - 1) / kRedT : 0;

  if (tid == 0) {
    for (int s = 0; s < kRedStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ready[s], kRedMath);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(mma_done, 1);
    mbar_init(comb_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kRedTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (kRope == kRopeTable && tid >= 64) build_rope_table(p.rope, rope_tab, tid - 64, kRedMath);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);
  // Everything above overlaps the previous kernel's tail; global memory is
  // touched only after it has completed. Then the next kernel may launch.
  pdl_wait();
  if (tid == 0) pdl_trigger();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % kRedStages;
        const uint32_t ph = (i / kRedStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, &g_tc_error, kErrWait)) break;
        mbar_arrive_expect_tx(&full[s], kRedStageBytes);
        uint8_t* st = smem + RedSmem::stages + s * kRedStageBytes;
        const int y = n_begin + i * kRedT;
        tma_load_3d(st, &tm_k, &full[s], h0 * 32, y, b);
        tma_load_3d(st + kRedBox, &tm_k, &full[s], h0 * 32 + 64, y, b);
        tma_load_3d(st + 2 * kRedBox, &tm_v, &full[s], h0 * 32, y, b);
        tma_load_3d(st + 3 * kRedBox, &tm_v, &full[s], h0 * 32 + 64, y, b);
        issued = i + 1;
      }
      // drain: every load issued must have landed before the CTA exits
      for (int i = max(0, issued - kRedStages); i < issued; ++i)
        mbar_wait(&full[i % kRedStages], (i / kRedStages) & 1, abort_flag, nullptr, 0);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128, 1, 1);
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % kRedStages;
        const uint32_t ph = (i / kRedStages) & 1;
        if (!mbar_wait(&ready[s], ph, abort_flag, &g_tc_error, kErrWait)) break;
        tc_fence_after();
        const uint32_t st = sbase + RedSmem::stages + s * kRedStageBytes;
#pragma unroll
        for (int kk = 0; kk < kRedT / 16; ++kk) {
          // 16 tokens = two 8-row groups of 128 bytes
          const uint64_t ad = smem_desc_sw128(st + kk * 2048, kRedBox, 1024);
          const uint64_t bd = smem_desc_sw128(st + 2 * kRedBox + kk * 2048, kRedBox, 1024);
          mma_bf16(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
      }
      mma_commit(acc_full);
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, abort_flag, nullptr, 0);
    }
  } else {
    // ------------------------------------------------- feature map + key sum
    const int wt = tid - 64;
    const int c = wt & 15;        // 16-byte chunk column: box c/8, chunk c%8 of the row
    const int rg = wt >> 4;       // row group: rows rg and rg + 32 of every stage
    const int box = c >> 3, cc = c & 7;
    const int dpos = (cc & 3) * 8;  // first dim of the chunk inside its head
    float2 zacc[4] = {};
    // this thread's tokens are n_begin + rg + 32 j, j = 0, 1, ...; its chunk
    // holds RoPE pairs j0 .. j0+3 (fixed per thread)
    TokPos tp = {0, 0, 0};
    if (kRope != kNoRope) tp = token_pos(p.rope, n_begin + rg);
    const int j0 = dpos / 2;
    int sel[4], off[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      sel[q] = pair_axis(j0 + q);
      off[q] = pair_off(j0 + q);
    }
    for (int i = 0; i < ntiles; ++i) {
      const int s = i % kRedStages;
      const uint32_t ph = (i / kRedStages) & 1;
      if (!mbar_wait(&full[s], ph, abort_flag, &g_tc_error, kErrWait)) break;
      const uint32_t kb = sbase + RedSmem::stages + s * kRedStageBytes + box * kRedBox;
      const int y0 = n_begin + i * kRedT;
#pragma unroll
      for (int k = 0; k < kRedT / 32; ++k) {
        const int r = rg + 32 * k;
        const uint32_t addr = kb + sw128_offset(r, cc);
        uint4 u = ld_shared_v4(addr);
        u.x = relu_bf16x2(u.x);
        u.y = relu_bf16x2(u.y);
        u.z = relu_bf16x2(u.z);
        u.w = relu_bf16x2(u.w);
        float x[8];
        unpack8(u, x);
#pragma unroll
        for (int e = 0; e < 4; ++e) zacc[e] = __fadd2_rn(zacc[e], make_float2(x[2 * e], x[2 * e + 1]));
        if (kRope != kNoRope) {
          if (y0 + r < p.N) {
            const RopeBases rb = rope_bases(p.rope, tp);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float2 cs;
              if (kRope == kRopeTable) {
                cs = rope_tab[(sel[q] == 0 ? rb.t : (sel[q] == 1 ? rb.h : rb.w)) + off[q]];
              } else {
                const int pos = sel[q] == 0 ? p.rope.t_offset + tp.t : (sel[q] == 1 ? tp.h : tp.w);
                rope_cos_sin(pos, p.rope.inv_freq[j0 + q], cs.x, cs.y);
              }
              const float2 t = __fmul2_rn(make_float2(x[2 * q + 1], x[2 * q + 1]),
                                          make_float2(-cs.y, cs.x));
              const float2 y = __ffma2_rn(make_float2(x[2 * q], x[2 * q]), cs, t);
              x[2 * q] = y.x;
              x[2 * q + 1] = y.y;
            }
            u = pack8(x);
          }
          token_pos_advance(p.rope, tp, 32);
        }
        st_shared_v4(addr, u);
      }
      fence_proxy_async_smem();
      mbar_arrive(&ready[s]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      zred[wt * 8 + 2 * e] = zacc[e].x;
      zred[wt * 8 + 2 * e + 1] = zacc[e].y;
    }
    named_bar_sync(1, kRedMath);

    // state of the four heads: the 32x32 diagonal blocks of the accumulator
    if (warp >= 2 && warp < 6) {
      const int q = warp & 3;  // TMEM lane quadrant = head in the group
      float v[32];
      bool ok = ntiles > 0 && mbar_wait(acc_full, 0, abort_flag, &g_tc_error, kErrWait);
      ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld is warp-collective
      if (ok) {
        tc_fence_after();
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * q) << 16) + 32 * q, v);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0.0f;
      }
      const int h = h0 + q;
      if (h < p.H) {
        float* dst = partials +
                     ((static_cast<size_t>(b) * p.H + h) * p.splits + split) * kStateFloats +
                     lane * kD;
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
      }
    }
    if (wt < 128) {
      // key sum of dim wt of the group: 32 row groups, in order
      const int q = wt >> 5, d = wt & 31;
      const int col = wt >> 3, e = wt & 7;  // chunk column and element holding this dim
      float s = 0.0f;
      for (int r = 0; r < kRedMath / 16; ++r) s += zred[(r * 16 + col) * 8 + e];
      const int h = h0 + q;
      if (h < p.H)
        partials[((static_cast<size_t>(b) * p.H + h) * p.splits + split) * kStateFloats +
                 kD * kD + d] = s;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kRedTmemCols);
  }
  if (*abort_flag) return;  // partials incomplete: leave the counter alone
  finish_reduce_bulk(p, b, h0, partials, counters, out, smem, comb_full, abort_flag);
}

// ================================================================= apply

constexpr int kApT = 128;                          // tokens per tile
constexpr int kApStages = 5;
constexpr int kApBox = kApT * 128;                 // [128 tokens][64 dims] bf16
constexpr int kApStageBytes = 2 * kApBox;
constexpr int kApTmemCols = 512;                   // kApWG 128-column accumulators

// A stage holds a tile's Q, then phi(Q) for the MMA, then the tile's O for the
// TMA store: it is released to the producer once the store has read it.
struct ApSmem {
  static constexpr int stages = 0;
  static constexpr int bop = stages + kApStages * kApStageBytes;       // [2 pairs][32][128 B]
  static constexpr int zs = bop + 2 * 32 * 128;                        // [4][32] float
  static constexpr int rope = zs + kGroupHeads * kD * 4;               // float2[kRopeTableMax]
  static constexpr int bars = rope + kRopeTableMax * 8;
  static constexpr int nbars = 3 * kApStages + 2 * kApWG + 2;
  static constexpr int misc = bars + nbars * 8;
  static constexpr int bytes = misc + 16;
};
constexpr int kApSmemBytes = ApSmem::bytes + 1024;

template <int kRope>
__global__ void __launch_bounds__(kThreads, 1)
apply_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
         const Problem p, const RopeTable rt, const float* __restrict__ S,
         const float* __restrict__ z, int tiles_per_cta, int q_before_wait) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + ApSmem::bars);
  uint64_t* q_ready = q_full + kApStages;
  uint64_t* q_empty = q_ready + kApStages;
  uint64_t* t_full = q_empty + kApStages;   // [kApWG]
  uint64_t* t_empty = t_full + kApWG;       // [kApWG]
  uint64_t* mma_done = t_empty + kApWG;
  uint64_t* b_ready = mma_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + ApSmem::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + ApSmem::misc + 4);
  float* zs = reinterpret_cast<float*>(smem + ApSmem::zs);
  float2* rope_tab = reinterpret_cast<float2*>(smem + ApSmem::rope);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int group = blockIdx.y, b = blockIdx.z;
  const int h0 = group * kGroupHeads;
  const int ntiles_all = (p.N + kApT - 1) / kApT;
  const int tile_begin = blockIdx.x * tiles_per_cta;
  const int ntiles = max(0, min(ntiles_all, tile_begin + tiles_per_cta) - tile_begin);

  if (tid == 0) {
    for (int s = 0; s < kApStages; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_ready[s], 128);
      mbar_init(&q_empty[s], 1);
    }
    for (int a = 0; a < kApWG; ++a) {
      mbar_init(&t_full[a], 1);
      mbar_init(&t_empty[a], 128);
    }
    mbar_init(mma_done, 1);
    mbar_init(b_ready, kMathThreads);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kApTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_o);
  }
  if (kRope == kRopeTable && tid >= 64) build_rope_table(p.rope, rope_tab, tid - 64, kMathThreads);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);

  // Programmatic dependent launch: S and z come from the previous kernel, so
  // they are read only after pdl_wait(). Q may be fetched before it when the
  // caller knows the previous kernel does not write Q (q_before_wait).
  if (warp == 0 && !q_before_wait) pdl_wait();
  if (tid >= 64) {
    pdl_wait();
    if (tid == 64) pdl_trigger();
    const int mt = tid - 64;
    // B operands: for head pair j, row e holds S[h][0..31][e] of heads 2j and
    // 2j+1 as bf16 (K-major, 128-byte swizzled)
    for (int idx = mt; idx < 2 * 32 * 8; idx += kMathThreads) {
      const int j = idx >> 8, e = (idx >> 3) & 31, c = idx & 7;
      const int hh = 2 * j + (c >> 2), d0 = (c & 3) * 8;
      const int h = h0 + hh;
      float x[8];
      if (h < p.H) {
        const float* src = S + ((static_cast<size_t>(b) * p.H + h) * kD + d0) * kD + e;
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = src[k * kD];
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = 0.0f;
      }
      st_shared_v4(smem_u32(smem + ApSmem::bop + j * 4096) + sw128_offset(e, c), pack8(x));
    }
    for (int idx = mt; idx < kGroupHeads * kD; idx += kMathThreads) {
      const int h = h0 + idx / kD;
      zs[idx] = h < p.H ? z[(static_cast<size_t>(b) * p.H + h) * kD + idx % kD] : 0.0f;
    }
    fence_proxy_async_smem();
    mbar_arrive(b_ready);
    named_bar_sync(1 + kApWG, kMathThreads);  // zs visible to every math thread
  }

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % kApStages;
        const uint32_t ph = (i / kApStages) & 1;
        if (!mbar_wait(&q_empty[s], ph ^ 1, abort_flag, &g_tc_error, kErrWait)) break;
        mbar_arrive_expect_tx(&q_full[s], kApStageBytes);
        uint8_t* st = smem + ApSmem::stages + s * kApStageBytes;
        const int y = (tile_begin + i) * kApT;
        tma_load_3d(st, &tm_q, &q_full[s], h0 * 32, y, b);
        tma_load_3d(st + kApBox, &tm_q, &q_full[s], h0 * 32 + 64, y, b);
        issued = i + 1;
      }
      for (int i = max(0, issued - kApStages); i < issued; ++i)
        mbar_wait(&q_full[i % kApStages], (i / kApStages) & 1, abort_flag, nullptr, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 32, 0, 0);
      const uint32_t bop = sbase + ApSmem::bop;
      const bool have_b = ntiles == 0 || mbar_wait(b_ready, 0, abort_flag, &g_tc_error, kErrWait);
      for (int i = 0; have_b && i < ntiles; ++i) {
        const int s = i % kApStages;
        const uint32_t ph = (i / kApStages) & 1;
        const int a = i % kApWG;
        if (!mbar_wait(&q_ready[s], ph, abort_flag, &g_tc_error, kErrWait)) break;
        if (!mbar_wait(&t_empty[a], ((i / kApWG) & 1) ^ 1, abort_flag, &g_tc_error, kErrWait))
          break;
        tc_fence_after();
        const uint32_t st = sbase + ApSmem::stages + s * kApStageBytes;
#pragma unroll
        for (int hh = 0; hh < kGroupHeads; ++hh) {
          const uint32_t koff = (hh & 1) * 64;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint64_t ad = smem_desc_sw128(st + (hh >> 1) * kApBox + koff + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(bop + (hh >> 1) * 4096 + koff + kk * 32, 16, 1024);
            mma_bf16(tmem + a * 128 + hh * 32, ad, bd, idesc, kk);
          }
        }
        mma_commit(&t_full[a]);
      }
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, abort_flag, nullptr, 0);
    }
  } else {
    const int wg = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const bool leader = (warp == 2 + 4 * wg) && lane == 0;
    for (int i = wg; i < ntiles; i += kApWG) {
      const int s = i % kApStages;
      const uint32_t ph = (i / kApStages) & 1;
      bool ok = mbar_wait(&q_full[s], ph, abort_flag, &g_tc_error, kErrWait);
      if (bar_any(1 + wg, 128, !ok || *abort_flag)) break;
      const int n0 = (tile_begin + i) * kApT;
      const int n = n0 + row;
      float2 cs[16];
      if (kRope != kNoRope) {
        const TokPos tp = token_pos(p.rope, min(n, p.N - 1));
        const RopeBases rb = rope_bases(p.rope, tp);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (kRope == kRopeTable) {
            const int a = pair_axis(j);
            cs[j] = rope_tab[(a == 0 ? rb.t : (a == 1 ? rb.h : rb.w)) + pair_off(j)];
          } else {
            const int a = pair_axis(j);
            const int pos = a == 0 ? p.rope.t_offset + tp.t : (a == 1 ? tp.h : tp.w);
            rope_cos_sin(pos, p.rope.inv_freq[j], cs[j].x, cs[j].y);
          }
        }
      }
      float den[kGroupHeads] = {0.0f, 0.0f, 0.0f, 0.0f};
      const uint32_t st = sbase + ApSmem::stages + s * kApStageBytes;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int hh = c >> 2, d0 = (c & 3) * 8;
        const uint32_t addr = st + (c >> 3) * kApBox + sw128_offset(row, c & 7);
        uint4 u = ld_shared_v4(addr);
        u.x = relu_bf16x2(u.x);
        u.y = relu_bf16x2(u.y);
        u.z = relu_bf16x2(u.z);
        u.w = relu_bf16x2(u.w);
        float x[8];
        unpack8(u, x);
        const float4 za = *reinterpret_cast<const float4*>(zs + hh * kD + d0);
        const float4 zb = *reinterpret_cast<const float4*>(zs + hh * kD + d0 + 4);
        den[hh] = fmaf(x[0], za.x, den[hh]);
        den[hh] = fmaf(x[1], za.y, den[hh]);
        den[hh] = fmaf(x[2], za.z, den[hh]);
        den[hh] = fmaf(x[3], za.w, den[hh]);
        den[hh] = fmaf(x[4], zb.x, den[hh]);
        den[hh] = fmaf(x[5], zb.y, den[hh]);
        den[hh] = fmaf(x[6], zb.z, den[hh]);
        den[hh] = fmaf(x[7], zb.w, den[hh]);
        if (kRope != kNoRope) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 r = cs[d0 / 2 + q];
            const float2 t = __fmul2_rn(make_float2(x[2 * q + 1], x[2 * q + 1]),
                                        make_float2(-r.y, r.x));
            const float2 y = __ffma2_rn(make_float2(x[2 * q], x[2 * q]), r, t);
            x[2 * q] = y.x;
            x[2 * q + 1] = y.y;
          }
          u = pack8(x);
        }
        st_shared_v4(addr, u);
      }
      fence_proxy_async_smem();
      mbar_arrive(&q_ready[s]);

      // epilogue: O = num / den, written over the tile in shared memory (the
      // MMA has finished reading it), stored with TMA
      const int a = wg;
      ok = mbar_wait(&t_full[a], (i / kApWG) & 1, abort_flag, &g_tc_error, kErrWait);
      tc_fence_after();
      if (bar_any(1 + wg, 128, !ok || *abort_flag)) break;
#pragma unroll
      for (int hh = 0; hh < kGroupHeads; ++hh) {
        float v[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + a * 128 + hh * 32,
                           v);
        const float inv = 1.0f / (den[hh] + p.eps);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = v[8 * k + e] * inv;
          st_shared_v4(st + (hh >> 1) * kApBox + sw128_offset(row, (hh & 1) * 4 + k), pack8(x));
        }
      }
      tc_fence_before();
      mbar_arrive(&t_empty[a]);
      fence_proxy_async_smem();
      named_bar_sync(1 + wg, 128);
      if (leader) {
        uint8_t* tile = smem + ApSmem::stages + s * kApStageBytes;
        tma_store_3d(&tm_o, tile, h0 * 32, n0, b);
        tma_store_3d(&tm_o, tile + kApBox, h0 * 32 + 64, n0, b);
        bulk_commit();
        bulk_wait_read<0>();      // the store has read the stage
        mbar_arrive(&q_empty[s]);  // hand the stage back to the producer
      }
    }
    if (leader) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kApTmemCols);
  }
}

// ============================================================== host side

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
bool g_attr_set[6][kMaxDev] = {};
std::mutex g_attr_mu;

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

}  // namespace

// Launch with programmatic dependent launch: the kernel's prologue may
// overlap the previous kernel in the stream; its pdl_wait() orders every
// access to global memory after that kernel.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, int threads, int smem,
                       cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

cudaError_t launch_reduce_tc(const Problem& p, const void* K, const void* V, float* partials,
                             unsigned* counters, const StateOut& out, cudaStream_t s) {
  CUtensorMap mk, mv;
  cudaError_t e;
  if ((e = make_map(&mk, K, p, kRedT)) != cudaSuccess) return e;
  if ((e = make_map(&mv, V, p, kRedT)) != cudaSuccess) return e;
  const RopeTable rt = rope_table_for(p);
  const int mode = !rt.enabled ? kNoRope : (rt.on_the_fly ? kRopeOnTheFly : kRopeTable);
  void (*kern)(CUtensorMap, CUtensorMap, Problem, RopeTable, float*, unsigned*, StateOut) =
      mode == kNoRope ? reduce_tc<kNoRope>
                      : (mode == kRopeTable ? reduce_tc<kRopeTable> : reduce_tc<kRopeOnTheFly>);
  if ((e = ensure_smem_attr(mode, reinterpret_cast<const void*>(kern), kRedSmemBytes)) !=
      cudaSuccess)
    return e;
  const dim3 grid(p.splits, (p.H + kGroupHeads - 1) / kGroupHeads, p.B);
  e = launch_pdl(kern, grid, kRedThreads, kRedSmemBytes, s, mk, mv, p, rt, partials, counters,
                 out);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_apply_tc(const Problem& p, const void* Q, const float* S, const float* z,
                            void* O, bool after_own_reduce, cudaStream_t s) {
  CUtensorMap mq, mo;
  cudaError_t e;
  if ((e = make_map(&mq, Q, p, kApT)) != cudaSuccess) return e;
  if ((e = make_map(&mo, O, p, kApT)) != cudaSuccess) return e;
  const int groups = (p.H + kGroupHeads - 1) / kGroupHeads;
  const int ntiles = (p.N + kApT - 1) / kApT;
  const long long units = static_cast<long long>(groups) * p.B;
  int ctas_per_unit =
      static_cast<int>(std::max<long long>(1, kNumSMs / std::max<long long>(1, units)));
  ctas_per_unit = std::min(ctas_per_unit, ntiles);
  const int tiles_per_cta = (ntiles + ctas_per_unit - 1) / ctas_per_unit;
  ctas_per_unit = (ntiles + tiles_per_cta - 1) / tiles_per_cta;
  const RopeTable rt = rope_table_for(p);
  const int mode = !rt.enabled ? kNoRope : (rt.on_the_fly ? kRopeOnTheFly : kRopeTable);
  void (*kern)(CUtensorMap, CUtensorMap, Problem, RopeTable, const float*, const float*, int,
               int) = mode == kNoRope ? apply_tc<kNoRope>
                                      : (mode == kRopeTable ? apply_tc<kRopeTable>
                                                            : apply_tc<kRopeOnTheFly>);
  if ((e = ensure_smem_attr(3 + mode, reinterpret_cast<const void*>(kern), kApSmemBytes)) !=
      cudaSuccess)
    return e;
  const dim3 grid(ctas_per_unit, groups, p.B);
  // Q may be read before the previous kernel completes only when that kernel
  // is this library's own state reduce, which does not write Q and itself
  // started reading only after everything before it had completed.
  e = launch_pdl(kern, grid, kThreads, kApSmemBytes, s, mq, mo, p, rt, S, z, tiles_per_cta,
                 after_own_reduce ? 1 : 0);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t read_device_error(unsigned* code, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(code, g_tc_error, sizeof(unsigned));
  if (e == cudaSuccess && reset) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(unsigned));
  }
  return e;
}

}  // namespace la
