// Token-causal linear attention on the tensor cores with independent chunks
// (bf16 I/O, no RoPE): query n sees keys 0..n ("SANA-Video: Efficient Video
// Generation with Block Linear Diffusion Transformer", section 2.3, with the
// sum over earlier j read at token granularity).
//
// Three launches. (1) The state reduce in its chunk form (layer_tc, la_tc.cu)
// writes every 128-token chunk's own state (dS_c, dz_c). (2) chunk_prefix
// replaces them, per head and in chunk order, by the exclusive prefix
//   P_c = carry + sum_{c' < c} (dS_c', dz_c'),
// and folds the whole sequence into the carry when asked. (3) causal_chunk_tc
// computes every chunk on its own:
//   O_i = (sum_{j <= i in chunk} (phi(q_i).phi(k_j)) v_j + phi(q_i) S_P)
//         / (sum_{j <= i in chunk} phi(q_i).phi(k_j) + phi(q_i).z_P + eps)
// with (S_P, z_P) the chunk's prefix (without RoPE the denominator's
// ReLU(q).ReLU(k) is the numerator's weight itself, so one matrix serves
// both). No state travels from chunk to chunk inside the last launch, so a
// CTA's chunks overlap: the next chunk's loads, ReLU and P run while the
// current chunk's products and output complete.
//
// causal_chunk_tc: a CTA owns two heads (one 64-dim TMA box per tensor) of one
// batch element and a range of chunks; 320 threads (TMA warp, MMA warp, one
// warpgroup per head). Per chunk, with three stages of Q, K, V and the
// chunk's prefix state in flight:
//   P   = phi(Q_h) phi(K_h)^T            M = N = 128, K = 32   (TMEM)
//   the head's warpgroup masks P to j <= i, sums its rows, and writes P back
//   into the same TMEM columns as two bf16 parts (the rounded value and the
//   rounded remainder: about 16 bits of each weight), 32 columns per block
//   of 32 keys (16 of each part);
//   O_h = P_hi V + P_lo V                 A from TMEM, B = V (MN-major, N = 64)
//       + phi(Q_h) (S_hi + S_lo)           S of the prefix in two bf16 parts
// and the warpgroup divides by the denominator and writes O over the Q box,
// which the TMA warp stores. Every wait is bounded.
#include <algorithm>

#include "la_tc_common.cuh"

namespace la {

// Device error word of the chunked token-causal kernels.
__device__ unsigned g_causal_chunk_error;

namespace {

constexpr int kXT = 128;                    // tokens per chunk
constexpr int kXBox = kXT * 128;            // [128 tokens][64 dims] bf16 = 16 KB
constexpr int kXStages = 3;
constexpr int kXMath = 256;                 // two warpgroups, one per head
constexpr int kXThreads = 64 + kXMath;
constexpr int kXTmemCols = 512;
constexpr int kBarBothX = 1;                // named barrier over both warpgroups

// Stage layout: Q, K, V boxes, then the S operand of the chunk's prefix in two
// bf16 parts ([hi, lo][32 rows e][128 B]: head h in bytes [64h, 64h + 64) of
// a row), then the prefix state as copied ([2 heads][32*32 + 32] f32).
struct XStage {
  static constexpr int q = 0;
  static constexpr int k = q + kXBox;
  static constexpr int v = k + kXBox;
  static constexpr int bop = v + kXBox;               // 2 x 4 KB
  static constexpr int state = bop + 2 * 4096;        // 2 x 4224 B
  static constexpr int bytes = state + 2 * kStateFloats * 4;
  static constexpr int stride = (bytes + 1023) / 1024 * 1024;
};

// TMEM columns: P of head h at 128 h; O of head h at kColO + 64 h (N = 64
// over both heads' V columns; head h's numerator is its columns 32 h ..).
constexpr uint32_t kColO = 256;

struct XSmem {
  static constexpr int stages = 0;
  static constexpr int bars = stages + kXStages * XStage::stride;
  // full[3] ready[3] bop_ready[3] o_done[3] p_full pm_ready[2] o_full[2] mma_done
  static constexpr int nbars = 4 * kXStages + 6;
  static constexpr int misc = bars + nbars * 8;
  static constexpr int bytes = misc + 16;
};
constexpr int kXSmemBytes = XSmem::bytes + 1024;
static_assert(kXSmemBytes <= 232448, "shared memory per CTA");

struct ChunkArgs {
  const float* prefix;  // [B*H][nchunks][kStateFloats]: each chunk's exclusive prefix state
  int nchunks;          // ceil(N / 128)
  int chunks_per_cta;
};

// D[tmem] (+)= A[tmem] * B[smem]: bf16 A read from tensor memory (K-major,
// two 16-bit values per 32-bit column), fp32 accumulation.
__device__ __forceinline__ void mma_bf16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns from registers to TMEM (thread i
// writes lane base + i); waits until the stores are done.
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__global__ void __launch_bounds__(kXThreads, 1)
causal_chunk_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                const Problem p, const ChunkArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + XSmem::bars);
  uint64_t* ready = full + kXStages;        // Q and K of the chunk ReLU'd (256 arrivals)
  uint64_t* bop_ready = ready + kXStages;   // the prefix's S operand built (256)
  uint64_t* o_done = bop_ready + kXStages;  // O written over the Q box (256)
  uint64_t* p_full = o_done + kXStages;     // P of both heads in TMEM (1)
  uint64_t* pm_ready = p_full + 1;          // [head] P masked, in two parts, in TMEM (128)
  uint64_t* o_full = pm_ready + 2;          // [head] O in TMEM (1)
  uint64_t* mma_done = o_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + XSmem::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + XSmem::misc + 4);
  unsigned* err = &g_causal_chunk_error;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pair = blockIdx.y, b = blockIdx.z;
  const int h0 = pair * 2;
  const size_t cidx = static_cast<size_t>(b) * p.H + h0;
  const int c_begin = blockIdx.x * a.chunks_per_cta;
  const int nC = max(0, min(a.nchunks, c_begin + a.chunks_per_cta) - c_begin);
  const int heads = min(2, p.H - h0);

  if (tid == 0) {
    for (int i = 0; i < kXStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&ready[i], kXMath);
      mbar_init(&bop_ready[i], kXMath);
      mbar_init(&o_done[i], kXMath);
    }
    mbar_init(p_full, 1);
    mbar_init(&pm_ready[0], 128);
    mbar_init(&pm_ready[1], 128);
    mbar_init(&o_full[0], 1);
    mbar_init(&o_full[1], 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kXTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_o);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);
  pdl_wait();
  if (tid == 64) pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      // stage c % 3 holds chunk c; before it takes chunk c the output of
      // chunk c - 3 (written over its Q box) is stored and has been read
      auto store_o = [&](int c) -> bool {
        const int s = c % kXStages;
        if (!mbar_wait(&o_done[s], (c / kXStages) & 1, abort_flag, err, kErrWait)) return false;
        tma_store_3d(&tm_o, smem + XSmem::stages + s * XStage::stride + XStage::q, h0 * 32,
                     (c_begin + c) * kXT, b);
        bulk_commit();
        bulk_wait_read<0>();
        return true;
      };
      bool ok = true;
      int c = 0;
      for (; ok && c < nC; ++c) {
        const int s = c % kXStages;
        if (c >= kXStages && !(ok = store_o(c - kXStages))) break;
        uint8_t* st = smem + XSmem::stages + s * XStage::stride;
        mbar_arrive_expect_tx(&full[s], 3 * kXBox + heads * kStateFloats * 4);
        const int y = (c_begin + c) * kXT;
        tma_load_3d(st + XStage::q, &tm_q, &full[s], h0 * 32, y, b);
        tma_load_3d(st + XStage::k, &tm_k, &full[s], h0 * 32, y, b);
        tma_load_3d(st + XStage::v, &tm_v, &full[s], h0 * 32, y, b);
        for (int hh = 0; hh < heads; ++hh)
          bulk_load(st + XStage::state + hh * kStateFloats * 4,
                    a.prefix + ((cidx + hh) * a.nchunks + c_begin + c) * kStateFloats,
                    kStateFloats * 4, &full[s]);
      }
      for (int k = max(0, c - kXStages); ok && k < c; ++k) ok = store_o(k);
      for (int k = max(0, c - kXStages); k < c; ++k)
        mbar_drain(&full[k % kXStages], (k / kXStages) & 1, err, kErrWait);
      bulk_wait<0>();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t id_p = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_pv = idesc_bf16_f32(128, 64, 0, 1);
      const uint32_t id_qs = idesc_bf16_f32(128, 32, 0, 0);
      bool ok = true;
      for (int c = 0; ok && c < nC; ++c) {
        const int s = c % kXStages;
        const uint32_t par = (c / kXStages) & 1;
        const uint32_t st = sbase + XSmem::stages + s * XStage::stride;
        const uint32_t qb = st + XStage::q, kb = st + XStage::k, vb = st + XStage::v;
        const uint32_t bop = st + XStage::bop;
        if (!(ok = mbar_wait(&ready[s], par, abort_flag, err, kErrWait))) break;
        // P of chunk c overwrites the P columns the previous chunk's P.V MMAs
        // read; those were issued earlier by this thread and run in order
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_bf16(tmem + 128 * h, smem_desc_sw128(qb + h * 64 + kk * 32, 16, 1024),
                     smem_desc_sw128(kb + h * 64 + kk * 32, 16, 1024), id_p, kk);
        mma_commit(p_full);
        for (int h = 0; ok && h < 2; ++h) {
          // O_h = P_hi V + P_lo V (A from TMEM: keys 16 kk .. of block kk / 2)
          if (!(ok = mbar_wait(&pm_ready[h], c & 1, abort_flag, err, kErrWait))) break;
          tc_fence_after();
#pragma unroll
          for (int part = 0; part < 2; ++part)
#pragma unroll
            for (int kk = 0; kk < kXT / 16; ++kk)
              mma_bf16_tmem_a(tmem + kColO + 64 * h,
                              tmem + 128 * h + 32 * (kk >> 1) + 16 * part + 8 * (kk & 1),
                              smem_desc_sw128(vb + kk * 2048, kXBox, 1024), id_pv,
                              (part > 0 || kk > 0) ? 1u : 0u);
          // + phi(Q_h) S of the prefix, S = S_hi + S_lo
          if (h == 0 && !(ok = mbar_wait(&bop_ready[s], par, abort_flag, err, kErrWait))) break;
#pragma unroll
          for (int part = 0; part < 2; ++part)
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
              mma_bf16(tmem + kColO + 64 * h + 32 * h,
                       smem_desc_sw128(qb + h * 64 + kk * 32, 16, 1024),
                       smem_desc_sw128(bop + part * 4096 + h * 64 + kk * 32, 16, 1024), id_qs, 1u);
          mma_commit(&o_full[h]);
        }
      }
      mma_commit(mma_done);
      mbar_drain(mma_done, 0, err, kErrWait);
    }
  } else {
    // ------------------------------------------------- math: one warpgroup per head
    const int mt = tid - 64;
    const int h = mt >> 7;           // head of the pair owned by this warpgroup
    const int wt = mt & 127;
    const int quad = warp & 3;       // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;
    const uint32_t lq = static_cast<uint32_t>(quad * 32) << 16;
    // The loads, ReLU and S operand of chunk c + 1 are done between chunk c's
    // mask and its output, so the MMA warp can compute chunk c + 1's P right
    // behind chunk c's products and the next mask starts without a gap.
    auto stage_of = [&](int c) { return sbase + XSmem::stages + (c % kXStages) * XStage::stride; };
    auto prefix_of = [&](int c) {
      return reinterpret_cast<const float*>(smem + XSmem::stages + (c % kXStages) * XStage::stride +
                                            XStage::state) + h * kStateFloats;
    };
    // ReLU of this head's Q and K columns of chunk c in place, then the
    // prefix's S as the B operand: row e holds S[0..31][e] of this head in two
    // bf16 parts (thread wt: row e = wt / 4, dims 8 (wt % 4) ..). False when
    // a wait gave up (decided by both warpgroups together).
    auto prepare = [&](int c) -> bool {
      const int s = c % kXStages;
      const bool ok = mbar_wait(&full[s], (c / kXStages) & 1, abort_flag, err, kErrWait);
      if (bar_any(kBarBothX, kXMath, !ok || *abort_flag)) return false;
      const uint32_t st = stage_of(c);
      const uint32_t qb = st + XStage::q, kb = st + XStage::k;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const uint32_t aq = qb + sw128_offset(row, h * 4 + c4);
        uint4 u = ld_shared_v4(aq);
        u.x = relu_bf16x2(u.x); u.y = relu_bf16x2(u.y); u.z = relu_bf16x2(u.z); u.w = relu_bf16x2(u.w);
        st_shared_v4(aq, u);
        const uint32_t ak = kb + sw128_offset(row, h * 4 + c4);
        uint4 w = ld_shared_v4(ak);
        w.x = relu_bf16x2(w.x); w.y = relu_bf16x2(w.y); w.z = relu_bf16x2(w.z); w.w = relu_bf16x2(w.w);
        st_shared_v4(ak, w);
      }
      fence_proxy_async_smem();
      mbar_arrive(&ready[s]);
      {
        const float* pre = prefix_of(c);
        const int e = wt >> 2, c4 = wt & 3;
        float x[8], lo[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = h < heads ? pre[(c4 * 8 + k) * kD + e] : 0.0f;
        const uint4 hi = pack8(x);
        float hx[8];
        unpack8(hi, hx);
#pragma unroll
        for (int k = 0; k < 8; ++k) lo[k] = x[k] - hx[k];
        const uint32_t bop = st + XStage::bop;
        st_shared_v4(bop + sw128_offset(e, h * 4 + c4), hi);
        st_shared_v4(bop + 4096 + sw128_offset(e, h * 4 + c4), pack8(lo));
      }
      fence_proxy_async_smem();
      mbar_arrive(&bop_ready[s]);
      return true;
    };

    bool alive = nC == 0 || prepare(0);
    for (int c = 0; alive && c < nC; ++c) {
      const int s = c % kXStages;
      const uint32_t qb = stage_of(c) + XStage::q;
      const float* pre = prefix_of(c);

      // ---- P: mask j <= i, row sums, two bf16 parts back into TMEM
      bool ok = mbar_wait(p_full, c & 1, abort_flag, err, kErrWait);
      tc_fence_after();
      if (bar_any(kBarBothX, kXMath, !ok || *abort_flag)) break;
      float psum = 0.0f;
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        float v[32];
        tmem_ld_32x32b_x32(tmem + lq + 128 * h + 32 * q, v);
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int j = q * 32 + 2 * e;
          const float x0 = j <= row ? v[2 * e] : 0.0f;
          const float x1 = j + 1 <= row ? v[2 * e + 1] : 0.0f;
          psum += x0 + x1;
          hi[e] = pack_bf16x2(x0, x1);
          const float h0f = __uint_as_float(hi[e] << 16), h1f = __uint_as_float(hi[e] & 0xffff0000u);
          lo[e] = pack_bf16x2(x0 - h0f, x1 - h1f);
        }
        tmem_st_32x32b_x16(tmem + lq + 128 * h + 32 * q, hi);
        tmem_st_32x32b_x16(tmem + lq + 128 * h + 32 * q + 16, lo);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&pm_ready[h]);
      // the denominator: the masked row sum plus ReLU(q) . z of the prefix
      float den = psum + p.eps;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        float x[8];
        unpack8(ld_shared_v4(qb + sw128_offset(row, h * 4 + c4)), x);
#pragma unroll
        for (int k = 0; k < 8; ++k) den = fmaf(x[k], h < heads ? pre[kD * kD + c4 * 8 + k] : 0.0f, den);
      }

      // ---- the next chunk, ahead of this chunk's output
      if (c + 1 < nC && !prepare(c + 1)) break;

      // ---- O = numerator / den over this head's columns of the Q box
      ok = mbar_wait(&o_full[h], c & 1, abort_flag, err, kErrWait);
      tc_fence_after();
      if (bar_any(kBarBothX, kXMath, !ok || *abort_flag)) break;
      {
        float v[32];
        tmem_ld_32x32b_x32(tmem + lq + kColO + 64 * h + 32 * h, v);
        const float inv = 1.0f / den;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          float x[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) x[k] = v[c4 * 8 + k] * inv;
          st_shared_v4(qb + sw128_offset(row, h * 4 + c4), pack8(x));
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(&o_done[s]);  // the TMA warp stores the tile once both heads are in
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kXTmemCols);
  }
}

// Exclusive prefix over the chunks, per head and float4 column, in chunk
// order: chunk c's state becomes carry + the sum of the chunks before it.
// update: the carry becomes carry + the sum of all chunks.
__global__ void __launch_bounds__(256)
chunk_prefix(float* states, int bh_count, int nchunks, float* S_carry, float* z_carry, int update) {
  constexpr int kVec = kStateFloats / 4;
  const long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  pdl_wait();
  if (threadIdx.x == 0) pdl_trigger();
  if (g >= static_cast<long long>(bh_count) * kVec) return;
  const int bh = static_cast<int>(g / kVec), i = static_cast<int>(g % kVec) * 4;
  const bool is_s = i < kD * kD;
  float* carry = S_carry == nullptr ? nullptr
                                    : (is_s ? S_carry + static_cast<size_t>(bh) * kD * kD + i
                                            : z_carry + static_cast<size_t>(bh) * kD + (i - kD * kD));
  float4 acc = carry != nullptr ? *reinterpret_cast<const float4*>(carry)
                                : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  float4* col = reinterpret_cast<float4*>(states + static_cast<size_t>(bh) * nchunks * kStateFloats + i);
  constexpr int kStride = kStateFloats / 4;  // float4 between consecutive chunks
  // 16 chunks' loads in flight at a time (the chain of adds is in chunk order)
  constexpr int kBatch = 16;
  int c = 0;
  for (; c + kBatch <= nchunks; c += kBatch) {
    float4 d[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) d[k] = __ldcg(col + static_cast<size_t>(c + k) * kStride);
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      __stcg(col + static_cast<size_t>(c + k) * kStride, acc);
      acc = make_float4(acc.x + d[k].x, acc.y + d[k].y, acc.z + d[k].z, acc.w + d[k].w);
    }
  }
  for (; c < nchunks; ++c) {
    const float4 d = __ldcg(col + static_cast<size_t>(c) * kStride);
    __stcg(col + static_cast<size_t>(c) * kStride, acc);
    acc = make_float4(acc.x + d.x, acc.y + d.y, acc.z + d.z, acc.w + d.w);
  }
  if (update && carry != nullptr) *reinterpret_cast<float4*>(carry) = acc;
}

cudaError_t launch_pdl_x(const void* fn, void** args, dim3 grid, dim3 block, int smem,
                         cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace

bool causal_chunk_supported(const Problem& p) {
  return p.io == LA_IO_BF16 && p.N > 0 && !p.rope.enabled;
}

size_t causal_chunk_state_bytes(const Problem& p) {
  const size_t nchunks = static_cast<size_t>((p.N + kXT - 1) / kXT);
  return static_cast<size_t>(p.B) * p.H * nchunks * kStateFloats * sizeof(float);
}

cudaError_t launch_causal_chunks(const Problem& p, const void* Q, const void* K, const void* V,
                                 float* states, float* S_carry, float* z_carry, int update,
                                 void* O, cudaStream_t s) {
  if (!causal_chunk_supported(p)) return cudaErrorNotSupported;
  const int nchunks = (p.N + kXT - 1) / kXT;
  // (1) every chunk's own state
  cudaError_t e = launch_chunk_states_tc(p, K, V, states, nchunks, s);
  if (e != cudaSuccess) return e;
  // (2) the exclusive prefix over the chunks (and the carry update)
  {
    int bh = p.B * p.H;
    int nc = nchunks;
    float* st = states;
    float* sc = S_carry;
    float* zc = z_carry;
    int up = update;
    void* args[] = {&st, &bh, &nc, &sc, &zc, &up};
    const long long threads = static_cast<long long>(bh) * (kStateFloats / 4);
    const dim3 grid(static_cast<unsigned>((threads + 255) / 256));
    e = launch_pdl_x(reinterpret_cast<const void*>(chunk_prefix), args, grid, dim3(256), 0, s);
    if (e != cudaSuccess) return e;
  }
  // (3) every chunk on its own
  CUtensorMap mq, mk, mv, mo;
  if ((e = make_map(&mq, Q, p, kXT)) != cudaSuccess) return e;
  if ((e = make_map(&mk, K, p, kXT)) != cudaSuccess) return e;
  if ((e = make_map(&mv, V, p, kXT)) != cudaSuccess) return e;
  if ((e = make_map(&mo, O, p, kXT)) != cudaSuccess) return e;
  if ((e = ensure_smem_attr(0, reinterpret_cast<const void*>(causal_chunk_tc), kXSmemBytes)) !=
      cudaSuccess)
    return e;
  const int pairs = (p.H + 1) / 2;
  const long long units = static_cast<long long>(pairs) * p.B;
  int ctas = static_cast<int>(std::max<long long>(1, kNumSMs / std::max<long long>(1, units)));
  ctas = std::min(ctas, nchunks);
  ChunkArgs a = {};
  a.prefix = states;
  a.nchunks = nchunks;
  a.chunks_per_cta = (nchunks + ctas - 1) / ctas;
  ctas = (nchunks + a.chunks_per_cta - 1) / a.chunks_per_cta;
  Problem pc = p;
  void* args[] = {&mq, &mk, &mv, &mo, &pc, &a};
  e = launch_pdl_x(reinterpret_cast<const void*>(causal_chunk_tc), args, dim3(ctas, pairs, p.B),
                   dim3(kXThreads), kXSmemBytes, s);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t read_device_error_causal_chunk(unsigned* code, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(code, g_causal_chunk_error, sizeof(unsigned));
  if (e == cudaSuccess && reset) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_causal_chunk_error, &zero, sizeof(unsigned));
  }
  return e;
}

}  // namespace la
