// Token-causal linear attention on the tensor cores with independent chunks
// (bf16 I/O): query n sees keys 0..n ("SANA-Video: Efficient Video Generation
// with Block Linear Diffusion Transformer", section 2.3, with the sum over
// earlier j read at token granularity).
//
// Three launches without RoPE, four with it. (1) The state reduce in its chunk
// form (layer_tc, la_tc.cu) writes every 128-token chunk's own state (dS_c,
// dz_c); with RoPE its keys are rotated, and chunk_key_sums forms dz_c from
// the plain ReLU(k). (2) chunk_prefix replaces the states, per head and in
// chunk order, by the exclusive prefix
//   P_c = carry + sum_{c' < c} (dS_c', dz_c'),
// and folds the whole sequence into the carry when asked. (3) causal_chunk_tc
// (or causal_chunk_rope_tc, further down) computes every chunk on its own:
//   O_i = (sum_{j <= i in chunk} (phi(q_i).phi(k_j)) v_j + phi(q_i) S_P)
//         / (sum_{j <= i in chunk} ReLU(q_i).ReLU(k_j) + ReLU(q_i).z_P + eps)
// with (S_P, z_P) the chunk's prefix (without RoPE the denominator's
// ReLU(q).ReLU(k) is the numerator's weight itself, so one matrix serves
// both). No state travels from chunk to chunk inside the last launch, so a
// CTA's chunks overlap: the next chunk's loads, ReLU and P run while the
// current chunk's products and output complete.
//
// causal_chunk_tc: a CTA owns two heads (one 64-dim TMA box per tensor) of one
// batch element and a range of chunks; 352 threads (TMA warp, one warpgroup
// per head, and one MMA-issuing warp per head: warps 1 and 10). Per chunk,
// with three stages of Q, K, V and the chunk's prefix state in flight:
//   P   = phi(Q_h) phi(K_h)^T            M = N = 128, K = 32   (TMEM)
//   the head's warpgroup masks P to j <= i, sums its rows, and writes P back
//   into the same TMEM columns as two bf16 parts (the rounded value and the
//   rounded remainder: about 16 bits of each weight), 32 columns per block
//   of 32 keys (16 of each part);
//   O_h = P_hi V_h + P_lo V_h              A from TMEM, B = V_h (MN-major, N = 32)
//       + phi(Q_h) (S_hi + S_lo)           S of the prefix in two bf16 parts
// and the warpgroup divides by the denominator and writes O over its head's
// half of the Q box, which the TMA warp stores once both halves are in. The
// two heads run as separate pipelines (their own barriers and MMA issuers:
// a tcgen05.mma costs tens of cycles to issue, and one issuer would make each
// head's products wait behind the other's). Every wait is bounded.
#include <algorithm>

#include "la_tc_common.cuh"

namespace la {

// Device error word of the chunked token-causal kernels.
__device__ unsigned g_causal_chunk_error;

namespace {

constexpr int kXT = 128;                    // tokens per chunk
constexpr int kXBox = kXT * 128;            // [128 tokens][64 dims] bf16 = 16 KB
constexpr int kXVBox = kXT * 64;            // [128 tokens][32 dims] bf16 = 8 KB
constexpr int kXStages = 3;
constexpr int kXMath = 256;                 // two warpgroups, one per head
constexpr int kXThreads = 64 + kXMath;
constexpr int kRThreads = kXThreads + 32;   // + a second MMA-issuing warp (warp 10)
constexpr int kXTmemCols = 512;
constexpr int kBarHeadX = 1;                // named barriers kBarHeadX + h: one warpgroup

// Stage layout: Q and K boxes (both heads, 128-byte swizzle), V as one box
// per head ([128 tokens][32 dims], 64-byte swizzle, so that each head's P.V
// has N = 32), then the S operand of the chunk's prefix in two bf16 parts
// ([hi, lo][32 rows e][128 B]: head h in bytes [64h, 64h + 64) of a row),
// then the prefix state as copied ([2 heads][32*32 + 32] f32).
struct XStage {
  static constexpr int q = 0;
  static constexpr int k = q + kXBox;
  static constexpr int v = k + kXBox;
  static constexpr int bop = v + kXBox;               // 2 x 4 KB
  static constexpr int state = bop + 2 * 4096;        // 2 x 4224 B
  static constexpr int bytes = state + 2 * kStateFloats * 4;
  static constexpr int stride = (bytes + 1023) / 1024 * 1024;
};

// TMEM columns: P of head h at 128 h; O of head h at kColO + 32 h.
constexpr uint32_t kColO = 256;

struct XSmem {
  static constexpr int stages = 0;
  static constexpr int bars = stages + kXStages * XStage::stride;
  // full[3] ready[3][2] o_done[3] p_full[2] pm_ready[2] o_full[2] mma_done[2]
  static constexpr int nbars = 4 * kXStages + 8;
  static constexpr int misc = bars + nbars * 8;
  static constexpr int bytes = misc + 16;
};
constexpr int kXSmemBytes = XSmem::bytes + 1024;
static_assert(kXSmemBytes <= 232448, "shared memory per CTA");

struct ChunkArgs {
  const float* prefix;  // [B*H][nchunks][kStateFloats]: each chunk's exclusive prefix state
  int nchunks;          // ceil(N / 128)
  int chunks_per_cta;
  int adv_w, adv_h, adv_t;  // RoPE: 128 tokens as a step of the (t, h, w) grid (w, h below W, Hh)
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

// 32 lanes x 32 consecutive fp32 columns without the wait (tmem_ld_wait
// completes every load issued before it).
__device__ __forceinline__ void tmem_ld_32x32b_x32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 64-byte swizzle, MN-major operand of 32
// elements along MN (one swizzle atom, tile base 512-aligned): sbo is the
// distance between 8-row K groups (8 x 64 B).
__device__ __forceinline__ uint64_t smem_desc_sw64_mn32(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFF) >> 4);
  d |= static_cast<uint64_t>((kXVBox >> 4) & 0x3FFF) << 16;  // between MN atoms (one here)
  d |= static_cast<uint64_t>((512 >> 4) & 0x3FFF) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version for sm_100
  d |= static_cast<uint64_t>(4) << 61;  // 64-byte swizzle
  return d;
}

// Eight floats as two bf16 parts: hi = the values truncated to bf16 (their
// upper 16 bits), lo = the exact remainders rounded to bf16; hi + lo keeps
// about 16 bits of each value.
__device__ __forceinline__ void split_bf16x8(const float* x, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t u0 = __float_as_uint(x[2 * k]), u1 = __float_as_uint(x[2 * k + 1]);
    h[k] = __byte_perm(u0, u1, 0x7632);
    l[k] = pack_bf16x2(x[2 * k] - __uint_as_float(u0 & 0xffff0000u),
                       x[2 * k + 1] - __uint_as_float(u1 & 0xffff0000u));
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// The causal mask and split of one head's P in TMEM (warp of lane quadrant
// `quad`: rows 32 quad + lane): key block q < quad is kept whole, the
// diagonal block q = quad keeps keys j <= row, blocks q > quad become zeros
// (not loaded); the loads of blocks (0, 1) and of (2, 3) are issued together.
// Each block goes back as 16 columns of rounded bf16 pairs and 16 of the
// rounded remainders. Returns the sum of the kept weights.
__device__ __forceinline__ float mask_split_p(uint32_t taddr, int quad, int lane) {
  float psum = 0.0f;
#pragma unroll
  for (int q2 = 0; q2 < 4; q2 += 2) {
    uint32_t r[2][32];
    if (q2 <= quad) {
#pragma unroll
      for (int t = 0; t < 2; ++t)
        if (q2 + t <= quad) tmem_ld_32x32b_x32_nowait(taddr + 32 * (q2 + t), r[t]);
      tmem_ld_wait();
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int q = q2 + t;
      uint32_t hi[16], lo[16];
      if (q > quad) {
#pragma unroll
        for (int e = 0; e < 16; ++e) hi[e] = lo[e] = 0u;
      } else {
        const int lim = q < quad ? 32 : lane + 1;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float x0 = 2 * e < lim ? __uint_as_float(r[t][2 * e]) : 0.0f;
          const float x1 = 2 * e + 1 < lim ? __uint_as_float(r[t][2 * e + 1]) : 0.0f;
          psum += x0 + x1;
          hi[e] = pack_bf16x2(x0, x1);
          const float h0f = __uint_as_float(hi[e] << 16), h1f = __uint_as_float(hi[e] & 0xffff0000u);
          lo[e] = pack_bf16x2(x0 - h0f, x1 - h1f);
        }
      }
      tmem_st_32x32b_x16(taddr + 32 * q, hi);
      tmem_st_32x32b_x16(taddr + 32 * q + 16, lo);
    }
  }
  return psum;
}

__global__ void __launch_bounds__(kRThreads, 1)
causal_chunk_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                const Problem p, const ChunkArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + XSmem::bars);
  uint64_t* ready = full + kXStages;          // [stage][head] Q, K ReLU'd, S operand built (128)
  uint64_t* o_done = ready + 2 * kXStages;    // [stage] O written over the Q box (256)
  uint64_t* p_full = o_done + kXStages;       // [head] P in TMEM (1)
  uint64_t* pm_ready = p_full + 2;            // [head] P masked, in two parts, in TMEM (128)
  uint64_t* o_full = pm_ready + 2;            // [head] O in TMEM (1)
  uint64_t* mma_done = o_full + 2;            // [head] this head's MMAs drained (1)
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
      mbar_init(&ready[2 * i], 128);
      mbar_init(&ready[2 * i + 1], 128);
      mbar_init(&o_done[i], kXMath);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&p_full[h], 1);
      mbar_init(&pm_ready[h], 128);
      mbar_init(&o_full[h], 1);
    }
    mbar_init(&mma_done[0], 1);
    mbar_init(&mma_done[1], 1);
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
        tma_load_3d(st + XStage::v + kXVBox, &tm_v, &full[s], h0 * 32 + 32, y, b);
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
  } else if (warp == 1 || warp == kRThreads / 32 - 1) {
    // ------------------------------------------------------------ MMA, one head per warp
    if (lane == 0) {
      const int hm = warp == 1 ? 0 : 1;
      const uint32_t id_p = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_pv = idesc_bf16_f32(128, 32, 0, 1);
      const uint32_t id_qs = idesc_bf16_f32(128, 32, 0, 0);
      auto stage_addr = [&](int c) { return sbase + XSmem::stages + (c % kXStages) * XStage::stride; };
      // The issue path is kept short (one tcgen05.mma costs tens of cycles to
      // issue, about as long as a small MMA runs): a stage's descriptors are
      // built once, and each MMA adds a constant offset (in 16-byte units) to
      // the start-address field, which cannot carry out of its 14 bits below
      // 256 KB.
      //
      // P_h = phi(Q_h) phi(K_h)^T of chunk c. It overwrites the P columns that
      // head h's P.V of chunk c - 1 read; those were issued earlier by this
      // thread and run in order.
      auto issue_p = [&](int c, int h) -> bool {
        const int s = c % kXStages;
        if (!mbar_wait(&ready[2 * s + h], (c / kXStages) & 1, abort_flag, err, kErrWait)) return false;
        tc_fence_after();
        const uint32_t st = stage_addr(c);
        const uint64_t dq = smem_desc_sw128(st + XStage::q, 16, 1024);
        const uint64_t dk = smem_desc_sw128(st + XStage::k, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_bf16(tmem + 128 * h, dq + (h * 64 + kk * 32) / 16, dk + (h * 64 + kk * 32) / 16, id_p, kk);
        mma_commit(&p_full[h]);
        return true;
      };
      // O_h = P_hi V_h + P_lo V_h (A from TMEM: keys 16 kk .. of block kk / 2)
      //     + phi(Q_h) (S_hi + S_lo) of the prefix
      auto issue_pv = [&](int c, int h) -> bool {
        if (!mbar_wait(&pm_ready[h], c & 1, abort_flag, err, kErrWait)) return false;
        tc_fence_after();
        const uint32_t st = stage_addr(c);
        const uint64_t dv = smem_desc_sw64_mn32(st + XStage::v + h * kXVBox);
        const uint64_t dq = smem_desc_sw128(st + XStage::q, 16, 1024);
        const uint64_t db = smem_desc_sw128(st + XStage::bop, 16, 1024);
        const uint32_t d = tmem + kColO + 32 * h;
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int kk = 0; kk < kXT / 16; ++kk)
            mma_bf16_tmem_a(d, tmem + 128 * h + 32 * (kk >> 1) + 16 * part + 8 * (kk & 1),
                            dv + kk * 1024 / 16, id_pv, (part > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_bf16(d, dq + (h * 64 + kk * 32) / 16, db + (part * 4096 + h * 64 + kk * 32) / 16,
                     id_qs, 1u);
        mma_commit(&o_full[h]);
        return true;
      };
      bool ok = true;
      if (hm == 0) {
        for (int c = 0; ok && c < nC; ++c) ok = issue_p(c, 0) && issue_pv(c, 0);
      } else {
        for (int c = 0; ok && c < nC; ++c) ok = issue_p(c, 1) && issue_pv(c, 1);
      }
      mma_commit(&mma_done[hm]);
      mbar_drain(&mma_done[hm], 0, err, kErrWait);
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
    // bf16 parts (thread wt: row e = wt % 32, dims 8 (wt / 32) ..). False when
    // a wait gave up (decided by the warpgroup together).
    auto prepare = [&](int c) -> bool {
      const int s = c % kXStages;
      const bool ok = mbar_wait(&full[s], (c / kXStages) & 1, abort_flag, err, kErrWait);
      if (bar_any(kBarHeadX + h, 128, !ok || *abort_flag)) return false;
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
      {
        const float* pre = prefix_of(c);
        const int e = wt & 31, c4 = wt >> 5;  // a warp reads 32 consecutive floats
        float x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = h < heads ? pre[(c4 * 8 + k) * kD + e] : 0.0f;
        uint4 hi, lo;
        split_bf16x8(x, hi, lo);
        const uint32_t bop = st + XStage::bop;
        st_shared_v4(bop + sw128_offset(e, h * 4 + c4), hi);
        st_shared_v4(bop + 4096 + sw128_offset(e, h * 4 + c4), lo);
      }
      fence_proxy_async_smem();
      mbar_arrive(&ready[2 * s + h]);
      return true;
    };

    bool alive = nC == 0 || prepare(0);
    for (int c = 0; alive && c < nC; ++c) {
      const int s = c % kXStages;
      const uint32_t qb = stage_of(c) + XStage::q;
      const float* pre = prefix_of(c);

      // ---- P: mask j <= i, row sums, two bf16 parts back into TMEM
      bool ok = mbar_wait(&p_full[h], c & 1, abort_flag, err, kErrWait);
      tc_fence_after();
      if (bar_any(kBarHeadX + h, 128, !ok || *abort_flag)) break;
      const float psum = mask_split_p(tmem + lq + 128 * h, quad, lane);
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
      if (bar_any(kBarHeadX + h, 128, !ok || *abort_flag)) break;
      {
        float v[32];
        tmem_ld_32x32b_x32(tmem + lq + kColO + 32 * h, v);
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

// ---------------------------------------------------------------------------
// With RoPE. The numerator takes the rotated features, the denominator the
// unrotated ones (SANA-Video, section 2.2):
//   num_i = sum_{j <= i in chunk} (R_i phi(q_i) . R_j phi(k_j)) v_j + R_i phi(q_i) S_P
//   den_i = ReLU(q_i) . (z_P + Z_i) + eps,   Z_i = sum_{j <= i in chunk} ReLU(k_j)
// with S_P the prefix state of rotated keys and z_P that of plain key sums.
// Z = L ReLU(K_h) is a tensor-core product with L the 128 x 128 lower
// triangle of ones (kept in TMEM as an A operand). The rotated q and k enter
// their products in two bf16 parts each (the value truncated to bf16 and the
// rounded remainder: P = q_hi.k_hi + q_hi.k_lo + q_lo.k_hi, and likewise
// q.S), so the weights keep about 16 bits as in the unrotated kernel.
//
// Stage layout (two stages): the Q box, overwritten with the rotated q's
// high part; the low part; the K box, overwritten with the rotated k's high
// part; its low part; plain ReLU(k) per head ([128][32] bf16, 64-byte
// swizzle, the B operand of Z); V per head; the prefix S operand (hi, lo).
// The prefix state itself is copied into one buffer shared by the stages.
struct RStage {
  static constexpr int q = 0;
  static constexpr int qlo = q + kXBox;
  static constexpr int k = qlo + kXBox;
  static constexpr int klo = k + kXBox;
  static constexpr int kp = klo + kXBox;     // 2 x 8 KB
  static constexpr int v = kp + kXBox;       // 2 x 8 KB
  static constexpr int bop = v + kXBox;      // 2 x 4 KB
  static constexpr int bytes = bop + 2 * 4096;
  static constexpr int stride = (bytes + 1023) / 1024 * 1024;
};
constexpr int kRStages = 2;

struct RSmem {
  static constexpr int stages = 0;
  static constexpr int state = stages + kRStages * RStage::stride;  // [2 heads][1056] f32
  static constexpr int rope = state + 2 * kStateFloats * 4;         // RoPE (cos, sin) table
  static constexpr int bars = rope + kRopeTableMax * 8;
  // full[2] ready[2][2] o_done[2] st_full st_empty p_full[2] pm_ready[2] o_full[2] mma_done[2]
  static constexpr int nbars = 2 * kRStages + 2 * kRStages + kRStages + 2 + 8;
  static constexpr int misc = bars + nbars * 8;
  static constexpr int bytes = misc + 16;
};
constexpr int kRSmemBytes = RSmem::bytes + 1024;
static_assert(kRSmemBytes <= 232448, "shared memory per CTA");

// TMEM columns of the RoPE kernel: P of head h at 128 h, O at 256 + 32 h, Z at
// 320 + 32 h, L (bf16 pairs) at 384 .. 447.
constexpr uint32_t kRColO = 256, kRColZ = 320, kRColL = 384;

// Physical byte offset of 16-byte chunk c of row r in a 64-byte-swizzled tile
// of 64-byte rows (512-aligned base).
__device__ __forceinline__ uint32_t sw64_offset(uint32_t r, uint32_t c) {
  return r * 64u + ((c ^ ((r >> 1) & 3u)) << 4);
}

// Every chunk's key sum z_c = sum over its tokens of ReLU(k), into the z slot
// of the chunk-state buffer (the chunk-state reduce leaves it alone with
// RoPE). Block (x, c, b): 32 consecutive 16-byte vectors of a token row (head
// vec / 4, dims 8 (vec % 4) ..) over chunk c, eight warps taking 16 tokens
// each; the eight partial sums are added in warp order.
__global__ void __launch_bounds__(256)
chunk_key_sums(const __nv_bfloat16* K, float* states, int N, int H, int nchunks) {
  __shared__ float part[8][32][8];
  const int lane = threadIdx.x & 31, slice = threadIdx.x >> 5;
  const int vec = blockIdx.x * 32 + lane;
  const int c = blockIdx.y, b = blockIdx.z;
  pdl_wait();
  if (threadIdx.x == 0) pdl_trigger();
  const bool live = vec < H * 4;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
  if (live) {
    const int n0 = c * kXT + slice * 16;
    const int cnt = min(16, N - n0);  // tokens of this slice inside the sequence
    const size_t stride = static_cast<size_t>(H) * kD;
    const uint4* src = reinterpret_cast<const uint4*>(
        K + (static_cast<size_t>(b) * N + max(0, min(n0, N - 1))) * stride + vec * 8);
    uint4 u[16];
    if (cnt == 16) {  // all 16 loads in flight
#pragma unroll
      for (int t = 0; t < 16; ++t) u[t] = __ldg(src + t * stride / 8);
    } else {
#pragma unroll
      for (int t = 0; t < 16; ++t) u[t] = t < cnt ? __ldg(src + t * stride / 8) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      float x[8];
      unpack8(u[t], x);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += fmaxf(x[e], 0.0f);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[slice][lane][e] = acc[e];
  __syncthreads();
  if (slice == 0 && live) {
    float z[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) z[e] = part[0][lane][e];
    for (int t = 1; t < 8; ++t)
#pragma unroll
      for (int e = 0; e < 8; ++e) z[e] += part[t][lane][e];
    float* dst = states + ((static_cast<size_t>(b) * H + vec / 4) * nchunks + c) * kStateFloats +
                 kD * kD + (vec % 4) * 8;
    *reinterpret_cast<float4*>(dst) = make_float4(z[0], z[1], z[2], z[3]);
    *reinterpret_cast<float4*>(dst + 4) = make_float4(z[4], z[5], z[6], z[7]);
  }
}

// causal_chunk_rope_tc: the same CTA shape, roles and head pipelines as
// causal_chunk_tc. Per chunk and head, after the warpgroup has prepared the
// stage (ReLU, rotation, the two parts, plain ReLU(k), the S operand):
//   Z_h = L ReLU(K_h)                    M = 128, N = 32, K = 128 (A = L in TMEM)
//   P_h = three products of the parts    M = N = 128, K = 32
// then the mask and split of P as without RoPE, and
//   O_h = P_hi V_h + P_lo V_h + (q_hi S_hi + q_hi S_lo + q_lo S_hi)
// The warpgroup keeps ReLU(q) of its row (16 registers) from the preparation
// to the denominator.
template <int kRopeMode>
__global__ void __launch_bounds__(kRThreads, 1)
causal_chunk_rope_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                     const Problem p, const ChunkArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + RSmem::bars);
  uint64_t* ready = full + kRStages;          // [stage][head] stage prepared (128)
  uint64_t* o_done = ready + 2 * kRStages;    // [stage] O written over the Q box (256)
  uint64_t* st_full = o_done + kRStages;      // the chunk's prefix state copied in (1)
  uint64_t* st_empty = st_full + 1;           // the prefix state read (256)
  uint64_t* p_full = st_empty + 1;            // [head] Z and P in TMEM (1)
  uint64_t* pm_ready = p_full + 2;            // [head] P masked, in two parts (128)
  uint64_t* o_full = pm_ready + 2;            // [head] O in TMEM (1)
  uint64_t* mma_done = o_full + 2;           // [head] this head's MMAs drained (1)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + RSmem::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + RSmem::misc + 4);
  float2* rope_tab = reinterpret_cast<float2*>(smem + RSmem::rope);
  unsigned* err = &g_causal_chunk_error;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pair = blockIdx.y, b = blockIdx.z;
  const int h0 = pair * 2;
  const size_t cidx = static_cast<size_t>(b) * p.H + h0;
  const int c_begin = blockIdx.x * a.chunks_per_cta;
  const int nC = max(0, min(a.nchunks, c_begin + a.chunks_per_cta) - c_begin);
  const int heads = min(2, p.H - h0);

  if (tid == 0) {
    for (int i = 0; i < kRStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&ready[2 * i], 128);
      mbar_init(&ready[2 * i + 1], 128);
      mbar_init(&o_done[i], kXMath);
    }
    mbar_init(st_full, 1);
    mbar_init(st_empty, kXMath);
    for (int h = 0; h < 2; ++h) {
      mbar_init(&p_full[h], 1);
      mbar_init(&pm_ready[h], 128);
      mbar_init(&o_full[h], 1);
      mbar_init(&mma_done[h], 1);
    }
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
  if (kRopeMode == kRopeTable && tid >= 64) build_rope_table(p.rope, rope_tab, tid - 64, kXMath);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);
  if (tid >= 64 && tid < 64 + 128) {
    // L into TMEM: row i holds keys j <= i as bf16 ones (pairs per column)
    const int quad = warp & 3, row = quad * 32 + lane;
    const uint32_t lq = static_cast<uint32_t>(quad * 32) << 16;
#pragma unroll
    for (int cb = 0; cb < 4; ++cb) {
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int j = 32 * cb + 2 * e;
        pk[e] = (j <= row ? 0x3F80u : 0u) | (j + 1 <= row ? 0x3F800000u : 0u);
      }
      tmem_st_32x32b_x16(tmem + lq + kRColL + 16 * cb, pk);
    }
    tmem_st_wait();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  if (tid == 64) pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      auto stage_ptr = [&](int c) { return smem + RSmem::stages + (c % kRStages) * RStage::stride; };
      auto store_o = [&](int c) -> bool {
        if (!mbar_wait(&o_done[c % kRStages], (c / kRStages) & 1, abort_flag, err, kErrWait))
          return false;
        tma_store_3d(&tm_o, stage_ptr(c) + RStage::q, h0 * 32, (c_begin + c) * kXT, b);
        bulk_commit();
        bulk_wait_read<0>();
        return true;
      };
      bool ok = true;
      int c = 0;
      for (; ok && c < nC; ++c) {
        const int s = c % kRStages;
        if (c >= kRStages && !(ok = store_o(c - kRStages))) break;
        // the shared state buffer takes chunk c once chunk c - 1's has been read
        if (c > 0 && !(ok = mbar_wait(st_empty, (c - 1) & 1, abort_flag, err, kErrWait))) break;
        uint8_t* st = stage_ptr(c);
        const int y = (c_begin + c) * kXT;
        mbar_arrive_expect_tx(&full[s], 3 * kXBox);
        tma_load_3d(st + RStage::q, &tm_q, &full[s], h0 * 32, y, b);
        tma_load_3d(st + RStage::k, &tm_k, &full[s], h0 * 32, y, b);
        tma_load_3d(st + RStage::v, &tm_v, &full[s], h0 * 32, y, b);
        tma_load_3d(st + RStage::v + kXVBox, &tm_v, &full[s], h0 * 32 + 32, y, b);
        mbar_arrive_expect_tx(st_full, heads * kStateFloats * 4);
        for (int hh = 0; hh < heads; ++hh)
          bulk_load(smem + RSmem::state + hh * kStateFloats * 4,
                    a.prefix + ((cidx + hh) * a.nchunks + c_begin + c) * kStateFloats,
                    kStateFloats * 4, st_full);
      }
      for (int k = max(0, c - kRStages); ok && k < c; ++k) ok = store_o(k);
      for (int k = max(0, c - kRStages); k < c; ++k)
        mbar_drain(&full[k % kRStages], (k / kRStages) & 1, err, kErrWait);
      if (c > 0) mbar_drain(st_full, (c - 1) & 1, err, kErrWait);
      bulk_wait<0>();
    }
  } else if (warp == 1 || warp == kRThreads / 32 - 1) {
    // ------------------------------------------------------------ MMA, one head per warp
    if (lane == 0) {
      const int hm = warp == 1 ? 0 : 1;
      const uint32_t id_z = idesc_bf16_f32(128, 32, 0, 1);
      const uint32_t id_p = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_pv = idesc_bf16_f32(128, 32, 0, 1);
      const uint32_t id_qs = idesc_bf16_f32(128, 32, 0, 0);
      auto stage_addr = [&](int c) { return sbase + RSmem::stages + (c % kRStages) * RStage::stride; };
      auto issue_p = [&](int c, int h) -> bool {
        const int s = c % kRStages;
        if (!mbar_wait(&ready[2 * s + h], (c / kRStages) & 1, abort_flag, err, kErrWait)) return false;
        tc_fence_after();
        const uint32_t st = stage_addr(c);
        // Z_h = L ReLU(K_h): keys 16 kk .. 16 kk + 15 are columns 8 kk .. of L
        const uint64_t dkp = smem_desc_sw64_mn32(st + RStage::kp + h * kXVBox);
#pragma unroll
        for (int kk = 0; kk < kXT / 16; ++kk)
          mma_bf16_tmem_a(tmem + kRColZ + 32 * h, tmem + kRColL + 8 * kk, desc_at(dkp, kk * 1024),
                          id_z, kk > 0 ? 1u : 0u);
        // P_h = q_hi.k_hi + q_hi.k_lo + q_lo.k_hi (P of chunk c - 1 was read
        // by this thread's earlier P.V MMAs, which run first)
        const uint64_t dq = smem_desc_sw128(st + RStage::q, 16, 1024);
        const uint64_t dql = smem_desc_sw128(st + RStage::qlo, 16, 1024);
        const uint64_t dk = smem_desc_sw128(st + RStage::k, 16, 1024);
        const uint64_t dkl = smem_desc_sw128(st + RStage::klo, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_bf16(tmem + 128 * h, desc_at(dq, h * 64 + kk * 32), desc_at(dk, h * 64 + kk * 32), id_p,
                   kk);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_bf16(tmem + 128 * h, desc_at(dq, h * 64 + kk * 32), desc_at(dkl, h * 64 + kk * 32),
                   id_p, 1u);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_bf16(tmem + 128 * h, desc_at(dql, h * 64 + kk * 32), desc_at(dk, h * 64 + kk * 32),
                   id_p, 1u);
        mma_commit(&p_full[h]);
        return true;
      };
      auto issue_pv = [&](int c, int h) -> bool {
        if (!mbar_wait(&pm_ready[h], c & 1, abort_flag, err, kErrWait)) return false;
        tc_fence_after();
        const uint32_t st = stage_addr(c);
        const uint64_t dv = smem_desc_sw64_mn32(st + RStage::v + h * kXVBox);
        const uint32_t d = tmem + kRColO + 32 * h;
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int kk = 0; kk < kXT / 16; ++kk)
            mma_bf16_tmem_a(d, tmem + 128 * h + 32 * (kk >> 1) + 16 * part + 8 * (kk & 1),
                            desc_at(dv, kk * 1024), id_pv, (part > 0 || kk > 0) ? 1u : 0u);
        const uint64_t dq = smem_desc_sw128(st + RStage::q, 16, 1024);
        const uint64_t dql = smem_desc_sw128(st + RStage::qlo, 16, 1024);
        const uint64_t db = smem_desc_sw128(st + RStage::bop, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const uint32_t off = h * 64 + kk * 32;
          mma_bf16(d, desc_at(dq, off), desc_at(db, off), id_qs, 1u);
          mma_bf16(d, desc_at(dq, off), desc_at(db, 4096 + off), id_qs, 1u);
          mma_bf16(d, desc_at(dql, off), desc_at(db, off), id_qs, 1u);
        }
        mma_commit(&o_full[h]);
        return true;
      };
      bool ok = true;
      if (hm == 0) {
        for (int c = 0; ok && c < nC; ++c) ok = issue_p(c, 0) && issue_pv(c, 0);
      } else {
        for (int c = 0; ok && c < nC; ++c) ok = issue_p(c, 1) && issue_pv(c, 1);
      }
      mma_commit(&mma_done[hm]);
      mbar_drain(&mma_done[hm], 0, err, kErrWait);
    }
  } else {
    // ------------------------------------------------- math: one warpgroup per head
    const int mt = tid - 64;
    const int h = mt >> 7;
    const int wt = mt & 127;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lq = static_cast<uint32_t>(quad * 32) << 16;
    auto stage_of = [&](int c) { return sbase + RSmem::stages + (c % kRStages) * RStage::stride; };
    const float* state_h = reinterpret_cast<const float*>(smem + RSmem::state) + h * kStateFloats;
    uint32_t qp[16];    // ReLU(q) of this row, bf16 pairs: kept for the denominator
    float dpre = 0.0f;  // ReLU(q) . z_P + eps
    // grid position of this row's token in the next chunk to prepare, moved
    // on by one chunk (128 tokens) per preparation without divisions
    TokPos tp = token_pos(p.rope, min(c_begin * kXT + row, p.N - 1));
    // Chunk c's stage for this head: ReLU of q and k; plain ReLU(k) for Z;
    // q and k rotated by the row's token position and written back as two
    // bf16 parts (the value truncated to bf16, and the remainder rounded);
    // ReLU(q) . z_P; the prefix's S operand. Rows past the end of the
    // sequence are zeros (TMA fill) and are not rotated. False when a wait
    // gave up (decided by the warpgroup together).
    auto prepare = [&](int c) -> bool {
      const int s = c % kRStages;
      const int n = (c_begin + c) * kXT + row;
      const TokPos tpc = tp;
      tp.w += a.adv_w;
      tp.h += a.adv_h;
      tp.t += a.adv_t;
      if (tp.w >= p.rope.W) {
        tp.w -= p.rope.W;
        ++tp.h;
      }
      if (tp.h >= p.rope.Hh) {
        tp.h -= p.rope.Hh;
        ++tp.t;
      }
      bool ok = mbar_wait(&full[s], (c / kRStages) & 1, abort_flag, err, kErrWait);
      ok = ok && mbar_wait(st_full, c & 1, abort_flag, err, kErrWait);
      if (bar_any(kBarHeadX + h, 128, !ok || *abort_flag)) return false;
      const uint32_t st = stage_of(c);
      float2 cs0[8], cs1[8];  // (cos, sin) of the row's 16 pairs
      // q: ReLU (kept for the denominator), ReLU(q) . z_P, rotation, two parts
      {
        float x[2][16];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint4 u = ld_shared_v4(st + RStage::q + sw128_offset(row, h * 4 + c4));
          u.x = relu_bf16x2(u.x); u.y = relu_bf16x2(u.y); u.z = relu_bf16x2(u.z); u.w = relu_bf16x2(u.w);
          qp[4 * c4] = u.x; qp[4 * c4 + 1] = u.y; qp[4 * c4 + 2] = u.z; qp[4 * c4 + 3] = u.w;
          float t[8];
          unpack8(u, t);
#pragma unroll
          for (int k = 0; k < 8; ++k) x[c4 >> 1][(c4 & 1) * 8 + k] = t[k];
        }
        float dz[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // four partial sums
        const float4* z4 = reinterpret_cast<const float4*>(state_h + kD * kD);
#pragma unroll
        for (int d4 = 0; d4 < kD / 4; ++d4) {
          const float4 z = h < heads ? z4[d4] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          const float* xv = &x[d4 >> 2][(d4 & 3) * 4];
          dz[0] = fmaf(xv[0], z.x, dz[0]);
          dz[1] = fmaf(xv[1], z.y, dz[1]);
          dz[2] = fmaf(xv[2], z.z, dz[2]);
          dz[3] = fmaf(xv[3], z.w, dz[3]);
        }
        dpre = ((dz[0] + dz[1]) + (dz[2] + dz[3])) + p.eps;
        if (n < p.N) {
          if (kRopeMode == kRopeTable) {
            const RopeBases rbs = rope_bases(p.rope, tpc);
            rope_table8<0>(rope_tab, rbs, cs0);
            rope_table8<1>(rope_tab, rbs, cs1);
          } else {
            rope_fly8<0>(p.rope, tpc, cs0);
            rope_fly8<1>(p.rope, tpc, cs1);
          }
          rotate8(x[0], cs0);
          rotate8(x[1], cs1);
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint4 hi, lo;
          split_bf16x8(&x[c4 >> 1][(c4 & 1) * 8], hi, lo);
          st_shared_v4(st + RStage::q + sw128_offset(row, h * 4 + c4), hi);
          st_shared_v4(st + RStage::qlo + sw128_offset(row, h * 4 + c4), lo);
        }
      }
      // k: ReLU (plain copy for Z), rotation, two parts
      {
        float x[2][16];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint4 w = ld_shared_v4(st + RStage::k + sw128_offset(row, h * 4 + c4));
          w.x = relu_bf16x2(w.x); w.y = relu_bf16x2(w.y); w.z = relu_bf16x2(w.z); w.w = relu_bf16x2(w.w);
          st_shared_v4(st + RStage::kp + h * kXVBox + sw64_offset(row, c4), w);
          float t[8];
          unpack8(w, t);
#pragma unroll
          for (int k = 0; k < 8; ++k) x[c4 >> 1][(c4 & 1) * 8 + k] = t[k];
        }
        if (n < p.N) {
          rotate8(x[0], cs0);
          rotate8(x[1], cs1);
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint4 hi, lo;
          split_bf16x8(&x[c4 >> 1][(c4 & 1) * 8], hi, lo);
          st_shared_v4(st + RStage::k + sw128_offset(row, h * 4 + c4), hi);
          st_shared_v4(st + RStage::klo + sw128_offset(row, h * 4 + c4), lo);
        }
      }
      {
        // the prefix's S as the B operand: row e holds S[0..31][e] of this
        // head in two bf16 parts (thread wt: row e = wt % 32, dims 8 (wt / 32) ..;
        // the state reads of a warp are then 32 consecutive floats)
        const int e = wt & 31, c4 = wt >> 5;
        float x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = h < heads ? state_h[(c4 * 8 + k) * kD + e] : 0.0f;
        uint4 hi, lo;
        split_bf16x8(x, hi, lo);
        st_shared_v4(st + RStage::bop + sw128_offset(e, h * 4 + c4), hi);
        st_shared_v4(st + RStage::bop + 4096 + sw128_offset(e, h * 4 + c4), lo);
      }
      fence_proxy_async_smem();
      tc_fence_before();  // this thread's TMEM reads of the previous chunk come first
      mbar_arrive(&ready[2 * s + h]);
      mbar_arrive(st_empty);
      return true;
    };

    bool alive = nC == 0 || prepare(0);
    for (int c = 0; alive && c < nC; ++c) {
      const int s = c % kRStages;
      const uint32_t qb = stage_of(c) + RStage::q;

      // ---- P: mask j <= i, two bf16 parts back into TMEM
      bool ok = mbar_wait(&p_full[h], c & 1, abort_flag, err, kErrWait);
      tc_fence_after();
      if (bar_any(kBarHeadX + h, 128, !ok || *abort_flag)) break;
      mask_split_p(tmem + lq + 128 * h, quad, lane);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&pm_ready[h]);

      // ---- den = ReLU(q) . (z_P + Z_i) + eps
      float den = dpre;
      {
        float zr[32];
        tmem_ld_32x32b_x32(tmem + lq + kRColZ + 32 * h, zr);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          float x[8];
          unpack8(make_uint4(qp[4 * c4], qp[4 * c4 + 1], qp[4 * c4 + 2], qp[4 * c4 + 3]), x);
#pragma unroll
          for (int k = 0; k < 8; ++k) den = fmaf(x[k], zr[c4 * 8 + k], den);
        }
      }

      // ---- the next chunk, ahead of this chunk's output
      if (c + 1 < nC && !prepare(c + 1)) break;

      // ---- O = numerator / den over this head's columns of the Q box
      ok = mbar_wait(&o_full[h], c & 1, abort_flag, err, kErrWait);
      tc_fence_after();
      if (bar_any(kBarHeadX + h, 128, !ok || *abort_flag)) break;
      {
        float v[32];
        tmem_ld_32x32b_x32(tmem + lq + kRColO + 32 * h, v);
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
      mbar_arrive(&o_done[s]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kXTmemCols);
  }
}
// Exclusive prefix over the chunks, per head and float4 column: chunk c's
// state becomes carry + the sum of the chunks before it (update: the carry
// becomes carry + the sum of all chunks). The chunk axis is cut into `segs`
// segments (a power of two, so that a segment holds about kPrefBatch chunks);
// a block covers 256 / segs consecutive float4 columns, each warp's lanes
// consecutive columns of one segment. Each thread sums its segment, the block
// exchanges the segment totals in shared memory, and each thread writes
// carry + the earlier segments' totals + the earlier chunks of its own
// segment. The sum order is fixed by the shape.
constexpr int kPrefThreads = 256, kPrefMaxSeg = 16, kPrefBatch = 8;

int prefix_segments(int nchunks) {
  int segs = 1;
  while (segs < kPrefMaxSeg && segs * kPrefBatch < nchunks) segs *= 2;
  return segs;
}

__global__ void __launch_bounds__(kPrefThreads, 4)
chunk_prefix(float* states, int bh_count, int nchunks, int segs, float* S_carry, float* z_carry,
             int update) {
  constexpr int kVec = kStateFloats / 4;
  constexpr int kStride = kStateFloats / 4;  // float4 between consecutive chunks
  __shared__ float4 seg_total[kPrefThreads];
  const int cpb = kPrefThreads / segs;
  const int col = threadIdx.x % cpb, seg = threadIdx.x / cpb;
  const long long g = static_cast<long long>(blockIdx.x) * cpb + col;
  pdl_wait();
  if (threadIdx.x == 0) pdl_trigger();
  const bool live = g < static_cast<long long>(bh_count) * kVec;
  const int bh = live ? static_cast<int>(g / kVec) : 0;
  const int i = live ? static_cast<int>(g % kVec) * 4 : 0;
  const bool is_s = i < kD * kD;
  float* carry = !live || S_carry == nullptr
                     ? nullptr
                     : (is_s ? S_carry + static_cast<size_t>(bh) * kD * kD + i
                             : z_carry + static_cast<size_t>(bh) * kD + (i - kD * kD));
  float4* colp = reinterpret_cast<float4*>(states + static_cast<size_t>(bh) * nchunks * kStateFloats + i);
  const int len = (nchunks + segs - 1) / segs;
  const int c0 = min(nchunks, seg * len), c1 = live ? min(nchunks, c0 + len) : c0;
  auto add4 = [](float4 x, float4 y) { return make_float4(x.x + y.x, x.y + y.y, x.z + y.z, x.w + y.w); };
  const float4 zero = make_float4(0.0f, 0.0f, 0.0f, 0.0f);

  // the segment's sum (kept in registers when the segment is one batch)
  float4 d[kPrefBatch];
  float4 sum = zero;
  for (int c = c0; c < c1; c += kPrefBatch) {
#pragma unroll
    for (int k = 0; k < kPrefBatch; ++k)
      d[k] = c + k < c1 ? __ldcg(colp + static_cast<size_t>(c + k) * kStride) : zero;
#pragma unroll
    for (int k = 0; k < kPrefBatch; ++k) sum = add4(sum, d[k]);
  }
  seg_total[threadIdx.x] = sum;
  __syncthreads();
  float4 acc = carry != nullptr ? *reinterpret_cast<const float4*>(carry) : zero;
  for (int t = 0; t < seg; ++t) acc = add4(acc, seg_total[t * cpb + col]);

  // the exclusive prefixes of the segment's chunks (a second read only when
  // the segment is longer than one batch)
  const bool one_batch = c1 - c0 <= kPrefBatch;
  for (int c = c0; c < c1; c += kPrefBatch) {
    if (!one_batch) {
#pragma unroll
      for (int k = 0; k < kPrefBatch; ++k)
        d[k] = c + k < c1 ? __ldcg(colp + static_cast<size_t>(c + k) * kStride) : zero;
    }
#pragma unroll
    for (int k = 0; k < kPrefBatch; ++k)
      if (c + k < c1) {
        __stcg(colp + static_cast<size_t>(c + k) * kStride, acc);
        acc = add4(acc, d[k]);
      }
  }
  // the last segment ends on the sum of everything (an empty one adds nothing)
  if (update && carry != nullptr && seg == segs - 1) *reinterpret_cast<float4*>(carry) = acc;
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

// V as [B][N][H*32] bf16 with a box of one head: 32 dims x 128 tokens x 1,
// 64-byte swizzle.
cudaError_t make_map_head(CUtensorMap* m, const void* base, const Problem& p) {
  cudaError_t e = get_encoder();
  if (e != cudaSuccess) return e;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(p.H) * kD, static_cast<cuuint64_t>(p.N),
                              static_cast<cuuint64_t>(p.B)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(p.H) * kD * 2,
                                 static_cast<cuuint64_t>(p.N) * p.H * kD * 2};
  const cuuint32_t box[3] = {kD, static_cast<cuuint32_t>(kXT), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

bool causal_chunk_supported(const Problem& p) { return p.io == LA_IO_BF16 && p.N > 0; }

size_t causal_chunk_state_bytes(const Problem& p) {
  const size_t nchunks = static_cast<size_t>((p.N + kXT - 1) / kXT);
  return static_cast<size_t>(p.B) * p.H * nchunks * kStateFloats * sizeof(float);
}

cudaError_t launch_causal_chunks(const Problem& p, const void* Q, const void* K, const void* V,
                                 float* states, float* S_carry, float* z_carry, int update,
                                 void* O, cudaStream_t s) {
  if (!causal_chunk_supported(p)) return cudaErrorNotSupported;
  const int nchunks = (p.N + kXT - 1) / kXT;
  // (1) every chunk's own state (with RoPE its key sums come from a second kernel)
  cudaError_t e = launch_chunk_states_tc(p, K, V, states, nchunks, s);
  if (e != cudaSuccess) return e;
  if (p.rope.enabled) {
    const __nv_bfloat16* kp = static_cast<const __nv_bfloat16*>(K);
    float* st = states;
    int n = p.N, hh = p.H, nc = nchunks;
    void* args[] = {&kp, &st, &n, &hh, &nc};
    const dim3 grid(static_cast<unsigned>((p.H * 4 + 31) / 32), static_cast<unsigned>(nchunks),
                    static_cast<unsigned>(p.B));
    e = launch_pdl_x(reinterpret_cast<const void*>(chunk_key_sums), args, grid, dim3(256), 0, s);
    if (e != cudaSuccess) return e;
  }
  // (2) the exclusive prefix over the chunks (and the carry update)
  {
    int bh = p.B * p.H;
    int nc = nchunks;
    float* st = states;
    float* sc = S_carry;
    float* zc = z_carry;
    int up = update;
    int segs = prefix_segments(nchunks);
    void* args[] = {&st, &bh, &nc, &segs, &sc, &zc, &up};
    const long long cols = static_cast<long long>(bh) * (kStateFloats / 4);
    const int cpb = kPrefThreads / segs;
    const dim3 grid(static_cast<unsigned>((cols + cpb - 1) / cpb));
    e = launch_pdl_x(reinterpret_cast<const void*>(chunk_prefix), args, grid, dim3(kPrefThreads),
                     0, s);
    if (e != cudaSuccess) return e;
  }
  // (3) every chunk on its own
  CUtensorMap mq, mk, mv, mo;
  if ((e = make_map(&mq, Q, p, kXT)) != cudaSuccess) return e;
  if ((e = make_map(&mk, K, p, kXT)) != cudaSuccess) return e;
  if ((e = make_map_head(&mv, V, p)) != cudaSuccess) return e;
  if ((e = make_map(&mo, O, p, kXT)) != cudaSuccess) return e;
  const RopeTable rt = rope_table_for(p);
  const int mode = rope_mode(rt);
  const void* kern = mode == kNoRope      ? reinterpret_cast<const void*>(causal_chunk_tc)
                     : mode == kRopeTable ? reinterpret_cast<const void*>(causal_chunk_rope_tc<kRopeTable>)
                                          : reinterpret_cast<const void*>(causal_chunk_rope_tc<kRopeOnTheFly>);
  const int smem_bytes = mode == kNoRope ? kXSmemBytes : kRSmemBytes;
  if ((e = ensure_smem_attr(mode, kern, smem_bytes)) != cudaSuccess) return e;
  const int pairs = (p.H + 1) / 2;
  const long long units = static_cast<long long>(pairs) * p.B;
  int ctas = static_cast<int>(std::max<long long>(1, kNumSMs / std::max<long long>(1, units)));
  ctas = std::min(ctas, nchunks);
  ChunkArgs a = {};
  a.prefix = states;
  a.nchunks = nchunks;
  a.chunks_per_cta = (nchunks + ctas - 1) / ctas;
  if (p.rope.enabled) {
    a.adv_w = kXT % p.rope.W;
    a.adv_h = (kXT / p.rope.W) % p.rope.Hh;
    a.adv_t = (kXT / p.rope.W) / p.rope.Hh;
  }
  ctas = (nchunks + a.chunks_per_cta - 1) / a.chunks_per_cta;
  Problem pc = p;
  void* args[] = {&mq, &mk, &mv, &mo, &pc, &a};
  e = launch_pdl_x(kern, args, dim3(ctas, pairs, p.B), dim3(kRThreads), smem_bytes, s);
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
