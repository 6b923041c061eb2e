// Token-causal linear attention on the tensor cores (bf16 I/O, no RoPE):
// query n sees keys 0..n ("SANA-Video: Efficient Video Generation with Block
// Linear Diffusion Transformer", section 2.3, with the sum over earlier j read
// at token granularity). With phi = ReLU and the running state R (carry plus
// every earlier token):
//
//   O_i = (sum_{j<=i in chunk} (phi(q_i).phi(k_j)) v_j + phi(q_i) R_S)
//         / (sum_{j<=i in chunk} phi(q_i).phi(k_j) + phi(q_i).R_z + eps)
//
// (without RoPE the denominator's ReLU(q).ReLU(k) is the numerator's weight
// itself, so one matrix serves both).
//
// A CTA owns two heads (one 64-dim TMA box per tensor) of one batch element
// and one token split, and walks it in 128-token chunks (two stages of Q, K
// and V in flight). Per chunk and head, on the tensor cores:
//   P   = phi(Q) phi(K)^T        M = N = 128 tokens, K = 32      (TMEM)
//   O   = mask(P) V + phi(Q) R   M = 128, N = 64 / 32, K = 128 / 32 (TMEM)
//   R  += phi(K)^T V             the reduce's M = 128 (dims), N = 64 form
// and on CUDA cores, one warpgroup per head (thread = token row): the mask
// j <= i, the row sums of P (the denominator), P to shared memory for the
// second MMA, 1 / den, and R back to shared memory as the next chunk's B
// operand. P and R enter their MMAs as the sum of two bf16 numbers (the
// rounded value and the rounded remainder, one MMA each), so the weights keep
// about 16 bits: one bf16 rounding (2^-9) of the weights of a few
// near-cancelling values would otherwise exceed the output tolerance. The two
// heads take turns through one such pair of shared-memory P tiles. The split starts from the carry plus the earlier splits' partial
// states (left in the workspace by the state reduce), summed in split order.
#include <algorithm>

#include "la_tc_common.cuh"

namespace la {

// Device error word of the token-causal kernel (bounded waits that gave up).
__device__ unsigned g_causal_tc_error;

namespace {

constexpr int kCT = 128;                 // tokens per chunk
constexpr int kCBox = kCT * 128;         // [128 tokens][64 dims] bf16 = 16 KB
constexpr int kCStage = 3 * kCBox;       // Q, K, V boxes
constexpr int kCStages = 2;
constexpr int kCMath = 256;              // two warpgroups, one per head
constexpr int kCThreads = 64 + kCMath;
constexpr int kCTmemCols = 512;
constexpr int kBarBoth = 1;              // named barrier over both warpgroups
constexpr int kBarHead0 = 2;             // + head

// TMEM columns
constexpr uint32_t kColP = 0;            // P of head h at kColP + 128 h
constexpr uint32_t kColO = 256;          // O of head h at kColO + 64 h
constexpr uint32_t kColR = 384;          // running-state accumulator (64 columns)

struct CSmem {
  static constexpr int stages = 0;                              // [2][Q, K, V]
  static constexpr int pmat = stages + kCStages * kCStage;      // [hi, lo][2 boxes][128][128 B]
  static constexpr int bop = pmat + 2 * 2 * kCBox;              // R as B operand: [hi, lo][32][128 B]
  static constexpr int prefix = bop + 2 * 4096;                 // [2][32][32] f32
  static constexpr int rz = prefix + 2 * kD * kD * 4;           // [2][32] f32: running z
  static constexpr int zwarp = rz + 2 * kD * 4;                 // [8 warps][32] f32: key sums
  static constexpr int rtmp = zwarp + 8 * kD * 4;               // [2][32][33] f32
  static constexpr int bars = rtmp + 2 * kD * (kD + 1) * 4;
  // full[2] empty[2] ready[2] p_full[2] pm_ready[2] o_full[2] st_full bop_ready mma_done pm_free
  static constexpr int nbars = 6 * 2 + 4;
  static constexpr int misc = bars + nbars * 8;
  static constexpr int bytes = misc + 16;
};
constexpr int kCSmemBytes = CSmem::bytes + 1024;
static_assert(kCSmemBytes <= 232448, "shared memory per CTA");

struct CausalArgs {
  const float* partials;  // [B*H][splits][kStateFloats]: each split's own state
  float* S_carry;         // may be null (zero carry)
  float* z_carry;
  int update;             // fold the whole sequence into the carry
  unsigned* counters;     // [B*H] arrival words (index b*H + h0), left zero
};

// lo[k] = x[k] - (the bf16 value in hi): the remainder of rounding x to bf16,
// itself rounded to bf16 when it is stored.
__device__ __forceinline__ void split_lo(const uint4& hi, const float (&x)[8], float (&lo)[8]) {
  float h8[8];
  unpack8(hi, h8);
#pragma unroll
  for (int k = 0; k < 8; ++k) lo[k] = x[k] - h8[k];
}

// Sum of 32 values held one per lane over the 32 lanes, for 32 different
// quantities at once: lane l ends with the total of quantity l (31 shuffles).
__device__ __forceinline__ float warp_transpose_sum(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      // keep the half of the quantities this lane is responsible for
      const float send = upper ? v[i] : v[i + w];
      const float keep = upper ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return v[0];
}

__global__ void __launch_bounds__(kCThreads, 1)
causal_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
          const Problem p, const CausalArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + CSmem::bars);
  uint64_t* empty = full + 2;      // 2 arrivals: the MMAs and the O store are done with the stage
  uint64_t* ready = empty + 2;     // the chunk's Q and K are ReLU'd (256 arrivals)
  uint64_t* p_full = ready + 2;    // [head] P in TMEM
  uint64_t* pm_ready = p_full + 2; // [head] masked P in shared memory, O columns free (128)
  uint64_t* o_full = pm_ready + 2; // [head] O in TMEM
  uint64_t* st_full = o_full + 2;  // the chunk's state MMA is done
  uint64_t* bop_ready = st_full + 1;  // R of the next chunk in shared memory (256 arrivals)
  uint64_t* mma_done = bop_ready + 1;
  uint64_t* pm_free = mma_done + 1;   // the P tiles' last reader (an MMA) is done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + CSmem::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + CSmem::misc + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + CSmem::misc + 8);
  float* prefix = reinterpret_cast<float*>(smem + CSmem::prefix);
  float* rz = reinterpret_cast<float*>(smem + CSmem::rz);
  float* zwarp = reinterpret_cast<float*>(smem + CSmem::zwarp);
  float* rtmp = reinterpret_cast<float*>(smem + CSmem::rtmp);
  unsigned* err = &g_causal_tc_error;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pair = blockIdx.y, b = blockIdx.z, split = blockIdx.x;
  const int h0 = pair * 2;
  const size_t cidx = static_cast<size_t>(b) * p.H + h0;
  const int n_begin = split * p.chunk;
  const int n_end = min(p.N, n_begin + p.chunk);
  const int nC = n_end > n_begin ? (n_end - n_begin + kCT - 1) / kCT : 0;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 2);
      mbar_init(&ready[i], kCMath);
      mbar_init(&p_full[i], 1);
      mbar_init(&pm_ready[i], 128);
      mbar_init(&o_full[i], 1);
    }
    mbar_init(st_full, 1);
    mbar_init(bop_ready, kCMath);
    mbar_init(mma_done, 1);
    mbar_init(pm_free, 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kCTmemCols);
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
    // ------------------------------------------------------------ TMA loads
    if (lane == 0) {
      int c = 0;
      for (; c < nC; ++c) {
        const int s = c & 1;
        if (!mbar_wait(&empty[s], ((c >> 1) & 1) ^ 1, abort_flag, err, kErrWait)) break;
        mbar_arrive_expect_tx(&full[s], kCStage);
        uint8_t* st = smem + CSmem::stages + s * kCStage;
        const int y = n_begin + c * kCT;
        tma_load_3d(st, &tm_q, &full[s], h0 * 32, y, b);
        tma_load_3d(st + kCBox, &tm_k, &full[s], h0 * 32, y, b);
        tma_load_3d(st + 2 * kCBox, &tm_v, &full[s], h0 * 32, y, b);
      }
      for (int q = max(0, c - kCStages); q < c; ++q)
        mbar_drain(&full[q & 1], (q >> 1) & 1, err, kErrWait);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t id_p = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_pv = idesc_bf16_f32(128, 64, 0, 1);
      const uint32_t id_qr = idesc_bf16_f32(128, 32, 0, 0);
      const uint32_t id_st = idesc_bf16_f32(128, 64, 1, 1);
      const uint32_t bop = sbase + CSmem::bop;
      bool ok = true;
      for (int c = 0; ok && c < nC; ++c) {
        const int s = c & 1;
        const uint32_t par = c & 1;
        const uint32_t st = sbase + CSmem::stages + s * kCStage;
        const uint32_t qb = st, kb = st + kCBox, vb = st + 2 * kCBox;
        if (!(ok = mbar_wait(&ready[s], (c >> 1) & 1, abort_flag, err, kErrWait))) break;
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // P = phi(Q) phi(K)^T
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_bf16(tmem + kColP + 128 * h, smem_desc_sw128(qb + h * 64 + kk * 32, 16, 1024),
                     smem_desc_sw128(kb + h * 64 + kk * 32, 16, 1024), id_p, kk);
          mma_commit(&p_full[h]);
        }
        for (int h = 0; ok && h < 2; ++h) {
          if (!(ok = mbar_wait(&pm_ready[h], par, abort_flag, err, kErrWait))) break;
          if (h == 0 && !(ok = mbar_wait(bop_ready, par, abort_flag, err, kErrWait))) break;
          tc_fence_after();
#pragma unroll
          for (int part = 0; part < 2; ++part) {  // O = mask(P) V, P = P_hi + P_lo
            const uint32_t pm = sbase + CSmem::pmat + part * 2 * kCBox;
#pragma unroll
            for (int kk = 0; kk < kCT / 16; ++kk)  // (both heads' V columns)
              mma_bf16(tmem + kColO + 64 * h,
                       smem_desc_sw128(pm + (kk >> 2) * kCBox + (kk & 3) * 32, 16, 1024),
                       smem_desc_sw128(vb + kk * 2048, kCBox, 1024), id_pv,
                       (part > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(pm_free);
#pragma unroll
          for (int part = 0; part < 2; ++part)  // O += phi(Q) R, R = R_hi + R_lo
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)  // (this head's columns)
              mma_bf16(tmem + kColO + 64 * h + 32 * h,
                       smem_desc_sw128(qb + h * 64 + kk * 32, 16, 1024),
                       smem_desc_sw128(bop + part * 4096 + h * 64 + kk * 32, 16, 1024), id_qr,
                       1u);
          mma_commit(&o_full[h]);
        }
        if (!ok) break;
#pragma unroll
        for (int kk = 0; kk < kCT / 16; ++kk)  // R += phi(K)^T V (rows 64..127 unused)
          mma_bf16(tmem + kColR, smem_desc_sw128(kb + kk * 2048, kCBox, 1024),
                   smem_desc_sw128(vb + kk * 2048, kCBox, 1024), id_st,
                   (c > 0 || kk > 0) ? 1u : 0u);
        mma_commit(st_full);
        mma_commit(&empty[s]);
      }
      mma_commit(mma_done);
      mbar_drain(mma_done, 0, err, kErrWait);
    }
  } else {
    // ------------------------------------------------- math: one warpgroup per head
    const int mt = tid - 64;
    const int h = mt >> 7;           // head of the pair owned by this warpgroup
    const int quad = warp & 3;       // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;
    const int wiw = (warp - 2) & 3;  // warp index inside the warpgroup
    bool alive = true;
    float* pre = prefix + h * kD * kD;
    float* rzh = rz + h * kD;
    float* rt = rtmp + h * kD * (kD + 1);

    // ---- starting state: carry + the earlier splits' partials, in split order
    for (int i = mt; i < 2 * kStateFloats; i += kCMath) {
      const int hh = i / kStateFloats, k = i % kStateFloats;
      float acc = 0.0f;
      if (h0 + hh < p.H) {
        const size_t bh = cidx + hh;
        if (a.S_carry != nullptr)
          acc = k < kD * kD ? a.S_carry[bh * kD * kD + k] : a.z_carry[bh * kD + k - kD * kD];
        const float* src = a.partials + bh * p.splits * kStateFloats + k;
        for (int s2 = 0; s2 < split; ++s2) acc += __ldcg(src + static_cast<size_t>(s2) * kStateFloats);
      }
      if (k < kD * kD) prefix[hh * kD * kD + k] = acc;
      else rz[hh * kD + k - kD * kD] = acc;
    }
    named_bar_sync(kBarBoth, kCMath);
    // ---- the last CTA of the head pair to have read the carry folds the
    // whole sequence into it
    if (a.update) {
      if (mt == 0) {
        fence_acq_rel_gpu();
        const unsigned prev = atomicAdd(&a.counters[cidx], 1u);
        *last_flag = prev == gridDim.x - 1;
        if (*last_flag) fence_acq_rel_gpu();
      }
      named_bar_sync(kBarBoth, kCMath);
      if (*last_flag) {
        for (int i = mt; i < 2 * kStateFloats; i += kCMath) {
          const int hh = i / kStateFloats, k = i % kStateFloats;
          if (h0 + hh >= p.H) continue;
          const size_t bh = cidx + hh;
          float* dst = k < kD * kD ? a.S_carry + bh * kD * kD + k : a.z_carry + bh * kD + k - kD * kD;
          float acc = *dst;
          const float* src = a.partials + bh * p.splits * kStateFloats + k;
          for (int s2 = 0; s2 < p.splits; ++s2) acc += __ldcg(src + static_cast<size_t>(s2) * kStateFloats);
          *dst = acc;
        }
        if (mt == 0) a.counters[cidx] = 0u;
      }
    }

    // ---- R of chunk 0 as the B operand: row e holds R_h[0..31][e] in bf16
    auto build_bop = [&](bool with_acc) {
      if (quad == h) {  // the warp that can read TMEM lanes 32h..32h+31 (state rows of head h)
        float v[32];
        if (with_acc) {
          tmem_ld_32x32b_x32(tmem + kColR + (static_cast<uint32_t>(32 * h) << 16) + 32 * h, v);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0.0f;
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) rt[lane * (kD + 1) + e] = v[e] + pre[lane * kD + e];
        __syncwarp();
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          float x[8], lo[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) x[k] = rt[(c4 * 8 + k) * (kD + 1) + lane];
          const uint4 hi = pack8(x);
          split_lo(hi, x, lo);
          st_shared_v4(sbase + CSmem::bop + sw128_offset(lane, h * 4 + c4), hi);
          st_shared_v4(sbase + CSmem::bop + 4096 + sw128_offset(lane, h * 4 + c4), pack8(lo));
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(bop_ready);
    };
    build_bop(false);

    for (int c = 0; c < nC; ++c) {
      const int s = c & 1;
      const uint32_t par = c & 1;
      const uint32_t st = sbase + CSmem::stages + s * kCStage;
      const uint32_t qb = st, kb = st + kCBox;
      bool ok = mbar_wait(&full[s], (c >> 1) & 1, abort_flag, err, kErrWait);
      if (bar_any(kBarBoth, kCMath, !ok || *abort_flag)) {
        alive = false;
        break;
      }

      // ---- ReLU in place on this head's Q and K columns; the chunk's key sum
      float kp[32];
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
        float x[8];
        unpack8(w, x);
#pragma unroll
        for (int e = 0; e < 8; ++e) kp[c4 * 8 + e] = x[e];
      }
      fence_proxy_async_smem();
      mbar_arrive(&ready[s]);
      zwarp[(h * 4 + wiw) * kD + lane] = warp_transpose_sum(kp, lane);

      // ---- P: mask j <= i, row sums (the denominator), bf16 into shared memory
      // every break decision is taken by both warpgroups together, so neither
      // is left waiting in a barrier the other has skipped
      ok = mbar_wait(&p_full[h], par, abort_flag, err, kErrWait);
      tc_fence_after();
      if (bar_any(kBarBoth, kCMath, !ok || *abort_flag)) {
        alive = false;
        break;
      }
      // the P tiles are free once the other head's (or the previous chunk's)
      // PV MMAs have run: head 0 of chunk c waits for completion 2c - 1 of
      // pm_free, head 1 for completion 2c (each waits for its phases in order)
      // (a wait that gives up raises the abort flag, which the next decision
      // point of both warpgroups acts on)
      ok = mbar_wait(pm_free, h == 0 ? 1u : 0u, abort_flag, err, kErrWait);
      if (!ok) alive = false;
      const uint32_t pm = sbase + CSmem::pmat;
      float psum = 0.0f;
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        float v[32];
        tmem_ld_32x32b_x32(tmem + kColP + 128 * h + (static_cast<uint32_t>(quad * 32) << 16) + 32 * q, v);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = q * 32 + c4 * 8 + e;
            x[e] = j <= row ? v[c4 * 8 + e] : 0.0f;
            psum += x[e];
          }
          const int cj = q * 4 + c4;  // 16-byte chunk of the 256-byte row
          float lo[8];
          const uint4 hi = pack8(x);
          split_lo(hi, x, lo);
          st_shared_v4(pm + (cj >> 3) * kCBox + sw128_offset(row, cj & 7), hi);
          st_shared_v4(pm + 2 * kCBox + (cj >> 3) * kCBox + sw128_offset(row, cj & 7), pack8(lo));
        }
      }
      float den = psum + p.eps;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        float x[8];
        unpack8(ld_shared_v4(qb + sw128_offset(row, h * 4 + c4)), x);
#pragma unroll
        for (int e = 0; e < 8; ++e) den = fmaf(x[e], rzh[c4 * 8 + e], den);
      }
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(&pm_ready[h]);
      // the chunk's keys join the running key sum (after its denominators)
      named_bar_sync(kBarHead0 + h, 128);
      if (wiw == 0) {
        float zsum = 0.0f;
#pragma unroll
        for (int w2 = 0; w2 < 4; ++w2) zsum += zwarp[(h * 4 + w2) * kD + lane];
        rzh[lane] += zsum;
      }

      // ---- O = (mask(P) V + phi(Q) R) / den, over this head's columns of the Q tile
      ok = mbar_wait(&o_full[h], par, abort_flag, err, kErrWait);
      tc_fence_after();
      if (bar_any(kBarBoth, kCMath, !ok || *abort_flag)) {
        alive = false;
        break;
      }
      {
        float v[32];
        tmem_ld_32x32b_x32(tmem + kColO + 64 * h + 32 * h + (static_cast<uint32_t>(quad * 32) << 16), v);
        const float inv = 1.0f / den;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = v[c4 * 8 + e] * inv;
          st_shared_v4(qb + sw128_offset(row, h * 4 + c4), pack8(x));
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      named_bar_sync(kBarBoth, kCMath);
      if (mt == 0) {
        tma_store_3d(&tm_o, smem + CSmem::stages + s * kCStage, h0 * 32, n_begin + c * kCT, b);
        bulk_commit();
        bulk_wait_read<0>();
        mbar_arrive(&empty[s]);
      }

      // ---- R after this chunk, as the next chunk's B operand
      ok = mbar_wait(st_full, par, abort_flag, err, kErrWait);
      tc_fence_after();
      if (bar_any(kBarBoth, kCMath, !ok || *abort_flag)) {
        alive = false;
        break;
      }
      if (c + 1 < nC) build_bop(true);
      tc_fence_before();
    }
    if (mt == 0) bulk_wait<0>();
    (void)alive;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCTmemCols);
  }
}

}  // namespace

bool causal_tc_supported(const Problem& p) { return p.io == LA_IO_BF16 && p.N > 0 && !p.rope.enabled; }

cudaError_t launch_causal_tc(const Problem& p, const void* Q, const void* K, const void* V,
                             const float* partials, float* S_carry, float* z_carry, int update,
                             unsigned* counters, void* O, cudaStream_t s) {
  if (!causal_tc_supported(p)) return cudaErrorNotSupported;
  CUtensorMap mq, mk, mv, mo;
  cudaError_t e;
  if ((e = make_map(&mq, Q, p, kCT)) != cudaSuccess) return e;
  if ((e = make_map(&mk, K, p, kCT)) != cudaSuccess) return e;
  if ((e = make_map(&mv, V, p, kCT)) != cudaSuccess) return e;
  if ((e = make_map(&mo, O, p, kCT)) != cudaSuccess) return e;
  if ((e = ensure_smem_attr(0, reinterpret_cast<const void*>(causal_tc), kCSmemBytes)) !=
      cudaSuccess)
    return e;
  CausalArgs a = {};
  a.partials = partials;
  a.S_carry = S_carry;
  a.z_carry = z_carry;
  a.update = update;
  a.counters = counters;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.splits, (p.H + 1) / 2, p.B);
  cfg.blockDim = dim3(kCThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(kCSmemBytes);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, causal_tc, mq, mk, mv, mo, p, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t read_device_error_causal(unsigned* code, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(code, g_causal_tc_error, sizeof(unsigned));
  if (e == cudaSuccess && reset) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_causal_tc_error, &zero, sizeof(unsigned));
  }
  return e;
}

}  // namespace la
