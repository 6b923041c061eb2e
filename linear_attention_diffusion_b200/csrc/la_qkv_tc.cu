// QKV projection fused with the state reduce, on tcgen05 tensor cores.
//
// "Sana: Efficient High-Resolution Image Synthesis with Linear Diffusion
// Transformers", section Infra: the deployment kernel of the QKV projection
// also forms ReLU(K)^T V, so that the keys and values are never written to
// memory and read back. Here the projection stays in bf16 (the precision of
// the rest of the path) and the state is the one la_state_reduce forms:
//
//   [q_n, k_n, v_n] = bf16(W x_n + b)         (each rounded as stored)
//   S = sum_n phi(k_n)^T v_n,  z = sum_n ReLU(k_n)
//
// with phi = ReLU, or 3D RoPE after ReLU ("SANA-Video: Efficient Video
// Generation with Block Linear Diffusion Transformer", section 2.2). Only the
// queries leave the operation.
//
// One persistent CTA per SM walks a contiguous range of output tiles of
// 128 tokens x 256 columns (M = 128, N = 256, K = 64 per stage, both operands
// K-major straight from 128-byte-swizzled TMA tiles; the accumulator is 256
// TMEM columns). A column tile is either 256 query features, written to Q,
// or the 128 key and 128 value features of a group of four heads. For a
// key/value tile the epilogue rounds k and v to bf16, applies ReLU (and RoPE)
// to k, sums ReLU(k) over the tile's tokens on CUDA cores, and writes phi(k)
// and v to a shared-memory staging buffer in two rounds of 64 tokens; each
// round is one more MMA, phi(K)^T V (M = 128 key dims x N = 128 value dims,
// K = 64 tokens, both MN-major), accumulated in TMEM over the CTA's
// consecutive tiles of the same head group (a "run"). The four 32 x 32
// diagonal blocks of that accumulator are the heads' states. At the end of a
// run they go to a partial slot; a second kernel sums each head's slots in a
// fixed order, so S and z are bitwise reproducible.
//
// Tile order: token tiles are cut into chunks of L tiles; chunk by chunk, all
// column tiles of the chunk, each over the chunk's tokens. With L = tiles per
// CTA, the CTAs running at any moment read few distinct token rows of X, so
// X comes from HBM about once and W stays in L2.
//
// Warp roles (320 threads): warps 0-7 epilogue (warp w reads TMEM lanes
// 32 (w % 4) .. + 31, i.e. token rows; warps 0-3 the first 128 columns,
// 4-7 the last 128), warp 8 TMA producer, warp 9 TMEM allocation and the MMA
// issuer (one thread). Every wait is bounded; a wait that gives up raises the
// CTA's abort flag and the device error word, and the CTA drains its copies
// and MMAs before it frees tensor memory.
#include <algorithm>

#include "la_tc_common.cuh"

namespace la {

// Device error word of this kernel: bit 0 = a bounded wait gave up.
__device__ unsigned g_qkv_error;

namespace {

using namespace sm100;

constexpr int kQkvEpiWarps = 8;
constexpr int kQkvThreads = (kQkvEpiWarps + 2) * 32;  // 320
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr int kTok = 128;                  // tokens per tile (MMA M)
constexpr int kCols = 256;                 // output columns per tile (MMA N)
constexpr int kKBlk = 64;                  // hidden channels per stage
constexpr int kQStages = 4;
constexpr int kBoxBytes = 128 * 128;       // [128 rows][64 bf16], 128-byte swizzle
constexpr int kQStageBytes = 3 * kBoxBytes;  // X box + two W boxes (256 rows)
constexpr int kHalfTok = 64;               // tokens per state round
constexpr int kStgBox = kHalfTok * 128;    // [64 tokens][64 dims] bf16
constexpr int kStgBytes = 4 * kStgBox;     // phi(K) dims 0-63, 64-127; V the same
constexpr int kTmemState = 256;            // state accumulators at columns 256 and 384
constexpr int kQkvTmemCols = 512;
// One partial slot: the state of 4 heads (4 x 32 x 32), then the key sums of
// every TMEM lane quadrant ([4 quadrants][4 heads][32]); the quadrant sums are
// added in the combine, in quadrant order.
constexpr int kPartS = 4 * kD * kD;
constexpr int kPartFloats = kPartS + 4 * 4 * kD;

struct QSmem {  // byte offsets from the 1024-aligned base
  static constexpr int stages = 0;
  static constexpr int stg = stages + kQStages * kQStageBytes;
  static constexpr int bars = stg + kStgBytes;
  // full[S] empty[S] acc_full acc_empty stg_full stg_empty[2] state_full[2] mma_done
  static constexpr int nbars = 2 * kQStages + 8;
  static constexpr int misc = bars + nbars * 8;  // tmem base, abort flag
  static constexpr int bytes = misc + 16;
};
constexpr int kQSmemBytes = QSmem::bytes + 1024;
static_assert(kQSmemBytes <= 232448, "dynamic shared memory of one CTA");

// The static schedule, a function of (B, N, H, C) only.
struct QkvSched {
  int B, N, H, C, HD;
  int NT;     // token tiles per batch element
  int G;      // head groups of 4 (key/value column tiles)
  int QC;     // query column tiles of 256
  int CT;     // column tiles: G key/value, then QC query
  int KB;     // K-blocks of 64 channels
  int L;      // token tiles per chunk
  int NK;     // chunks per batch element
  int J;      // partial slots per (batch, group, chunk)
  int total;  // tiles
  int ctas, q, r;  // total = q * ctas + r; CTA c owns [c q + min(c, r), ...)
};

__host__ __device__ inline int sched_begin(const QkvSched& s, int c) {
  return c * s.q + (c < s.r ? c : s.r);
}

__host__ __device__ inline int sched_owner(const QkvSched& s, int i) {
  const int big = s.r * (s.q + 1);
  return i < big ? i / (s.q + 1) : s.r + (i - big) / s.q;
}

// First tile of chunk k of batch element b, and the chunk's length.
__host__ __device__ inline int chunk_begin(const QkvSched& s, int b, int k) {
  return b * s.NT * s.CT + k * s.L * s.CT;
}
__host__ __device__ inline int chunk_len(const QkvSched& s, int k) {
  const int rest = s.NT - k * s.L;
  return rest < s.L ? rest : s.L;
}

struct Tile {
  int kv;     // 1: key/value columns of head group g; 0: query column tile
  int b, nt;  // batch element, token tile
  int col;    // g or the query column tile
  int k;      // chunk
  int run0;   // kv: first tile of the run's (b, k, g) block
  int first;  // kv: first tile of its run in this CTA
  int last;   // kv: last tile of its run in this CTA
};

__device__ __forceinline__ Tile decode(const QkvSched& s, int i, int i_begin, int i_end) {
  Tile t;
  t.b = i / (s.NT * s.CT);
  int rem = i - t.b * s.NT * s.CT;
  t.k = rem / (s.L * s.CT);
  rem -= t.k * s.L * s.CT;
  const int len = chunk_len(s, t.k);
  const int ct = rem / len;
  t.nt = t.k * s.L + (rem - ct * len);
  t.kv = ct < s.G;
  t.col = t.kv ? ct : ct - s.G;
  t.run0 = chunk_begin(s, t.b, t.k) + ct * len;
  t.first = t.kv && i == max(i_begin, t.run0);
  t.last = t.kv && i == min(i_end, t.run0 + len) - 1;
  return t;
}

// Column sums of a warp: x[j] of lane l holds element (row l, column j); on
// return x[0] of lane l holds the sum over the warp's rows of column l. 31
// shuffles; the pairing, and with it the rounding, is fixed.
template <int kOff>
__device__ __forceinline__ void colsum_step(float (&x)[32], int lane) {
  const bool up = (lane & kOff) != 0;
#pragma unroll
  for (int i = 0; i < kOff; ++i) {
    const float send = up ? x[i] : x[i + kOff];
    const float keep = up ? x[i + kOff] : x[i];
    x[i] = keep + __shfl_xor_sync(0xffffffffu, send, kOff);
  }
}
__device__ __forceinline__ float warp_colsum(float (&x)[32], int lane) {
  colsum_step<16>(x, lane);
  colsum_step<8>(x, lane);
  colsum_step<4>(x, lane);
  colsum_step<2>(x, lane);
  colsum_step<1>(x, lane);
  return x[0];
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <int kRope>
__global__ void __launch_bounds__(kQkvThreads, 1)
qkv_state_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
             const QkvSched sc, const Rope rope, const __nv_bfloat16* __restrict__ bias,
             __nv_bfloat16* __restrict__ Q, float* __restrict__ part) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + QSmem::bars);
  uint64_t* empty = full + kQStages;
  uint64_t* acc_full = empty + kQStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* stg_full = acc_empty + 1;
  uint64_t* stg_empty = stg_full + 1;   // [2]: round 0, round 1
  uint64_t* state_full = stg_empty + 2;  // [2]: run parity
  uint64_t* mma_done = state_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + QSmem::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + QSmem::misc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;
  const int i_begin = sched_begin(sc, cta), i_end = sched_begin(sc, cta + 1);

  if (tid == 0) {
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kQkvEpiWarps * 32);
    mbar_init(stg_full, 4 * 32);  // the four warps of one round's token rows
    mbar_init(&stg_empty[0], 1);
    mbar_init(&stg_empty[1], 1);
    mbar_init(&state_full[0], 1);
    mbar_init(&state_full[1], 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, kQkvTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == kWarpTma && lane == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_w);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);

  // Programmatic dependent launch: global memory only after the previous grid
  // has completed; the combine may then be scheduled.
  pdl_wait();
  if (tid == 0) pdl_trigger();

  if (warp == kWarpTma) {
    // ---------------------------------------------------------- TMA loads
    if (lane == 0) {
      int pos = 0;
      bool ok = true;
      for (int i = i_begin; ok && i < i_end; ++i) {
        const Tile t = decode(sc, i, i_begin, i_end);
        const int y = t.nt * kTok;
        // key/value tile: the group's 128 key rows and 128 value rows of W;
        // query tile: 256 consecutive query rows. Rows past H*32 of a section
        // read as zero.
        const int wy0 = t.kv ? t.col * 128 : t.col * kCols;
        const int wy1 = t.kv ? t.col * 128 : t.col * kCols + 128;
        const int wz0 = t.kv ? 1 : 0, wz1 = t.kv ? 2 : 0;
        for (int kb = 0; kb < sc.KB; ++kb, ++pos) {
          const int s = pos % kQStages;
          if (!(ok = mbar_wait(&empty[s], ((pos / kQStages) & 1) ^ 1, abort_flag, &g_qkv_error,
                               kErrWait)))
            break;
          mbar_arrive_expect_tx(&full[s], kQStageBytes);
          uint8_t* st = smem + QSmem::stages + s * kQStageBytes;
          const int x = kb * kKBlk;
          tma_load_3d(st, &tm_x, &full[s], x, y, t.b);
          tma_load_3d(st + kBoxBytes, &tm_w, &full[s], x, wy0, wz0);
          tma_load_3d(st + 2 * kBoxBytes, &tm_w, &full[s], x, wy1, wz1);
        }
      }
      // every load issued must have landed before the CTA exits
      for (int qq = max(0, pos - kQStages); qq < pos; ++qq)
        mbar_drain(&full[qq % kQStages], (qq / kQStages) & 1, &g_qkv_error, kErrWait);
    }
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id_gemm = idesc_bf16_f32(kTok, kCols, 0, 0);
      const uint32_t id_state = idesc_bf16_f32(128, 128, 1, 1);
      const uint32_t stg = sbase + QSmem::stg;
      int pending = 0;  // state rounds whose accumulator tile has been committed
      int u = 0;        // state rounds issued so far
      int svc_i = i_begin, svc_r = 0, run = -1;
      bool have = false;
      Tile svc{};
      // Issue the next state round if its staging is written. Rounds are
      // issued in tile order, between the GEMM's K-blocks.
      auto service = [&]() -> bool {
        if (pending == 0 || !mbar_try_wait(stg_full, u & 1)) return false;
        if (!have) {
          while (svc_i < i_end) {
            svc = decode(sc, svc_i, i_begin, i_end);
            if (svc.kv) break;
            ++svc_i;
          }
          have = true;
          if (svc.first) ++run;
        }
        tc_fence_after();
        const uint32_t acc = tmem + kTmemState + (run & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < kHalfTok / 16; ++kk) {
          // 16 tokens = two 8-row groups; LBO = the second 64-dim box
          const uint64_t ad = smem_desc_sw128(stg + kk * 2048, kStgBox, 1024);
          const uint64_t bd = smem_desc_sw128(stg + 2 * kStgBox + kk * 2048, kStgBox, 1024);
          mma_bf16(acc, ad, bd, id_state, (svc.first && svc_r == 0 && kk == 0) ? 0u : 1u);
        }
        mma_commit(&stg_empty[svc_r]);
        if (svc_r == 1) {
          if (svc.last) mma_commit(&state_full[run & 1]);
          have = false;
          ++svc_i;
          svc_r = 0;
        } else {
          svc_r = 1;
        }
        ++u;
        --pending;
        return true;
      };
      // Bounded wait for a barrier phase (or, with bar == nullptr, for every
      // pending state round) that keeps issuing state rounds meanwhile: the
      // epilogue's next accumulator read may be waiting for one.
      auto wait_svc = [&](uint64_t* bar, uint32_t parity) -> bool {
        uint64_t t0 = globaltimer_ns();
        while (true) {
          if (bar != nullptr ? mbar_try_wait(bar, parity) : pending == 0) return true;
          if (service()) {
            t0 = globaltimer_ns();
            continue;
          }
          if (*abort_flag) return false;
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicOr(&g_qkv_error, kErrWait);
            return false;
          }
        }
      };
      int pos = 0;
      bool ok = true;
      for (int i = i_begin; ok && i < i_end; ++i) {
        const int tl = i - i_begin;
        const bool kv = decode(sc, i, i_begin, i_end).kv;
        // the epilogue has read the previous tile's accumulator
        if (!(ok = wait_svc(acc_empty, (tl & 1) ^ 1))) break;
        tc_fence_after();
        for (int kb = 0; kb < sc.KB; ++kb, ++pos) {
          const int s = pos % kQStages;
          if (!(ok = wait_svc(&full[s], (pos / kQStages) & 1))) break;
          tc_fence_after();
          const uint32_t st = sbase + QSmem::stages + s * kQStageBytes;
#pragma unroll
          for (int kk = 0; kk < kKBlk / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(st + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(st + kBoxBytes + kk * 32, 16, 1024);
            mma_bf16(tmem, ad, bd, id_gemm, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
          service();
        }
        if (!ok) break;
        mma_commit(acc_full);
        if (kv) pending += 2;
      }
      if (ok) wait_svc(nullptr, 0);
      mma_commit(mma_done);
      mbar_drain(mma_done, 0, &g_qkv_error, kErrWait);
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int quad = warp & 3;       // TMEM lane quadrant: token rows 32 quad ..
    const int hf = warp >> 2;        // 0: columns 0-127 (keys), 1: 128-255 (values)
    const int row = quad * 32 + lane;
    const int rnd = quad >> 1;       // state round of this row
    const int srow = row - rnd * kHalfTok;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t stg = sbase + QSmem::stg + (hf ? 2 * kStgBox : 0);
    float zacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    int kv_seen = 0, run = -1;
    for (int i = i_begin; i < i_end; ++i) {
      const Tile t = decode(sc, i, i_begin, i_end);
      const int tl = i - i_begin;
      bool ok = mbar_wait(acc_full, tl & 1, abort_flag, &g_qkv_error, kErrWait);
      if (!__all_sync(0xffffffffu, ok)) break;  // tcgen05.ld is warp-collective
      tc_fence_after();
      const int n = t.nt * kTok + row;
      const bool valid = n < sc.N;
      // first feature (row of W, entry of the bias) of this warp's 128 columns
      const int f0 = t.kv ? (1 + hf) * sc.HD + t.col * 128 : t.col * kCols + hf * 128;
      const int f_end = t.kv ? (2 + hf) * sc.HD : sc.HD;
      uint32_t pk[64];  // the row's 128 features: bf16(acc + bias), in pairs
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        float v[32];
        tmem_ld_32x32b_x32(tmem + lane_base + hf * 128 + ch * 32, v);
        const int f = f0 + ch * 32;
        if (f < f_end) {  // H*32 is a multiple of 32: a chunk is all in or all out
          if (bias != nullptr) {
            const uint4* bp = reinterpret_cast<const uint4*>(bias + f);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint4 w4 = __ldg(bp + k);
              const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                v[8 * k + 2 * e] += bf16_lo(w[e]);
                v[8 * k + 2 * e + 1] += bf16_hi(w[e]);
              }
            }
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[ch * 16 + e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[ch * 16 + e] = 0u;
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty);  // the accumulator may take the next tile

      if (!t.kv) {
        // ---- query tile: the row's features straight to Q
        if (valid) {
          __nv_bfloat16* dst = Q + (static_cast<size_t>(t.b) * sc.N + n) * sc.HD + f0;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            if (f0 + ch * 32 >= sc.HD) break;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              *reinterpret_cast<uint4*>(dst + ch * 32 + 8 * k) =
                  make_uint4(pk[ch * 16 + 4 * k], pk[ch * 16 + 4 * k + 1],
                             pk[ch * 16 + 4 * k + 2], pk[ch * 16 + 4 * k + 3]);
          }
        }
        continue;
      }

      // ---- key/value tile
      if (t.first) ++run;
      if (!valid) {
#pragma unroll
        for (int e = 0; e < 64; ++e) pk[e] = 0u;
      }
      if (hf == 0) {
        // keys: ReLU (exact on bf16), key sums of the unrotated ReLU(k)
#pragma unroll
        for (int e = 0; e < 64; ++e) pk[e] = relu_bf16x2(pk[e]);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          float x[32];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            x[2 * e] = bf16_lo(pk[ch * 16 + e]);
            x[2 * e + 1] = bf16_hi(pk[ch * 16 + e]);
          }
          zacc[ch] += warp_colsum(x, lane);
        }
        if (kRope != kNoRope && valid) {
          // phi(k) = R(t, h, w) ReLU(k): pair j of every head turns by the
          // token's position on the pair's axis times inv_freq[j]
          const TokPos tp = token_pos(rope, n);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int ax = pair_axis(j);
            const int pp = ax == 0 ? rope.t_offset + tp.t : (ax == 1 ? tp.h : tp.w);
            float2 r;
            rope_cos_sin(pp, rope.inv_freq[j], r.x, r.y);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {  // the same angle for every head
              const uint32_t w = pk[ch * 16 + j];
              const float x0 = bf16_lo(w), x1 = bf16_hi(w);
              const float2 tt = __fmul2_rn(make_float2(x1, x1), make_float2(-r.y, r.x));
              const float2 yy = __ffma2_rn(make_float2(x0, x0), r, tt);
              pk[ch * 16 + j] = pack_bf16x2(yy.x, yy.y);
            }
          }
        }
      }
      // staging: wait until the previous round's MMA has read it. Each round
      // has its own barrier, which completes once per key/value tile: round 0
      // waits for round 1 of the previous tile, round 1 for round 0 of this
      // one. (With one barrier for both rounds a writer could be two phases
      // ahead of it, which a parity wait cannot tell from the phase it wants.)
      ok = rnd == 0 ? mbar_wait(&stg_empty[1], (kv_seen & 1) ^ 1, abort_flag, &g_qkv_error,
                                kErrWait)
                    : mbar_wait(&stg_empty[0], kv_seen & 1, abort_flag, &g_qkv_error, kErrWait);
      if (!__all_sync(0xffffffffu, ok)) break;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          st_shared_v4(stg + (ch >> 1) * kStgBox + sw128_offset(srow, (ch & 1) * 4 + k),
                       make_uint4(pk[ch * 16 + 4 * k], pk[ch * 16 + 4 * k + 1],
                                  pk[ch * 16 + 4 * k + 2], pk[ch * 16 + 4 * k + 3]));
      fence_proxy_async_smem();
      mbar_arrive(stg_full);
      ++kv_seen;

      if (t.last && hf == 0) {
        // ---- end of a run: head `quad`'s state block and this quadrant's
        // key sums go to the run's partial slot
        const int a = run & 1;
        ok = mbar_wait(&state_full[a], (run >> 1) & 1, abort_flag, &g_qkv_error, kErrWait);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
        float s[32];
        tmem_ld_32x32b_x32(tmem + lane_base + kTmemState + a * 128 + quad * 32, s);
        tc_fence_before();
        const int g = t.col;
        const int slot = cta - sched_owner(sc, t.run0);
        float* dst = part + ((static_cast<size_t>(t.b * sc.G + g) * sc.NK + t.k) * sc.J + slot) *
                                kPartFloats;
        float* ds = dst + quad * kD * kD + lane * kD;
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(ds + e) = make_float4(s[e], s[e + 1], s[e + 2], s[e + 3]);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          dst[kPartS + quad * 4 * kD + ch * kD + lane] = zacc[ch];
          zacc[ch] = 0.0f;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kQkvTmemCols);
  }
}

// Sum of the partial slots of one (batch, head group) in a fixed order:
// chunk, then slot, then (for z) TMEM lane quadrant.
__global__ void __launch_bounds__(256)
qkv_combine(const QkvSched sc, const float* __restrict__ part, float* __restrict__ S,
            float* __restrict__ z) {
  pdl_wait();
  const int bg = blockIdx.x;
  const int b = bg / sc.G, g = bg - b * sc.G;
  const float* base = part + static_cast<size_t>(bg) * sc.NK * sc.J * kPartFloats;
  for (int v = threadIdx.x; v < (kPartS + 4 * kD) / 4; v += blockDim.x) {
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int k = 0; k < sc.NK; ++k) {
      const int len = chunk_len(sc, k);
      const int run0 = chunk_begin(sc, b, k) + g * len;
      const int nslots = sched_owner(sc, run0 + len - 1) - sched_owner(sc, run0) + 1;
      for (int j = 0; j < nslots; ++j) {
        const float* src = base + (static_cast<size_t>(k) * sc.J + j) * kPartFloats;
        if (v < kPartS / 4) {
          const float4 t = __ldcg(reinterpret_cast<const float4*>(src) + v);
          acc.x += t.x;
          acc.y += t.y;
          acc.z += t.z;
          acc.w += t.w;
        } else {
#pragma unroll
          for (int qd = 0; qd < 4; ++qd) {
            const float4 t = __ldcg(reinterpret_cast<const float4*>(src + kPartS + qd * 4 * kD) +
                                    (v - kPartS / 4));
            acc.x += t.x;
            acc.y += t.y;
            acc.z += t.z;
            acc.w += t.w;
          }
        }
      }
    }
    if (v < kPartS / 4) {
      const int hh = v / (kD * kD / 4), h = 4 * g + hh;
      if (h < sc.H)
        *reinterpret_cast<float4*>(S + (static_cast<size_t>(b) * sc.H + h) * kD * kD +
                                   (v - hh * (kD * kD / 4)) * 4) = acc;
    } else {
      const int w = v - kPartS / 4;  // head w / 8, dims 4 (w % 8) ..
      const int hh = w >> 3, h = 4 * g + hh;
      if (h < sc.H)
        *reinterpret_cast<float4*>(z + (static_cast<size_t>(b) * sc.H + h) * kD + (w & 7) * 4) =
            acc;
    }
  }
}

// ============================================================== host side

QkvSched make_sched(int B, int N, int H, int C) {
  QkvSched s{};
  s.B = B;
  s.N = N;
  s.H = H;
  s.C = C;
  s.HD = H * kD;
  s.NT = (N + kTok - 1) / kTok;
  s.G = (H + 3) / 4;
  s.QC = (s.HD + kCols - 1) / kCols;
  s.CT = s.G + s.QC;
  s.KB = (C + kKBlk - 1) / kKBlk;
  const long long total = 1LL * B * s.NT * s.CT;
  s.total = static_cast<int>(total);
  s.ctas = static_cast<int>(std::min<long long>(kNumSMs, std::max<long long>(1, total)));
  s.q = std::max(1, s.total / s.ctas);
  s.r = s.total - s.q * s.ctas;
  s.L = std::max(1, std::min(s.NT, s.q));
  s.NK = (s.NT + s.L - 1) / s.L;
  s.J = std::min(s.L, (s.L - 1) / s.q + 2);
  return s;
}

// [d2][d1][d0] bf16 viewed as a 3D tensor; box = 64 x 128 x 1, 128-byte swizzle.
cudaError_t make_map_qkv(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1,
                         uint64_t d2) {
  cudaError_t e = get_encoder();
  if (e != cudaSuccess) return e;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

using QkvKernel = void (*)(CUtensorMap, CUtensorMap, QkvSched, Rope, const __nv_bfloat16*,
                           __nv_bfloat16*, float*);

}  // namespace

size_t qkv_workspace_floats(int B, int N, int H, int C) {
  if (N <= 0 || B <= 0 || H <= 0) return 0;
  const QkvSched s = make_sched(B, N, H, C);
  return static_cast<size_t>(B) * s.G * s.NK * s.J * kPartFloats;
}

cudaError_t launch_qkv_state(const Problem& p, int C, const void* X, const void* W,
                             const void* bias, void* Q, float* S, float* z, float* part,
                             cudaStream_t s) {
  const QkvSched sc = make_sched(p.B, p.N, p.H, C);
  CUtensorMap mx, mw;
  cudaError_t e;
  if ((e = make_map_qkv(&mx, X, C, p.N, p.B)) != cudaSuccess) return e;
  if ((e = make_map_qkv(&mw, W, C, static_cast<uint64_t>(p.H) * kD, 3)) != cudaSuccess) return e;
  const int mode = p.rope.enabled ? kRopeOnTheFly : kNoRope;
  QkvKernel kern = mode == kNoRope ? qkv_state_tc<kNoRope> : qkv_state_tc<kRopeOnTheFly>;
  if ((e = ensure_smem_attr(mode == kNoRope ? 0 : 1, reinterpret_cast<const void*>(kern),
                            kQSmemBytes)) != cudaSuccess)
    return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sc.ctas, 1, 1);
  cfg.blockDim = dim3(kQkvThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(kQSmemBytes);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, mx, mw, sc, p.rope,
                         static_cast<const __nv_bfloat16*>(bias), static_cast<__nv_bfloat16*>(Q),
                         part);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg2 = {};
  cfg2.gridDim = dim3(p.B * sc.G, 1, 1);
  cfg2.blockDim = dim3(256, 1, 1);
  cfg2.stream = s;
  cfg2.attrs = attr;
  cfg2.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg2, qkv_combine, sc, static_cast<const float*>(part), S, z);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t read_device_error_qkv(unsigned* code, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(code, g_qkv_error, sizeof(unsigned));
  if (e == cudaSuccess && reset) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_qkv_error, &zero, sizeof(unsigned));
  }
  return e;
}

}  // namespace la
