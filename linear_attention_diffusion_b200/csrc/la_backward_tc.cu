// Tensor-core (tcgen05) backward of the bf16 layer. What it computes is the
// gradient of the Sana Linear DiT's ReLU linear attention ("Sana: Efficient
// High-Resolution Image Synthesis with Linear Diffusion Transformers", section
// Infra: the attention is trained with a fused forward and backward kernel),
// with the RoPE-after-ReLU numerator of "SANA-Video: Efficient Video
// Generation with Block Linear Diffusion Transformer", section 2.2. With
// den_n = ReLU(q_n) . z + eps and R_n the token's rotation:
//
//   dnum_n = dO_n / den_n,   t_n = S dnum_n^T,   u_n = R_n^T t_n
//   dden_n = -(ReLU(q_n) . u_n) / den_n      (= -(dO_n . O_n) / den_n)
//   dQ_n   = [u_n + dden_n z] * [q_n > 0]
//   dS     = sum_n phi(q_n)^T dnum_n,        dz = sum_n dden_n ReLU(q_n)
//   dK_n   = [R_n^T (dS v_n^T) + dz] * [k_n > 0],   dV_n = phi(k_n) dS
//
// Query side (one launch, grid = token splits x head pairs x batch): per
// 128-token tile of a head pair (one 64-dim TMA box per tensor),
//   transform  Q -> ReLU(Q) and dO -> dnum (bf16) in place in shared memory;
//   MMA 1      t = dnum S^T per head (M = 128 tokens, N = 32, K = 32) into TMEM;
//   epilogue   dden, dQ, dz on CUDA cores;
//   rewrite    ReLU(Q) -> phi(Q) in place (RoPE only);
//   MMA 2      dS += phi(Q)^T dnum (the reduce's MN-major form, M = 128 with
//              the upper 64 rows unused, N = 64, K = 16 tokens; the two 32x32
//              diagonal blocks are the heads' dS).
// Without RoPE phi(Q) = ReLU(Q) is ready after the transform, so MMA 1 and
// MMA 2 are issued together; dQ then goes over the dnum box in shared memory
// and out with one TMA store. With RoPE, MMA 2 waits for the rewrite and dQ
// is stored from registers.
// The split partials of (dS, dz) are combined by the last CTA of each head
// pair in split order, as in the state reduce: deterministic.
//
// Key side (one launch, grid = tile ranges x head pairs x batch): per tile,
//   transform  K -> phi(K) in place (the sign mask stays in registers);
//   MMA 1      dphi(K) = V dS^T per head; epilogue dK = R^T dphi(K) + dz,
//              masked, written over the V tile (MMA 1 has read it);
//   MMA 2      dV = phi(K) dS per head, in the same TMEM columns; dV written
//              over the K tile; dK and dV stored with TMA.
//
// Warp roles: warp 0 TMA, warp 1 MMA (one elected lane), warps 2..13 three
// math warpgroups. Six stages of 32 KB: tile j uses stage j mod 6 and TMEM
// columns [64 s, 64 s + 64), and belongs to warpgroup j mod 3, so each
// warpgroup owns two stages (its next tile loads while it works on the
// current one) and every mbarrier has one consumer that waits for its phases
// in order (a parity wait cannot tell phase k from k + 2). Two heads per CTA
// keep the tiles small enough for six stages; the split count (query side)
// and tile ranges (key side) are chosen for head pairs so the grid still
// covers the SMs in one wave. Every wait is bounded and raises the device
// error word when it gives up.
#include <algorithm>

#include "la_tc_common.cuh"

namespace la {

// Device error word of the backward kernels (same meaning as the forward's).
__device__ unsigned g_bwd_tc_error;

namespace {

constexpr int kBT = 128;                // tokens per tile
constexpr int kBBox = kBT * 128;        // [128 tokens][64 dims] bf16 = 16 KB
constexpr int kBTile = 2 * kBBox;       // two tensors = 32 KB
constexpr int kBStages = 6;
constexpr int kBWG = 3;                 // math warpgroups (two stages each)
constexpr int kPair = 2;                // heads per CTA
constexpr uint32_t kColDS = 64 * kBStages;  // query side: dS accumulator (64 columns)
constexpr int kBMath = kBWG * 128;
constexpr int kBThreads = 64 + kBMath;
constexpr int kBTmemCols = 512;
constexpr int kBarAll = 1;              // named barrier over the math threads
constexpr int kBarW0 = 2;               // + warpgroup

struct QSmem {  // query side, byte offsets from the 1024-aligned base
  static constexpr int stages = 0;                          // [6][Q box, dO box]
  static constexpr int bop = stages + kBStages * kBTile;    // S as B operand: [32 rows][128 B]
  static constexpr int zs = bop + 4096;                     // [2][32] f32
  static constexpr int dden = zs + 256;                     // [3][128 rows][2] f32
  static constexpr int sraw = dden + kBWG * kBT * kPair * 4;  // S of the pair as copied: [2][32][32] f32
  static constexpr int rope = sraw + kPair * kD * kD * 4;     // float2[kRopeTableMax]
  static constexpr int bars = rope + kRopeTableMax * 8;
  // full[6] empty[6] ready_t[6] ready_s[6] t_full[6] o_full[6] s2_done[6]
  // acc_full mma_done b_ready s_full
  static constexpr int nbars = 7 * kBStages + 4;
  static constexpr int misc = bars + nbars * 8;
  static constexpr int bytes = misc + 16;
};
struct KVSmem {  // key side
  static constexpr int stages = 0;                          // [6][K box, V box]
  static constexpr int bop1 = stages + kBStages * kBTile;   // dS rows d (K = e)
  static constexpr int bop2 = bop1 + 4096;                  // dS^T rows e (K = d)
  static constexpr int zs = bop2 + 4096;                    // dz [2][32] f32
  static constexpr int rope = zs + 256;
  static constexpr int bars = rope + kRopeTableMax * 8;
  // full[6] empty[6] ready[6] t_full[6] t_empty[6] b_ready mma_done
  static constexpr int nbars = 5 * kBStages + 2;
  static constexpr int misc = bars + nbars * 8;
  static constexpr int bytes = misc + 16;
};
constexpr int kQSmemBytes = QSmem::bytes + 1024;
constexpr int kKVSmemBytes = KVSmem::bytes + 1024;
static_assert(kQSmemBytes <= 232448 && kKVSmemBytes <= 232448, "shared memory per CTA");

struct BwdArgs {
  float* partials;        // query side: [B*H][splits][kStateFloats]
  unsigned* arrive;       // query side: per head-pair arrival counters (index b*H + h0)
  StateOut out;           // query side: where the combined (dS, dz) goes
  const float* S;         // query side: the forward state; key side: dS
  const float* z;         // query side: z; key side: dz
  __nv_bfloat16* dQ;      // query side output
  int tiles_per_cta;      // key side
  int kv_before_wait;     // key side: K, V may be fetched before the previous grid completes
};

// (cos, sin) of the 16 pairs of token n (the row's RoPE rotation).
template <int kRope>
__device__ __forceinline__ void row_angles(const Problem& p, const float2* tab, int n,
                                           float2 (&cs)[16]) {
  const TokPos tp = token_pos(p.rope, min(n, p.N - 1));
  const RopeBases rb = rope_bases(p.rope, tp);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int ax = pair_axis(j);
    if (kRope == kRopeTable) {
      cs[j] = tab[(ax == 0 ? rb.t : (ax == 1 ? rb.h : rb.w)) + pair_off(j)];
    } else {
      const int pp = ax == 0 ? p.rope.t_offset + tp.t : (ax == 1 ? tp.h : tp.w);
      rope_cos_sin(pp, p.rope.inv_freq[j], cs[j].x, cs[j].y);
    }
  }
}

// x <- R x (sign = +1) or R^T x (sign = -1) for the 4 pairs of a chunk whose
// first pair is j0.
template <int kSign>
__device__ __forceinline__ void rotate_chunk(const float2 (&cs)[16], int j0, float (&x)[8]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 r = cs[j0 + q];
    const float sn = kSign > 0 ? r.y : -r.y;
    const float2 t = __fmul2_rn(make_float2(x[2 * q + 1], x[2 * q + 1]), make_float2(-sn, r.x));
    const float2 y = __ffma2_rn(make_float2(x[2 * q], x[2 * q]), make_float2(r.x, sn), t);
    x[2 * q] = y.x;
    x[2 * q + 1] = y.y;
  }
}

// Build a head pair's B operand in shared memory from a float32 [heads][32][32]
// global array M: row r holds M[h][r][0..31] (transpose = 0) or M[h][0..31][r]
// (transpose = 1) of heads h0 and h0 + 1, in bf16, K-major with the 128-byte
// swizzle. A missing head is zero.
__device__ __forceinline__ void build_bop(uint32_t bop, const float* M, size_t cidx, int h0,
                                          int H, bool transpose, int mt, int nthreads) {
  for (int idx = mt; idx < 32 * 8; idx += nthreads) {
    const int r = idx >> 3, c = idx & 7;
    const int hh = c >> 2, k0 = (c & 3) * 8;
    float x[8];
    if (h0 + hh < H) {
      const float* m = M + (cidx + hh) * kD * kD;
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] = transpose ? __ldcg(m + (k0 + k) * kD + r) : __ldcg(m + r * kD + k0 + k);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] = 0.0f;
    }
    st_shared_v4(bop + sw128_offset(r, c), pack8(x));
  }
}

// ================================================================ query side

template <int kRope>
__global__ void __launch_bounds__(kBThreads, 1)
bwd_q_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_g,
         const __grid_constant__ CUtensorMap tm_dq, const Problem p, const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + QSmem::bars);
  uint64_t* empty = full + kBStages;
  uint64_t* ready_t = empty + kBStages;   // tile transformed (128 arrivals)
  uint64_t* ready_s = ready_t + kBStages; // phi(Q) in place, dz done (128 arrivals)
  uint64_t* t_full = ready_s + kBStages;  // t of the stage's tile is in TMEM
  uint64_t* o_full = t_full + kBStages;   // dQ of the stage's tile in its dO box
  uint64_t* s2_done = o_full + kBStages;  // RoPE: MMA 2 of the stage's tile done
  uint64_t* acc_full = s2_done + kBStages;
  uint64_t* mma_done = acc_full + 1;
  uint64_t* b_ready = mma_done + 1;
  uint64_t* s_full = b_ready + 1;         // S and z of the pair copied in
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + QSmem::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + QSmem::misc + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + QSmem::misc + 8);
  float* zs = reinterpret_cast<float*>(smem + QSmem::zs);
  float* dden_buf = reinterpret_cast<float*>(smem + QSmem::dden);
  float2* rope_tab = reinterpret_cast<float2*>(smem + QSmem::rope);
  unsigned* err = &g_bwd_tc_error;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pair = blockIdx.y, b = blockIdx.z;
  const int h0 = pair * kPair;
  const size_t cidx = static_cast<size_t>(b) * p.H + h0;
  const int n_begin = blockIdx.x * p.chunk;
  const int n_end = min(p.N, n_begin + p.chunk);
  const int nT = n_end > n_begin ? (n_end - n_begin + kBT - 1) / kBT : 0;

  if (tid == 0) {
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&ready_t[s], 128);
      mbar_init(&ready_s[s], 128);
      mbar_init(&t_full[s], 1);
      mbar_init(&o_full[s], 1);
      mbar_init(&s2_done[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(mma_done, 1);
    mbar_init(b_ready, 1);
    mbar_init(s_full, 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kBTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_g);
    prefetch_tmap(&tm_dq);
  }
  if (kRope == kRopeTable && tid >= 64) build_rope_table(p.rope, rope_tab, tid - 64, kBMath);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);
  pdl_wait();
  if (tid == 64) pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA loads
    if (lane == 0) {
      // S and z of the pair first, ahead of the tiles in the memory queues
      const int heads = min(kPair, p.H - h0);
      mbar_arrive_expect_tx(s_full, heads * (kD * kD + kD) * 4);
      bulk_load(smem + QSmem::sraw, a.S + cidx * kD * kD, heads * kD * kD * 4, s_full);
      bulk_load(smem + QSmem::zs, a.z + cidx * kD, heads * kD * 4, s_full);
      // The warpgroups leave dQ in the tile's dO box (o_full) once both MMAs
      // have read the stage, and this thread stores it with TMA before it
      // reloads the stage.
      auto store_dq = [&](int k) -> bool {
        const int ks = k % kBStages;
        if (!mbar_wait(&o_full[ks], (k / kBStages) & 1, abort_flag, err, kErrWait)) return false;
        tma_store_3d(&tm_dq, smem + QSmem::stages + ks * kBTile + kBBox, h0 * 32, n_begin + k * kBT, b);
        bulk_commit();
        bulk_wait_read<0>();
        return true;
      };
      int i = 0;
      bool ok = true;
      for (; i < nT; ++i) {
        const int s = i % kBStages;
        if (i >= kBStages) {
          if (!(ok = store_dq(i - kBStages))) break;
        } else if (!mbar_wait(&empty[s], ((i / kBStages) & 1) ^ 1, abort_flag, err, kErrWait)) {
          break;
        }
        mbar_arrive_expect_tx(&full[s], kBTile);
        uint8_t* st = smem + QSmem::stages + s * kBTile;
        const int y = n_begin + i * kBT;
        tma_load_3d(st, &tm_q, &full[s], h0 * 32, y, b);
        tma_load_3d(st + kBBox, &tm_g, &full[s], h0 * 32, y, b);
      }
      for (int k = max(0, i - kBStages); ok && k < i; ++k) ok = store_dq(k);
      for (int q = max(0, i - kBStages); q < i; ++q)
        mbar_drain(&full[q % kBStages], (q / kBStages) & 1, err, kErrWait);
      bulk_wait<0>();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      bool ok = nT == 0 || mbar_wait(b_ready, 0, abort_flag, err, kErrWait);
      const uint32_t id_t = idesc_bf16_f32(128, 32, 0, 0);
      const uint32_t id_s = idesc_bf16_f32(128, 64, 1, 1);
      const uint64_t bop0 = smem_desc_sw128(sbase + QSmem::bop, 16, 1024);
      // Without RoPE, phi(Q) = ReLU(Q) is in place after the transform, so both
      // MMAs of a tile go at once and the epilogue may then write dQ over the
      // dnum box. With RoPE, MMA 2 of tile i - 1 (after the warpgroup has
      // rotated Q in place) is issued after MMA 1 of tile i.
      for (int i = 0; kRope == kNoRope && ok && i < nT; ++i) {
        const int s = i % kBStages;
        if (!(ok = mbar_wait(&ready_t[s], (i / kBStages) & 1, abort_flag, err, kErrWait))) break;
        tc_fence_after();
        const uint32_t st = sbase + QSmem::stages + s * kBTile;
        const uint64_t g0 = smem_desc_sw128(st + kBBox, 16, 1024);
#pragma unroll
        for (int hh = 0; hh < kPair; ++hh)
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_bf16(tmem + 64 * s + hh * 32, desc_at(g0, hh * 64 + kk * 32),
                     desc_at(bop0, hh * 64 + kk * 32), id_t, kk);
        const uint64_t a0 = smem_desc_sw128(st, kBBox, 1024);
        const uint64_t b0 = smem_desc_sw128(st + kBBox, kBBox, 1024);
#pragma unroll
        for (int kk = 0; kk < kBT / 16; ++kk)
          mma_bf16(tmem + kColDS, desc_at(a0, kk * 2048), desc_at(b0, kk * 2048), id_s,
                   (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&t_full[s]);
      }
      for (int i = 0; kRope != kNoRope && ok && i <= nT; ++i) {
        if (i < nT) {
          const int s = i % kBStages;
          if (!(ok = mbar_wait(&ready_t[s], (i / kBStages) & 1, abort_flag, err, kErrWait))) break;
          tc_fence_after();
          const uint64_t g0 = smem_desc_sw128(sbase + QSmem::stages + s * kBTile + kBBox, 16, 1024);
#pragma unroll
          for (int hh = 0; hh < kPair; ++hh) {
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              const uint64_t ad = desc_at(g0, hh * 64 + kk * 32);
              const uint64_t bd = desc_at(bop0, hh * 64 + kk * 32);
              mma_bf16(tmem + 64 * s + hh * 32, ad, bd, id_t, kk);
            }
          }
          mma_commit(&t_full[s]);
        }
        const int k = i - 1;
        if (k >= 0) {
          const int s = k % kBStages;
          if (!(ok = mbar_wait(&ready_s[s], (k / kBStages) & 1, abort_flag, err, kErrWait))) break;
          tc_fence_after();
          const uint32_t st = sbase + QSmem::stages + s * kBTile;
          // A: phi(Q) as M = 128 dims; its second 64-dim atom (LBO) is the
          // dO box, whose rows of the product are not used
          const uint64_t a0 = smem_desc_sw128(st, kBBox, 1024);
          const uint64_t b0 = smem_desc_sw128(st + kBBox, kBBox, 1024);
#pragma unroll
          for (int kk = 0; kk < kBT / 16; ++kk) {
            const uint64_t ad = desc_at(a0, kk * 2048);
            const uint64_t bd = desc_at(b0, kk * 2048);
            mma_bf16(tmem + kColDS, ad, bd, id_s, (k > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&s2_done[s]);  // the warpgroup then writes dQ over the dnum box
        }
      }
      mma_commit(acc_full);
      mma_commit(mma_done);
      mbar_drain(mma_done, 0, err, kErrWait);
    }
  } else {
    // ---------------------------------------------------------- math warps
    const int mt = tid - 64;
    const int wg = mt >> 7, wt = mt & 127;
    const int quad = warp & 3;            // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;     // token row of the tile (thread = row)
    bool alive = true;

    // S as the B operand of MMA 1 (rows d, K = e), z of the two heads: the
    // TMA warp has copied the pair's S and z in (a missing head is zero)
    {
      const int heads = min(kPair, p.H - h0);
      if (mt >= heads * kD && mt < kPair * kD) zs[mt] = 0.0f;
      if (!mbar_wait(s_full, 0, abort_flag, err, kErrWait)) alive = false;
      const float* sr = reinterpret_cast<const float*>(smem + QSmem::sraw);
      for (int idx = mt; idx < 32 * 8; idx += kBMath) {
        const int r = idx >> 3, c = idx & 7;
        const int hh = c >> 2, k0 = (c & 3) * 8;
        float x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = hh < heads ? sr[hh * kD * kD + r * kD + k0 + k] : 0.0f;
        st_shared_v4(sbase + QSmem::bop + sw128_offset(r, c), pack8(x));
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(kBarAll, kBMath);
    if (mt == 0) mbar_arrive(b_ready);

    // dz of dims [(c&3)*8, +8) of head c>>2 over rows rg, rg + 16, ...
    const int zc = wt & 7, zrg = wt >> 3;
    float zacc[8] = {};
    float* my_dden = dden_buf + wg * kBT * kPair;

    for (int j = wg; j < nT; j += kBWG) {
      const int s = j % kBStages;  // wg or wg + 3
      const uint32_t par = (j / kBStages) & 1;
      bool ok = mbar_wait(&full[s], par, abort_flag, err, kErrWait);
      if (bar_any(kBarW0 + wg, 128, !ok || *abort_flag)) {
        alive = false;
        break;
      }
      const uint32_t st = sbase + QSmem::stages + s * kBTile;
      const int n0 = n_begin + j * kBT;
      const int n = n0 + row;
      float2 cs[16];
      if (kRope != kNoRope) row_angles<kRope>(p, rope_tab, n, cs);

      // ---- transform: ReLU(Q) in place, den, dnum = dO / den in place.
      // Without RoPE a head's eight shared-memory loads go first (a store
      // orders every later access after it) and den is four partial sums;
      // with RoPE (short of registers) one 16-byte chunk at a time.
      float inv[kPair];
      if (kRope == kNoRope) {
#pragma unroll
        for (int hh = 0; hh < kPair; ++hh) {
          uint4 uq[4], ug[4];
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uq[c4] = ld_shared_v4(st + sw128_offset(row, hh * 4 + c4));
            ug[c4] = ld_shared_v4(st + kBBox + sw128_offset(row, hh * 4 + c4));
          }
          float dp[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uq[c4].x = relu_bf16x2(uq[c4].x);
            uq[c4].y = relu_bf16x2(uq[c4].y);
            uq[c4].z = relu_bf16x2(uq[c4].z);
            uq[c4].w = relu_bf16x2(uq[c4].w);
            float x[8];
            unpack8(uq[c4], x);
            const float* zz = zs + hh * kD + c4 * 8;
#pragma unroll
            for (int e = 0; e < 8; ++e) dp[e & 3] = fmaf(x[e], zz[e], dp[e & 3]);
          }
          inv[hh] = 1.0f / (((dp[0] + dp[1]) + (dp[2] + dp[3])) + p.eps);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            st_shared_v4(st + sw128_offset(row, hh * 4 + c4), uq[c4]);
            float x[8];
            unpack8(ug[c4], x);
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] *= inv[hh];
            st_shared_v4(st + kBBox + sw128_offset(row, hh * 4 + c4), pack8(x));
          }
        }
      } else {
#pragma unroll
        for (int hh = 0; hh < kPair; ++hh) {
          float den = 0.0f;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int c = hh * 4 + c4;
            const uint32_t addr = st + sw128_offset(row, c);
            uint4 u = ld_shared_v4(addr);
            u.x = relu_bf16x2(u.x);
            u.y = relu_bf16x2(u.y);
            u.z = relu_bf16x2(u.z);
            u.w = relu_bf16x2(u.w);
            float x[8];
            unpack8(u, x);
            const float* zz = zs + hh * kD + c4 * 8;
#pragma unroll
            for (int e = 0; e < 8; ++e) den = fmaf(x[e], zz[e], den);
            st_shared_v4(addr, u);
          }
          inv[hh] = 1.0f / (den + p.eps);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int c = hh * 4 + c4;
            const uint32_t addr = st + kBBox + sw128_offset(row, c);
            float x[8];
            unpack8(ld_shared_v4(addr), x);
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] *= inv[hh];
            st_shared_v4(addr, pack8(x));
          }
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&ready_t[s]);

      // ---- epilogue: u = R^T t, dden, dQ, per head
      ok = mbar_wait(&t_full[s], par, abort_flag, err, kErrWait);
      tc_fence_after();
      if (bar_any(kBarW0 + wg, 128, !ok || *abort_flag)) {
        alive = false;
        break;
      }
      uint4 dq[kPair][4];  // RoPE: this row's dQ until MMA 2 has read the stage
#pragma unroll
      for (int hh = 0; hh < kPair; ++hh) {
        float t[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + 64 * s + hh * 32, t);
        if (kRope != kNoRope) {
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = t[c4 * 8 + e];
            rotate_chunk<-1>(cs, c4 * 4, y);
#pragma unroll
            for (int e = 0; e < 8; ++e) t[c4 * 8 + e] = y[e];
          }
        }
        // ReLU(q) of the row: without RoPE the four loads go together and
        // are kept for dQ; with RoPE (short of registers) one chunk at a time,
        // read again below
        uint4 uq[4];
        if (kRope == kNoRope) {
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) uq[c4] = ld_shared_v4(st + sw128_offset(row, hh * 4 + c4));
        }
        float dot;
        if (kRope == kNoRope) {
          float dp[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            float x[8];
            unpack8(uq[c4], x);
#pragma unroll
            for (int e = 0; e < 8; ++e) dp[e & 3] = fmaf(x[e], t[c4 * 8 + e], dp[e & 3]);
          }
          dot = (dp[0] + dp[1]) + (dp[2] + dp[3]);
        } else {
          dot = 0.0f;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            float x[8];
            unpack8(ld_shared_v4(st + sw128_offset(row, hh * 4 + c4)), x);
#pragma unroll
            for (int e = 0; e < 8; ++e) dot = fmaf(x[e], t[c4 * 8 + e], dot);
          }
        }
        const float dden = -dot * inv[hh];
        my_dden[row * kPair + hh] = dden;
        if (kRope == kNoRope) {
          // both MMAs are done: dQ goes over the dnum box, stored with TMA
          // (rows and heads beyond the tensor are clipped by the store)
          const float* zz = zs + hh * kD;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int c = hh * 4 + c4;
            float x[8];
            unpack8(uq[c4], x);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int d = c4 * 8 + e;
              x[e] = x[e] > 0.0f ? fmaf(dden, zz[d], t[d]) : 0.0f;
            }
            st_shared_v4(st + kBBox + sw128_offset(row, c), pack8(x));
          }
        } else {
          // MMA 2 still reads the dnum box: dQ waits in registers
          const float* zz = zs + hh * kD;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int c = hh * 4 + c4;
            float x[8];
            unpack8(ld_shared_v4(st + sw128_offset(row, c)), x);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int d = c4 * 8 + e;
              x[e] = x[e] > 0.0f ? fmaf(dden, zz[d], t[d]) : 0.0f;
            }
            dq[hh][c4] = pack8(x);
          }
        }
      }
      tc_fence_before();
      if (kRope == kNoRope) fence_proxy_async_smem();  // dQ in shared memory, for the store
      named_bar_sync(kBarW0 + wg, 128);

      // ---- dz over the tile's rows (fixed order per thread)
      {
        const int hh = zc >> 2;
#pragma unroll 4
        for (int r = zrg; r < kBT; r += 16) {
          float x[8];
          unpack8(ld_shared_v4(st + sw128_offset(r, zc)), x);
          const float dd = my_dden[r * kPair + hh];
#pragma unroll
          for (int e = 0; e < 8; ++e) zacc[e] = fmaf(dd, x[e], zacc[e]);
        }
      }
      named_bar_sync(kBarW0 + wg, 128);

      if (kRope == kNoRope) {
        // the stage is done with: the TMA warp stores dQ and reloads it
        if (wt == 0) mbar_arrive(&o_full[s]);
        continue;
      }
      // ---- rewrite ReLU(Q) -> phi(Q) for MMA 2
      if (kRope != kNoRope) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t addr = st + sw128_offset(row, c);
          float x[8];
          unpack8(ld_shared_v4(addr), x);
          rotate_chunk<1>(cs, (c & 3) * 4, x);
          st_shared_v4(addr, pack8(x));
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&ready_s[s]);
      // ---- once MMA 2 has read the stage, dQ goes over the dnum box and the
      // TMA warp stores it (rows and heads beyond the tensor are clipped)
      ok = mbar_wait(&s2_done[s], par, abort_flag, err, kErrWait);
      if (bar_any(kBarW0 + wg, 128, !ok || *abort_flag)) {
        alive = false;
        break;
      }
#pragma unroll
      for (int hh = 0; hh < kPair; ++hh)
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
          st_shared_v4(st + kBBox + sw128_offset(row, hh * 4 + c4), dq[hh][c4]);
      fence_proxy_async_smem();
      named_bar_sync(kBarW0 + wg, 128);
      if (wt == 0) mbar_arrive(&o_full[s]);
    }

    // ---- partial (dS, dz) of this split
    alive = !bar_any(kBarAll, kBMath, !alive || *abort_flag);
    float* scratch = reinterpret_cast<float*>(smem + QSmem::stages);  // [kBMath][8] after the MMAs
    if (warp >= 2 && warp < 6 && (warp & 3) < kPair) {  // TMEM lanes of head q's dS rows
      const int q = warp & 3;
      float v[32];
      bool got = alive && nT > 0 && mbar_wait(acc_full, 0, abort_flag, err, kErrWait);
      got = __all_sync(0xffffffffu, got);
      if (got) {
        tc_fence_after();
        tmem_ld_32x32b_x32(tmem + kColDS + (static_cast<uint32_t>(32 * q) << 16) + 32 * q, v);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0.0f;
      }
      if (h0 + q < p.H) {
        float* dst = a.partials + ((cidx + q) * p.splits + blockIdx.x) * kStateFloats + lane * kD;
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
      }
    }
    // every MMA has completed (acc_full) before the stages are reused as scratch
    bool drained = !alive || nT == 0 || mbar_wait(acc_full, 0, abort_flag, err, kErrWait);
    alive = !bar_any(kBarAll, kBMath, !drained || *abort_flag) && alive;
    if (alive) {
#pragma unroll
      for (int e = 0; e < 8; ++e) scratch[mt * 8 + e] = zacc[e];
    }
    named_bar_sync(kBarAll, kBMath);
    if (alive && mt < kPair * kD) {
      const int q = mt >> 5, d = mt & 31;
      const int col = q * 4 + (d >> 3), e = d & 7;
      float sum = 0.0f;
      for (int w = 0; w < kBWG; ++w)
        for (int rg = 0; rg < 16; ++rg) sum += scratch[(w * 128 + rg * 8 + col) * 8 + e];
      if (h0 + q < p.H)
        a.partials[((cidx + q) * p.splits + blockIdx.x) * kStateFloats + kD * kD + d] = sum;
    }
    tc_fence_before();

    // ---- last CTA of the head group: sum the splits in order
    named_bar_sync(kBarAll, kBMath);
    if (mt == 0) {
      fence_acq_rel_gpu();
      const unsigned prev = atomicAdd(&a.arrive[cidx], 1u);
      *last_flag = prev == gridDim.x - 1;
      if (*last_flag) fence_acq_rel_gpu();
    }
    named_bar_sync(kBarAll, kBMath);
    const bool last = *last_flag != 0;
    if (last && alive) combine_from_global<kBMath, kPair>(p, b, h0, mt, a.partials, a.out);
    named_bar_sync(kBarAll, kBMath);
    if (mt == 0 && last) a.arrive[cidx] = 0u;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBTmemCols);
  }
}

// ================================================================== key side

template <int kRope>
__global__ void __launch_bounds__(kBThreads, 1)
bwd_kv_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
          const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
          const Problem p, const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + KVSmem::bars);
  uint64_t* empty = full + kBStages;
  uint64_t* ready = empty + kBStages;    // tile transformed (128 arrivals)
  uint64_t* t_full = ready + kBStages;   // MMA 1, then MMA 2, of the stage's tile done
  uint64_t* t_empty = t_full + kBStages; // their results read out of TMEM
  uint64_t* b_ready = t_empty + kBStages;
  uint64_t* mma_done = b_ready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + KVSmem::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + KVSmem::misc + 4);
  float* zs = reinterpret_cast<float*>(smem + KVSmem::zs);
  float2* rope_tab = reinterpret_cast<float2*>(smem + KVSmem::rope);
  unsigned* err = &g_bwd_tc_error;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pair = blockIdx.y, b = blockIdx.z;
  const int h0 = pair * kPair;
  const size_t cidx = static_cast<size_t>(b) * p.H + h0;
  const int ntiles_all = (p.N + kBT - 1) / kBT;
  const int tile_begin = blockIdx.x * a.tiles_per_cta;
  const int nT = max(0, min(ntiles_all, tile_begin + a.tiles_per_cta) - tile_begin);

  if (tid == 0) {
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&ready[s], 128);
      mbar_init(&t_full[s], 1);
      mbar_init(&t_empty[s], 1);
    }
    mbar_init(b_ready, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kBTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_dk);
    prefetch_tmap(&tm_dv);
  }
  if (kRope == kRopeTable && tid >= 64) build_rope_table(p.rope, rope_tab, tid - 64, kBMath);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);
  // K and V are inputs the query side does not write: the TMA warp may fetch
  // them before that grid completes; dS and dz are read after the wait.
  if (!(warp == 0 && a.kv_before_wait)) pdl_wait();
  if (tid == 64) pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      int i = 0;
      for (; i < nT; ++i) {
        const int s = i % kBStages;
        if (!mbar_wait(&empty[s], ((i / kBStages) & 1) ^ 1, abort_flag, err, kErrWait)) break;
        mbar_arrive_expect_tx(&full[s], kBTile);
        uint8_t* st = smem + KVSmem::stages + s * kBTile;
        const int y = (tile_begin + i) * kBT;
        tma_load_3d(st, &tm_k, &full[s], h0 * 32, y, b);
        tma_load_3d(st + kBBox, &tm_v, &full[s], h0 * 32, y, b);
      }
      for (int q = max(0, i - kBStages); q < i; ++q)
        mbar_drain(&full[q % kBStages], (q / kBStages) & 1, err, kErrWait);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = nT == 0 || mbar_wait(b_ready, 0, abort_flag, err, kErrWait);
      const uint32_t id = idesc_bf16_f32(128, 32, 0, 0);
      const uint64_t bop1d = smem_desc_sw128(sbase + KVSmem::bop1, 16, 1024);
      const uint64_t bop2d = smem_desc_sw128(sbase + KVSmem::bop2, 16, 1024);
      // t_empty[s] completes twice per tile (MMA 1's and MMA 2's results
      // read), so the waits alternate parity 1 (before MMA 1) and 0 (before
      // MMA 2). MMA 2 of tile i - 1 is issued after MMA 1 of tile i.
      for (int i = 0; ok && i <= nT; ++i) {
        if (i < nT) {
          const int s = i % kBStages;
          if (!(ok = mbar_wait(&ready[s], (i / kBStages) & 1, abort_flag, err, kErrWait))) break;
          if (!(ok = mbar_wait(&t_empty[s], 1, abort_flag, err, kErrWait))) break;
          tc_fence_after();
          const uint64_t v0 = smem_desc_sw128(sbase + KVSmem::stages + s * kBTile + kBBox, 16, 1024);
#pragma unroll
          for (int hh = 0; hh < kPair; ++hh) {
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              // dphi(K)[n][d] = sum_e V[n][e] dS[d][e]
              const uint64_t av = desc_at(v0, hh * 64 + kk * 32);
              const uint64_t bd = desc_at(bop1d, hh * 64 + kk * 32);
              mma_bf16(tmem + s * 64 + hh * 32, av, bd, id, kk);
            }
          }
          mma_commit(&t_full[s]);
        }
        const int k = i - 1;
        if (k >= 0) {
          const int s = k % kBStages;
          if (!(ok = mbar_wait(&t_empty[s], 0, abort_flag, err, kErrWait))) break;
          tc_fence_after();
          const uint64_t k0 = smem_desc_sw128(sbase + KVSmem::stages + s * kBTile, 16, 1024);
#pragma unroll
          for (int hh = 0; hh < kPair; ++hh) {
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              // dV[n][e] = sum_d phi(K)[n][d] dS[d][e]
              const uint64_t ak = desc_at(k0, hh * 64 + kk * 32);
              const uint64_t bd = desc_at(bop2d, hh * 64 + kk * 32);
              mma_bf16(tmem + s * 64 + hh * 32, ak, bd, id, kk);
            }
          }
          mma_commit(&t_full[s]);
        }
      }
      mma_commit(mma_done);
      mbar_drain(mma_done, 0, err, kErrWait);
    }
  } else {
    const int mt = tid - 64;
    const int wg = mt >> 7, wt = mt & 127;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const bool leader = wt == 0;

    build_bop(sbase + KVSmem::bop1, a.S, cidx, h0, p.H, false, mt, kBMath);
    build_bop(sbase + KVSmem::bop2, a.S, cidx, h0, p.H, true, mt, kBMath);
    if (mt < kPair * kD) zs[mt] = h0 + mt / kD < p.H ? __ldcg(a.z + cidx * kD + mt) : 0.0f;
    fence_proxy_async_smem();
    named_bar_sync(kBarAll, kBMath);
    if (mt == 0) mbar_arrive(b_ready);

    for (int j = wg; j < nT; j += kBWG) {
      const int s = j % kBStages;  // wg or wg + 3
      bool ok = mbar_wait(&full[s], (j / kBStages) & 1, abort_flag, err, kErrWait);
      if (bar_any(kBarW0 + wg, 128, !ok || *abort_flag)) break;
      const uint32_t st = sbase + KVSmem::stages + s * kBTile;
      const int n0 = (tile_begin + j) * kBT;
      float2 cs[16];
      if (kRope != kNoRope) row_angles<kRope>(p, rope_tab, n0 + row, cs);

      // ---- transform: K -> phi(K) in place; keep the sign mask of K
      uint32_t mask[kPair] = {0u, 0u};
      // without RoPE a head's four loads go first (a store orders every later
      // access after it); with RoPE (short of registers) one chunk at a time
#pragma unroll
      for (int hh = 0; hh < kPair; ++hh) {
        uint4 kv[4];
        if (kRope == kNoRope) {
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) kv[c4] = ld_shared_v4(st + sw128_offset(row, hh * 4 + c4));
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int c = hh * 4 + c4;
          uint4 v = kRope == kNoRope ? kv[c4] : ld_shared_v4(st + sw128_offset(row, c));
          v.x = relu_bf16x2(v.x);
          v.y = relu_bf16x2(v.y);
          v.z = relu_bf16x2(v.z);
          v.w = relu_bf16x2(v.w);
          float x[8];
          unpack8(v, x);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if (x[e] > 0.0f) mask[hh] |= 1u << (c4 * 8 + e);
          if (kRope != kNoRope) {
            rotate_chunk<1>(cs, c4 * 4, x);
            v = pack8(x);
          }
          st_shared_v4(st + sw128_offset(row, c), v);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&ready[s]);

      const uint32_t tcol = tmem + (static_cast<uint32_t>(quad * 32) << 16) + s * 64;
      // ---- dK = R^T dphi(K) + dz, masked, over the V tile (MMA 1 has read it)
      ok = mbar_wait(&t_full[s], 0, abort_flag, err, kErrWait);
      tc_fence_after();
      if (bar_any(kBarW0 + wg, 128, !ok || *abort_flag)) break;
#pragma unroll
      for (int hh = 0; hh < kPair; ++hh) {
        float g[32];
        tmem_ld_32x32b_x32(tcol + hh * 32, g);
        const float* zz = zs + hh * kD;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = g[c4 * 8 + e];
          if (kRope != kNoRope) rotate_chunk<-1>(cs, c4 * 4, x);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int d = c4 * 8 + e;
            x[e] = (mask[hh] >> d) & 1u ? x[e] + zz[d] : 0.0f;
          }
          const int c = hh * 4 + c4;
          st_shared_v4(st + kBBox + sw128_offset(row, c), pack8(x));
        }
      }
      tc_fence_before();
      named_bar_sync(kBarW0 + wg, 128);
      if (leader) mbar_arrive(&t_empty[s]);

      // ---- dV over the K tile (MMA 2 has read phi(K)), then both stores
      ok = mbar_wait(&t_full[s], 1, abort_flag, err, kErrWait);
      tc_fence_after();
      if (bar_any(kBarW0 + wg, 128, !ok || *abort_flag)) break;
#pragma unroll
      for (int hh = 0; hh < kPair; ++hh) {
        float g[32];
        tmem_ld_32x32b_x32(tcol + hh * 32, g);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = g[c4 * 8 + e];
          const int c = hh * 4 + c4;
          st_shared_v4(st + sw128_offset(row, c), pack8(x));
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      named_bar_sync(kBarW0 + wg, 128);
      if (leader) {
        mbar_arrive(&t_empty[s]);
        uint8_t* tile = smem + KVSmem::stages + s * kBTile;
        tma_store_3d(&tm_dk, tile + kBBox, h0 * 32, n0, b);
        tma_store_3d(&tm_dv, tile, h0 * 32, n0, b);
        bulk_commit();
        bulk_wait_read<0>();
        mbar_arrive(&empty[s]);
      }
    }
    if (leader) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBTmemCols);
  }
}

// ============================================================== host side

// Launch with programmatic dependent launch: the prologue (barriers, TMEM,
// RoPE table) may overlap the previous kernel in the stream.
template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel kern, dim3 grid, int smem, cudaStream_t s, const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kBThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace

cudaError_t launch_backward_q_tc(const Problem& p, const void* Q, const void* dO, const float* S,
                                 const float* z, void* dQ, float* partials, unsigned* counters,
                                 const StateOut& out, cudaStream_t s) {
  CUtensorMap mq, mg, mdq;
  cudaError_t e;
  if ((e = make_map(&mq, Q, p, kBT)) != cudaSuccess) return e;
  if ((e = make_map(&mg, dO, p, kBT)) != cudaSuccess) return e;
  if ((e = make_map(&mdq, dQ, p, kBT)) != cudaSuccess) return e;
  const int mode = rope_mode(rope_table_for(p));
  auto kern = mode == kNoRope ? bwd_q_tc<kNoRope>
                              : (mode == kRopeTable ? bwd_q_tc<kRopeTable> : bwd_q_tc<kRopeOnTheFly>);
  if ((e = ensure_smem_attr(mode, reinterpret_cast<const void*>(kern), kQSmemBytes)) != cudaSuccess)
    return e;
  BwdArgs a = {};
  a.partials = partials;
  a.arrive = counters;
  a.out = out;
  a.S = S;
  a.z = z;
  a.dQ = static_cast<__nv_bfloat16*>(dQ);
  // token splits for head pairs (one wave); never more than the state
  // reduce's, for which the workspace is sized
  const int pairs = (p.H + kPair - 1) / kPair;
  Problem pb = p;
  const long long units = static_cast<long long>(pairs) * p.B;
  int splits = static_cast<int>(std::max<long long>(1, kNumSMs / std::max<long long>(1, units)));
  splits = std::min(splits, std::min(p.splits, (p.N + kBT - 1) / kBT));
  pb.chunk = ((p.N + splits - 1) / splits + kBT - 1) / kBT * kBT;
  pb.splits = (p.N + pb.chunk - 1) / pb.chunk;
  const dim3 grid(pb.splits, pairs, p.B);
  e = launch_pdl(kern, grid, kQSmemBytes, s, mq, mg, mdq, pb, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_backward_kv_tc(const Problem& p, const void* K, const void* V, const float* dS,
                                  const float* dz, void* dK, void* dV, bool after_own_q,
                                  cudaStream_t s) {
  CUtensorMap mk, mv, mdk, mdv;
  cudaError_t e;
  if ((e = make_map(&mk, K, p, kBT)) != cudaSuccess) return e;
  if ((e = make_map(&mv, V, p, kBT)) != cudaSuccess) return e;
  if ((e = make_map(&mdk, dK, p, kBT)) != cudaSuccess) return e;
  if ((e = make_map(&mdv, dV, p, kBT)) != cudaSuccess) return e;
  const int mode = rope_mode(rope_table_for(p));
  auto kern = mode == kNoRope
                  ? bwd_kv_tc<kNoRope>
                  : (mode == kRopeTable ? bwd_kv_tc<kRopeTable> : bwd_kv_tc<kRopeOnTheFly>);
  if ((e = ensure_smem_attr(3 + mode, reinterpret_cast<const void*>(kern), kKVSmemBytes)) !=
      cudaSuccess)
    return e;
  const int groups = (p.H + kPair - 1) / kPair;
  const int ntiles = (p.N + kBT - 1) / kBT;
  const long long units = static_cast<long long>(groups) * p.B;
  int ctas = static_cast<int>(std::max<long long>(1, kNumSMs / std::max<long long>(1, units)));
  ctas = std::min(ctas, ntiles);
  const int tpc = (ntiles + ctas - 1) / ctas;
  ctas = (ntiles + tpc - 1) / tpc;
  BwdArgs a = {};
  a.S = dS;
  a.z = dz;
  a.tiles_per_cta = tpc;
  a.kv_before_wait = after_own_q ? 1 : 0;
  const dim3 grid(ctas, groups, p.B);
  e = launch_pdl(kern, grid, kKVSmemBytes, s, mk, mv, mdk, mdv, p, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t read_device_error_bwd(unsigned* code, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(code, g_bwd_tc_error, sizeof(unsigned));
  if (e == cudaSuccess && reset) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_bwd_tc_error, &zero, sizeof(unsigned));
  }
  return e;
}

}  // namespace la
